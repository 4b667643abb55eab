"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them element by element."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

# Tolerances of the matching rule: fp32 configurations max-abs 1e-4; bf16
# configurations max-abs relative to max|ref| 2e-2.
TOL_F32_ABS = 1e-4
TOL_BF16_REL = 2e-2
# conf is fp32 on the GPU, fp64 in the oracle; the sum over V terms carries
# at most a few 1e-7 relative error, so 1e-5 bounds it with margin.
CONF_TOL = 1e-5


def dtype_name(t: torch.Tensor) -> str:
    return {torch.float32: "f32", torch.bfloat16: "bf16"}[t.dtype]


def assert_close(gpu, ref, dtype, what):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite values from the GPU"
    err = np.abs(gpu - ref).max() if gpu.size else 0.0
    if dtype == "f32":
        assert err <= TOL_F32_ABS, f"{what}: max-abs error {err:.3e} > {TOL_F32_ABS}"
    else:
        scale = np.abs(ref).max() if ref.size else 0.0
        assert err <= TOL_BF16_REL * scale, \
            f"{what}: max-abs error {err:.3e} > {TOL_BF16_REL} * max|ref| = {TOL_BF16_REL * scale:.3e}"
    return err


def oracle_fused(inp: dict, H: int, dh: int, rope_base: float, dtype: str):
    f = O.to_f64
    return O.fused_step(f(inp["x"]), inp["q_idx"].numpy(), f(inp["w_qkv"]), rope_base,
                        f(inp["k_cache"]), f(inp["v_cache"]), H, dh, dtype)


def oracle_verify(inp: dict, H: int, dh: int, rope_base: float, dtype: str, causal=False):
    f = O.to_f64
    return O.verify_step(f(inp["x_rows"]), inp["pos"].numpy(), inp["view"].numpy(),
                         inp["rank"].numpy(), f(inp["w_qkv"]), rope_base, f(inp["k_cache"]),
                         f(inp["v_cache"]), f(inp["k_side"]), f(inp["v_side"]), H, dh, dtype,
                         causal)


def check_cache_update(k_gpu, k_in, k_ref, q_idx, dtype, what):
    """Slots outside Q must be bit-identical to the input; slots in Q must match
    the oracle's rounded k/v within tolerance.  k_gpu, k_in: torch CPU tensors
    [B, H, N, dh]; k_ref: float64 [B, H, N, dh]; q_idx: int [B, nq]."""
    B, H, N, dh = k_gpu.shape
    for b in range(B):
        inq = np.zeros(N, bool)
        inq[q_idx[b]] = True
        rest = torch.from_numpy(~inq)
        assert torch.equal(k_gpu[b][:, rest], k_in[b][:, rest]), \
            f"{what}: a slot outside Q changed in sequence {b}"
        assert_close(O.to_f64(k_gpu[b][:, torch.from_numpy(inq)]), k_ref[b][:, inq], dtype,
                     f"{what} written slots, sequence {b}")


def check_outside_q_on_device(k_dev, k_in, idx, what, written_mask=None):
    """Every slot of every sequence outside its written set is bit-identical to
    the input, compared on the device.  k_dev: the cache after the call (CUDA,
    [B, H, N, dh]); k_in: the input cache (CPU); idx: int [B, n] the written
    slots (entries outside [0, N) ignored), or written_mask: bool [B, N]."""
    B, H, N, dh = k_dev.shape
    if written_mask is None:
        written_mask = np.zeros((B, N), bool)
        ix = np.asarray(idx)
        for b in range(B):
            ok = ix[b][(ix[b] >= 0) & (ix[b] < N)]
            written_mask[b, ok] = True
    for b in range(B):
        keep = torch.from_numpy(~written_mask[b]).to(k_dev.device)
        ref = k_in[b].to(k_dev.device)
        assert torch.equal(k_dev[b][:, keep], ref[:, keep]), \
            f"{what}: a slot outside the written set changed in sequence {b}"


def run_fused_gpu(F, inp_dev: dict, rope_base: float):
    x = inp_dev["x"]
    B, N, D = x.shape
    H, dh = inp_dev["k_cache"].shape[1], inp_dev["k_cache"].shape[3]
    nq = inp_dev["q_idx"].shape[1]
    out = torch.empty((B, nq, H * dh), dtype=x.dtype, device=x.device)
    ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(B, N, D, H, dh, nq, x.dtype), x.device)
    F.fdllm_fused_step(x, inp_dev["q_idx"], inp_dev["w_qkv"], inp_dev["k_cache"],
                       inp_dev["v_cache"], out, ws, rope_base=rope_base)
    st = F.fdllm_get_status(ws)
    return out, ws, st


def run_verify_gpu(F, inp_dev: dict, rope_base: float, causal=False):
    x = inp_dev["x_rows"]
    B, R, D = x.shape
    H, N, dh = inp_dev["k_cache"].shape[1], inp_dev["k_cache"].shape[2], inp_dev["k_cache"].shape[3]
    S_max = inp_dev["k_side"].shape[2]
    out = torch.empty((B, R, H * dh), dtype=x.dtype, device=x.device)
    ws = F.alloc_workspace(F.fdllm_verify_step_workspace_bytes(B, N, D, H, dh, R, S_max, x.dtype),
                           x.device)
    F.fdllm_verify_step(x, inp_dev["pos"], inp_dev["view"], inp_dev["rank"], inp_dev["w_qkv"],
                        inp_dev["k_cache"], inp_dev["v_cache"], inp_dev["k_side"],
                        inp_dev["v_side"], out, ws, rope_base=rope_base, causal_cross=causal)
    st = F.fdllm_get_status(ws)
    return out, ws, st


def run_accept_gpu(F, logits, kind, ref_tok, rank, eps, gamma):
    B, R, V = logits.shape
    dev = logits.device
    top1 = torch.empty((B, R), dtype=torch.int32, device=dev)
    conf = torch.empty((B, R), dtype=torch.float32, device=dev)
    flags = torch.empty((B, R), dtype=torch.uint8, device=dev)
    n_acc = torch.empty((B,), dtype=torch.int32, device=dev)
    ws = F.alloc_workspace(F.fdllm_accept_workspace_bytes(B, R, V), dev)
    F.fdllm_accept(logits, kind, ref_tok, rank, top1, conf, flags, n_acc, ws, eps=eps, gamma=gamma)
    torch.cuda.synchronize()
    return top1.cpu().numpy(), conf.cpu().numpy(), flags.cpu().numpy(), n_acc.cpu().numpy(), ws


def check_accept(gpu, ref, kind, rank, eps, gamma):
    """top1 bit-exact; conf within CONF_TOL; flags and n_accept exact except where
    the oracle's confidence lies within CONF_TOL of a threshold (both decisions
    are then correct); there the GPU's flags must agree with its own confidence
    and the prefix rule must hold on the GPU's own pass bits."""
    t_g, c_g, f_g, n_g = gpu
    t_r, c_r, f_r, n_r = ref
    np.testing.assert_array_equal(t_g, t_r)
    assert np.abs(c_g - c_r).max() <= CONF_TOL, np.abs(c_g - c_r).max()
    amb = ((kind == 1) & (np.abs(c_r - eps) < CONF_TOL)) | ((kind == 2) & (np.abs(c_r - gamma) < CONF_TOL))
    B, R = kind.shape
    seq_amb = amb.any(axis=1)
    for b in range(B):
        if not seq_amb[b]:
            np.testing.assert_array_equal(f_g[b], f_r[b])
            assert n_g[b] == n_r[b]
        else:  # valid on its own terms
            pas = (f_g[b] & O.FLAG_PASS) > 0
            fails = [rank[b, r] for r in range(R) if kind[b, r] == 2 and not pas[r]]
            ff = min(fails) if fails else np.inf
            acc = np.array([(kind[b, r] == 2) and rank[b, r] < ff for r in range(R)])
            np.testing.assert_array_equal((f_g[b] & O.FLAG_ACCEPT) > 0, acc)
            assert n_g[b] == acc.sum()
    return int(amb.sum())


def check_track(track, mass, ref, cand, beta_t, dt):
    """A tracked-set selection from the GPU (track [B, beta_t], mass [B, N]) is
    valid against the oracle's masses ref [B, N]: the masses match within the
    tolerance; the first min(beta_t, candidates) entries are distinct
    candidates in the GPU's own order (mass descending, equal mass to the lower
    slot) and the rest are -1; and no candidate left out is heavier than a
    chosen one beyond what the tolerance allows.  The GPU ranks by its own
    masses, each within tol of the oracle's, so a chosen slot may be up to
    2 tol lighter (in the oracle's masses) than one left out."""
    scale = max(float(np.abs(ref).max()), 1e-30)
    tol = (1e-4 if dt == "f32" else 2e-2) * scale
    err = float(np.abs(mass - ref).max())
    assert err <= tol, f"mass max error {err:.3e} > {tol:.3e}"
    B, N = ref.shape
    for b in range(B):
        cands = np.nonzero(cand[b])[0]
        k = min(beta_t, cands.size)
        sel = track[b, :k]
        assert (track[b, k:] == -1).all(), "padding past the candidates must be -1"
        assert len(set(sel.tolist())) == k, "selected slots must be distinct"
        assert all(cand[b, j] for j in sel), "selected slots must be candidates"
        for t in range(k - 1):
            a0, a1 = mass[b, sel[t]], mass[b, sel[t + 1]]
            assert a0 > a1 or (a0 == a1 and sel[t] < sel[t + 1]), "order"
        rest = np.setdiff1d(cands, sel)
        if k and rest.size:
            assert ref[b, sel].min() >= ref[b, rest].max() - 2 * tol, \
                "a heavier candidate was left out"
