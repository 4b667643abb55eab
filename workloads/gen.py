"""Seeded synthetic workloads for the fused KV-cache step.

Every tensor is drawn from its own PCG64 substream keyed by (seed, tensor tag,
sequence index), so one sequence of a large batch can be regenerated on its own
(the oracle checks sampled sequences of the big configurations this way) and
the values do not depend on how many sequences were asked for.

Shapes follow the method's workloads (Flash-dLLM review, "Performance
Validation: Key Results", Experimental Setup: generation lengths 256/512,
beta_m up to 64, batch up to 32) scaled to the five synthetic configurations.
No dataset or trained weight is involved: hidden states and cache entries are
N(0,1), W_qkv is N(0, 1/D).

Draws are made in float32 and rounded once (round to nearest even, by torch) to
the storage dtype.  Rows of x outside the query set are never read by the step;
they are left at zero here (and a parity test poisons them with NaN).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

# name -> configuration.  kind "fused": query set Q = T (tracked) + front
# beta_m masks; kind "verify": rows [T_v | draft view over S | mask view over S].
CONFIGS = {
    "tiny_fp32": dict(kind="fused", B=1, N=64, n_prompt=32, D=256, H=4, dh=64,
                      n_track=2, beta_m=2, dtype="f32", seed=0, rope_base=10000.0),
    "single_bf16": dict(kind="fused", B=1, N=1024, n_prompt=512, D=4096, H=32,
                        dh=128, n_track=16, beta_m=16, dtype="bf16", seed=1,
                        rope_base=10000.0),
    "verify_bf16": dict(kind="verify", B=8, N=2048, n_prompt=1536, D=4096, H=32,
                        dh=128, n_tv=8, n_s=16, dtype="bf16", seed=2,
                        rope_base=10000.0, vocab=126464),
    "long_bf16": dict(kind="fused", B=1, N=16384, n_prompt=15360, D=4096, H=32,
                      dh=128, n_track=32, beta_m=32, dtype="bf16", seed=3,
                      rope_base=10000.0),
    "batch_bf16": dict(kind="fused", B=64, N=4096, n_prompt=3584, D=4096, H=32,
                       dh=128, n_track=16, beta_m=16, dtype="bf16", seed=4,
                       rope_base=10000.0),
}

_TAGS = {"w": 1, "x": 2, "k": 3, "v": 4, "idx": 5, "xr": 6, "ks": 7, "vs": 8,
         "logit": 9, "spike": 10}

_THREADS = max(1, min(32, os.cpu_count() or 1))


def _rng(seed: int, tag: str, b: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAGS[tag], b])))


def _store(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def _torch_dtype(dtype: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]


def _normal(seed, tag, b, shape, scale=1.0):
    a = _rng(seed, tag, b).standard_normal(int(np.prod(shape)), dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a.reshape(shape)


def _per_seq(fn, seqs):
    if len(seqs) <= 1:
        return [fn(b) for b in seqs]
    with ThreadPoolExecutor(_THREADS) as ex:
        return list(ex.map(fn, seqs))


def weights(cfg: dict) -> torch.Tensor:
    """W_qkv [3*H*dh, D]: rows are the q block, then k, then v; head-major inside a block."""
    E = cfg["H"] * cfg["dh"]
    D = cfg["D"]
    return _store(_normal(cfg["seed"], "w", 0, (3 * E, D), 1.0 / math.sqrt(D)), cfg["dtype"])


def cache(cfg: dict, seqs, tag: str, n_slots: int | None = None) -> torch.Tensor:
    """A K or V cache [len(seqs), H, n_slots, dh] of N(0,1) entries."""
    H, dh = cfg["H"], cfg["dh"]
    n = cfg["N"] if n_slots is None else n_slots
    out = torch.empty((len(seqs), H, n, dh), dtype=_torch_dtype(cfg["dtype"]))

    def one(i_b):
        i, b = i_b
        out[i] = _store(_normal(cfg["seed"], tag, b, (H, n, dh)), cfg["dtype"])

    _per_seq(one, list(enumerate(seqs)))
    return out


def query_positions(cfg: dict, b: int):
    """Query set of sequence b: (tracked T, front beta_m masks M), both in the generation region.

    The generation region is [n_prompt, N).  A random front start s leaves
    [n_prompt, s) decoded; each later slot is still masked with probability
    0.75.  M is the first beta_m masked slots; T is drawn from the decoded gen
    slots (Flash-dLLM review, "How It Works": Q = T u M^{beta_m})."""
    N, P = cfg["N"], cfg["n_prompt"]
    n_track = cfg.get("n_track", cfg.get("n_tv"))
    beta_m = cfg.get("beta_m", cfg.get("n_s"))
    L = N - P
    if n_track + beta_m > L:
        raise ValueError("query set larger than the generation region")
    g = _rng(cfg["seed"], "idx", b)
    s = P + int(g.integers(n_track, L - beta_m + 1))
    masked = g.random(N - s) < 0.75
    if masked.sum() < beta_m:
        need = beta_m - int(masked.sum())
        for j in range(N - s):
            if not masked[j]:
                masked[j] = True
                need -= 1
                if need == 0:
                    break
    masked_pos = s + np.nonzero(masked)[0]
    M = masked_pos[:beta_m]
    decoded = np.setdiff1d(np.arange(P, N), masked_pos)
    T = g.choice(decoded, size=n_track, replace=False)
    return np.sort(T).astype(np.int32), M.astype(np.int32), g


def fused_inputs(cfg: dict, seqs=None) -> dict:
    """Inputs of one fused step: x [B,N,D], q_idx [B,nq] int32, w_qkv, K, V [B,H,N,dh]."""
    seqs = list(range(cfg["B"])) if seqs is None else list(seqs)
    N, D = cfg["N"], cfg["D"]
    nq = cfg["n_track"] + cfg["beta_m"]
    q_idx = np.empty((len(seqs), nq), np.int32)
    x = torch.zeros((len(seqs), N, D), dtype=_torch_dtype(cfg["dtype"]))

    def one(i_b):
        i, b = i_b
        T, M, g = query_positions(cfg, b)
        q = np.concatenate([T, M])
        q = q[g.permutation(nq)]
        q_idx[i] = q
        x[i, torch.from_numpy(q.astype(np.int64))] = _store(
            _normal(cfg["seed"], "x", b, (nq, D)), cfg["dtype"])

    _per_seq(one, list(enumerate(seqs)))
    return dict(x=x, q_idx=torch.from_numpy(q_idx), w_qkv=weights(cfg),
                k_cache=cache(cfg, seqs, "k"), v_cache=cache(cfg, seqs, "v"))


def verify_inputs(cfg: dict, seqs=None) -> dict:
    """Inputs of one verify pass.

    Rows per sequence: n_tv tracked rows (view 0), then n_s draft-view rows
    (view 1) and n_s mask-view rows (view 2) over the same positions S, in the
    same order (Flash-dLLM review, "How It Works", Step 1: Verification: the
    query block is [track, D, S draft, S mask]).  rank is the decoding order of
    S (a seeded permutation), shared by the two views; view-0 rows carry -1."""
    seqs = list(range(cfg["B"])) if seqs is None else list(seqs)
    D = cfg["D"]
    n_tv, n_s = cfg["n_tv"], cfg["n_s"]
    R = n_tv + 2 * n_s
    pos = np.empty((len(seqs), R), np.int32)
    view = np.empty((len(seqs), R), np.int8)
    rank = np.empty((len(seqs), R), np.int32)
    x_rows = torch.empty((len(seqs), R, D), dtype=_torch_dtype(cfg["dtype"]))

    def one(i_b):
        i, b = i_b
        T, S, g = query_positions(cfg, b)
        r = g.permutation(n_s).astype(np.int32)
        pos[i] = np.concatenate([T, S, S])
        view[i] = np.array([0] * n_tv + [1] * n_s + [2] * n_s, np.int8)
        rank[i] = np.concatenate([np.full(n_tv, -1, np.int32), r, r])
        x_rows[i] = _store(_normal(cfg["seed"], "xr", b, (R, D)), cfg["dtype"])

    _per_seq(one, list(enumerate(seqs)))
    return dict(x_rows=x_rows, pos=torch.from_numpy(pos), view=torch.from_numpy(view),
                rank=torch.from_numpy(rank), w_qkv=weights(cfg),
                k_cache=cache(cfg, seqs, "k"), v_cache=cache(cfg, seqs, "v"),
                k_side=cache(cfg, seqs, "ks", n_s), v_side=cache(cfg, seqs, "vs", n_s),
                S_max=n_s)


def accept_inputs(cfg: dict, seqs=None, spike: str = "spread", p_agree: float = 0.8) -> dict:
    """Logits [B, R, V] fp32 for the acceptance reduction of a verify pass.

    Each row is N(0,1) plus one spike on a random token.  spike="spread" sizes
    the spike as ln(V) + 1/2 + logit(u), u ~ U(0.3, 0.99), so the row's max
    softmax probability lands near u (the sum of exp over V standard normals is
    about V*e^(1/2)); spike="literal" adds +6, which at V=126464 leaves every
    confidence near 0.002.  Mask-view rows are kind 2 with ref_tok equal to the
    spike token with probability p_agree (else another token); other rows are
    kind 0.  rank is the verify rank of the row."""
    seqs = list(range(cfg["B"])) if seqs is None else list(seqs)
    V = cfg["vocab"]
    n_tv, n_s = cfg["n_tv"], cfg["n_s"]
    R = n_tv + 2 * n_s
    logits = np.empty((len(seqs), R, V), np.float32)
    kind = np.empty((len(seqs), R), np.int8)
    ref_tok = np.empty((len(seqs), R), np.int32)
    rank = np.empty((len(seqs), R), np.int32)

    def one(i_b):
        i, b = i_b
        logits[i] = _normal(cfg["seed"], "logit", b, (R, V))
        g = _rng(cfg["seed"], "spike", b)
        tok = g.integers(0, V, size=R)
        u = g.uniform(0.3, 0.99, size=R)
        if spike == "spread":
            a = math.log(V) + 0.5 + np.log(u / (1.0 - u))
        elif spike == "literal":
            a = np.full(R, 6.0)
        else:
            raise ValueError(spike)
        logits[i, np.arange(R), tok] += a.astype(np.float32)
        _, _, gq = query_positions(cfg, b)
        r = gq.permutation(n_s).astype(np.int32)
        kind[i] = np.array([0] * (n_tv + n_s) + [2] * n_s, np.int8)
        rank[i] = np.concatenate([np.full(n_tv, -1, np.int32), r, r])
        agree = g.random(R) < p_agree
        other = (tok + 1 + g.integers(0, V - 1, size=R)) % V
        rt = np.where(agree, tok, other).astype(np.int32)
        rt[kind[i] != 2] = -1
        ref_tok[i] = rt

    _per_seq(one, list(enumerate(seqs)))
    return dict(logits=torch.from_numpy(logits), kind=torch.from_numpy(kind),
                ref_tok=torch.from_numpy(ref_tok), rank=torch.from_numpy(rank))


def to_device(inputs: dict, device="cuda") -> dict:
    """Copy every tensor of an input dict to `device` (other values unchanged)."""
    return {k: (v.to(device).contiguous() if isinstance(v, torch.Tensor) else v)
            for k, v in inputs.items()}


# ---------------------------------------------------------------------------
# general shapes for edge-case tests (same distributions, any sizes)

def random_fused(B, N, D, H, dh, nq=None, q_idx=None, dtype="bf16", seed=100, x_outside=0.0):
    """A fused-step input of any shape.  q_idx (int array [B, nq]) may be given;
    otherwise nq distinct slots per sequence are drawn uniformly from [0, N).
    Rows of x outside Q are filled with x_outside (NaN poisons them)."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 77])))
    if q_idx is None:
        q_idx = np.stack([g.choice(N, nq, replace=False) for _ in range(B)]).astype(np.int32)
    q_idx = np.asarray(q_idx, np.int32)
    nq = q_idx.shape[1]
    x = np.full((B, N, D), x_outside, np.float32)
    for b in range(B):
        ok = (q_idx[b] >= 0) & (q_idx[b] < N)
        x[b, q_idx[b][ok]] = g.standard_normal((int(ok.sum()), D), dtype=np.float32)
    E = H * dh
    w = g.standard_normal((3 * E, D), dtype=np.float32) / np.float32(math.sqrt(D))
    k = g.standard_normal((B, H, N, dh), dtype=np.float32)
    v = g.standard_normal((B, H, N, dh), dtype=np.float32)
    return dict(x=_store(x, dtype), q_idx=torch.from_numpy(q_idx), w_qkv=_store(w, dtype),
                k_cache=_store(k, dtype), v_cache=_store(v, dtype))


def random_verify(B, N, D, H, dh, n_tv, n_s, S_max=None, dtype="bf16", seed=200,
                  with_views=True):
    """A verify-pass input of any shape: rows [T_v (n_tv) | draft (n_s) | mask (n_s)]
    at distinct random positions, ranks a random permutation per sequence."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 78])))
    S_max = n_s if S_max is None else S_max
    R = n_tv + (2 * n_s if with_views else 0)
    pos = np.empty((B, R), np.int32)
    view = np.empty((B, R), np.int8)
    rank = np.empty((B, R), np.int32)
    for b in range(B):
        p = g.choice(N, n_tv + n_s, replace=False)
        T, S = p[:n_tv], p[n_tv:]
        r = g.permutation(n_s)
        if with_views:
            pos[b] = np.concatenate([T, S, S])
            view[b] = [0] * n_tv + [1] * n_s + [2] * n_s
            rank[b] = np.concatenate([np.full(n_tv, -1), r, r])
        else:
            pos[b], view[b], rank[b] = T, 0, -1
    x_rows = g.standard_normal((B, R, D), dtype=np.float32)
    E = H * dh
    w = g.standard_normal((3 * E, D), dtype=np.float32) / np.float32(math.sqrt(D))
    k = g.standard_normal((B, H, N, dh), dtype=np.float32)
    v = g.standard_normal((B, H, N, dh), dtype=np.float32)
    ks = g.standard_normal((B, H, max(S_max, 1), dh), dtype=np.float32)[:, :, :S_max]
    vs = g.standard_normal((B, H, max(S_max, 1), dh), dtype=np.float32)[:, :, :S_max]
    return dict(x_rows=_store(x_rows, dtype), pos=torch.from_numpy(pos),
                view=torch.from_numpy(view), rank=torch.from_numpy(rank), w_qkv=_store(w, dtype),
                k_cache=_store(k, dtype), v_cache=_store(v, dtype), k_side=_store(ks, dtype),
                v_side=_store(vs, dtype), S_max=S_max)


def random_logits(B, R, V, seed=300, spike_lo=2.0, spike_hi=12.0):
    """fp32 logits [B, R, V]: N(0,1) plus one spike of U(spike_lo, spike_hi) per row."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 79])))
    l = g.standard_normal((B, R, V), dtype=np.float32)
    tok = g.integers(0, V, (B, R))
    l[np.arange(B)[:, None], np.arange(R)[None, :], tok] += g.uniform(
        spike_lo, spike_hi, (B, R)).astype(np.float32)
    return torch.from_numpy(l), tok.astype(np.int32)
