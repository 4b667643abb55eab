"""GPU parity of the tracked-set selection ([review], "How It Works", Step 1:
Cache selection) against the fp64 oracle, through the C ABI.

The GPU ranks fp32 masses computed from the step's bf16/fp32 queries, the oracle
fp64 masses from exact queries, so two slots whose masses are closer than the
tolerance may trade places: the selection is checked for validity against the
oracle's masses (every chosen slot at least as heavy as every slot left out, up
to the tolerance), and exactly where the masses are exact (all zero)."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity import check_track, dtype_name

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_attention_fdllm_b200 as F
    return F


def _masks(B, N, nq, q_idx, seed, p_masked=0.5, p_cand=0.6):
    rng = np.random.default_rng(seed)
    masked = (rng.random((B, nq)) < p_masked).astype(np.int8)
    masked[:, 0] = 1
    cand = (rng.random((B, N)) < p_cand).astype(np.int8)
    # some of the slots resolved in this step are candidates too
    for b in range(B):
        cand[b, q_idx[b, : nq // 2]] = 1
    return masked, cand


def _run(F, inp, masked, cand, beta_t, rope_base=10000.0):
    dev = W.to_device(inp)
    x, q_idx, w = dev["x"], dev["q_idx"], dev["w_qkv"]
    B, N, D = x.shape
    H, dh = dev["k_cache"].shape[1], dev["k_cache"].shape[3]
    nq = q_idx.shape[1]
    ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(B, N, D, H, dh, nq, x.dtype), "cuda")
    out = torch.empty((B, nq, H * dh), dtype=x.dtype, device="cuda")
    F.fdllm_fused_step(x, q_idx, w, dev["k_cache"], dev["v_cache"], out, ws, rope_base=rope_base)
    track = torch.full((B, beta_t), -7, dtype=torch.int32, device="cuda")
    mass = torch.empty((B, N), dtype=torch.float32, device="cuda")
    F.fdllm_track_select(torch.from_numpy(masked).cuda(), torch.from_numpy(cand).cuda(),
                         dev["k_cache"], track, ws, mass=mass)
    st = F.fdllm_get_status(ws)
    assert st == F.OK, f"device status {st}"
    return track.cpu().numpy(), mass.cpu().numpy(), dev


def _oracle_mass(inp, masked, rope_base=10000.0):
    dt = dtype_name(inp["x"])
    H, dh = inp["k_cache"].shape[1], inp["k_cache"].shape[3]
    f = O.to_f64
    K2, _, _ = O.fused_step(f(inp["x"]), inp["q_idx"].numpy(), f(inp["w_qkv"]), rope_base,
                            f(inp["k_cache"]), f(inp["v_cache"]), H, dh, dt)
    return O.attention_mass(f(inp["x"]), inp["q_idx"].numpy(), f(inp["w_qkv"]), rope_base, K2,
                            H, dh, masked), dt


@pytest.mark.parametrize("cfg_name", ["tiny_fp32", "single_bf16"])
def test_track_select_configs(F, cfg_name):
    cfg = W.CONFIGS[cfg_name]
    inp = W.fused_inputs(cfg)
    B, nq = inp["q_idx"].shape
    N = inp["x"].shape[1]
    masked, cand = _masks(B, N, nq, inp["q_idx"].numpy(), seed=31)
    beta_t = min(80, N)
    track, mass, _ = _run(F, inp, masked, cand, beta_t, cfg["rope_base"])
    ref, dt = _oracle_mass(inp, masked, cfg["rope_base"])
    check_track(track, mass, ref, cand, beta_t, dt)


@pytest.mark.parametrize("shape", [
    (2, 300, 128, 40, 64, 9),     # 80 (sequence, head) items: the stream-K merge
    (1, 4096, 128, 2, 128, 40),   # items split over clusters of 8 CTAs, NQ = 64
    (3, 385, 192, 3, 128, 37),    # ragged
])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_track_select_shapes(F, shape, dtype):
    B, N, D, H, dh, nq = shape
    inp = W.random_fused(B, N, D, H, dh, nq=nq, dtype=dtype, seed=N + nq)
    masked, cand = _masks(B, N, nq, inp["q_idx"].numpy(), seed=N)
    track, mass, _ = _run(F, inp, masked, cand, 16)
    ref, dt = _oracle_mass(inp, masked)
    check_track(track, mass, ref, cand, 16, dt)


def test_track_select_exact_cases(F):
    """No masked row: every mass is exactly 0, so T is the first beta_t
    candidates in slot order.  No candidate: all -1.  beta_t above the number
    of candidates: the tail is -1.  Two calls give identical bits."""
    inp = W.random_fused(2, 200, 128, 2, 64, nq=6, seed=3)
    B, nq = inp["q_idx"].shape
    N = inp["x"].shape[1]
    masked, cand = _masks(B, N, nq, inp["q_idx"].numpy(), seed=4)
    zero = np.zeros_like(masked)
    track, mass, _ = _run(F, inp, zero, cand, 12)
    assert not mass.any()
    expect = O.track_select(np.zeros((B, N)), cand, 12)
    assert (track == expect).all()
    track, _, _ = _run(F, inp, masked, np.zeros_like(cand), 5)
    assert (track == -1).all()
    few = np.zeros_like(cand)
    few[:, [3, 50, 199]] = 1
    track, mass, _ = _run(F, inp, masked, few, 7)
    assert (track[:, 3:] == -1).all() and set(track[0, :3].tolist()) == {3, 50, 199}
    t1, m1, _ = _run(F, inp, masked, cand, 9)
    t2, m2, _ = _run(F, inp, masked, cand, 9)
    assert (t1 == t2).all() and (m1.view(np.uint32) == m2.view(np.uint32)).all()


def test_track_select_rejects_bad_beta(F):
    inp = W.random_fused(1, 64, 64, 2, 64, nq=4, seed=1)
    dev = W.to_device(inp)
    ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(1, 64, 64, 2, 64, 4, torch.bfloat16), "cuda")
    q_m = torch.ones((1, 4), dtype=torch.int8, device="cuda")
    cand = torch.ones((1, 64), dtype=torch.int8, device="cuda")
    for bad in (0, 1025):
        track = torch.empty((1, bad), dtype=torch.int32, device="cuda")
        with pytest.raises(F.FdllmError):
            F.fdllm_track_select(q_m, cand, dev["k_cache"], track, ws)
