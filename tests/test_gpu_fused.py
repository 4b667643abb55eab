"""GPU parity of the fused KV-cache step against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity import (assert_close, check_cache_update, check_outside_q_on_device, dtype_name,
                    oracle_fused, run_fused_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_attention_fdllm_b200 as F
    return F


def _check_fused(F, inp, rope_base=10000.0, seqs_for_oracle=None, inp_oracle=None):
    dev = W.to_device(inp)
    k_in, v_in = inp["k_cache"].clone(), inp["v_cache"].clone()
    out, ws, st = run_fused_gpu(F, dev, rope_base)
    assert st == F.OK, f"device status {st}"
    # every sequence, sampled for the oracle or not: slots outside Q bit-identical
    check_outside_q_on_device(dev["k_cache"], inp["k_cache"], inp["q_idx"], "k_cache")
    check_outside_q_on_device(dev["v_cache"], inp["v_cache"], inp["q_idx"], "v_cache")
    dt = dtype_name(inp["x"])
    H, dh = inp["k_cache"].shape[1], inp["k_cache"].shape[3]
    sel = list(range(inp["x"].shape[0])) if seqs_for_oracle is None else list(seqs_for_oracle)
    ref_inp = inp if inp_oracle is None else inp_oracle
    if inp_oracle is None and seqs_for_oracle is not None:
        ref_inp = {k: v[sel] for k, v in inp.items() if k != "w_qkv"}
        ref_inp["w_qkv"] = inp["w_qkv"]
    K2, V2, ref_out = oracle_fused(ref_inp, H, dh, rope_base, dt)
    out_c = out.cpu()[sel]
    err = assert_close(O.to_f64(out_c), ref_out, dt, "attention output")
    qi = ref_inp["q_idx"].numpy()
    check_cache_update(dev["k_cache"].cpu()[sel], k_in[sel], K2, qi, dt, "k_cache")
    check_cache_update(dev["v_cache"].cpu()[sel], v_in[sel], V2, qi, dt, "v_cache")
    return err, out, dev


def test_tiny_fp32_config(F):
    cfg = W.CONFIGS["tiny_fp32"]
    _check_fused(F, W.fused_inputs(cfg), cfg["rope_base"])


def test_single_bf16_config(F):
    cfg = W.CONFIGS["single_bf16"]
    _check_fused(F, W.fused_inputs(cfg), cfg["rope_base"])


def test_long_bf16_config(F):
    cfg = W.CONFIGS["long_bf16"]
    _check_fused(F, W.fused_inputs(cfg), cfg["rope_base"])


def test_batch_bf16_config_sampled(F):
    """Full-size B=64 batch; the oracle recomputes sampled sequences one by one
    from their own input substreams (the first, a middle one, the last)."""
    cfg = W.CONFIGS["batch_bf16"]
    inp = W.fused_inputs(cfg)
    seqs = [0, 37, 63]
    _check_fused(F, inp, cfg["rope_base"], seqs_for_oracle=seqs,
                 inp_oracle=W.fused_inputs(cfg, seqs=seqs))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dh", [64, 128])
@pytest.mark.parametrize("shape", [(2, 200, 128, 2, 5), (1, 130, 256, 3, 1), (3, 385, 192, 1, 37)])
def test_ragged_shapes(F, dtype, dh, shape):
    """Several KV tiles with a ragged tail, ragged query counts, B > 1."""
    B, N, D, H, nq = shape
    inp = W.random_fused(B, N, D, H, dh, nq=nq, dtype=dtype, seed=hash((shape, dh)) % 1000)
    _check_fused(F, inp)


# (B, N, D, H, dh, nq, work split the attention must take on 148 SMs); items =
# B * H * query chunks of up to 64 rows.  Above SMs / 2 items, whole-item mode
# takes one or two waves when they are no slower than stream-K's share plus its
# merge and boundaries; stream-K takes the rest.
SPLIT_SHAPES = [
    pytest.param(9, 1000, 128, 32, 64, 20, "whole", id="whole-288items-nq32-dh64"),
    pytest.param(9, 700, 128, 32, 128, 12, "whole", id="whole-288items-nq16-dh128"),
    pytest.param(9, 1024, 128, 32, 128, 32, "whole", id="whole-288items-nq32-dh128"),
    pytest.param(9, 1000, 128, 32, 128, 40, "whole", id="whole-288items-nq48-dh128"),
    pytest.param(5, 1000, 128, 32, 64, 20, "stream", id="streamk-160items-nq32-dh64"),
    pytest.param(12, 700, 128, 16, 128, 12, "stream", id="streamk-192items-nq16-dh128"),
    pytest.param(8, 1024, 128, 32, 128, 32, "stream", id="streamk-256items-nq32-dh128"),
    pytest.param(5, 1000, 128, 32, 128, 40, "stream", id="streamk-160items-nq48-dh128"),
    pytest.param(3, 900, 128, 32, 128, 60, "whole", id="whole-96items-nq64-dh128"),
    pytest.param(3, 900, 128, 32, 64, 44, "whole", id="whole-96items-nq48-dh64"),
    pytest.param(2, 800, 128, 32, 64, 100, "whole", id="whole-128items-2chunks-dh64"),
    pytest.param(5, 900, 128, 32, 128, 60, "stream", id="streamk-160items-nq64-dh128"),
    pytest.param(5, 900, 128, 32, 64, 44, "stream", id="streamk-160items-nq48-dh64"),
    pytest.param(12, 600, 128, 32, 64, 30, "stream", id="streamk-384items-nq32-dh64"),
    pytest.param(5, 800, 128, 32, 64, 100, "stream", id="streamk-320items-2chunks-dh64"),
    pytest.param(16, 1024, 128, 32, 128, 32, "stream", id="streamk-512items-nq32-dh128"),
    # one- and two-tile items: a CTA's range holds several short segments, each
    # finished while later ones run (whole ones and split ones)
    pytest.param(16, 100, 128, 32, 128, 8, "stream", id="streamk-512items-1tile"),
    pytest.param(16, 200, 128, 32, 64, 12, "stream", id="streamk-512items-2tiles-dh64"),
]
_SPLIT_CODE = {"stream": 1, "whole": 2, "cluster": 3}


def _assert_split(F, B, N, H, dh, rows, want, S_max=0, verify=False):
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the shapes are chosen for 148 SMs")
    mode, _ = F.fdllm_attention_split(B, N, H, dh, rows, S_max, verify)
    assert mode == _SPLIT_CODE[want], f"attention split {mode}, expected {want}"


@pytest.mark.parametrize("B,N,D,H,dh,nq,split", SPLIT_SHAPES)
def test_attention_work_splits(F, B, N, D, H, dh, nq, split):
    """Every way the attention spreads (sequence, head, chunk) items over the SMs
    gives the oracle's result; the oracle checks up to four sequences (first,
    last and two between), the cache outside Q is checked on all of them."""
    _assert_split(F, B, N, H, dh, nq, split)
    inp = W.random_fused(B, N, D, H, dh, nq=nq, seed=31 + B + N)
    seqs = sorted({0, B // 3, (2 * B) // 3, B - 1})
    _check_fused(F, inp, seqs_for_oracle=seqs)


@pytest.mark.parametrize("B,N,D,H,dh,nq", [(12, 600, 128, 32, 64, 30), (5, 900, 128, 32, 128, 40),
                                            (5, 900, 128, 32, 128, 60)])
def test_stream_k_deterministic(F, B, N, D, H, dh, nq):
    """Stream-K merges a split item in CTA order by its last contributor: two
    runs give the same bits whatever order the contributors finish in."""
    _assert_split(F, B, N, H, dh, nq, "stream")
    inp = W.random_fused(B, N, D, H, dh, nq=nq, seed=57)
    a, b = W.to_device(inp), W.to_device(inp)
    oa, _, sa = run_fused_gpu(F, a, 10000.0)
    ob, _, sb = run_fused_gpu(F, b, 10000.0)
    assert sa == F.OK and sb == F.OK
    assert torch.equal(oa, ob)
    assert torch.equal(a["k_cache"], b["k_cache"]) and torch.equal(a["v_cache"], b["v_cache"])


@pytest.mark.parametrize("shape", [(1, 4096, 128, 1, 128, 20), (1, 6000, 128, 2, 64, 40)])
def test_item_split_over_many_ctas(F, shape):
    """Few (sequence, head) items and a long cache: each item's key tiles are
    spread over dozens of CTAs, so the partial merge runs in several batches."""
    B, N, D, H, dh, nq = shape
    _check_fused(F, W.random_fused(B, N, D, H, dh, nq=nq, seed=N + H))


def test_edge_slots_and_single_query(F):
    N = 257
    q_idx = np.array([[0, N - 1, 128], [N - 1, 5, 0]], np.int32)
    _check_fused(F, W.random_fused(2, N, 128, 2, 128, q_idx=q_idx, seed=5))
    _check_fused(F, W.random_fused(1, N, 128, 2, 128, q_idx=np.array([[N - 1]]), seed=6))


def test_query_set_covers_whole_cache(F):
    N = 96
    q_idx = np.stack([np.random.default_rng(1).permutation(N)]).astype(np.int32)
    _check_fused(F, W.random_fused(1, N, 64 * 2, 2, 64, q_idx=q_idx, seed=7))


def test_rows_outside_q_are_never_read(F):
    """x rows outside Q are NaN: the step must not use them."""
    inp = W.random_fused(2, 300, 128, 2, 128, nq=9, seed=8, x_outside=float("nan"))
    _, out, _ = _check_fused(F, inp)
    assert torch.isfinite(out).all()


def test_deterministic(F):
    inp = W.random_fused(2, 700, 256, 4, 128, nq=33, seed=9)
    a = W.to_device(inp)
    b = W.to_device(inp)
    oa, _, _ = run_fused_gpu(F, a, 10000.0)
    ob, _, _ = run_fused_gpu(F, b, 10000.0)
    assert torch.equal(oa, ob) and torch.equal(a["k_cache"], b["k_cache"])


def test_out_of_range_index_sets_status_and_skips_row(F):
    inp = W.random_fused(1, 100, 128, 2, 64, q_idx=np.array([[3, 100, 7]]), seed=10)
    dev = W.to_device(inp)
    k_in = dev["k_cache"].clone()
    out, ws, st = run_fused_gpu(F, dev, 10000.0)
    assert st == F.ERR_BAD_INDEX
    changed = (dev["k_cache"] != k_in).any(dim=3).any(dim=1)[0]
    assert set(torch.nonzero(changed).flatten().tolist()) <= {3, 7}
    assert F.fdllm_get_status(ws) == F.OK  # read-and-clear


def test_repeated_index_sets_status(F):
    """Q is a set; a repeated slot is reported through the status word."""
    inp = W.random_fused(2, 100, 128, 2, 64, q_idx=np.array([[3, 9, 3], [5, 6, 7]]), seed=11)
    dev = W.to_device(inp)
    out, ws, st = run_fused_gpu(F, dev, 10000.0)
    assert st == F.ERR_BAD_INDEX
    inp = W.random_fused(2, 100, 128, 2, 64, q_idx=np.array([[3, 9, 4], [5, 6, 7]]), seed=11)
    out, ws, st = run_fused_gpu(F, W.to_device(inp), 10000.0)
    assert st == F.OK


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_guard_sequences_around_the_buffers_stay_intact(F, dtype):
    """The caches and the output sit inside larger allocations whose extra
    sequences before and after are filled with a NaN pattern: the call must
    leave them bit-identical (no write past its own buffers)."""
    B, N, D, H, dh, nq = 2, 300, 128, 2, 64, 9
    inp = W.random_fused(B, N, D, H, dh, nq=nq, dtype=dtype, seed=12)
    dev = W.to_device(inp)
    t = dev["k_cache"].dtype
    guard = float("nan")
    kb = torch.full((B + 2, H, N, dh), guard, dtype=t, device="cuda")
    vb = torch.full((B + 2, H, N, dh), guard, dtype=t, device="cuda")
    ob = torch.full((B + 2, nq, H * dh), guard, dtype=t, device="cuda")
    kb[1:B + 1].copy_(dev["k_cache"])
    vb[1:B + 1].copy_(dev["v_cache"])
    before = [kb.clone(), vb.clone(), ob.clone()]
    k, v, o = kb[1:B + 1], vb[1:B + 1], ob[1:B + 1]
    assert k.is_contiguous() and o.is_contiguous()
    ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(B, N, D, H, dh, nq, t), "cuda")
    F.fdllm_fused_step(dev["x"], dev["q_idx"], dev["w_qkv"], k, v, o, ws)
    assert F.fdllm_get_status(ws) == F.OK
    for now, was in zip((kb, vb, ob), before):
        for g in (0, B + 1):
            a = now[g].contiguous().view(torch.int16 if t == torch.bfloat16 else torch.int32)
            b = was[g].contiguous().view(torch.int16 if t == torch.bfloat16 else torch.int32)
            assert torch.equal(a, b), "a guard sequence changed"
    assert not torch.isnan(o).any()


def test_empty_batch_is_a_no_op(F):
    x = torch.zeros((0, 10, 64), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((0, 2), dtype=torch.int32, device="cuda")
    w = torch.zeros((3 * 64, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((0, 1, 10, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    ws = F.alloc_workspace(4096, "cuda")
    F.fdllm_fused_step(x, q, w, k, k.clone(), out, ws)
    assert F.fdllm_get_status(ws) == F.OK


def test_stage_calls_equal_fused_call(F):
    inp = W.random_fused(2, 300, 256, 2, 128, nq=11, seed=12)
    a, b = W.to_device(inp), W.to_device(inp)
    out_f, _, _ = run_fused_gpu(F, a, 500.0)
    B, N, D = b["x"].shape
    H, dh, nq = 2, 128, 11
    ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(B, N, D, H, dh, nq, torch.bfloat16), "cuda")
    q = torch.empty((B, nq, H, dh), dtype=torch.bfloat16, device="cuda")
    out_s = torch.empty_like(out_f)
    F.fdllm_qkv_rope_scatter(b["x"], b["q_idx"], b["w_qkv"], b["k_cache"], b["v_cache"], q, ws,
                             rope_base=500.0)
    F.fdllm_attend(q, b["k_cache"], b["v_cache"], out_s, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_f, out_s) and torch.equal(a["k_cache"], b["k_cache"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H,dh,nq", [(3, 400, 2, 128, 21), (16, 1024, 32, 128, 32)])
def test_fused_step_rows_equals_fused_step(F, dtype, B, N, H, dh, nq):
    """fdllm_fused_step_rows (x[Q] given packed) runs the same kernels on the same
    rows as fdllm_fused_step: the same bits, caches included."""
    inp = W.random_fused(B, N, 128, H, dh, nq=nq, dtype=dtype, seed=81 + B)
    a, b = W.to_device(inp), W.to_device(inp)
    out_f, _, st = run_fused_gpu(F, a, 10000.0)
    assert st == F.OK
    x_rows = torch.stack([b["x"][i, b["q_idx"][i].long()] for i in range(B)]).contiguous()
    ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(B, N, 128, H, dh, nq, x_rows.dtype),
                           "cuda")
    out_r = torch.empty_like(out_f)
    F.fdllm_fused_step_rows(x_rows, b["q_idx"], b["w_qkv"], b["k_cache"], b["v_cache"], out_r, ws)
    assert F.fdllm_get_status(ws) == F.OK
    assert torch.equal(out_f, out_r)
    assert torch.equal(a["k_cache"], b["k_cache"]) and torch.equal(a["v_cache"], b["v_cache"])


def test_fused_step_rows_reports_repeated_and_out_of_range_indices(F):
    for q_idx in ([[3, 9, 3], [5, 6, 7]], [[3, 100, 7], [5, 6, 7]]):
        inp = W.random_fused(2, 100, 128, 2, 64, q_idx=np.array([[3, 9, 4], [5, 6, 7]]), seed=11)
        d = W.to_device(inp)
        x_rows = torch.stack([d["x"][i, d["q_idx"][i].long()] for i in range(2)]).contiguous()
        qi = torch.tensor(q_idx, dtype=torch.int32, device="cuda")
        ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(2, 100, 128, 2, 64, 3,
                                                                  torch.bfloat16), "cuda")
        out = torch.empty((2, 3, 128), dtype=torch.bfloat16, device="cuda")
        F.fdllm_fused_step_rows(x_rows, qi, d["w_qkv"], d["k_cache"], d["v_cache"], out, ws)
        assert F.fdllm_get_status(ws) == F.ERR_BAD_INDEX


@pytest.mark.parametrize("B,N,D,H,dh,nq", [
    pytest.param(2, 300, 192, 2, 64, 65, id="M130-whole-tile-one-mma"),
    pytest.param(3, 400, 128, 3, 128, 100, id="M300-whole-tile-two-mmas-ragged"),
    pytest.param(2, 500, 256, 5, 128, 100, id="M200-H5-whole-tiles-past-F"),
    pytest.param(1, 1200, 128, 2, 128, 512, id="M512-whole-tile-two-mmas"),
    pytest.param(13, 300, 192, 4, 64, 80, id="M1040-five-token-tiles-ragged-k"),
    pytest.param(6, 500, 256, 5, 128, 100, id="M600-H5-last-pair-past-F"),
])
def test_projection_on_cta_pairs(F, B, N, D, H, dh, nq):
    """128 or more projection rows run on CTA pairs (256 features per MMA, each
    CTA holding half of the token rows).  Up to 512 rows a pair takes one whole
    tile of all the rows (two MMAs past 256); the shapes reach a tile padded
    past M, several token tiles with a short last k-step, and a last feature
    pair that runs past F with the q/k block boundary between its two CTAs."""
    _check_fused(F, W.random_fused(B, N, D, H, dh, nq=nq, seed=91 + nq))
