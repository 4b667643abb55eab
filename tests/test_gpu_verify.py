"""GPU parity of the Flash-Verify pass against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity import (assert_close, check_outside_q_on_device, dtype_name, oracle_verify,
                    run_verify_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_attention_fdllm_b200 as F
    return F


def _check_verify(F, inp, rope_base=10000.0, causal=False, seqs=None, inp_oracle=None):
    dev = W.to_device(inp)
    k_in, v_in = inp["k_cache"].clone(), inp["v_cache"].clone()
    out, ws, st = run_verify_gpu(F, dev, rope_base, causal)
    assert st == F.OK, f"device status {st}"
    # every sequence, sampled for the oracle or not: cache slots outside the
    # T_v and draft positions, and side slots past the mask rows, bit-identical
    pos_all, view_all = inp["pos"].numpy(), inp["view"].numpy()
    Bn, Nn = inp["k_cache"].shape[0], inp["k_cache"].shape[2]
    wmask = np.zeros((Bn, Nn), bool)
    for b in range(Bn):
        wmask[b, pos_all[b][(view_all[b] == 0) | (view_all[b] == 1)]] = True
    check_outside_q_on_device(dev["k_cache"], inp["k_cache"], None, "k_cache", wmask)
    check_outside_q_on_device(dev["v_cache"], inp["v_cache"], None, "v_cache", wmask)
    for b in range(Bn):
        n_side = int((view_all[b] == 2).sum())
        for name in ("k_side", "v_side"):
            assert torch.equal(dev[name][b][:, n_side:].cpu(), inp[name][b][:, n_side:]), \
                f"{name}: an unused side slot changed in sequence {b}"
    dt = dtype_name(inp["x_rows"])
    H, dh = inp["k_cache"].shape[1], inp["k_cache"].shape[3]
    sel = list(range(inp["x_rows"].shape[0])) if seqs is None else list(seqs)
    ref_inp = inp if inp_oracle is None else inp_oracle
    K2, V2, KS, VS, ref_out = oracle_verify(ref_inp, H, dh, rope_base, dt, causal)
    assert_close(O.to_f64(out.cpu()[sel]), ref_out, dt, "verify output")
    kc, vc = dev["k_cache"].cpu()[sel], dev["v_cache"].cpu()[sel]
    pos, view = ref_inp["pos"].numpy(), ref_inp["view"].numpy()
    N = kc.shape[2]
    for i in range(len(sel)):
        written = np.zeros(N, bool)
        written[pos[i][(view[i] == 0) | (view[i] == 1)]] = True
        keep = torch.from_numpy(~written)
        assert torch.equal(kc[i][:, keep], k_in[sel[i]][:, keep])
        assert torch.equal(vc[i][:, keep], v_in[sel[i]][:, keep])
        assert_close(O.to_f64(kc[i][:, torch.from_numpy(written)]), K2[i][:, written], dt, "k written")
        assert_close(O.to_f64(vc[i][:, torch.from_numpy(written)]), V2[i][:, written], dt, "v written")
        n_side = int((view[i] == 2).sum())
        ks, vs = dev["k_side"].cpu()[sel[i]], dev["v_side"].cpu()[sel[i]]
        assert_close(O.to_f64(ks[:, :n_side]), KS[i][:, :n_side], dt, "k side")
        assert_close(O.to_f64(vs[:, :n_side]), VS[i][:, :n_side], dt, "v side")
        assert torch.equal(ks[:, n_side:], inp["k_side"][sel[i]][:, n_side:])
    return out


_SPLIT_CODE = {"stream": 1, "whole": 2, "cluster": 3}

# (B, N, D, H, dh, |T_v|, |S|, split the attention must take on 148 SMs):
# R = |T_v| + 2 |S| rows per sequence, query chunks of 16, 32 or 64 rows
VERIFY_SPLITS = [
    pytest.param(5, 700, 128, 32, 128, 4, 6, "stream", id="streamk-160items-nq16-dh128"),
    pytest.param(5, 700, 128, 32, 128, 6, 12, "stream", id="streamk-160items-nq32-dh128"),
    pytest.param(5, 700, 128, 32, 128, 8, 20, "stream", id="streamk-160items-nq48-dh128"),
    pytest.param(5, 700, 128, 32, 128, 8, 26, "stream", id="streamk-160items-nq64-dh128"),
    pytest.param(5, 700, 128, 32, 64, 8, 20, "stream", id="streamk-160items-nq48-dh64"),
    pytest.param(5, 700, 128, 32, 128, 20, 40, "stream", id="streamk-320items-2chunks-dh128"),
    pytest.param(3, 700, 128, 32, 128, 4, 6, "whole", id="whole-96items-nq16-dh128"),
    pytest.param(3, 700, 128, 32, 128, 8, 26, "whole", id="whole-96items-nq64-dh128"),
    pytest.param(2, 700, 128, 32, 128, 20, 40, "whole", id="whole-128items-2chunks-dh128"),
    pytest.param(5, 1000, 128, 32, 128, 8, 16, "stream", id="streamk-160items-nq48-dh128"),
    pytest.param(5, 1000, 128, 32, 128, 8, 26, "stream", id="streamk-160items-nq64-dh128"),
    pytest.param(9, 1000, 128, 32, 128, 8, 16, "whole", id="whole-288items-nq48-dh128"),
    pytest.param(9, 1000, 128, 32, 128, 8, 26, "whole", id="whole-288items-nq64-dh128"),
    pytest.param(16, 100, 128, 32, 128, 4, 6, "stream", id="streamk-512items-2tiles-side"),
]


def _assert_split(F, B, N, H, dh, R, S_max, want):
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the shapes are chosen for 148 SMs")
    mode, _ = F.fdllm_attention_split(B, N, H, dh, R, S_max, True)
    assert mode == _SPLIT_CODE[want], f"attention split {mode}, expected {want}"


@pytest.mark.parametrize("causal", [False, True], ids=["mutual", "causal"])
@pytest.mark.parametrize("B,N,D,H,dh,n_tv,n_s,split", VERIFY_SPLITS)
def test_verify_work_splits(F, B, N, D, H, dh, n_tv, n_s, split, causal):
    """The view predicate under every work split of the attention, in both
    visibility readings, against the oracle on every sequence."""
    _assert_split(F, B, N, H, dh, n_tv + 2 * n_s, n_s, split)
    inp = W.random_verify(B, N, D, H, dh, n_tv=n_tv, n_s=n_s, seed=61 + B + n_s)
    _check_verify(F, inp, causal=causal)


@pytest.mark.parametrize("causal", [False, True], ids=["mutual", "causal"])
def test_verify_stream_k_deterministic(F, causal):
    """Two stream-K verify passes on the same inputs give the same bits."""
    B, N, D, H, dh, n_tv, n_s = 5, 700, 128, 32, 128, 8, 20
    _assert_split(F, B, N, H, dh, n_tv + 2 * n_s, n_s, "stream")
    inp = W.random_verify(B, N, D, H, dh, n_tv=n_tv, n_s=n_s, seed=67)
    a, b = W.to_device(inp), W.to_device(inp)
    oa, _, sa = run_verify_gpu(F, a, 10000.0, causal)
    ob, _, sb = run_verify_gpu(F, b, 10000.0, causal)
    assert sa == F.OK and sb == F.OK
    assert torch.equal(oa, ob)
    for k in ("k_cache", "v_cache", "k_side", "v_side"):
        assert torch.equal(a[k], b[k]), k


def test_verify_bf16_config_sampled(F):
    cfg = W.CONFIGS["verify_bf16"]
    inp = W.verify_inputs(cfg)
    seqs = [0, 5]
    _check_verify(F, inp, cfg["rope_base"], seqs=seqs, inp_oracle=W.verify_inputs(cfg, seqs=seqs))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype,dh", [("bf16", 128), ("bf16", 64), ("f32", 64)])
def test_verify_ragged(F, causal, dtype, dh):
    inp = W.random_verify(2, 333, 128, 2, dh, n_tv=5, n_s=7, S_max=9, dtype=dtype, seed=21)
    _check_verify(F, inp, causal=causal)


def test_verify_many_views_spanning_tiles(F):
    inp = W.random_verify(1, 1000, 128, 2, 128, n_tv=3, n_s=70, S_max=140, seed=22)
    _check_verify(F, inp)
    _check_verify(F, inp, causal=True)


def test_verify_without_views_equals_fused(F):
    inp = W.random_verify(2, 250, 128, 2, 128, n_tv=6, n_s=0, S_max=0, seed=23, with_views=False)
    out_v = _check_verify(F, inp)
    fin = dict(x=torch.zeros((2, 250, 128), dtype=torch.bfloat16), q_idx=inp["pos"],
               w_qkv=inp["w_qkv"], k_cache=inp["k_cache"], v_cache=inp["v_cache"])
    for b in range(2):
        fin["x"][b, inp["pos"][b].long()] = inp["x_rows"][b]
    from parity import run_fused_gpu
    dev = W.to_device(fin)
    out_f, _, st = run_fused_gpu(F, dev, 10000.0)
    assert st == F.OK
    assert torch.equal(out_f, out_v)


def test_single_s_position_modes_coincide(F):
    inp = W.random_verify(2, 200, 128, 2, 128, n_tv=2, n_s=1, seed=24)
    a = _check_verify(F, inp, causal=False)
    b = _check_verify(F, inp, causal=True)
    assert torch.equal(a, b)


def test_side_overflow_sets_status(F):
    inp = W.random_verify(1, 120, 128, 2, 64, n_tv=2, n_s=5, S_max=3, seed=25)
    dev = W.to_device(inp)
    out, ws, st = run_verify_gpu(F, dev, 10000.0)
    assert st == F.ERR_BAD_INDEX


@pytest.mark.parametrize("causal", [False, True], ids=["mutual", "causal"])
def test_verify_projection_on_cta_pairs(F, causal):
    """A verify pass of 520 rows projects on CTA pairs: view-2 rows write side
    slots, the others cache slots, from both CTAs of a pair."""
    inp = W.random_verify(13, 400, 128, 4, 64, n_tv=8, n_s=16, seed=73)
    _check_verify(F, inp, causal=causal)
