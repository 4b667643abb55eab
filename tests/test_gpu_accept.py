"""GPU parity of the acceptance reduction against the fp64 oracle (through the C ABI)."""
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity import check_accept, run_accept_gpu

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.txt")


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_attention_fdllm_b200 as F
    return F


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = [s.strip() for s in line.split("=", 1)]
            vals[k] = v.split()
    return vals


def _run_both(F, logits, kind, ref_tok, rank, eps, gamma):
    dev = logits.device
    gpu = run_accept_gpu(F, logits, kind.to(dev), ref_tok.to(dev), rank.to(dev), eps, gamma)[:4]
    ref = O.accept(O.to_f64(logits.cpu()), kind.numpy(), ref_tok.numpy(), rank.numpy(), eps, gamma)
    return gpu, ref


def test_worked_example(F):
    g = _golden()
    eps, gamma = float(g["eps"][0]), float(g["gamma"][0])
    probs = np.stack([np.array(g[k], np.float64) for k in ("q_2", "q_3", "p_3")])
    logits = torch.from_numpy(np.log(probs).astype(np.float32))[None].cuda()
    kind = torch.tensor([[1, 1, 2]], dtype=torch.int8)
    A = g["vocab"].index(g["xhat_3"][0])
    ref_tok = torch.tensor([[-1, -1, A]], dtype=torch.int32)
    rank = torch.tensor([[-1, -1, 0]], dtype=torch.int32)
    gpu, ref = _run_both(F, logits, kind, ref_tok, rank, eps, gamma)
    t, c, f, n = gpu
    assert list(t[0]) == [A, A, A]
    np.testing.assert_allclose(c[0], [0.92, 0.70, 0.85], atol=1e-6)
    assert f[0, 0] & O.FLAG_COMMIT and not f[0, 1] & O.FLAG_COMMIT   # D_1 = {2}, S_1 = {3}
    assert f[0, 2] & O.FLAG_ACCEPT and n[0] == 1                      # position 3 accepted
    check_accept(gpu, ref, kind.numpy(), rank.numpy(), eps, gamma)


def test_verify_config_logits(F):
    cfg = W.CONFIGS["verify_bf16"]
    a = W.accept_inputs(cfg)
    logits = a["logits"].cuda()
    gpu, ref = _run_both(F, logits, a["kind"], a["ref_tok"], a["rank"], 0.9, 0.8)
    check_accept(gpu, ref, a["kind"].numpy(), a["rank"].numpy(), 0.9, 0.8)
    # the spread makes the prefix rule non-trivial: some sequences accept part of S
    n = gpu[3]
    assert n.min() < cfg["n_s"] and n.max() > 0


def test_literal_spike_variant(F):
    cfg = W.CONFIGS["verify_bf16"]
    a = W.accept_inputs(cfg, seqs=[0, 1], spike="literal")
    gpu, ref = _run_both(F, a["logits"].cuda(), a["kind"], a["ref_tok"], a["rank"], 0.9, 0.8)
    check_accept(gpu, ref, a["kind"].numpy(), a["rank"].numpy(), 0.9, 0.8)


@pytest.mark.parametrize("V", [1, 3, 5, 1000, 4097, 50001])
def test_ragged_vocab_and_kinds(F, V):
    B, R = 3, 9
    logits, tok = W.random_logits(B, R, V, seed=V)
    g = np.random.default_rng(V)
    kind = torch.from_numpy(g.integers(0, 3, (B, R)).astype(np.int8))
    ref = torch.from_numpy(np.where(g.random((B, R)) < 0.7, tok, (tok + 1) % V).astype(np.int32))
    rank = torch.from_numpy(np.stack([g.permutation(R) for _ in range(B)]).astype(np.int32))
    gpu, refr = _run_both(F, logits.cuda(), kind, ref, rank, 0.6, 0.5)
    check_accept(gpu, refr, kind.numpy(), rank.numpy(), 0.6, 0.5)


def test_ties_all_pass_all_fail(F):
    B, R, V = 2, 4, 777
    l = torch.zeros((B, R, V))
    l[:, :, 10] = 5.0
    l[:, :, 400] = 5.0                     # tie: the lowest index wins
    kind = torch.full((B, R), 2, dtype=torch.int8)
    rank = torch.tensor([[0, 1, 2, 3], [3, 2, 1, 0]], dtype=torch.int32)
    ok = torch.full((B, R), 10, dtype=torch.int32)
    gpu, ref = _run_both(F, l.cuda(), kind, ok, rank, 0.9, 0.01)
    assert (gpu[0] == 10).all() and (gpu[3] == R).all()          # all pass
    check_accept(gpu, ref, kind.numpy(), rank.numpy(), 0.9, 0.01)
    gpu, ref = _run_both(F, l.cuda(), kind, ok + 1, rank, 0.9, 0.01)
    assert (gpu[3] == 0).all()                                    # all fail
    check_accept(gpu, ref, kind.numpy(), rank.numpy(), 0.9, 0.01)


def test_repeated_calls_reuse_workspace(F):
    """Counters are left at zero, so the same workspace serves many calls."""
    B, R, V = 4, 6, 30000
    logits, tok = W.random_logits(B, R, V, seed=3)
    kind = torch.full((B, R), 2, dtype=torch.int8)
    rank = torch.arange(R, dtype=torch.int32).repeat(B, 1)
    ref_tok = torch.from_numpy(tok)
    d = logits.cuda()
    top1 = torch.empty((B, R), dtype=torch.int32, device="cuda")
    conf = torch.empty((B, R), dtype=torch.float32, device="cuda")
    flags = torch.empty((B, R), dtype=torch.uint8, device="cuda")
    n = torch.empty((B,), dtype=torch.int32, device="cuda")
    ws = F.alloc_workspace(F.fdllm_accept_workspace_bytes(B, R, V), "cuda")
    res = []
    for _ in range(3):
        F.fdllm_accept(d, kind.cuda(), ref_tok.cuda(), rank.cuda(), top1, conf, flags, n, ws)
        res.append((top1.clone(), conf.clone(), flags.clone(), n.clone()))
    for r in res[1:]:
        assert all(torch.equal(x, y) for x, y in zip(r, res[0]))


@pytest.mark.parametrize("B,R,V", [(2, 160, 4096), (3, 7, 60001), (1, 25, 126464), (4, 80, 9000)])
def test_long_rows_split_over_ctas(F, B, R, V):
    """Rows split over several CTAs, many rows per sequence, and a vocabulary
    that is not a multiple of four (rows start off 16-byte boundaries)."""
    logits, tok = W.random_logits(B, R, V, seed=B * R + V)
    g = np.random.default_rng(V)
    kind = torch.from_numpy(g.integers(0, 3, (B, R)).astype(np.int8))
    ref = torch.from_numpy(np.where(g.random((B, R)) < 0.7, tok, (tok + 1) % V).astype(np.int32))
    rank = torch.from_numpy(np.stack([g.permutation(R) for _ in range(B)]).astype(np.int32))
    gpu, refr = _run_both(F, logits.cuda(), kind, ref, rank, 0.6, 0.5)
    check_accept(gpu, refr, kind.numpy(), rank.numpy(), 0.6, 0.5)


def test_ties_across_splits_and_masked_logits(F):
    """The largest logit tied at two places of a row that different CTAs hold
    (the lower index wins), the maximum in a row's last element, and -inf
    logits (a masked vocabulary entry adds nothing to the sum)."""
    B, R, V = 1, 40, 126464
    g = torch.Generator().manual_seed(9)
    l = torch.randn((B, R, V), generator=g)
    l[0, 0, 5] = 9.0
    l[0, 0, V - 7] = 9.0                   # same value far apart: index 5 wins
    l[0, 1, V - 1] = 12.0                  # the maximum in the last element
    l[0, 2, ::3] = -float("inf")           # a third of the row masked out
    l[0, 3, :] = -float("inf")
    l[0, 3, 77] = 0.0                      # one finite logit: confidence 1
    kind = torch.ones((B, R), dtype=torch.int8)
    gpu, ref = _run_both(F, l.cuda(), kind, torch.zeros((B, R), dtype=torch.int32),
                         torch.zeros((B, R), dtype=torch.int32), 0.9, 0.8)
    assert gpu[0][0, 0] == 5 and gpu[0][0, 1] == V - 1 and gpu[0][0, 3] == 77
    assert gpu[1][0, 3] == 1.0
    assert np.isfinite(gpu[1]).all()
    check_accept(gpu, ref, kind.numpy(), np.zeros((B, R), np.int64), 0.9, 0.8)


def test_long_rows_deterministic(F):
    B, R, V = 8, 40, 126464
    logits, tok = W.random_logits(B, R, V, seed=17)
    kind = torch.full((B, R), 2, dtype=torch.int8).cuda()
    rank = torch.arange(R, dtype=torch.int32).repeat(B, 1).cuda()
    ref_tok = torch.from_numpy(tok).cuda()
    d = logits.cuda()
    a = run_accept_gpu(F, d, kind, ref_tok, rank, 0.9, 0.8)[:4]
    b = run_accept_gpu(F, d, kind, ref_tok, rank, 0.9, 0.8)[:4]
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
