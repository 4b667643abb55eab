"""The parity checkers reject what they must (CPU only).

The GPU parity tests decide through the helpers in `parity.py`.  Each helper
here gets the oracle's own result in place of the GPU's, which it must accept,
and then that result with one planted mistake, made on the CPU, which it must
reject: a value just past the tolerance, a non-finite value, a changed slot
outside Q, a missed or misplaced scatter, a wrong token, confidence, flag or
accepted count, a prefix that runs past a failure, a tracked set that is out of
order, repeats a slot, holds a non-candidate, pads wrongly or leaves out a
heavier candidate.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity import (CONF_TOL, TOL_BF16_REL, TOL_F32_ABS, assert_close, check_accept,
                    check_cache_update, check_track, oracle_fused)


def test_assert_close_bounds():
    ref = np.linspace(-3.0, 3.0, 101)
    for dtype, tol in (("f32", TOL_F32_ABS), ("bf16", TOL_BF16_REL * 3.0)):
        g = ref.copy()
        g[50] += 0.9 * tol
        assert_close(g, ref, dtype, "inside")
        g[50] = ref[50] + 1.1 * tol          # one element past the bound
        with pytest.raises(AssertionError):
            assert_close(g, ref, dtype, "outside")
    g = ref.copy()
    g[7] = np.nan
    with pytest.raises(AssertionError):
        assert_close(g, ref, "f32", "nan")
    with pytest.raises(AssertionError):
        assert_close(ref[:-1], ref, "f32", "shape")


def _bf16(a):
    """bf16 tensor of float64 values that are already bf16 values (exact)."""
    t = torch.from_numpy(a).to(torch.bfloat16)
    assert np.array_equal(O.to_f64(t), a)
    return t


def test_check_cache_update_rejects_planted_mistakes():
    B, N, D, H, dh = 2, 48, 64, 2, 64
    inp = W.random_fused(B, N, D, H, dh, nq=5, dtype="bf16", seed=11)
    K2, _, _ = oracle_fused(inp, H, dh, 10000.0, "bf16")
    q = inp["q_idx"].numpy()
    k_in = inp["k_cache"]
    good = _bf16(K2)
    check_cache_update(good, k_in, K2, q, "bf16", "k")

    bad = good.clone()
    outside = np.setdiff1d(np.arange(N), q[1])[3]
    bad.view(torch.int16)[1, 0, outside, 5] ^= 1          # one bit outside Q
    with pytest.raises(AssertionError, match="outside Q"):
        check_cache_update(bad, k_in, K2, q, "bf16", "k")

    bad = good.clone()
    bad[0, :, q[0, 2]] = k_in[0, :, q[0, 2]]               # a write that never landed
    with pytest.raises(AssertionError):
        check_cache_update(bad, k_in, K2, q, "bf16", "k")

    bad = good.clone()
    a, c = int(q[0, 0]), int(q[0, 1])
    bad[0, :, [a, c]] = good[0, :, [c, a]]                 # two scatter targets swapped
    with pytest.raises(AssertionError):
        check_cache_update(bad, k_in, K2, q, "bf16", "k")


def _as_gpu(ref):
    """The oracle's acceptance result in the GPU's output types."""
    t, c, f, n = ref
    return t.astype(np.int32), c.astype(np.float32), f.copy(), n.astype(np.int32)


def _accept_case():
    B, R, V = 2, 12, 50
    logits, tok = W.random_logits(B, R, V, seed=5)
    kind = np.tile(np.array([0, 0, 1, 1, 1, 1, 2, 2, 2, 2, 2, 2], np.int8), (B, 1))
    g = np.random.default_rng(1)
    rank = np.stack([np.r_[[-1] * 6, g.permutation(6)] for _ in range(B)]).astype(np.int32)
    ref_tok = np.where(kind == 2, tok, -1).astype(np.int32)
    ref_tok[1, 8] = (tok[1, 8] + 1) % V                    # one draft the check rejects
    l64 = logits.numpy().astype(np.float64)
    return l64, kind, ref_tok, rank


def test_check_accept_rejects_planted_mistakes():
    l64, kind, ref_tok, rank = _accept_case()
    eps, gamma = 0.9, 0.8
    ref = O.accept(l64, kind, ref_tok, rank, eps, gamma)
    assert check_accept(_as_gpu(ref), ref, kind, rank, eps, gamma) == 0   # no row near a threshold
    assert ref[3][1] < (kind[1] == 2).sum()                              # sequence 1 stops early

    def planted(edit):
        gpu = list(_as_gpu(ref))
        edit(gpu)
        with pytest.raises(AssertionError):
            check_accept(tuple(gpu), ref, kind, rank, eps, gamma)

    planted(lambda g: g[0].__setitem__((0, 3), (g[0][0, 3] + 1) % l64.shape[2]))
    planted(lambda g: g[1].__setitem__((1, 5), g[1][1, 5] + 2 * CONF_TOL))
    kind1 = int(np.nonzero(kind[0] == 1)[0][0])
    planted(lambda g: g[2].__setitem__((0, kind1), g[2][0, kind1] ^ O.FLAG_COMMIT))
    planted(lambda g: g[2].__setitem__((1, 8), g[2][1, 8] | O.FLAG_ACCEPT))
    planted(lambda g: g[3].__setitem__(1, g[3][1] + 1))


def _logit_for(conf):
    return math.log(conf / (1.0 - conf))


def test_check_accept_near_a_threshold():
    """A row whose oracle confidence is within CONF_TOL of gamma may go either
    way; the GPU's flags must then follow from its own pass bits."""
    gamma, eps = 0.8, 0.9
    confs = [0.95, gamma + 3e-6, 0.95]                    # the middle row is ambiguous
    l32 = np.zeros((1, 3, 2), np.float32)
    l32[0, :, 0] = [_logit_for(c) for c in confs]
    l64 = l32.astype(np.float64)
    kind = np.full((1, 3), 2, np.int8)
    ref_tok = np.zeros((1, 3), np.int32)
    rank = np.array([[0, 1, 2]], np.int32)
    ref = O.accept(l64, kind, ref_tok, rank, eps, gamma)
    assert ref[3][0] == 3
    P, A = O.FLAG_PASS, O.FLAG_ACCEPT

    def gpu(flags, n, c_mid):
        c = ref[1].astype(np.float32).copy()
        c[0, 1] = c_mid
        return (ref[0].astype(np.int32), c, np.array([flags], np.uint8), np.array([n], np.int32))

    # the oracle's decision, and the other one taken consistently: both valid
    assert check_accept(gpu([P | A, P | A, P | A], 3, gamma + 3e-6), ref, kind, rank, eps, gamma) == 1
    assert check_accept(gpu([P | A, 0, P], 1, gamma - 1e-6), ref, kind, rank, eps, gamma) == 1
    # the middle row failed on the GPU, yet the prefix runs past it
    with pytest.raises(AssertionError):
        check_accept(gpu([P | A, 0, P | A], 2, gamma - 1e-6), ref, kind, rank, eps, gamma)
    with pytest.raises(AssertionError):
        check_accept(gpu([P | A, 0, P], 2, gamma - 1e-6), ref, kind, rank, eps, gamma)


def test_check_track_rejects_planted_mistakes():
    B, N, D, H, dh, nq, beta_t = 2, 40, 64, 3, 64, 6, 8
    inp = W.random_fused(B, N, D, H, dh, nq=nq, dtype="f32", seed=12)
    K2, _, _ = oracle_fused(inp, H, dh, 10000.0, "f32")
    g = np.random.default_rng(13)
    masked = (g.random((B, nq)) < 0.5).astype(np.int8)
    masked[:, 0] = 1
    cand = (g.random((B, N)) < 0.6).astype(np.int8)
    f = O.to_f64
    ref = O.attention_mass(f(inp["x"]), inp["q_idx"].numpy(), f(inp["w_qkv"]), 10000.0, K2, H,
                           dh, masked)
    good = O.track_select(ref, cand, beta_t).astype(np.int32)
    check_track(good, ref, ref, cand, beta_t, "f32")
    tol = 1e-4 * np.abs(ref).max()

    def planted(track=None, mass=None, cnd=cand):
        with pytest.raises(AssertionError):
            check_track(good if track is None else track, ref if mass is None else mass, ref,
                        cnd, beta_t, "f32")

    t = good.copy()
    t[0, [1, 2]] = t[0, [2, 1]]                            # out of order
    planted(track=t)
    t = good.copy()
    t[1, 3] = t[1, 2]                                      # a slot twice
    planted(track=t)
    t = good.copy()
    t[0, -1] = int(np.nonzero(cand[0] == 0)[0][0])         # not a decoded slot
    planted(track=t)
    t = good.copy()
    rest = np.setdiff1d(np.nonzero(cand[0])[0], good[0])
    light = rest[np.argmin(ref[0, rest])]
    assert ref[0, good[0, -1]] - ref[0, light] > 2 * tol   # a real gap, not a near tie
    t[0, -1] = light                                       # still in descending order
    planted(track=t)
    m = ref.copy()
    m[1, 7] += 1.5 * tol                                   # a mass past the tolerance
    planted(mass=m)
    few = np.zeros_like(cand)
    few[:, [2, 9, 30]] = 1
    short = O.track_select(ref, few, beta_t).astype(np.int32)
    check_track(short, ref, ref, few, beta_t, "f32")
    t = short.copy()
    t[0, 3:] = 0                                           # padding must be -1
    planted(track=t, cnd=few)
