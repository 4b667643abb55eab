"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test ties one part of the oracle to something it does not compute itself:
the pages' worked example, a library routine (torch's bfloat16 conversion and
scaled-dot-product attention), hand-evaluated closed forms, or a structural
invariant of the method.  Each is chosen so that a plausible slip (a dropped
term, a wrong sign or index, a transposed operand, swapped q/k/v blocks) fails.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        k, v = [s.strip() for s in line.split("=", 1)]
        vals[k] = v.split()
    return vals


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_on_float32_values():
    g = np.random.default_rng(0)
    x = np.concatenate([g.standard_normal(20000), g.standard_normal(2000) * 1e-30,
                        g.standard_normal(2000) * 1e30]).astype(np.float32)
    # exact ties: a float32 whose low 16 bits are 0x8000
    ties = ((g.integers(0x3f00, 0x4100, 500).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x.astype(np.float64)), ref)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.bf16_bits(x.astype(np.float64)), bits)
    np.testing.assert_array_equal(O.bf16_bits_to_f64(bits), ref)


def test_round_bf16_hand_cases():
    # near 1 the bf16 step is 2^-7
    assert O.round_bf16(1 + 2**-8) == 1.0                   # tie -> even (1.0)
    assert O.round_bf16(1 + 3 * 2**-8) == 1 + 2**-6         # tie -> even
    # just above a tie rounds up; rounding via float32 first would give 1.0
    assert O.round_bf16(1 + 2**-8 + 2**-40) == 1 + 2**-7
    assert O.round_bf16(-1.0 - 2**-8 - 2**-40) == -(1 + 2**-7)
    assert O.round_bf16(0.0) == 0.0


def test_storage_decoding_and_f32_rounding_match_torch():
    """to_f64 widens stored bf16 and fp32 tensors exactly as torch does, and
    round_to(., "f32") is torch's float64 -> float32 conversion (the bf16
    branch is checked above on float32 inputs: torch's float64 -> bfloat16
    conversion goes through float32 and so rounds twice)."""
    g = np.random.default_rng(10)
    x = g.standard_normal(5000) * np.exp(g.uniform(-30, 30, 5000))
    t64 = torch.from_numpy(x)
    for dt in (torch.bfloat16, torch.float32):
        t = t64.to(dt)
        np.testing.assert_array_equal(O.to_f64(t), t.to(torch.float64).numpy())
    np.testing.assert_array_equal(O.round_to(x, "f32"),
                                  t64.to(torch.float32).to(torch.float64).numpy())
    assert not np.array_equal(O.round_to(x, "f32"), x)


# ---------------------------------------------------------------- RoPE

def test_rope_hand_values():
    # dh = 4, base = 10000: theta = [1, 10000^(-1/2)] = [1, 0.01]
    x = np.zeros((2, 1, 4))
    x[0, 0, 1] = 1.0           # second pair, first component
    x[1, 0, 0] = 1.0           # first pair, first component
    y = O.rope(x, np.array([100, 1]), 10000.0)
    c1, s1 = 0.5403023058681398, 0.8414709848078965        # cos 1, sin 1
    np.testing.assert_allclose(y[0, 0], [0, c1, 0, s1], atol=1e-15)
    np.testing.assert_allclose(y[1, 0], [c1, 0, s1, 0], atol=1e-15)


def test_rope_is_complex_rotation_and_relative():
    g = np.random.default_rng(1)
    n, H, dh, base = 7, 3, 8, 500.0
    x = g.standard_normal((n, H, dh))
    pos = g.integers(0, 4000, n)
    y = O.rope(x, pos, base)
    half = dh // 2
    theta = np.array([base ** (-k / half) for k in range(half)])   # base^(-2k/dh)
    z = (x[..., :half] + 1j * x[..., half:]) * np.exp(1j * pos[:, None, None] * theta)
    np.testing.assert_allclose(y[..., :half], z.real, atol=1e-12)
    np.testing.assert_allclose(y[..., half:], z.imag, atol=1e-12)
    np.testing.assert_allclose(O.rope(x, np.zeros(n, int), base), x, atol=0)
    # pair norms are kept; dot products depend on the position difference only
    np.testing.assert_allclose(np.hypot(y[..., :half], y[..., half:]),
                               np.hypot(x[..., :half], x[..., half:]), atol=1e-12)
    q, k = x[:1], x[1:2]
    d1 = (O.rope(q, np.array([37]), base) * O.rope(k, np.array([11]), base)).sum()
    d2 = (O.rope(q, np.array([1037]), base) * O.rope(k, np.array([1011]), base)).sum()
    assert abs(d1 - d2) < 1e-10


# ---------------------------------------------------------------- attention

def test_attend_closed_forms():
    g = np.random.default_rng(2)
    q = g.standard_normal((5, 16))
    K = g.standard_normal((40, 16))
    u = g.standard_normal(16)
    np.testing.assert_allclose(O.attend(q, K, np.tile(u, (40, 1))), np.tile(u, (5, 1)), atol=1e-12)
    V = g.standard_normal((40, 16))
    np.testing.assert_allclose(O.attend(np.zeros((2, 16)), K, V), np.tile(V.mean(0), (2, 1)), atol=1e-12)
    K2 = K.copy()
    K2[17] = 1e3 * q[0]          # one key dominates row 0
    np.testing.assert_allclose(O.attend(q[:1], K2, V), V[17:18], atol=1e-9)
    vis = np.ones((1, 40), bool)
    vis[0, 17] = False           # hiding it removes it exactly
    np.testing.assert_allclose(O.attend(q[:1], K2, V, vis),
                               O.attend(q[:1], np.delete(K2, 17, 0), np.delete(V, 17, 0)), atol=1e-12)


def _sdpa_full_sequence(x, w, H, dh, base):
    """Bidirectional self-attention over a whole sequence by an independent route:
    heads split with a reshape of W, RoPE as a complex rotation, torch SDPA."""
    N, D = x.shape
    W = torch.from_numpy(w).view(3, H, dh, D)
    X = torch.from_numpy(x)
    q, k, v = (torch.einsum("nd,hed->hne", X, W[i]) for i in range(3))
    half = dh // 2
    theta = torch.tensor([base ** (-j / half) for j in range(half)], dtype=torch.float64)
    rot = torch.polar(torch.ones(N, half, dtype=torch.float64),
                      torch.arange(N, dtype=torch.float64)[:, None] * theta)

    def rope_c(t):
        z = torch.complex(t[..., :half], t[..., half:]) * rot
        return torch.cat([z.real, z.imag], -1)

    q, k = rope_c(q), rope_c(k)
    o = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0]
    return o.permute(1, 0, 2).reshape(N, H * dh).numpy(), k.numpy(), v.numpy()


@pytest.mark.parametrize("dh", [8, 16])
def test_fused_step_equals_full_recompute(dh):
    g = np.random.default_rng(3)
    B, N, D, H, base = 2, 24, 32, 2, 10000.0
    x = g.standard_normal((B, N, D))
    w = g.standard_normal((3 * H * dh, D)) / math.sqrt(D)
    full = [_sdpa_full_sequence(x[b], w, H, dh, base) for b in range(B)]
    # (a) Q = every slot: every cache slot is overwritten, out is plain self-attention
    junk = g.standard_normal((B, H, N, dh))
    q_all = np.stack([g.permutation(N) for _ in range(B)])
    K2, V2, out = O.fused_step(x, q_all, w, base, junk, junk * 3, H, dh, "f64")
    for b in range(B):
        np.testing.assert_allclose(out[b], full[b][0][q_all[b]], atol=1e-12)
        np.testing.assert_allclose(K2[b], full[b][1], atol=1e-12)
        np.testing.assert_allclose(V2[b], full[b][2], atol=1e-12)
    # (b) consistent cache, Q a strict subset: same rows as the full recompute
    Kc = np.stack([f[1] for f in full])
    Vc = np.stack([f[2] for f in full])
    q_sub = np.stack([g.choice(N, 5, replace=False) for _ in range(B)])
    K3, V3, out3 = O.fused_step(x, q_sub, w, base, Kc, Vc, H, dh, "f64")
    for b in range(B):
        np.testing.assert_allclose(out3[b], full[b][0][q_sub[b]], atol=1e-12)
    np.testing.assert_allclose(K3, Kc, atol=1e-12)


def test_fused_step_touches_only_q_slots_and_rounds_once():
    g = np.random.default_rng(4)
    B, N, D, H, dh = 2, 30, 16, 2, 8
    x = g.standard_normal((B, N, D))
    w = g.standard_normal((3 * H * dh, D))
    K = O.round_bf16(g.standard_normal((B, H, N, dh)))
    V = O.round_bf16(g.standard_normal((B, H, N, dh)))
    q_idx = np.stack([g.choice(N, 4, replace=False) for _ in range(B)])
    K2, V2, _ = O.fused_step(x, q_idx, w, 100.0, K, V, H, dh, "bf16")
    K64, V64, _ = O.fused_step(x, q_idx, w, 100.0, K, V, H, dh, "f64")
    for b in range(B):
        rest = np.setdiff1d(np.arange(N), q_idx[b])
        assert np.array_equal(K2[b][:, rest].view(np.uint64), K[b][:, rest].view(np.uint64))
        assert np.array_equal(V2[b][:, rest].view(np.uint64), V[b][:, rest].view(np.uint64))
        Qb = q_idx[b]
        np.testing.assert_array_equal(K2[b][:, Qb], O.round_bf16(K64[b][:, Qb]))
        np.testing.assert_array_equal(V2[b][:, Qb], O.round_bf16(V64[b][:, Qb]))
        assert not np.array_equal(K2[b][:, Qb], K64[b][:, Qb])  # rounding did happen


# ---------------------------------------------------------------- verify pass

def _verify_case(g, n_tv=3, n_s=4, N=40, D=24, H=2, dh=8):
    pos_all = g.choice(N, n_tv + n_s, replace=False)
    T, S = pos_all[:n_tv], pos_all[n_tv:]
    r = g.permutation(n_s)
    pos = np.concatenate([T, S, S])[None]
    view = np.array([0] * n_tv + [1] * n_s + [2] * n_s)[None]
    rank = np.concatenate([-np.ones(n_tv, int), r, r])[None]
    R = pos.shape[1]
    x_rows = g.standard_normal((1, R, D))
    w = g.standard_normal((3 * H * dh, D)) / math.sqrt(D)
    K = g.standard_normal((1, H, N, dh))
    V = g.standard_normal((1, H, N, dh))
    KS = g.standard_normal((1, H, n_s + 2, dh))
    VS = g.standard_normal((1, H, n_s + 2, dh))
    return dict(x_rows=x_rows, pos=pos, view=view, rank=rank, w=w, K=K, V=V, KS=KS, VS=VS,
                H=H, dh=dh, n_tv=n_tv, n_s=n_s, T=T, S=S, N=N)


def _run_verify(c, causal=False, **over):
    a = dict(c)
    a.update(over)
    return O.verify_step(a["x_rows"], a["pos"], a["view"], a["rank"], a["w"], 10000.0,
                         a["K"], a["V"], a["KS"], a["VS"], a["H"], a["dh"], "f64", causal)


def test_verify_views_are_two_fused_steps():
    """Draft/T_v rows see the cache with the drafts written at S; mask rows see the
    same cache with the [MASK]-view keys at S instead.  Each equals a plain fused
    step over the corresponding state."""
    g = np.random.default_rng(5)
    c = _verify_case(g)
    K2, V2, KS, VS, out = _run_verify(c)
    n_tv, n_s, H, dh, N = c["n_tv"], c["n_s"], c["H"], c["dh"], c["N"]
    D = c["x_rows"].shape[2]
    for view_rows in (np.arange(n_tv + n_s), np.r_[np.arange(n_tv), n_tv + n_s + np.arange(n_s)]):
        x = np.zeros((1, N, D))
        Q = c["pos"][0, view_rows]
        x[0, Q] = c["x_rows"][0, view_rows]
        Kf, Vf, of = O.fused_step(x, Q[None], c["w"], 10000.0, c["K"], c["V"], H, dh, "f64")
        own = view_rows[n_tv:]
        np.testing.assert_allclose(out[0, own], of[0, n_tv:], atol=1e-12)
        if view_rows[-1] < n_tv + n_s:   # draft state: the cache itself matches
            np.testing.assert_allclose(K2, Kf, atol=1e-12)
            np.testing.assert_allclose(out[0, :n_tv], of[0, :n_tv], atol=1e-12)
        else:                             # mask state: side slots hold the mask-view keys
            np.testing.assert_allclose(KS[0, :, :n_s], Kf[0][:, c["S"]], atol=1e-12)
            np.testing.assert_allclose(VS[0, :, :n_s], Vf[0][:, c["S"]], atol=1e-12)
    # the unused side slots are untouched
    np.testing.assert_array_equal(KS[0, :, n_s:], c["KS"][0, :, n_s:])


def test_verify_views_cannot_see_each_other():
    g = np.random.default_rng(6)
    c = _verify_case(g)
    n_tv, n_s = c["n_tv"], c["n_s"]
    out = _run_verify(c)[4]
    xr = c["x_rows"].copy()
    xr[0, n_tv:n_tv + n_s] += 5.0            # perturb the draft view
    out_d = _run_verify(c, x_rows=xr)[4]
    np.testing.assert_allclose(out_d[0, n_tv + n_s:], out[0, n_tv + n_s:], atol=1e-12)
    assert np.abs(out_d[0, :n_tv] - out[0, :n_tv]).max() > 1e-3    # T_v does see drafts
    xr = c["x_rows"].copy()
    xr[0, n_tv + n_s:] -= 5.0                # perturb the mask view
    out_m = _run_verify(c, x_rows=xr)[4]
    np.testing.assert_allclose(out_m[0, :n_tv + n_s], out[0, :n_tv + n_s], atol=1e-12)


def test_verify_without_views_is_fused_step():
    g = np.random.default_rng(7)
    c = _verify_case(g)
    n = c["n_tv"]
    sub = dict(x_rows=c["x_rows"][:, :n], pos=c["pos"][:, :n], view=c["view"][:, :n],
               rank=c["rank"][:, :n])
    K2, V2, KS, VS, out = _run_verify(c, **sub)
    x = np.zeros((1, c["N"], c["x_rows"].shape[2]))
    x[0, c["T"]] = c["x_rows"][0, :n]
    Kf, Vf, of = O.fused_step(x, c["T"][None], c["w"], 10000.0, c["K"], c["V"], c["H"], c["dh"], "f64")
    np.testing.assert_allclose(out, of, atol=1e-12)
    np.testing.assert_allclose(K2, Kf, atol=0)
    np.testing.assert_array_equal(KS, c["KS"])


def test_causal_cross_special_cases():
    g = np.random.default_rng(8)
    # |S| = 1: the causal and mutual readings coincide (the worked example's case)
    c1 = _verify_case(g, n_s=1)
    np.testing.assert_allclose(_run_verify(c1, causal=True)[4], _run_verify(c1)[4], atol=0)
    c = _verify_case(g, n_s=5)
    n_tv, n_s = c["n_tv"], c["n_s"]
    mut = _run_verify(c)[4]
    cau = _run_verify(c, causal=True)[4]
    r = c["rank"][0, n_tv + n_s:]
    lo, hi = n_tv + n_s + np.argmin(r), n_tv + n_s + np.argmax(r)
    # the first mask row in decoding order conditions on no draft: same as mutual
    np.testing.assert_allclose(cau[0, lo], mut[0, lo], atol=1e-12)
    # the last one sees every other draft and only its own [MASK] key: a fused
    # step over the state "drafts everywhere in S except its own position"
    N, D = c["N"], c["x_rows"].shape[2]
    rows = np.r_[np.arange(n_tv), n_tv + np.arange(n_s)]
    rows = np.where(c["pos"][0, rows] == c["pos"][0, hi], hi, rows)
    x = np.zeros((1, N, D))
    Q = c["pos"][0, rows]
    x[0, Q] = c["x_rows"][0, rows]
    of = O.fused_step(x, Q[None], c["w"], 10000.0, c["K"], c["V"], c["H"], c["dh"], "f64")[2]
    np.testing.assert_allclose(cau[0, hi], of[0, list(rows).index(hi)], atol=1e-12)
    # the draft and T_v rows never depend on the mode
    np.testing.assert_allclose(cau[0, :n_tv + n_s], mut[0, :n_tv + n_s], atol=0)


# ---------------------------------------------------------------- acceptance

def test_accept_worked_example():
    gd = _golden()
    eps, gamma = float(gd["eps"][0]), float(gd["gamma"][0])
    vocab = gd["vocab"]
    q2 = np.array(gd["q_2"], float)
    q3 = np.array(gd["q_3"], float)
    p3 = np.array(gd["p_3"], float)
    # draft pass: rows for positions 2 and 3, kind 1
    logits = np.log(np.stack([q2, q3]))[None]
    top1, conf, flags, _ = O.accept(logits, np.array([[1, 1]]), np.array([[-1, -1]]),
                                    np.array([[-1, -1]]), eps, gamma)
    np.testing.assert_allclose(conf[0], [float(gd["c_2"][0]), float(gd["c_3"][0])], atol=1e-12)
    assert [vocab[t] for t in top1[0]] == [gd["xhat_2"][0], gd["xhat_3"][0]]
    D = [p for p, f in zip((2, 3), flags[0]) if f & O.FLAG_COMMIT]
    S = [p for p, f in zip((2, 3), flags[0]) if not f & O.FLAG_COMMIT]
    assert D == [int(gd["D_1"][0])] and S == [int(gd["S_1"][0])]
    # verification: the mask-view row of position 3 against the draft token A
    xhat3 = vocab.index(gd["xhat_3"][0])
    t, c, f, n = O.accept(np.log(p3)[None, None], np.array([[2]]), np.array([[xhat3]]),
                          np.array([[0]]), eps, gamma)
    assert vocab[t[0, 0]] == gd["xtilde_3"][0]
    assert abs(c[0, 0] - float(gd["ctilde_3"][0])) < 1e-12
    assert f[0, 0] & O.FLAG_ACCEPT and n[0] == 1 and int(gd["accepted"][0]) == 3
    # without verification position 3 would have been dropped: c_3 < eps
    assert conf[0, 1] < eps
    # perturbations: a stricter gamma, or a different draft token, rejects it
    assert O.accept(np.log(p3)[None, None], np.array([[2]]), np.array([[xhat3]]),
                    np.array([[0]]), eps, 0.9)[3][0] == 0
    assert O.accept(np.log(p3)[None, None], np.array([[2]]), np.array([[vocab.index("B")]]),
                    np.array([[0]]), eps, gamma)[3][0] == 0


def test_accept_prefix_stops_at_first_failure():
    # decoding order is given by rank, not by row order
    probs = np.array([[0.9, 0.02, 0.02, 0.02, 0.02, 0.02],     # passes
                      [0.5, 0.1, 0.1, 0.1, 0.1, 0.1],          # fails on confidence
                      [0.02, 0.9, 0.02, 0.02, 0.02, 0.02]])    # passes
    ref = np.array([[0, 0, 1]])
    for rank, expect in (([0, 1, 2], [1, 0, 0]), ([2, 1, 0], [0, 0, 1]), ([1, 2, 0], [1, 0, 1])):
        t, c, f, n = O.accept(np.log(probs)[None], np.array([[2, 2, 2]]), ref,
                              np.array([rank]), 0.9, 0.8)
        got = [int((int(x) & O.FLAG_ACCEPT) > 0) for x in f[0]]
        assert got == expect and n[0] == sum(expect)
        assert [(int(x) & O.FLAG_PASS) > 0 for x in f[0]] == [True, False, True]


def test_accept_thresholds_are_inclusive():
    """Two equal logits give a confidence of exactly 1/2.  At eps = gamma = 1/2
    the draft row is committed and the mask-view row passes (the worked
    example's margins leave the boundary open; the reading is c >= eps and
    c~ >= gamma).  One ulp above 1/2, neither."""
    l = np.zeros((1, 2, 2))
    kind, ref, rank = np.array([[1, 2]]), np.array([[-1, 0]]), np.array([[-1, 0]])
    _, c, f, n = O.accept(l, kind, ref, rank, 0.5, 0.5)
    assert c[0].tolist() == [0.5, 0.5]
    assert f[0, 0] & O.FLAG_COMMIT and f[0, 1] & O.FLAG_PASS and n[0] == 1
    up = float(np.nextafter(0.5, 1.0))
    _, _, f, n = O.accept(l, kind, ref, rank, up, up)
    assert not f[0, 0] & O.FLAG_COMMIT and not f[0, 1] & O.FLAG_PASS and n[0] == 0


def test_accept_ties_uniform_and_tv_bound():
    g = np.random.default_rng(9)
    l = np.zeros((1, 2, 50))
    l[0, 0, [7, 30]] = 3.0                 # tie -> lowest index
    t, c, _, _ = O.accept(l, np.zeros((1, 2), int), -np.ones((1, 2), int),
                          -np.ones((1, 2), int), 0.9, 0.8)
    assert t[0, 0] == 7 and t[0, 1] == 0
    assert abs(c[0, 1] - 1 / 50) < 1e-15    # uniform row
    assert abs(c[0, 0] - math.exp(3) / (2 * math.exp(3) + 48)) < 1e-15
    # TV bound of the accepted block: prod of accepted confidences >= gamma^m
    for trial in range(20):
        R, gamma = 12, 0.7
        logits = g.standard_normal((1, R, 40))
        tok = g.integers(0, 40, R)
        logits[0, np.arange(R), tok] += g.uniform(2, 9, R)
        ref = np.where(g.random(R) < 0.85, tok, (tok + 1) % 40)[None]
        rank = g.permutation(R)[None]
        t, c, f, n = O.accept(logits, np.full((1, R), 2), ref, rank, 0.9, gamma)
        acc = (f[0] & O.FLAG_ACCEPT) > 0
        m = int(acc.sum())
        assert m == n[0]
        assert np.prod(c[0, acc]) >= gamma ** m - 1e-15
        # the accepted set is a prefix in rank order
        order = np.argsort(rank[0])
        seq = acc[order]
        assert not np.any(seq[1:] & ~seq[:-1])


# ----------------------------------------------------------------------------
# tracked-set selection ([review], "How It Works", Step 1: Cache selection)


def _mass_case(seed, B=2, N=40, D=64, H=3, dh=64, nq=6):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, N, D))
    w = rng.standard_normal((3 * H * dh, D)) / np.sqrt(D)
    K = rng.standard_normal((B, H, N, dh))
    V = rng.standard_normal((B, H, N, dh))
    q_idx = np.stack([rng.choice(N, nq, replace=False) for _ in range(B)])
    masked = (rng.random((B, nq)) < 0.5).astype(np.int8)
    masked[:, 0] = 1
    K2, V2, _ = O.fused_step(x, q_idx, w, 10000.0, K, V, H, dh, "f64")
    return x, q_idx, w, K2, masked, H, dh


def test_attention_mass_is_sdpa_probabilities():
    """With V = the identity, torch's scaled-dot-product attention returns the
    softmax probabilities themselves; summed over the masked rows and heads
    they must equal the oracle's attention mass (catches a wrong scale, a
    softmax over the wrong axis or a transposed operand)."""
    x, q_idx, w, K2, masked, H, dh = _mass_case(21)
    a = O.attention_mass(x, q_idx, w, 10000.0, K2, H, dh, masked)
    B, N = a.shape
    for b in range(B):
        rows = np.nonzero(masked[b])[0]
        Q = q_idx[b][rows]
        q, _, _ = O.project_qkv(x[b, Q], w, H, dh)
        q = O.rope(q, Q, 10000.0)
        ref = np.zeros(N)
        eye = torch.eye(N, dtype=torch.float64)
        for h in range(H):
            p = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[:, h])[None], torch.from_numpy(K2[b, h])[None], eye[None])[0]
            ref += p.numpy().sum(axis=0)
        np.testing.assert_allclose(a[b], ref, rtol=1e-12, atol=1e-14)


def test_attention_mass_closed_forms():
    """Each masked row and head spreads probability 1 over the N slots: the
    mass sums to (masked rows) x H.  Equal keys give every slot the same
    share; no masked row gives no mass."""
    x, q_idx, w, K2, masked, H, dh = _mass_case(22)
    a = O.attention_mass(x, q_idx, w, 10000.0, K2, H, dh, masked)
    np.testing.assert_allclose(a.sum(axis=1), masked.sum(axis=1) * H, rtol=1e-12)
    Kc = np.broadcast_to(K2[:, :, :1, :], K2.shape).copy()
    a_eq = O.attention_mass(x, q_idx, w, 10000.0, Kc, H, dh, masked)
    N = K2.shape[2]
    np.testing.assert_allclose(a_eq, (masked.sum(axis=1) * H / N)[:, None] * np.ones((1, N)),
                               rtol=1e-12)
    assert not O.attention_mass(x, q_idx, w, 10000.0, K2, H, dh, np.zeros_like(masked)).any()


def test_track_select_order_ties_and_padding():
    a = np.array([[0.5, 2.0, 2.0, 0.1, 3.0, 2.0]])
    cand = np.array([[1, 1, 1, 1, 0, 1]])
    # slot 4 has the most mass but is not decoded; 1, 2, 5 tie: lower slot first
    assert O.track_select(a, cand, 4).tolist() == [[1, 2, 5, 0]]
    assert O.track_select(a, cand, 7).tolist() == [[1, 2, 5, 0, 3, -1, -1]]
    assert O.track_select(a, np.zeros_like(cand), 2).tolist() == [[-1, -1]]


def test_track_select_worked_example_rule():
    """The review's example: [BOS] + 4 masks, slot 0 decoded before the step,
    Q = {1, 2} (the front beta_m = 2 masks), both resolved by the step, beta_t
    = 1.  The resolved slots join the ranking, so T keeps exactly one slot, and
    it is the slot the masked queries attend to most.  The cache is built so
    that one key dominates every score (closed form: it takes all the mass)."""
    H, dh, N, D = 2, 64, 5, 64
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, N, D))
    w = rng.standard_normal((3 * H * dh, D)) / np.sqrt(D)
    q_idx = np.array([[1, 2]])
    masked = np.array([[1, 1]], dtype=np.int8)
    cand = np.array([[1, 1, 1, 0, 0]])  # slot 0 earlier; 1, 2 resolved now
    for target in (0, 2):
        K = rng.standard_normal((1, H, N, dh)) * 1e-3
        V = np.zeros((1, H, N, dh))
        K2, _, _ = O.fused_step(x, q_idx, w, 10000.0, K, V, H, dh, "f64")
        q, _, _ = O.project_qkv(x[0, q_idx[0]], w, H, dh)
        q = O.rope(q, q_idx[0], 10000.0)
        for h in range(H):
            # a key along the sum of the queries' directions, far above the rest
            K2[0, h, target] = 400.0 * (q[:, h] / np.linalg.norm(q[:, h], axis=1, keepdims=True)).sum(0)
            K2[0, h, 1:3] *= 1e-6 if target == 0 else 1.0
        a = O.attention_mass(x, q_idx, w, 10000.0, K2, H, dh, masked)
        assert a[0, target] > 0.999 * 2 * H
        assert O.track_select(a, cand, 1).tolist() == [[target]]
