"""The seeded input recipe holds what the tests rely on (CPU only).

Query sets are distinct slots of the generation region, T (tracked, decoded)
and M (the front masks) disjoint; rows of x outside Q are zero; verify rows are
[T_v | S drafts | S masks] over the same positions with one decoding order
shared by the two views; acceptance kinds follow the views; and one sequence
regenerated alone equals its slice of the full batch, which is what lets the
parity tests check sampled sequences of a large batch against the oracle."""
import numpy as np
import torch

import workloads as W

# the configurations' recipes at sizes that generate in milliseconds
SMALL_FUSED = dict(W.CONFIGS["batch_bf16"], B=4, N=300, n_prompt=200, D=64, H=2, dh=64)
SMALL_VERIFY = dict(W.CONFIGS["verify_bf16"], B=3, N=300, n_prompt=200, D=64, H=2, dh=64,
                    vocab=97)


def test_query_sets():
    for name in ("tiny_fp32", "single_bf16", "verify_bf16", "long_bf16", "batch_bf16"):
        cfg = W.CONFIGS[name]
        P, N = cfg["n_prompt"], cfg["N"]
        n_track = cfg.get("n_track", cfg.get("n_tv"))
        beta_m = cfg.get("beta_m", cfg.get("n_s"))
        for b in range(min(cfg["B"], 3)):
            T, M, _ = W.query_positions(cfg, b)
            assert len(T) == n_track and len(M) == beta_m
            assert len(set(T.tolist()) | set(M.tolist())) == n_track + beta_m, "T and M overlap"
            both = np.concatenate([T, M])
            assert both.min() >= P and both.max() < N, "outside the generation region"
            assert np.all(np.diff(M) > 0), "M is taken front to back"


def test_fused_inputs_layout():
    inp = W.fused_inputs(SMALL_FUSED)
    x, q = inp["x"], inp["q_idx"].numpy()
    B, N, D = x.shape
    assert q.shape == (B, SMALL_FUSED["n_track"] + SMALL_FUSED["beta_m"])
    for b in range(B):
        assert len(set(q[b].tolist())) == q.shape[1]
        T, M, _ = W.query_positions(SMALL_FUSED, b)
        assert sorted(q[b].tolist()) == sorted(np.concatenate([T, M]).tolist())
        outside = np.setdiff1d(np.arange(N), q[b])
        assert not x[b, torch.from_numpy(outside)].any(), "x rows outside Q must be zero"
        assert x[b, torch.from_numpy(q[b].astype(np.int64))].abs().sum(-1).min() > 0
    assert inp["k_cache"].shape == (B, SMALL_FUSED["H"], N, SMALL_FUSED["dh"])
    assert inp["w_qkv"].shape == (3 * SMALL_FUSED["H"] * SMALL_FUSED["dh"], D)


def test_verify_inputs_layout():
    inp = W.verify_inputs(SMALL_VERIFY)
    n_tv, n_s = SMALL_VERIFY["n_tv"], SMALL_VERIFY["n_s"]
    pos, view, rank = inp["pos"].numpy(), inp["view"].numpy(), inp["rank"].numpy()
    for b in range(SMALL_VERIFY["B"]):
        assert view[b].tolist() == [0] * n_tv + [1] * n_s + [2] * n_s
        S = pos[b, n_tv:n_tv + n_s]
        assert np.array_equal(pos[b, n_tv + n_s:], S), "the two views share positions"
        assert len(set(pos[b, :n_tv + n_s].tolist())) == n_tv + n_s, "cache rows distinct"
        assert (rank[b, :n_tv] == -1).all()
        r = rank[b, n_tv:n_tv + n_s]
        assert sorted(r.tolist()) == list(range(n_s)), "rank is a permutation"
        assert np.array_equal(rank[b, n_tv + n_s:], r), "the two views share the order"
    assert inp["k_side"].shape[2] == inp["S_max"] == n_s


def test_accept_inputs_follow_the_views():
    a = W.accept_inputs(SMALL_VERIFY)
    v = W.verify_inputs(SMALL_VERIFY)
    n_tv, n_s = SMALL_VERIFY["n_tv"], SMALL_VERIFY["n_s"]
    kind, ref, rank = a["kind"].numpy(), a["ref_tok"].numpy(), a["rank"].numpy()
    assert (kind == np.array([0] * (n_tv + n_s) + [2] * n_s)).all()
    assert ((ref >= 0) == (kind == 2)).all() and ref.max() < SMALL_VERIFY["vocab"]
    assert np.array_equal(rank, v["rank"].numpy())
    assert a["logits"].dtype == torch.float32
    assert a["logits"].shape == (SMALL_VERIFY["B"], n_tv + 2 * n_s, SMALL_VERIFY["vocab"])


def test_one_sequence_regenerates_alone():
    full_f = W.fused_inputs(SMALL_FUSED)
    full_v = W.verify_inputs(SMALL_VERIFY)
    full_a = W.accept_inputs(SMALL_VERIFY)
    for b in (0, 2):
        one = W.fused_inputs(SMALL_FUSED, seqs=[b])
        for k in ("x", "q_idx", "k_cache", "v_cache"):
            assert torch.equal(one[k][0], full_f[k][b]), k
        assert torch.equal(one["w_qkv"], full_f["w_qkv"])
        one = W.verify_inputs(SMALL_VERIFY, seqs=[b])
        for k in ("x_rows", "pos", "view", "rank", "k_cache", "v_cache", "k_side", "v_side"):
            assert torch.equal(one[k][0], full_v[k][b]), k
        one = W.accept_inputs(SMALL_VERIFY, seqs=[b])
        for k in ("logits", "kind", "ref_tok", "rank"):
            assert torch.equal(one[k][0], full_a[k][b]), k
