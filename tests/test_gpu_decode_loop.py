"""The synthetic multi-step decode loop runs every call of the path in sequence
(draft pass per layer, epsilon split, verify pass, gamma acceptance, tracked-set
selection) until the generated block is decoded."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
def test_decode_loop_decodes_everything(causal):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_attention_fdllm_b200 import decode_loop as DL
    cfg = DL.LoopConfig(B=2, n_prompt=32, n_gen=24, H=2, dh=64, L=2, beta_m=8, beta_t=4,
                        vocab=64, seed=3, max_steps=100, causal_cross=causal)
    r = DL.run(cfg)
    assert r["all_decoded"]
    assert r["tokens_decoded"] == cfg.B * cfg.n_gen
    assert 1 <= r["steps"] <= cfg.n_gen
    assert r["kernel_launches"] > 0
    assert r["draft_traffic_saving"] > 1.0


def test_first_step_replays_in_the_oracle():
    """The first step of the loop, call by call, against the fp64 oracle on the
    inputs each call got: the draft pass of layer 0 and of the middle layer
    (outputs and cache writes), the attention masses and the tracked set, the
    epsilon split, the verify pass of layer 0, the gamma acceptance, and the
    sets the step ends with (decoded slots, next tracked set).

    Flags, accepted counts, the decoded set and the tracked set must match bit
    for bit; only rows whose oracle confidence lies within the confidence
    tolerance of a threshold may take either decision (then the GPU's own
    flags must be consistent).  The tracked set is the exact selection rule
    applied to the GPU's masses, which must match the oracle's masses."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import numpy as np

    import oracle as O
    from kv_cache_attention_fdllm_b200 import decode_loop as DL
    from parity import assert_close, check_accept, check_cache_update, check_track

    cfg = DL.LoopConfig(B=2, n_prompt=64, n_gen=48, H=2, dh=64, L=2, beta_m=16, beta_t=8,
                        vocab=256, seed=5, max_steps=1)
    tr = {}
    DL.run(cfg, trace=tr)
    f = O.to_f64
    H, dh, base = cfg.H, cfg.dh, 10000.0
    q_idx = tr["q_idx"].numpy()

    # draft pass, layers 0 and L // 2
    for l, d in tr["draft"].items():
        K2, V2, ref = O.fused_step(f(d["x"]), q_idx, f(tr["W"][l]), base, f(d["k_in"]),
                                   f(d["v_in"]), H, dh, "bf16")
        assert_close(f(d["out"]), ref, "bf16", f"draft output, layer {l}")
        check_cache_update(d["k_out"], d["k_in"], K2, q_idx, "bf16", f"k_cache layer {l}")
        check_cache_update(d["v_out"], d["v_in"], V2, q_idx, "bf16", f"v_cache layer {l}")

    # attention masses and the tracked set (middle layer)
    t = tr["track"]
    dm = tr["draft"][t["layer"]]
    a_ref = O.attention_mass(f(dm["x"]), q_idx, f(tr["W"][t["layer"]]), base, f(dm["k_out"]),
                             H, dh, tr["q_masked"].numpy())
    cand = t["candidate"].numpy()
    track, mass = t["track"].numpy(), t["mass"].numpy()
    K_sel = track.shape[1]
    check_track(track, mass, a_ref, cand, K_sel, "bf16")
    np.testing.assert_array_equal(track, O.track_select(mass.astype(np.float64), cand, K_sel))

    # epsilon split of the masked rows
    sp = tr["split"]
    kind = sp["kind"].numpy()
    ref_s = O.accept(sp["logits"].numpy().astype(np.float64), kind, None, None, cfg.eps, cfg.gamma)
    B, R1 = kind.shape
    amb_s = check_accept((sp["top1"].numpy(), sp["conf"].numpy(), sp["flags"].numpy(),
                          np.zeros(B, np.int64)), ref_s, kind, np.zeros((B, R1), np.int64),
                         cfg.eps, cfg.gamma)

    # verify pass, layer 0, and the gamma acceptance
    assert tr["sets"]["n_s"] > 0, "the seed must leave exploratory rows"
    v = tr["verify"]
    K2, V2, KS, VS, ref_v = O.verify_step(f(v["x_rows"]), v["pos"].numpy(), v["view"].numpy(),
                                          v["rank"].numpy(), f(tr["W"][0]), base, f(v["k_in"]),
                                          f(v["v_in"]), f(v["ks_in"]), f(v["vs_in"]), H, dh,
                                          "bf16", cfg.causal_cross)
    assert_close(f(v["out"]), ref_v, "bf16", "verify output, layer 0")
    view, pos = v["view"].numpy(), v["pos"].numpy()
    for b in range(B):
        wr = pos[b][view[b] != 2]
        check_cache_update(v["k_out"][b:b + 1], v["k_in"][b:b + 1], K2[b:b + 1], wr[None], "bf16",
                           "verify k_cache")
        check_cache_update(v["v_out"][b:b + 1], v["v_in"][b:b + 1], V2[b:b + 1], wr[None], "bf16",
                           "verify v_cache")
        n_side = int((view[b] == 2).sum())
        assert_close(f(v["ks_out"][b][:, :n_side]), KS[b][:, :n_side], "bf16", "k side")
        assert_close(f(v["vs_out"][b][:, :n_side]), VS[b][:, :n_side], "bf16", "v side")
    g = tr["gamma"]
    kind_v, rank_v = g["kind"].numpy(), g["rank"].numpy()
    ref_g = O.accept(g["logits"].numpy().astype(np.float64), kind_v, g["ref_tok"].numpy(), rank_v,
                     cfg.eps, cfg.gamma)
    amb_g = check_accept((g["top1"].numpy(), g["conf"].numpy(), g["flags"].numpy(),
                          g["n_accept"].numpy()), ref_g, kind_v, rank_v, cfg.eps, cfg.gamma)

    # the sets the step ends with, from the oracle's decisions and the loop's policy
    st = tr["sets"]
    if amb_s == 0 and amb_g == 0 and not st["progress_forced"].any():
        front = tr["front"].numpy()
        valid = tr["q_masked"].numpy()[:, cfg.beta_t:] != 0
        newly = np.zeros_like(st["newly"].numpy())
        s_pos = g["s_pos"].numpy()
        for b in range(B):
            newly[b, front[b][((ref_s[2][b] & O.FLAG_COMMIT) != 0) & valid[b]]] = True
            newly[b, s_pos[b][(ref_g[2][b] & O.FLAG_ACCEPT) != 0]] = True
        newly &= ~tr["decoded_before"].numpy()
        np.testing.assert_array_equal(st["newly"].numpy(), newly)
        np.testing.assert_array_equal(st["decoded"].numpy(), tr["decoded_before"].numpy() | newly)
    T_next = DL.next_tracked(torch.from_numpy(track.astype(np.int32)), st["decoded"], cfg.beta_t)
    np.testing.assert_array_equal(st["T_next"].numpy(), T_next.numpy())
