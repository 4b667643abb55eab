"""The oracle's pins catch plausible slips (CPU only).

Each mutant below plants one mistake in one oracle function: a dropped term, a
wrong sign, scale, axis or index, a transposed or swapped operand, a missed
rounding, or a wrong reading of the visibility, threshold or prefix rules.  The
mistake is a textual edit of the function's own source, compiled in the oracle
module's namespace and patched in for the duration of one test.  The pins of
`test_oracle_pins` then run against the mutated oracle, and at least one of them
must fail with an assertion.  Each edit must match its function's source exactly
once, so a mutant cannot silently stop applying when the oracle changes.
"""
import __future__
import inspect
import textwrap

import pytest

import oracle
import oracle.fdllm_oracle as M
import test_oracle_pins as P

# (id, function, text in its source, replacement)
MUTANTS = [
    # bfloat16 storage
    ("bf16_truncates", "round_bf16", "np.rint(x / ulp)", "np.trunc(x / ulp)"),
    ("bf16_ties_up", "round_bf16", "np.rint(x / ulp)", "np.floor(x / ulp + 0.5)"),
    ("bf16_nine_bits", "round_bf16", "np.maximum(e - 8, -133)", "np.maximum(e - 9, -133)"),
    ("bf16_via_float32", "round_bf16", "x = np.asarray(x, dtype=np.float64)",
     "x = np.asarray(x, dtype=np.float32).astype(np.float64)"),
    ("bf16_decode_shift", "bf16_bits_to_f64", "<< np.uint32(16)", "<< np.uint32(15)"),
    ("bf16_tensor_read_as_integers", "to_f64",
     "bf16_bits_to_f64(t.contiguous().view(dtype=_torch_int16()).numpy().view(np.uint16))",
     "t.contiguous().view(dtype=_torch_int16()).numpy().astype(np.float64)"),
    ("f32_not_rounded", "round_to",
     "np.asarray(x, np.float64).astype(np.float32).astype(np.float64)", "np.asarray(x, np.float64)"),
    # RoPE
    ("rope_theta_exponent", "rope", "base ** (-2.0 * j / dh)", "base ** (-1.0 * j / dh)"),
    ("rope_theta_from_one", "rope", "j = np.arange(half, dtype=np.float64)",
     "j = np.arange(1, half + 1, dtype=np.float64)"),
    ("rope_rotation_sign", "rope", "x1 * c - x2 * s, x1 * s + x2 * c",
     "x1 * c + x2 * s, -x1 * s + x2 * c"),
    ("rope_interleaved_pairs", "rope", "x1 = x[..., :half]\n    x2 = x[..., half:]",
     "x1 = x[..., 0::2]\n    x2 = x[..., 1::2]"),
    ("rope_position_plus_one", "rope", "np.asarray(pos, np.float64)[:, None]",
     "(np.asarray(pos, np.float64) + 1)[:, None]"),
    # QKV projection layout
    ("qkv_k_v_swapped", "project_qkv",
     "y[:, E:2 * E].reshape(n, H, dh),\n            y[:, 2 * E:].reshape(n, H, dh)",
     "y[:, 2 * E:].reshape(n, H, dh),\n            y[:, E:2 * E].reshape(n, H, dh)"),
    ("qkv_q_k_swapped", "project_qkv",
     "return (y[:, :E].reshape(n, H, dh), y[:, E:2 * E].reshape(n, H, dh),",
     "return (y[:, E:2 * E].reshape(n, H, dh), y[:, :E].reshape(n, H, dh),"),
    ("qkv_head_minor", "project_qkv", "y[:, :E].reshape(n, H, dh)",
     "y[:, :E].reshape(n, dh, H).transpose(0, 2, 1)"),
    # attention
    ("attend_no_scale", "attend", "(q @ K.T) / np.sqrt(dh)", "(q @ K.T)"),
    ("attend_scale_1_over_dh", "attend", "(q @ K.T) / np.sqrt(dh)", "(q @ K.T) / dh"),
    ("attend_softmax_over_queries", "attend", "p = p / p.sum(axis=1, keepdims=True)",
     "p = p / p.sum(axis=0, keepdims=True)"),
    ("attend_ignores_visibility", "attend", "s = np.where(visible, s, -np.inf)", "s = s"),
    # the fused step
    ("step_k_not_rotated", "fused_step", "k = rope(k, Q, rope_base)", "k = k"),
    ("step_q_not_rotated", "fused_step", "q = rope(q, Q, rope_base)", "q = q"),
    ("step_q_rotated_at_row", "fused_step", "q = rope(q, Q, rope_base)",
     "q = rope(q, np.arange(len(Q)), rope_base)"),
    ("step_k_not_rounded", "fused_step", "round_to(k, dtype)", "k"),
    ("step_v_not_rounded", "fused_step", "round_to(v, dtype)", "v"),
    ("step_v_into_k_cache", "fused_step", "K2[b][:, Q, :] = round_to(k, dtype)",
     "K2[b][:, Q, :] = round_to(v, dtype)"),
    ("step_attends_old_cache", "fused_step", "attend(q[:, h], K2[b, h], V2[b, h])",
     "attend(q[:, h], k_cache[b, h], v_cache[b, h])"),
    # Flash-Verify visibility and writes
    ("verify_mask_sees_drafts", "verify_visibility", "vis[r, dpos] = False",
     "vis[r, dpos] = True"),
    ("verify_mask_misses_side", "verify_visibility", "vis[r, n_cache_pos:] = True",
     "vis[r, n_cache_pos:] = False"),
    ("verify_draft_sees_side", "verify_visibility",
     "if view[r] in (0, 1):\n            vis[r, :n_cache_pos] = True",
     "if view[r] in (0, 1):\n            vis[r, :] = True"),
    ("verify_causal_own_draft", "verify_visibility", "drank < rank[r]", "drank <= rank[r]"),
    ("verify_causal_own_mask", "verify_visibility", "side_rank >= rank[r]",
     "side_rank > rank[r]"),
    ("verify_mask_view_into_cache", "verify_step",
     "in_cache = np.nonzero((vw == 0) | (vw == 1))[0]", "in_cache = np.arange(len(vw))"),
    ("verify_side_order_reversed", "verify_step", "for s, r in enumerate(mask_rows):",
     "for s, r in enumerate(mask_rows[::-1]):"),
    ("verify_k_not_rotated", "verify_step", "k = rope(k, P, rope_base)", "k = k"),
    # acceptance
    ("accept_strict_eps", "accept", "conf[b, r] >= eps", "conf[b, r] > eps"),
    ("accept_strict_gamma", "accept", "conf[b, r] >= gamma", "conf[b, r] > gamma"),
    ("accept_ties_to_last", "accept", "int(np.argmax(l))",
     "int(len(l) - 1 - np.argmax(l[::-1]))"),
    ("accept_conf_unshifted", "accept", "np.exp(l - m).sum()", "np.exp(l).sum()"),
    ("accept_prefix_by_row", "accept", "first_fail = min(first_fail, rank[b, r])",
     "first_fail = min(first_fail, r)"),
    ("accept_no_prefix_stop", "accept", "if kind[b, r] == 2 and rank[b, r] < first_fail:",
     "if kind[b, r] == 2 and flags[b, r] & FLAG_PASS:"),
    ("accept_prefix_takes_failure", "accept", "rank[b, r] < first_fail",
     "rank[b, r] <= first_fail"),
    ("accept_pass_ignores_draft", "accept", "top1[b, r] == ref_tok[b, r] and ", ""),
    # tracked-set selection
    ("mass_no_scale", "attention_mass", "(q[:, h] @ k_cache2[b, h].T) / np.sqrt(dh)",
     "(q[:, h] @ k_cache2[b, h].T)"),
    ("mass_softmax_over_rows", "attention_mass", "p = p / p.sum(axis=1, keepdims=True)",
     "p = p / p.sum(axis=0, keepdims=True)"),
    ("mass_counts_unmasked_rows", "attention_mass",
     "rows = np.nonzero(np.asarray(masked_row[b]) != 0)[0]", "rows = np.arange(nq)"),
    ("mass_q_not_rotated", "attention_mass", "q = rope(q, Q[rows], rope_base)", "q = q"),
    ("track_ties_to_higher_slot", "track_select", "key=lambda j: (-a[b, j], j)",
     "key=lambda j: (-a[b, j], -j)"),
    ("track_ascending_mass", "track_select", "key=lambda j: (-a[b, j], j)",
     "key=lambda j: (a[b, j], j)"),
    ("track_ignores_candidates", "track_select", "if candidate[b, j] != 0", "if True"),
    ("track_pads_with_zero", "track_select", "np.full((B, beta_t), -1,", "np.full((B, beta_t), 0,"),
]


def _pin_calls():
    """Every pin of test_oracle_pins, one call per parametrization."""
    calls = []
    for name, fn in vars(P).items():
        if not (name.startswith("test_") and callable(fn)):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn, ()))
            continue
        assert len(marks) == 1, name
        argnames, values = marks[0].args[:2]
        single = isinstance(argnames, str) and "," not in argnames
        for v in values:
            calls.append((f"{name}[{v}]", fn, (v,) if single else tuple(v)))
    return calls


def _failing_pins():
    failed = []
    for name, fn, args in _pin_calls():
        try:
            fn(*args)
        except AssertionError:
            failed.append(name)
    return failed


def _mutate(fname, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(M, fname)))
    assert src.count(old) == 1, f"{fname}: the planted edit must match exactly once"
    ns = dict(vars(M))
    code = compile(src.replace(old, new), f"<mutant of {fname}>", "exec",
                   flags=__future__.annotations.compiler_flag, dont_inherit=True)
    exec(code, ns)
    return ns[fname]


def test_pins_pass_on_the_oracle():
    assert _failing_pins() == []


@pytest.mark.parametrize("mid,fname,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(monkeypatch, mid, fname, old, new):
    fn = _mutate(fname, old, new)
    monkeypatch.setattr(M, fname, fn)        # calls from inside the oracle
    monkeypatch.setattr(oracle, fname, fn)   # calls through the package
    assert _failing_pins(), f"no pin catches the mutant {mid}"
