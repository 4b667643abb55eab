"""fdllm_accept_noalloc: the acceptance call for callers that cannot allocate
device memory where they call the library (a plugin handed only its buffers, a
runtime whose memory is all reserved, a loop where cudaMalloc would stall).

It runs the same kernel as fdllm_accept, with the same split of each row, so
it must give the same bits on the same inputs, on two calls in a row (the
second call reuses the library's fixed scratch array, which still holds the
first call's partials).  A clean call leaves the array's counters at zero
itself; the call's own clearing of them guards only against an earlier launch
that was cut short, which these two calls do not exercise.  This file sorts
last so that a run stopping at the first failure has already run every other
test."""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def _outs(B, R):
    return (torch.empty((B, R), dtype=torch.int32, device="cuda"),
            torch.empty((B, R), dtype=torch.float32, device="cuda"),
            torch.empty((B, R), dtype=torch.uint8, device="cuda"),
            torch.empty((B,), dtype=torch.int32, device="cuda"))


def _compare(F, logits, kind, ref_tok, rank, eps, gamma):
    B, R, V = logits.shape
    ref = _outs(B, R)
    ws = F.alloc_workspace(F.fdllm_accept_workspace_bytes(B, R, V), "cuda")
    F.fdllm_accept(logits, kind, ref_tok, rank, *ref, ws, eps=eps, gamma=gamma)
    got = _outs(B, R)
    F.fdllm_accept_noalloc(logits, kind, ref_tok, rank, *got, eps=eps, gamma=gamma)
    torch.cuda.synchronize()
    assert torch.equal(got[0], ref[0])                                   # top1
    assert torch.equal(got[1], ref[1])                                   # conf, bit for bit
    assert torch.equal(got[2], ref[2]) and torch.equal(got[3], ref[3])   # flags, n_accept


def test_noalloc_matches_workspace_call_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_attention_fdllm_b200 as F
    # call 1: the verify configuration's logits (two sequences)
    a = W.accept_inputs(W.CONFIGS["verify_bf16"], seqs=[0, 1])
    _compare(F, a["logits"].cuda(), a["kind"].cuda(), a["ref_tok"].cuda(), a["rank"].cuda(),
             0.9, 0.8)
    # call 2: other shapes and kinds, with the array still holding call 1's contents
    B, R, V = 3, 7, 4097
    logits, tok = W.random_logits(B, R, V, seed=41)
    g = np.random.default_rng(41)
    kind = torch.from_numpy(g.integers(0, 3, (B, R)).astype(np.int8)).cuda()
    ref_tok = torch.from_numpy(np.where(g.random((B, R)) < 0.7, tok, (tok + 1) % V)
                               .astype(np.int32)).cuda()
    rank = torch.from_numpy(np.stack([g.permutation(R) for _ in range(B)]).astype(np.int32)).cuda()
    _compare(F, logits.cuda(), kind, ref_tok, rank, 0.6, 0.5)


def test_noalloc_rejects_calls_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_attention_fdllm_b200 as F
    B, R = 1, 300000   # B*R*20 bytes of scratch > FDLLM_ACCEPT_NOALLOC_SCRATCH_BYTES
    logits = torch.empty((B, R, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(F.FdllmError) as e:
        F.fdllm_accept_noalloc(logits, torch.zeros((B, R), dtype=torch.int8, device="cuda"),
                               None, None, *_outs(B, R))
    assert e.value.status == F.ERR_UNSUPPORTED
