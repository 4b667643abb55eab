"""The bounded wait every kernel uses on its mbarriers gives up cleanly.

fdllm_bounded_wait_selftest waits, with a short limit, on an mbarrier that
nothing completes (no copy or MMA is in flight, nothing faults): the wait must
end after about the limit with FDLLM_ERR_TIMEOUT in the status word, a second
wait in the same CTA must return at once, and the device must still run a full
step correctly afterwards."""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kv_cache_attention_fdllm_b200 as F
    return F


@pytest.mark.parametrize("limit_ms", [2, 20])
def test_bounded_wait_runs_out_and_returns(F, limit_ms):
    limit = limit_ms * 1_000_000
    ws = F.alloc_workspace(512, "cuda")
    done1, ns1, done2, ns2 = F.fdllm_bounded_wait_selftest(limit, ws)
    assert done1 == 0 and done2 == 0, "nothing completes the barrier"
    assert limit <= ns1 < limit + 50_000_000, f"first wait gave up after {ns1} ns"
    assert ns2 < min(limit, 5_000_000), f"the wait after the abort took {ns2} ns"
    assert F.fdllm_get_status(ws) == F.ERR_TIMEOUT
    assert F.fdllm_get_status(ws) == F.OK  # read and cleared


def test_device_still_runs_a_step_after_a_timeout(F):
    from test_gpu_fused import _check_fused
    ws = F.alloc_workspace(512, "cuda")
    F.fdllm_bounded_wait_selftest(1_000_000, ws)
    assert F.fdllm_get_status(ws) == F.ERR_TIMEOUT
    _check_fused(F, W.random_fused(2, 300, 128, 2, 128, nq=9, seed=71))


def test_limit_outside_range_is_rejected(F):
    ws = F.alloc_workspace(512, "cuda")
    for bad in (0, 999, 2_000_000_001):
        with pytest.raises(F.FdllmError) as e:
            F.fdllm_bounded_wait_selftest(bad, ws)
        assert e.value.status == F.ERR_INVALID_ARG
