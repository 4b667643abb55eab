"""The byte counts behind the benchmark's roofline fractions (CPU only).

The step's minimal bytes follow from the method's definition (W, the rows x[Q],
the untouched cache slots, the new k, v, the side slots, the output, the
logits).  They are compared with figures worked out independently from the
workload shapes: 117.96 MB (single sequence), 378.5 + 161.9 MB (verify pass and
acceptance), 370.15 MB (long context), 4429.2 MB (batch of 64).  The per-kernel
counts, which also hold the staged q and the attention's re-read of the slots
just written, are never smaller."""
import sys

import pytest

import workloads as W


@pytest.fixture(scope="module")
def bench():
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        import bench as B
    finally:
        sys.argv = argv
    return B


@pytest.mark.parametrize("name,mb", [("single_bf16", 117.96), ("verify_bf16", 378.5 + 161.9),
                                     ("long_bf16", 370.15), ("batch_bf16", 4429.2)])
def test_step_bytes_match_the_worked_figures(bench, name, mb):
    got = bench.step_bytes_min(W.CONFIGS[name]) / 1e6
    assert abs(got - mb) <= 0.05, (name, got, mb)


def test_kernel_bytes_bound_the_step_from_above(bench):
    for name in ("tiny_fp32", "single_bf16", "verify_bf16", "long_bf16", "batch_bf16"):
        cfg = W.CONFIGS[name]
        alg, _ = bench.algorithmic_bytes(cfg)
        assert sum(alg.values()) >= bench.step_bytes_min(cfg)


def test_traffic_record_is_used_only_for_the_captured_source(bench):
    """The ncu traffic of a kernel is reported only while its source still hashes to
    the capture's; unknown keys give None."""
    import hashlib
    import json
    import os
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for key, d in rec.items():
        src = os.path.join(bench.ROOT, d["source"])
        same = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] == d["source_sha256_16"]
        assert bench.traffic_for(key) == (d["bytes_per_launch"] if same else None)
    assert bench.traffic_for("no_such_workload:proj") is None
