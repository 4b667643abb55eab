"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
function include/fdllm.h declares, and rejects bad arguments before touching the
device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fdllm.h")


@pytest.fixture(scope="module")
def native():
    import __graft_entry__
    __graft_entry__.build()
    from kv_cache_attention_fdllm_b200 import _native
    return _native


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(fdllm_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_three_operations():
    names = declared_functions()
    for n in ("fdllm_fused_step", "fdllm_verify_step", "fdllm_accept", "fdllm_get_status"):
        assert n in names


def test_every_declared_symbol_is_exported(native):
    lib = ctypes.CDLL(native.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    # and the binding declares a signature for each of them
    assert sorted(native.SIGNATURES) == declared_functions()


def test_status_strings_and_version(native):
    lib = native.lib()
    assert lib.fdllm_version() >= 100
    for s in range(7):
        assert lib.fdllm_status_string(s)
    assert lib.fdllm_status_string(99) == b"unknown status"


def test_workspace_sizes(native):
    lib = native.lib()
    assert lib.fdllm_fused_step_workspace_bytes(1, 1024, 4096, 32, 128, 32, 1) > 0
    assert lib.fdllm_fused_step_workspace_bytes(1, 1024, 4096, 32, 96, 32, 1) == 0   # dh 96
    assert lib.fdllm_fused_step_workspace_bytes(1, 1024, 4000, 32, 128, 32, 1) == 0  # D % 64
    assert lib.fdllm_fused_step_workspace_bytes(1, 1024, 4000, 32, 128, 32, 0) > 0   # fp32 ok
    assert lib.fdllm_fused_step_workspace_bytes(1, 1024, 4096, 32, 128, 32, 7) == 0  # dtype
    assert lib.fdllm_verify_step_workspace_bytes(8, 2048, 4096, 32, 128, 40, 16, 1) > 0
    assert lib.fdllm_accept_workspace_bytes(8, 40, 126464) > 0
    assert lib.fdllm_accept_workspace_bytes(8, 40, 0) == 0


FAKE = ctypes.c_void_p(1 << 20)  # an aligned address that is never dereferenced


def test_workspace_sizes_grow_with_rows(native):
    """A workspace sized for the most rows serves every smaller row count (the
    decode loop sizes one verify workspace for its largest pass)."""
    lib = native.lib()
    for dt in (0, 1):
        prev = 0
        for R in range(1, 513):
            w = lib.fdllm_verify_step_workspace_bytes(8, 1024, 4096, 32, 128, R, 64, dt)
            assert w >= prev, (dt, R, w, prev)
            prev = w
        prev = 0
        for nq in range(1, 300):
            w = lib.fdllm_fused_step_workspace_bytes(8, 1024, 4096, 32, 128, nq, dt)
            assert w >= prev, (dt, nq, w, prev)
            prev = w


def test_bad_arguments_are_rejected_on_the_host(native):
    lib = native.lib()
    big = 1 << 40
    f = lib.fdllm_fused_step
    args = lambda dh=128, D=4096, dtype=1, ws=FAKE, wsb=big, x=FAKE, base=10000.0: (
        1, 1024, D, 32, dh, 32, dtype, x, FAKE, FAKE, base, FAKE, FAKE, FAKE, ws, wsb, None)
    assert f(*args(dh=96)) == 2                      # unsupported head size
    assert f(*args(D=100)) == 2                      # D not a multiple of 64 for bf16
    assert f(*args(dtype=5)) == 2
    assert f(*args(base=0.0)) == 1                   # rope base must be positive
    assert f(*args(ws=None)) == 6                    # no workspace
    assert f(*args(ws=ctypes.c_void_p((1 << 20) + 16))) == 6   # misaligned workspace
    assert f(*args(wsb=10)) == 6                     # too small
    assert f(*args(x=ctypes.c_void_p((1 << 20) + 2))) == 1     # misaligned tensor
    assert f(*args(x=None)) == 1                     # null tensor
    # B = 0 is a no-op that succeeds without touching the device
    assert f(0, 1024, 4096, 32, 128, 32, 1, None, None, None, 10000.0, None, None, None, FAKE,
             big, None) == 0
    v = lib.fdllm_verify_step
    assert v(1, 100, 128, 2, 128, 5000, 4, 1, FAKE, FAKE, FAKE, FAKE, FAKE, 10000.0, FAKE, FAKE,
             FAKE, FAKE, FAKE, 0, FAKE, big, None) == 2       # too many verify rows
    assert v(1, 100, 128, 2, 128, 5, 4, 1, FAKE, FAKE, FAKE, FAKE, FAKE, 10000.0, FAKE, FAKE,
             FAKE, FAKE, FAKE, 3, FAKE, big, None) == 1       # causal_cross must be 0/1
    a = lib.fdllm_accept
    assert a(1, 3, 0, FAKE, FAKE, None, None, 0.9, 0.8, FAKE, FAKE, FAKE, FAKE, FAKE, big,
             None) == 1                                       # V = 0
    assert a(1, 3, 3, FAKE, FAKE, None, None, 0.9, 0.8, FAKE, FAKE, FAKE, FAKE, FAKE, 0,
             None) == 6                                       # workspace too small


def test_track_select_rejects_bad_arguments_on_the_host(native):
    lib = native.lib()
    big = 1 << 40
    t = lib.fdllm_track_select
    args = lambda beta=80, dh=128, ws=FAKE, wsb=big, qm=FAKE, mass=None: (
        1, 1024, 32, dh, 32, 1, qm, FAKE, FAKE, beta, FAKE, mass, ws, wsb, None)
    assert t(*args(beta=0)) == 2                     # beta_t out of range
    assert t(*args(beta=1025)) == 2
    assert t(*args(dh=96)) == 2                      # unsupported head size
    assert t(*args(ws=None)) == 6                    # no workspace
    assert t(*args(wsb=10)) == 6                     # smaller than the fused step's
    assert t(*args(qm=None)) == 1                    # null tensor
    assert t(*args(mass=ctypes.c_void_p((1 << 20) + 4))) == 1   # misaligned optional output
    # the workspace a fused step of the same shape gets is large enough
    need = lib.fdllm_fused_step_workspace_bytes(1, 1024, 4096, 32, 128, 32, 1)
    assert need > 0
    assert t(0, 1024, 32, 128, 32, 1, None, None, None, 80, None, None, FAKE, need, None) == 0


def test_binding_launches_only_on_the_tensors_device(native, monkeypatch):
    """The library launches on the current CUDA device: the binding refuses
    tensors on another device, and a stream on another device (faked devices:
    no GPU is needed)."""
    import torch
    from kv_cache_attention_fdllm_b200 import api

    class FakeStream:
        def __init__(self, index, handle):
            self.device = torch.device("cuda", index)
            self.cuda_stream = handle

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: FakeStream(1, 0x1234))
    assert api._stream(None, torch.device("cuda", 1)).value == 0x1234
    assert api._stream(FakeStream(1, 0x99), torch.device("cuda", 1)).value == 0x99
    with pytest.raises(ValueError, match="current CUDA device"):
        api._stream(None, torch.device("cuda", 0))
    with pytest.raises(ValueError, match="the stream is on"):
        api._stream(FakeStream(0, 0x99), torch.device("cuda", 1))
    with pytest.raises(ValueError, match="not on a CUDA device"):
        api._stream(None, torch.device("cpu"))
