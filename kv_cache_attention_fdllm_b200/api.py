"""Python binding of the fdllm C ABI: argument marshalling only.

Each function has the name of the C entry point it calls (include/fdllm.h),
takes torch CUDA tensors, checks their dtype, shape, device and contiguity,
passes raw pointers and the current CUDA stream, and raises FdllmError on a
non-OK status.  The library launches on the current CUDA device, so the tensors
and the stream must be on it (a ValueError otherwise).  Every step of the
computation runs in the CUDA library.
"""
from __future__ import annotations

import ctypes

import torch

from ._native import lib

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_BAD_INDEX, ERR_TIMEOUT, ERR_WORKSPACE = range(7)
FLAG_COMMIT, FLAG_ACCEPT, FLAG_PASS = 1, 2, 4
_DT = {torch.float32: 0, torch.bfloat16: 1}


class FdllmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().fdllm_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


def _check(st: int, where: str):
    if st != OK:
        raise FdllmError(st, where)


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream, device):
    """The stream handle to launch on.  The library launches on the current CUDA
    device, so the tensors (on `device`) and the stream must both be on it."""
    if device.type != "cuda":
        raise ValueError(f"the tensors are on {device}, not on a CUDA device")
    cur = torch.cuda.current_device()
    if device.index != cur:
        raise ValueError(f"the tensors are on {device}, but the current CUDA device is "
                         f"cuda:{cur} (use torch.cuda.set_device)")
    s = torch.cuda.current_stream(device) if stream is None else stream
    if s.device != device:
        raise ValueError(f"the stream is on {s.device}, the tensors on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _dtype_code(t):
    if t.dtype not in _DT:
        raise ValueError(f"unsupported storage dtype {t.dtype}")
    return _DT[t.dtype]


# ---------------------------------------------------------------- workspace sizes

def fdllm_fused_step_workspace_bytes(B, N, D, H, dh, nq, dtype) -> int:
    return int(lib().fdllm_fused_step_workspace_bytes(B, N, D, H, dh, nq, _DT.get(dtype, dtype)))


def fdllm_verify_step_workspace_bytes(B, N, D, H, dh, R, S_max, dtype) -> int:
    return int(lib().fdllm_verify_step_workspace_bytes(B, N, D, H, dh, R, S_max,
                                                       _DT.get(dtype, dtype)))


def fdllm_accept_workspace_bytes(B, R, V) -> int:
    return int(lib().fdllm_accept_workspace_bytes(B, R, V))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled workspace of nbytes (the library requires zeros before first use)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- fused step

def _fused_shapes(x, q_idx, w_qkv, k_cache):
    B, N, D = x.shape
    nq = q_idx.shape[1]
    H, dh = k_cache.shape[1], k_cache.shape[3]
    return B, N, D, H, dh, nq


def _check_fused(x, q_idx, w_qkv, k_cache, v_cache):
    _need(x, "x")
    B, N, D, H, dh, nq = _fused_shapes(x, q_idx, w_qkv, k_cache)
    dt, dev = x.dtype, x.device
    _need(q_idx, "q_idx", torch.int32, (B, nq), dev)
    _need(w_qkv, "w_qkv", dt, (3 * H * dh, D), dev)
    _need(k_cache, "k_cache", dt, (B, H, N, dh), dev)
    _need(v_cache, "v_cache", dt, (B, H, N, dh), dev)
    return B, N, D, H, dh, nq


def fdllm_fused_step(x, q_idx, w_qkv, k_cache, v_cache, out, workspace, rope_base=10000.0,
                     stream=None):
    """One fused KV-cache step (see include/fdllm.h); k_cache/v_cache are updated in place."""
    B, N, D, H, dh, nq = _check_fused(x, q_idx, w_qkv, k_cache, v_cache)
    _need(out, "out", x.dtype, (B, nq, H * dh), x.device)
    _need(workspace, "workspace", torch.uint8, None, x.device)
    st = lib().fdllm_fused_step(B, N, D, H, dh, nq, _dtype_code(x), _p(x), _p(q_idx), _p(w_qkv),
                                float(rope_base), _p(k_cache), _p(v_cache), _p(out),
                                _p(workspace), workspace.numel(), _stream(stream, x.device))
    _check(st, "fdllm_fused_step")
    return out


def fdllm_fused_step_rows(x_rows, q_idx, w_qkv, k_cache, v_cache, out, workspace,
                          rope_base=10000.0, stream=None):
    """fdllm_fused_step with the rows x[Q] given packed, x_rows [B, nq, D]."""
    _need(x_rows, "x_rows")
    B, nq, D = x_rows.shape
    _need(k_cache, "k_cache")
    H, N, dh = k_cache.shape[1], k_cache.shape[2], k_cache.shape[3]
    dt, dev = x_rows.dtype, x_rows.device
    _need(q_idx, "q_idx", torch.int32, (B, nq), dev)
    _need(w_qkv, "w_qkv", dt, (3 * H * dh, D), dev)
    _need(k_cache, "k_cache", dt, (B, H, N, dh), dev)
    _need(v_cache, "v_cache", dt, (B, H, N, dh), dev)
    _need(out, "out", dt, (B, nq, H * dh), dev)
    _need(workspace, "workspace", torch.uint8, None, dev)
    st = lib().fdllm_fused_step_rows(B, N, D, H, dh, nq, _dtype_code(x_rows), _p(x_rows),
                                     _p(q_idx), _p(w_qkv), float(rope_base), _p(k_cache),
                                     _p(v_cache), _p(out), _p(workspace), workspace.numel(),
                                     _stream(stream, dev))
    _check(st, "fdllm_fused_step_rows")
    return out


def fdllm_qkv_rope_scatter(x, q_idx, w_qkv, k_cache, v_cache, q_out, workspace,
                           rope_base=10000.0, stream=None):
    B, N, D, H, dh, nq = _check_fused(x, q_idx, w_qkv, k_cache, v_cache)
    _need(q_out, "q_out", x.dtype, (B, nq, H, dh), x.device)
    _need(workspace, "workspace", torch.uint8, None, x.device)
    st = lib().fdllm_qkv_rope_scatter(B, N, D, H, dh, nq, _dtype_code(x), _p(x), _p(q_idx),
                                      _p(w_qkv), float(rope_base), _p(k_cache), _p(v_cache),
                                      _p(q_out), _p(workspace), workspace.numel(),
                                      _stream(stream, x.device))
    _check(st, "fdllm_qkv_rope_scatter")
    return q_out


def fdllm_attend(q, k_cache, v_cache, out, workspace, stream=None):
    _need(q, "q")
    B, nq, H, dh = q.shape
    N = k_cache.shape[2]
    _need(k_cache, "k_cache", q.dtype, (B, H, N, dh), q.device)
    _need(v_cache, "v_cache", q.dtype, (B, H, N, dh), q.device)
    _need(out, "out", q.dtype, (B, nq, H * dh), q.device)
    _need(workspace, "workspace", torch.uint8, None, q.device)
    st = lib().fdllm_attend(B, N, H, dh, nq, _dtype_code(q), _p(q), _p(k_cache), _p(v_cache),
                            _p(out), _p(workspace), workspace.numel(), _stream(stream, q.device))
    _check(st, "fdllm_attend")
    return out


# ---------------------------------------------------------------- verify pass

def _check_verify(x_rows, pos, view, w_qkv, k_cache, v_cache, k_side, v_side):
    _need(x_rows, "x_rows")
    B, R, D = x_rows.shape
    H, N, dh = k_cache.shape[1], k_cache.shape[2], k_cache.shape[3]
    dt, dev = x_rows.dtype, x_rows.device
    _need(pos, "pos", torch.int32, (B, R), dev)
    _need(view, "view", torch.int8, (B, R), dev)
    _need(w_qkv, "w_qkv", dt, (3 * H * dh, D), dev)
    _need(k_cache, "k_cache", dt, (B, H, N, dh), dev)
    _need(v_cache, "v_cache", dt, (B, H, N, dh), dev)
    S_max = k_side.shape[2]
    _need(k_side, "k_side", dt, (B, H, S_max, dh), dev)
    _need(v_side, "v_side", dt, (B, H, S_max, dh), dev)
    return B, N, D, H, dh, R, S_max


def fdllm_verify_step(x_rows, pos, view, rank, w_qkv, k_cache, v_cache, k_side, v_side, out,
                      workspace, rope_base=10000.0, causal_cross=False, stream=None):
    """One Flash-Verify pass (see include/fdllm.h); caches and side buffers updated in place."""
    B, N, D, H, dh, R, S_max = _check_verify(x_rows, pos, view, w_qkv, k_cache, v_cache, k_side,
                                             v_side)
    _need(rank, "rank", torch.int32, (B, R), x_rows.device)
    _need(out, "out", x_rows.dtype, (B, R, H * dh), x_rows.device)
    _need(workspace, "workspace", torch.uint8, None, x_rows.device)
    st = lib().fdllm_verify_step(B, N, D, H, dh, R, S_max, _dtype_code(x_rows), _p(x_rows),
                                 _p(pos), _p(view), _p(rank), _p(w_qkv), float(rope_base),
                                 _p(k_cache), _p(v_cache), _p(k_side), _p(v_side), _p(out),
                                 int(bool(causal_cross)), _p(workspace), workspace.numel(),
                                 _stream(stream, x_rows.device))
    _check(st, "fdllm_verify_step")
    return out


def fdllm_verify_qkv_rope_scatter(x_rows, pos, view, w_qkv, k_cache, v_cache, k_side, v_side,
                                  q_out, workspace, rope_base=10000.0, stream=None):
    B, N, D, H, dh, R, S_max = _check_verify(x_rows, pos, view, w_qkv, k_cache, v_cache, k_side,
                                             v_side)
    _need(q_out, "q_out", x_rows.dtype, (B, R, H, dh), x_rows.device)
    _need(workspace, "workspace", torch.uint8, None, x_rows.device)
    st = lib().fdllm_verify_qkv_rope_scatter(B, N, D, H, dh, R, S_max, _dtype_code(x_rows),
                                             _p(x_rows), _p(pos), _p(view), _p(w_qkv),
                                             float(rope_base), _p(k_cache), _p(v_cache),
                                             _p(k_side), _p(v_side), _p(q_out), _p(workspace),
                                             workspace.numel(), _stream(stream, x_rows.device))
    _check(st, "fdllm_verify_qkv_rope_scatter")
    return q_out


def fdllm_verify_attend(q, pos, view, rank, k_cache, v_cache, k_side, v_side, out, workspace,
                        causal_cross=False, stream=None):
    _need(q, "q")
    B, R, H, dh = q.shape
    N = k_cache.shape[2]
    S_max = k_side.shape[2]
    dev, dt = q.device, q.dtype
    _need(pos, "pos", torch.int32, (B, R), dev)
    _need(view, "view", torch.int8, (B, R), dev)
    _need(rank, "rank", torch.int32, (B, R), dev)
    _need(k_cache, "k_cache", dt, (B, H, N, dh), dev)
    _need(v_cache, "v_cache", dt, (B, H, N, dh), dev)
    _need(k_side, "k_side", dt, (B, H, S_max, dh), dev)
    _need(v_side, "v_side", dt, (B, H, S_max, dh), dev)
    _need(out, "out", dt, (B, R, H * dh), dev)
    _need(workspace, "workspace", torch.uint8, None, dev)
    st = lib().fdllm_verify_attend(B, N, H, dh, R, S_max, _dtype_code(q), _p(q), _p(pos),
                                   _p(view), _p(rank), _p(k_cache), _p(v_cache), _p(k_side),
                                   _p(v_side), _p(out), int(bool(causal_cross)), _p(workspace),
                                   workspace.numel(), _stream(stream, dev))
    _check(st, "fdllm_verify_attend")
    return out


# ---------------------------------------------------------------- acceptance

def fdllm_track_select(q_masked, candidate, k_cache, track, workspace, mass=None, dtype=None,
                       stream=None):
    """The next tracked set from the last fused step on `workspace` (see include/fdllm.h).

    q_masked int8 [B, nq], candidate int8 [B, N], k_cache [B, H, N, dh] as the
    step left it, track int32 [B, beta_t] (out), mass float32 [B, N] (out, optional)."""
    _need(q_masked, "q_masked", torch.int8)
    B, nq = q_masked.shape
    _need(k_cache, "k_cache")
    _, H, N, dh = k_cache.shape
    dev = k_cache.device
    _need(q_masked, "q_masked", torch.int8, (B, nq), dev)
    _need(candidate, "candidate", torch.int8, (B, N), dev)
    _need(track, "track", torch.int32, None, dev)
    if track.dim() != 2 or track.shape[0] != B:
        raise ValueError(f"track must be [B, beta_t] with B={B}, got {tuple(track.shape)}")
    if mass is not None:
        _need(mass, "mass", torch.float32, (B, N), dev)
    _need(workspace, "workspace", torch.uint8, None, dev)
    st = lib().fdllm_track_select(B, N, H, dh, nq, _dtype_code(k_cache), _p(q_masked),
                                  _p(candidate), _p(k_cache), track.shape[1], _p(track), _p(mass),
                                  _p(workspace), workspace.numel(), _stream(stream, dev))
    _check(st, "fdllm_track_select")
    return track, mass


def fdllm_accept(logits, kind, ref_tok, rank, top1, conf, flags, n_accept, workspace, eps=0.9,
                 gamma=0.8, stream=None):
    """Top-1, confidence, epsilon split and gamma prefix acceptance (see include/fdllm.h)."""
    _need(logits, "logits", torch.float32)
    B, R, V = logits.shape
    dev = logits.device
    _need(kind, "kind", torch.int8, (B, R), dev)
    if ref_tok is not None:
        _need(ref_tok, "ref_tok", torch.int32, (B, R), dev)
    if rank is not None:
        _need(rank, "rank", torch.int32, (B, R), dev)
    _need(top1, "top1", torch.int32, (B, R), dev)
    _need(conf, "conf", torch.float32, (B, R), dev)
    _need(flags, "flags", torch.uint8, (B, R), dev)
    _need(n_accept, "n_accept", torch.int32, (B,), dev)
    _need(workspace, "workspace", torch.uint8, None, dev)
    st = lib().fdllm_accept(B, R, V, _p(logits), _p(kind), _p(ref_tok), _p(rank), float(eps),
                            float(gamma), _p(top1), _p(conf), _p(flags), _p(n_accept),
                            _p(workspace), workspace.numel(), _stream(stream, dev))
    _check(st, "fdllm_accept")
    return top1, conf, flags, n_accept


def fdllm_accept_noalloc(logits, kind, ref_tok, rank, top1, conf, flags, n_accept, eps=0.9,
                         gamma=0.8, stream=None):
    """fdllm_accept without a workspace, for callers that cannot allocate device
    memory where they call the library (see include/fdllm.h): the scratch is a
    fixed device array inside the library, shared by every call on a device."""
    _need(logits, "logits", torch.float32)
    B, R, V = logits.shape
    dev = logits.device
    _need(kind, "kind", torch.int8, (B, R), dev)
    if ref_tok is not None:
        _need(ref_tok, "ref_tok", torch.int32, (B, R), dev)
    if rank is not None:
        _need(rank, "rank", torch.int32, (B, R), dev)
    _need(top1, "top1", torch.int32, (B, R), dev)
    _need(conf, "conf", torch.float32, (B, R), dev)
    _need(flags, "flags", torch.uint8, (B, R), dev)
    _need(n_accept, "n_accept", torch.int32, (B,), dev)
    st = lib().fdllm_accept_noalloc(B, R, V, _p(logits), _p(kind), _p(ref_tok), _p(rank),
                                    float(eps), float(gamma), _p(top1), _p(conf), _p(flags),
                                    _p(n_accept), _stream(stream, dev))
    _check(st, "fdllm_accept_noalloc")
    return top1, conf, flags, n_accept


SPLIT_STREAM_K, SPLIT_WHOLE_ITEMS, SPLIT_CLUSTERS = 1, 2, 3


def fdllm_attention_split(B, N, H, dh, rows, S_max=0, verify=False):
    """(split, cluster_size): how the bf16 attention spreads these shapes over the
    current device (SPLIT_STREAM_K, SPLIT_WHOLE_ITEMS or SPLIT_CLUSTERS; -1 if
    it does not run them).  A diagnostic: launches nothing."""
    cs = ctypes.c_int(0)
    mode = lib().fdllm_attention_split(B, N, H, dh, rows, S_max, int(bool(verify)),
                                       ctypes.byref(cs))
    return int(mode), int(cs.value)


def fdllm_bounded_wait_selftest(limit_ns, workspace, stream=None):
    """Runs the kernels' bounded mbarrier wait against a barrier nothing completes
    (see include/fdllm.h).  Returns the four result words (first wait completed,
    its ns, second wait completed, its ns) after synchronising the stream; the
    status word is left for fdllm_get_status."""
    _need(workspace, "workspace", torch.uint8, None, None)
    st = lib().fdllm_bounded_wait_selftest(int(limit_ns), _p(workspace), workspace.numel(),
                                           _stream(stream, workspace.device))
    _check(st, "fdllm_bounded_wait_selftest")
    torch.cuda.current_stream(workspace.device).synchronize() if stream is None else \
        stream.synchronize()
    return [int(v) for v in workspace[256:288].view(torch.int64).cpu().tolist()]


def fdllm_get_status(workspace, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status word."""
    return int(lib().fdllm_get_status(_p(workspace), _stream(stream, workspace.device)))
