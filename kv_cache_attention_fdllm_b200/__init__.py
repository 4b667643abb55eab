"""B200 (sm_100a) implementation of the Flash-dLLM fused KV-cache step.

The computation lives in libfdllm.so (hand-written CUDA behind the C ABI of
include/fdllm.h); this package only loads it and marshals torch tensors.
Importing the package fails when the library has not been built: there is no
CPU fallback.
"""
from ._native import LIB_PATH, lib

lib()  # fail loudly at import when the CUDA library is missing

from .api import (ERR_BAD_INDEX, ERR_CUDA, ERR_INVALID_ARG, ERR_TIMEOUT, ERR_UNSUPPORTED,  # noqa: E402
                  ERR_WORKSPACE, FLAG_ACCEPT, FLAG_COMMIT, FLAG_PASS, OK, FdllmError,
                  SPLIT_CLUSTERS, SPLIT_STREAM_K, SPLIT_WHOLE_ITEMS,
                  alloc_workspace, fdllm_accept, fdllm_accept_noalloc, fdllm_attention_split,
                  fdllm_bounded_wait_selftest,
                  fdllm_accept_workspace_bytes, fdllm_attend,
                  fdllm_fused_step, fdllm_fused_step_rows, fdllm_fused_step_workspace_bytes,
                  fdllm_get_status,
                  fdllm_qkv_rope_scatter, fdllm_verify_attend, fdllm_verify_qkv_rope_scatter,
                  fdllm_track_select, fdllm_verify_step, fdllm_verify_step_workspace_bytes)

from .shard import max_over_ranks, rank_sequences  # noqa: E402

__all__ = [n for n in dir() if n.startswith(("fdllm_", "FLAG_", "ERR_", "SPLIT_"))] + [
    "OK", "FdllmError", "alloc_workspace", "lib", "LIB_PATH", "max_over_ranks", "rank_sequences"]
