"""fp64 CPU oracle of the Flash-dLLM fused KV-cache step (test infrastructure only).

Only `tests/`, `__graft_entry__.smoke()` and the benchmark's CPU-baseline and
reference legs may import this package.  The CUDA library never does.
"""
from .fdllm_oracle import (FLAG_ACCEPT, FLAG_COMMIT, FLAG_PASS, accept, attend,
                           attention_mass, bf16_bits, bf16_bits_to_f64, fused_step,
                           project_qkv, rope, round_bf16, round_to, to_f64,
                           track_select, verify_step, verify_visibility)

__all__ = ["FLAG_ACCEPT", "FLAG_COMMIT", "FLAG_PASS", "accept", "attend", "attention_mass",
           "bf16_bits", "bf16_bits_to_f64", "fused_step", "project_qkv", "rope",
           "round_bf16", "round_to", "to_f64", "track_select", "verify_step",
           "verify_visibility"]
