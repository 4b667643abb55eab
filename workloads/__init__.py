"""Seeded synthetic inputs for the fused KV-cache step, its verify pass and the
acceptance reduction.

This package produces inputs only: random draws, index sets and their rounding
to the storage dtype.  It holds none of the step's arithmetic, so both the CUDA
path and the CPU oracle can take their inputs from it.
"""
from .gen import (CONFIGS, fused_inputs, verify_inputs, accept_inputs,
                  query_positions, random_fused, random_logits, random_verify,
                  to_device)

__all__ = ["CONFIGS", "fused_inputs", "verify_inputs", "accept_inputs",
           "query_positions", "random_fused", "random_logits", "random_verify",
           "to_device"]
