"""B200-native KDA (Kimi Delta Attention): a CUDA library for sm_100a with a C ABI.

Entry points (see include/kda.h): ``forward`` (chunkwise prefill),
``forward_varlen`` (prefill over packed sequences of different lengths),
``forward_scalar_gate`` / ``decode_step_scalar_gate`` (one retention factor per head:
Gated DeltaNet),
``forward_sequential`` (token-by-token schedule), ``decode_step`` (one token per
sequence, state updated in place).  ``inputs`` draws the seeded synthetic
workloads.  All arithmetic runs in ``libkda_b200.so``; build it with
``python -m gated_delta_rule_122_b200.build``.
"""
from .kda import (EXPORTED_SYMBOLS, KDAError, decode_step, decode_step_scalar_gate, forward,
                  forward_scalar_gate, forward_sequential, forward_varlen, library, library_path,
                  status_string, version)

__all__ = ["forward", "forward_varlen", "forward_scalar_gate", "forward_sequential", "decode_step",
           "decode_step_scalar_gate", "KDAError", "library", "library_path", "status_string",
           "version", "EXPORTED_SYMBOLS"]
