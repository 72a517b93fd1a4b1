"""B200-native KDA (Kimi Delta Attention): a CUDA library for sm_100a with a C ABI.

Entry points (see include/kda.h): ``forward`` (chunkwise prefill),
``forward_varlen`` / ``forward_varlen_raw`` / ``forward_varlen_gdn2`` (prefill over
packed sequences of different lengths), the same calls on host tensors go through the
host-buffer entry points,
``forward_scalar_gate`` / ``decode_step_scalar_gate`` (one retention factor per
head: Gated DeltaNet), ``forward_gdn2`` / ``decode_step_gdn2`` (decoupled erase
and write gates: GDN-2), ``forward_raw`` / ``decode_step_raw`` (input
preprocessing fused into the kernels: raw q and k, gate and beta logits),
``decode_tokens`` / ``state_copy`` (serving: several tokens per sequence over a
pool of state slots with per-token states for rollback; whole-state copies for
fork and rollback), ``forward_sequential`` (token-by-token schedule),
``decode_step`` (one token per sequence, state updated in place).
``set_schedule`` / ``schedule`` choose the prefill schedule (automatic: the tensor-core
chunk kernel where it applies, the column scan otherwise; or always chunkwise).  ``inputs``
draws the seeded synthetic workloads.  All arithmetic runs in
``libkda_b200.so``; build it with ``python -m gated_delta_rule_122_b200.build``.
"""
from .kda import (EXPORTED_SYMBOLS, KDAError, decode_step, decode_step_gdn2, decode_step_raw,
                  decode_step_scalar_gate, decode_tokens, forward, forward_gdn2, forward_raw,
                  forward_scalar_gate, forward_sequential, forward_varlen, forward_varlen_gdn2,
                  forward_varlen_raw, get_schedule, library, library_path, schedule, set_schedule,
                  selftest_bounded_wait, state_copy, status_string, version)

__all__ = ["forward", "forward_varlen", "forward_varlen_raw", "forward_varlen_gdn2", "forward_scalar_gate", "forward_gdn2", "forward_raw",
           "forward_sequential", "decode_step", "decode_step_scalar_gate", "decode_step_gdn2",
           "decode_step_raw", "decode_tokens", "state_copy", "selftest_bounded_wait", "set_schedule",
           "get_schedule", "schedule", "KDAError", "library",
           "library_path",
           "status_string", "version", "EXPORTED_SYMBOLS"]
