"""fp64 CPU oracle of the fused linear-head + KL-divergence loss.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use it.  It shares no code with the CUDA path.
"""
from .flkl_oracle import (REDUCTIONS, OracleError, ce_forward_backward, divisor, forward_backward,
                          forward_backward_loops, jsd_forward_backward, kl_terms,
                          log_softmax_rows, selective_logprob, selective_logprob_backward,
                          valid_rows)

__all__ = ["REDUCTIONS", "OracleError", "ce_forward_backward", "divisor", "forward_backward",
           "forward_backward_loops", "jsd_forward_backward", "kl_terms", "log_softmax_rows",
           "selective_logprob",
           "selective_logprob_backward", "valid_rows"]
