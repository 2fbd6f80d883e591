"""fp64 CPU oracle for the Cut Cross-Entropy hot path (test infrastructure only).

Only tests, the smoke check and the bench's CPU-baseline legs use this package;
the CUDA library never imports it.
"""
from .cce_oracle import (  # noqa: F401
    widen_bf16, as_f64, logits_rows, logsumexp_rows, forward, dlogits, backward,
    softmax_rows, dE_columns, full_pass, mean_loss, kahan_reference, kl_forward, kl_backward, SLICE_ROWS,
)
