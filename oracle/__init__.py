"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE. Only the tests, the package smoke check and the bench's
CPU-baseline / reference legs may import it. The library's own path never
touches it, and it shares no code with the CUDA kernels or their bindings.

Parity status of each function is stated in ``attention_ref``'s header.
"""
from .attention_ref import (  # noqa: F401
    attention_rows,
    bf16_bits_to_f64,
    combine_partials,
    gather_paged,
    ref_attention,
    ref_decode_paged,
    ref_prefill_paged,
    softmax_probs,
)
from .brute import brute_attention  # noqa: F401
