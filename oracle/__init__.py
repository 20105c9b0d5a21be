"""Float64 CPU oracle for scaled dot-product attention (test infrastructure only).

Only tests, the smoke check and the benchmark's CPU-baseline legs may import
this package; the product path never does.
"""
from .sdpa_ref import default_scale, sdpa, sdpa_packed  # noqa: F401
from .sdpa_bwd_ref import attention_weights, sdpa_backward, sdpa_backward_packed  # noqa: F401
from .paged_ref import gather_pages, sdpa_decode_paged  # noqa: F401
