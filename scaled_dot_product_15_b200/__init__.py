"""B200 (sm_100a) scaled dot-product attention.

``sdpa(query, key, value, ...)`` returns ``(out, lse)``: softmax(Q K^T * scale
+ mask) V and the per-row logsumexp; ``sdpa_backward(...)`` returns the input
gradients for an output gradient; ``attention(...)`` is the differentiable op
built from the two; ``sdpa_decode_paged(...)`` is decode attention over a
paged key/value cache.  Everything runs in the CUDA library built from ``csrc/``
(see include/sdpa15.h for the C ABI).
"""
from .api import (  # noqa: F401
    LIB_PATH,
    PreparedCall,
    SdpaError,
    attention,
    exported_symbols,
    last_launch_count,
    load_library,
    plan,
    sdpa,
    sdpa_backward,
    sdpa_decode_paged,
)
