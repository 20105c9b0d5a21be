"""B200 (sm_100a) scaled dot-product attention forward.

``sdpa(query, key, value, ...)`` returns ``(out, lse)``: softmax(Q K^T * scale
+ mask) V and the per-row logsumexp, computed by the CUDA library built from
``csrc/`` (see include/sdpa15.h for the C ABI).
"""
from .api import (  # noqa: F401
    LIB_PATH,
    PreparedCall,
    SdpaError,
    exported_symbols,
    last_launch_count,
    load_library,
    plan,
    sdpa,
)
