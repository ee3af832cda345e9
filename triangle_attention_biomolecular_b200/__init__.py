"""B200-native (sm_100a) triangle attention for AlphaFold3 / OpenFold3 Pairformers.

The computation lives in ``libtriattn.so`` (C ABI in ``include/tri_attn.h``);
this package is its thin Python binding plus seeded synthetic inputs.
Importing the package does not load the library; the first call does, and
raises if it is missing.
"""
from ._binding import (  # noqa: F401
    TRI_ATTN_BWD_NO_RESIDUAL,
    TriAttnError,
    tri_attn_abi_version,
    tri_attn_bwd,
    tri_attn_bwd_workspace_bytes,
    tri_attn_device_error,
    tri_attn_fwd,
    tri_attn_selftest_expire_wait,
    tri_attn_set_wait_limit_ns,
    tri_attn_strerror,
)
from .api import backward, forward, triangle_attention  # noqa: F401
