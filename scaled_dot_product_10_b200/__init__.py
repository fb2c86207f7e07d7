"""B200-native (sm_100a) fused scaled dot-product attention forward.

The compute path is a hand-written CUDA kernel behind a C ABI
(``include/attn_fwd.h``); :mod:`scaled_dot_product_10_b200.attn` is the thin
ctypes binding over it.  Importing this package does not load the CUDA
library; the first call does, and it fails loudly if the library is missing.
"""
from .attn import (  # noqa: F401
    ATTN_ERR_ALIGN, ATTN_ERR_CUDA, ATTN_ERR_INVALID, ATTN_ERR_TIMEOUT, ATTN_ERR_UNSUPPORTED,
    ATTN_OK, AttnError, attn_fwd, attn_fwd_host, attn_status, attn_strerror,
    host_workspace_bytes, library_path, load_library,
)
