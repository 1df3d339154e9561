"""B200-native block top-k sparse decode attention over a paged KV cache.

The compute lives in ``libvt.so`` (hand-written sm_100a CUDA behind the C ABI of
``include/vt.h``); this package is its ctypes binding plus the seeded synthetic
workload generator.  The library is loaded on first use and a missing or broken
library raises ``VtError`` -- there is no CPU or PyTorch fallback.
"""
from .binding import (  # noqa: F401
    EXPORTS,
    PAGE_SIZE,
    PreparedCall,
    VT_DEV_BAD_LEN,
    VT_DEV_BAD_ORDER,
    VT_DEV_BAD_PAGE,
    VT_DEV_BAD_SEL,
    VT_DEV_TIMEOUT,
    VtError,
    fused_workspace,
    decode_workspace,
    load_library,
    prepare_build_centroids,
    prepare_sparse_decode_fused,
    prepare_sparse_decode_step,
    vt_abi_version,
    vt_build_centroids,
    vt_fused_workspace_size,
    vt_plan_requests,
    vt_select_pages,
    vt_select_pages_approx,
    vt_sparse_decode,
    vt_sparse_decode_fused,
    vt_sparse_decode_step,
    vt_sparse_decode_fused_static,
)
