"""Gated DeltaNet recurrence on B200 (sm_100a): prefill, state-pool decode and the
causal conv1d that feeds them.

The compute lives in libgdn.so (hand-written CUDA, C ABI declared in
include/gdn.h); this package is its thin Python binding plus the seeded
synthetic workloads used by the tests and the benchmark.
"""
from ._binding import (  # noqa: F401
    GDN_BF16, GDN_DECODE_QK_L2NORM, GDN_DEV_BAD_SLOT, GDN_DISABLE_STATE_UPDATE, GDN_ERR_ALIAS,
    GDN_ERR_ALIGN, GDN_ERR_CUDA, GDN_ERR_DTYPE, GDN_ERR_NULL, GDN_ERR_SHAPE,
    GDN_ERR_UNSUPPORTED, GDN_F32, GDN_OK, GDN_PREFILL_SEQUENTIAL, EXPORTED, LIB_PATH, GdnError,
    GDN_F16, gdn_conv1d, gdn_decode, gdn_prefill, lib, prefill_uses_chunked, status_string,
    CHECKED_LIB_PATH, GDN_DEV_BOUNDS, GDN_DEV_TEST_STALL, GDN_DEV_TIMEOUT, use_library,
    GDN_DECAY_PER_KEY,
)

__all__ = ["gdn_prefill", "gdn_decode", "gdn_conv1d", "GdnError", "lib", "status_string"]
