"""B200-native STCA forward: stacked target cross attention over jagged user
histories with request-level batching.  The computation runs in libstca.so
(hand-written CUDA for sm_100a, C ABI in include/stca.h); this package is its
Python binding."""
from .stca import (  # noqa: F401
    EXPORTS,
    LIB_PATH,
    STCA_BF16,
    STCA_F32,
    STCA_OPT_ATTN_PATH,
    STCA_OPT_ENCODE_PATH,
    STCA_OPT_LAUNCHES,
    STCA_OPT_SPLIT_KEYS,
    STCA_OPT_STEP_PATH,
    STCA_OPT_TIMING,
    Stca,
    StcaError,
    stca_destroy,
    stca_device_status,
    stca_encode,
    stca_forward,
    stca_forward_static,
    stca_get_encoded,
    stca_get_option,
    stca_head,
    stca_kernel_times,
    stca_init,
    stca_last_error,
    stca_plan_attention,
    stca_run_host,
    stca_set_option,
    stca_validate_offsets,
)
