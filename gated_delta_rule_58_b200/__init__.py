"""B200-native (sm_100a) gated delta rule library.

The compute lives in libgdn.so (C ABI in include/gdn.h); this package is its
Python binding plus the seeded input generators used by tests and benchmarks.

    from gated_delta_rule_58_b200 import gdn_decode, gdn_chunk_prefill
"""
from ._lib import (  # noqa: F401
    GDN_BF16, GDN_F32, GDN_OK, GDN_ERR_CUDA, GDN_ERR_DEVICE_DATA, GDN_ERR_INVALID_ARG,
    GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_DEVERR_BAD_CU_SEQLENS,
    GDN_DEVERR_SLOT_OUT_OF_RANGE, GDN_DEVERR_TIMEOUT, GDN_PREFILL_AUTO, GDN_PREFILL_FUSED,
    GDN_PREFILL_SEQUENTIAL, GDN_PREFILL_TRANSFER, GDN_QK_L2NORM, GdnError, declared_functions,
    gdn_chunk_prefill, gdn_chunk_prefill_backward, gdn_chunk_prefill_backward_workspace_size,
    gdn_chunk_prefill_static_scratch, gdn_cp_combine, gdn_cp_finish, gdn_cp_local_state, gdn_cp_local_state_workspace_size, gdn_chunk_prefill_workspace_size, gdn_decode,
    gdn_decode_mtp,
    gdn_get_device_error, gdn_selftest_wait_timeout,
    gdn_last_error, gdn_version, lib,
)
from .cp import cp_chunk_prefill  # noqa: F401,E402
