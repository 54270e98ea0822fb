"""B200-native hashed n-gram embedding lookup (Engram / N-gram Embedding).

The computation lives in ``libengram.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/engram.h``).  This package is its thin Python binding; it never
computes a step itself and has no CPU fallback.
"""
from ._native import (  # noqa: F401
    ENGRAM_ERR_CUDA, ENGRAM_ERR_INVALID_ARG, ENGRAM_ERR_TIMEOUT,
    ENGRAM_ERR_UNSUPPORTED, ENGRAM_FORWARD_STAGES, ENGRAM_OK, ENGRAM_STATUS_BAD_ROW,
    ENGRAM_STATUS_BAD_TOKEN, ENGRAM_STATUS_WAIT_TIMEOUT, ENGRAM_TABLES_DEVICE,
    ENGRAM_TABLES_HOST_MAPPED, ENGRAM_NOALLOC_SCRATCH_BYTES, ENGRAM_FLAG_SINGLE_CTA_MMA,
    ENGRAM_FLAG_ROW_ORDER_GATHER, ENGRAM_FLAG_BULK_GATHER, ENGRAM_PATH_BULK_GATHER, ENGRAM_TABLE_BF16, ENGRAM_TABLE_FP8_E4M3, ENGRAM_PATH_FUSED_LOOKUP, ENGRAM_PATH_STAGED_ROWS, ENGRAM_PATH_SPLIT_K,
    ENGRAM_PATH_PAIR_MMA, ENGRAM_PATH_ROW_ORDER, EngramError, LIB_PATH, Plan, Weights, alloc_workspace,
    engram_advance_history, engram_device_status, engram_forward, engram_forward_path, engram_gate_conv,
    engram_gate_conv_noalloc, engram_gather, engram_hash, engram_selftest_wait_timeout, engram_stage_rows,
    engram_stage_rows_cached, engram_stage_rows_from_ids, engram_synchronize, RowCache,
    pack_weights, engram_packed_weights_size,
    engram_remap, engram_workspace_size, kernel_launches, last_error, lib, version,
)
