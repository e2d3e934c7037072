"""B200-native (sm_100a) HISA token-selection indexer.

The work happens in ``libhisa.so`` (hand-written CUDA kernels behind the C ABI
of ``include/hisa.h``); this package is its thin Python binding.  PyTorch only
provides device memory and streams.
"""

from .binding import (  # noqa: F401
    EXPORTED,
    HISA_ATT_DIM,
    HISA_BLOCK,
    HISA_INDEX_DIM,
    HISA_MAX_M,
    HISA_MAX_TOPK,
    HisaError,
    LIB_PATH,
    dsa_flat_select,
    dsa_flat_workspace_size,
    hisa_append_keys,
    hisa_block_sparse_select,
    hisa_block_sparse_workspace_size,
    hisa_decode_step,
    hisa_device_status,
    hisa_pool_blocks,
    hisa_fraction_blocks,
    hisa_select,
    hisa_select_varm,
    hisa_select_workspace_size,
    hisa_sparse_attention,
    hisa_test_fault,
    hisa_timing_collect,
    hisa_timing_enable,
    lib,
)
