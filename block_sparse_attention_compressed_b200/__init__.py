"""Block-sparse compressed-key decode attention for NVIDIA B200 (sm_100a).

The computation lives in ``libbsa.so`` (hand-written CUDA kernels behind the C ABI of
``include/bsa.h``); this package is its thin ctypes binding plus the seeded synthetic workloads
used by the tests and the benchmark.

    from block_sparse_attention_compressed_b200 import make_params, alloc_workspace, bsa_decode_step
"""
from ._abi import (  # noqa: F401
    BSA_BF16, BSA_ERR_CUDA, BSA_ERR_DEVICE_CHECK, BSA_ERR_INVALID_ARG, BSA_ERR_UNSUPPORTED,
    BSA_ERR_WORKSPACE, BSA_F32, BSA_MAX_LAYERS, BSA_OK, DEVERR_BLOCK_IDX, DEVERR_CAPACITY,
    DEVERR_N_SEL, DEVERR_SEQ_LEN, LIB_PATH, BsaError, Params, Sizes, alloc_workspace,
    bsa_abi_version, bsa_check_params, bsa_compress_append, bsa_compress_keys, bsa_decode_step,
    bsa_decode_step_anchored, bsa_decode_step_info, bsa_decode_step_lookahead, bsa_prefill,
    bsa_prefill_attend, bsa_prefill_tiles, bsa_decode_step_clsa, bsa_clsa_workspace_size, alloc_clsa_workspace,
    bsa_get_sizes, bsa_read_device_error, bsa_select_blocks, bsa_select_blocks_forecast,
    bsa_sparse_decode, bsa_sparse_decode_layers, bsa_sparse_decode_noalloc, bsa_workspace_init,
    bsa_workspace_size, lib, make_params, status_string,
)
