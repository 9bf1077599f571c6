"""B200 (sm_100a) Qwen Sparse Attention (QSA) layer forward.

The product is libqsa.so (C ABI in include/qsa.h); ``qsa`` is its ctypes binding.
"""

from .qsa import (  # noqa: F401
    QSA_OK, QSA_ERR_INVALID_ARG, QSA_ERR_WORKSPACE_TOO_SMALL, QSA_ERR_UNSUPPORTED, QSA_ERR_CUDA,
    QSA_MODE_DECODE, QSA_MODE_PREFILL, QSA_MODE_MIXED, QsaError, load, make_dims, status_string,
    qsa_workspace_bytes, qsa_workspace_init, qsa_read_device_status, qsa_pool_block_keys,
    qsa_index_scores, qsa_topk_blocks, qsa_sparse_attn, qsa_forward, qsa_sparse_attn_noalloc,
    qsa_sparse_attn_ex, qsa_select_blocks, QSA_DEV_BAD_PAGE, QSA_SEL_CAP, CP_PART_ROW,
    qsa_cp_workspace_bytes, qsa_cp_select_keys, qsa_cp_merge_keys, qsa_cp_attn_partial, qsa_cp_combine,
    qsa_attn_plan,
)
