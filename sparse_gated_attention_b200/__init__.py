"""Sparse Gated Attention (SGA) hot path for NVIDIA B200 (sm_100a).

The computation runs in ``libsga.so`` (hand-written CUDA kernels behind the C
ABI declared in ``include/sga.h``); this package is its Python binding.
"""
from ._binding import (  # noqa: F401
    EXPORTED,
    HEADS,
    INDEX_DIM,
    INDEX_HEADS,
    LIB_PATH,
    OP_FORWARD,
    OP_INDEX_SCORES,
    OP_SPARSE_MLA_ATTEND,
    OP_TOPK_SELECT,
    QK_DIM,
    TOP_K,
    V_DIM,
    Dims,
    SGAError,
    alloc_workspace,
    clear_device_status,
    device_status,
    forward,
    forward_fp8,
    index_scores,
    index_scores_fp8,
    load_library,
    make_dims,
    sparse_mla_attend,
    topk_select,
    topk_select_noalloc,
    workspace_size,
)
