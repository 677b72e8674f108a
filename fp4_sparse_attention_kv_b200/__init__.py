"""fp4_sparse_attention_kv_b200: decode-time sparse attention over an FP4 KV cache on B200.

The compute path is the C-ABI library ``libfp4kv.so`` (hand-written CUDA for sm_100a,
declared in ``include/fp4kv.h``); ``binding`` marshals torch tensors into it.
"""
from .binding import (  # noqa: F401
    E2M1Planes, Fp4kvError, KEY_BF16, KEY_E2M1, KEY_E4M3, OP_HIER_POOL_SELECT, OP_INDEXER_SCORES, OP_INDEXER_TOPK,
    OP_KV_QUANT, OP_REINDEX_TOPK, OP_SPARSE_ATTN, alloc_workspace, hier_pool_select,
    indexer_scores, indexer_topk, indexer_topk_noalloc, kv_quant_fp4, lib, lse_combine, noalloc_status, profile_enable,
    profile_read, selftest_wait_timeout, selftest_wait_timeout_noalloc, sparse_attn_decode, swa_quant_fp8, topk_merge, version, workspace_bytes, workspace_init,
    workspace_status)
