"""Exact top-k retrieval attention (RetrievalAttention's decode step with an exact device scan)
for B200 (sm_100a): CUDA kernels behind the C ABI of include/ra.h, and a ctypes binding."""
from .ra import (  # noqa: F401
    EXPORTS, LIB_PATH, KVCache, RA_ERR_ARG, RA_ERR_CAPACITY, RA_ERR_CUDA, RA_ERR_EMPTY, RA_ERR_SHAPE,
    RA_ERR_WORKSPACE, RA_OK, RaError, append_kv, check, decode_step, decode_workspace,
    dense_decode, dense_workspace, lib, ra_append_kv, ra_decode_step, ra_decode_workspace_bytes,
    ra_decode_step_static, ra_dense_decode, ra_dense_workspace_bytes, ra_kv, ra_last_error, ra_score_gqa,
    ra_select_attend, ra_sparse_attn, ra_status_str, ra_topk_select, ra_version,
    ra_prefill_workspace_bytes, ra_prefill_topk, ra_prefill_score, ra_prefill_select, prefill_topk,
    ra_decode_step_eps, decode_step_eps, pyramid_budgets, ra_paged_kv, PagedKVCache,
    paged_append_kv, paged_workspace, paged_decode_step, ra_ivf, IvfIndex, ivf_build,
    ivf_decode_step, ra_decode_step_append, ra_score_gqa_append, decode_step_append,
    ra_decode_step_append_host, ra_step_io,
)
