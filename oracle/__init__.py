"""Oracle (test infrastructure): fp64 CPU restatement of the decode step.

Importable only from tests/, __graft_entry__.smoke() and bench.py's CPU-baseline legs.
"""
from .retrieval_attention import (  # noqa: F401
    attend, attention_mass, bf16_to_f64, candidate_set, decode_head, decode_step,
    decode_head_eps, dense_decode, dense_head, gather_paged, merge_partials, partial_state,
    prefill_score_matrix, ivf_build, ivf_probe, ivf_decode_head, round_to_bf16,
    prefill_topk, pyramid_budgets, select_threshold,
    scores, select_topk,
    softmax_weights, static_set, threshold_set,
)
