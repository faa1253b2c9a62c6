"""Planted mistakes in the oracle (CPU only): each must make at least one pin fail.

The mistakes are planted by monkeypatching the oracle module for the duration of a test;
the oracle's files are never modified.
"""
import math

import numpy as np
import pytest

import oracle
import oracle.retrieval_attention as ra
import test_oracle_pins as pins


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(ra, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_wrong_score_scale_is_caught(monkeypatch):
    _patch(monkeypatch, "scores", lambda q, K: (K @ q) / q.shape[-1])
    assert _fails(pins.test_scores_match_exact_rationals, 64)


def test_transposed_or_dropped_term_is_caught(monkeypatch):
    _patch(monkeypatch, "scores", lambda q, K: (K[:, 1:] @ q[1:]) / math.sqrt(q.shape[-1]))
    assert _fails(pins.test_scores_match_exact_rationals, 128)


def test_ascending_selection_is_caught(monkeypatch):
    def bad(z, C, k):
        C = np.asarray(C, dtype=np.int64)
        order = np.lexsort((C, z[C]))
        return C[order[:min(k, C.size)]]
    _patch(monkeypatch, "select_topk", bad)
    assert _fails(pins.test_topk_brute_force_with_ties, 0)


def test_ties_to_higher_position_are_caught(monkeypatch):
    def bad(z, C, k):
        C = np.asarray(C, dtype=np.int64)
        order = np.lexsort((-C, -z[C]))
        return C[order[:min(k, C.size)]]
    _patch(monkeypatch, "select_topk", bad)
    assert any(_fails(pins.test_topk_brute_force_with_ties, t) for t in range(10))


def test_overlapping_static_and_dynamic_sets_are_caught(monkeypatch):
    _patch(monkeypatch, "candidate_set", lambda N, s, w: np.arange(N, dtype=np.int64))
    assert _fails(pins.test_topk_brute_force_with_ties, 1)


def test_window_off_by_one_is_caught(monkeypatch):
    def bad(N, n_sink, n_window):
        return np.union1d(np.arange(0, min(n_sink, N)), np.arange(max(0, N - n_window - 1), N))
    _patch(monkeypatch, "static_set", bad)
    assert _fails(pins.test_static_set_and_candidates)


def test_merge_without_rescale_is_caught(monkeypatch):
    def bad(parts):
        den = sum(ZS for _, ZS, _ in parts)
        return sum((ZS / den) * (NS / ZS) for _, ZS, NS in parts)
    _patch(monkeypatch, "merge_partials", bad)
    assert _fails(pins.test_merge_of_disjoint_parts_equals_union_softmax, 3)


def test_unnormalised_attention_is_caught(monkeypatch):
    def bad(z, V, U):
        U = np.asarray(U, dtype=np.int64)
        w = np.exp(z[U] - np.max(z[U]))
        return w @ V[U]
    _patch(monkeypatch, "attend", bad)
    assert _fails(pins.test_dense_matches_torch_sdpa_fp64, 7, 128)


# ---------------------------------------------------------------- IVF retrieval


def test_ivf_probe_of_the_lowest_centroids_is_caught(monkeypatch):
    def bad(q, centroids, nprobe):
        zc = centroids @ q
        return np.lexsort((np.arange(zc.size), zc))[:nprobe]
    _patch(monkeypatch, "ivf_probe", bad)
    assert _fails(pins.test_ivf_candidates_are_the_probed_clusters)


def test_ivf_probe_ties_to_the_higher_cluster_are_caught(monkeypatch):
    def bad(q, centroids, nprobe):
        zc = centroids @ q
        return np.lexsort((-np.arange(zc.size), -zc))[:nprobe]
    _patch(monkeypatch, "ivf_probe", bad)
    assert _fails(pins.test_ivf_candidates_are_the_probed_clusters)


def test_ivf_candidates_not_restricted_to_c_are_caught(monkeypatch):
    def bad(q_bits, K_bits, V_bits, pos, offsets, cent_bits, k, nprobe, n_sink, n_window):
        q, K, V = ra.bf16_to_f64(q_bits), ra.bf16_to_f64(K_bits), ra.bf16_to_f64(V_bits)
        z = ra.scores(q, K)
        probe = ra.ivf_probe(q, ra.bf16_to_f64(cent_bits), nprobe)
        cand = np.concatenate([pos[offsets[c]:offsets[c + 1]] for c in probe]).astype(np.int64)
        omega = ra.select_topk(z, cand, k)                 # W keys left among the candidates
        U = np.union1d(ra.static_set(K.shape[0], n_sink, n_window), omega)
        return ra.attend(z, V, U), omega, z, probe
    _patch(monkeypatch, "ivf_decode_head", bad)
    assert _fails(pins.test_ivf_probing_every_cluster_is_exact_retrieval)


# ---------------------------------------------------------------- budgets and paging


def test_threshold_weights_over_the_candidates_only_are_caught(monkeypatch):
    def bad(z, C, k, eps):
        C = np.asarray(C, dtype=np.int64)
        a = np.exp(z[C] - z[C].max())
        a = a / a.sum()                                   # softmax over C instead of all N
        return ra.select_topk(z, C[a > eps], k)
    _patch(monkeypatch, "select_threshold", bad)
    assert _fails(pins.test_threshold_weights_use_the_full_softmax)


def test_threshold_not_strict_is_caught(monkeypatch):
    def bad(z, C, k, eps):
        a = ra.softmax_weights(z)
        C = np.asarray(C, dtype=np.int64)
        return ra.select_topk(z, C[a[C] >= eps], k)      # a_i >= eps instead of a_i > eps
    _patch(monkeypatch, "select_threshold", bad)
    assert _fails(pins.test_threshold_two_keys_logistic_closed_form)


def test_budgets_growing_with_depth_are_caught(monkeypatch):
    good = ra.pyramid_budgets
    _patch(monkeypatch, "pyramid_budgets", lambda L, k, r: good(L, k, r)[::-1].copy())
    assert _fails(pins.test_pyramid_budgets_shape)


def test_paged_gather_off_by_one_page_is_caught(monkeypatch):
    def bad(pool, table, lens):
        P = pool.shape[2]
        out = []
        for b, n in enumerate(lens):
            rows = [pool[table[b][min(i // P + 1, table.shape[1] - 1)], :, i % P, :]
                    for i in range(int(n))]
            out.append(np.stack(rows, axis=1))
        return out
    _patch(monkeypatch, "gather_paged", bad)
    assert _fails(pins.test_gather_paged_inverts_a_scatter_by_the_definition)


def test_prefill_with_the_wrong_kv_head_is_caught(monkeypatch):
    def bad(Q_bits, K_bits, k, n_sink, n_window):
        B, Hq, M, _ = Q_bits.shape
        Hkv, N = K_bits.shape[1], K_bits.shape[2]
        C = ra.candidate_set(N, n_sink, n_window)
        return [[[ra.select_topk(ra.prefill_score_matrix(Q_bits[b, h], K_bits[b, h % Hkv])[m],
                                 C, k) for m in range(M)] for h in range(Hq)] for b in range(B)]
    _patch(monkeypatch, "prefill_topk", bad)    # query head h reading KV head h % Hkv
    assert any(_fails(pins.test_prefill_topk_brute_force, t) for t in range(6))


def test_prefill_with_a_causal_mask_is_caught(monkeypatch):
    def bad(Q_bits, K_bits, k, n_sink, n_window):
        B, Hq, M, _ = Q_bits.shape
        Hkv, N = K_bits.shape[1], K_bits.shape[2]
        G = Hq // Hkv
        C = ra.candidate_set(N, n_sink, n_window)
        out = [[[None] * M for _ in range(Hq)] for _ in range(B)]
        for b in range(B):
            for h in range(Hq):
                Z = ra.prefill_score_matrix(Q_bits[b, h], K_bits[b, h // G])
                for m in range(M):   # query m of the last M positions sees keys up to N - M + m
                    out[b][h][m] = ra.select_topk(Z[m], C[C <= N - M + m], k)
        return out
    _patch(monkeypatch, "prefill_topk", bad)
    # (with the window covering the last M positions the mask removes no candidate; the tiny
    # brute-force cases have windows of 0 or 1 token)
    assert any(_fails(pins.test_prefill_topk_brute_force, t) for t in range(6))


# ---------------------------------------------------------------- IVF index construction


def _kmeans(K_bits, nlist, iters, init=None, argmax=None, update=None, empty=None):
    """The oracle's spherical k-means with one step swapped for a planted mistake."""
    K = ra.bf16_to_f64(K_bits)
    N = K.shape[0]
    starts = init(N, nlist) if init else [(j * N) // nlist for j in range(nlist)]
    cent = np.stack([ra.unit_bf16(K[i]) for i in starts])
    for it in range(iters + 1):
        S = K @ ra.bf16_to_f64(cent).T
        assign = argmax(S) if argmax else np.argmax(S, axis=1)
        if it == iters:
            break
        for j in range(nlist):
            members = assign == j
            if np.any(members):
                s = np.sum(K[members], axis=0)
                cent[j] = update(s, members) if update else ra.unit_bf16(s)
            elif empty:
                cent[j] = empty(cent[j])
    pos = np.argsort(assign, kind="stable")
    offsets = np.concatenate([[0], np.cumsum(np.bincount(assign, minlength=nlist))])
    return cent, assign, pos, offsets


def test_ivf_ties_to_the_higher_centroid_are_caught(monkeypatch):
    last_max = lambda S: S.shape[1] - 1 - np.argmax(S[:, ::-1], axis=1)
    _patch(monkeypatch, "ivf_build", lambda K, n, it: _kmeans(K, n, it, argmax=last_max))
    assert _fails(pins.test_ivf_build_ties_go_to_the_lower_centroid)


def test_ivf_unnormalised_mean_is_caught(monkeypatch):
    mean = lambda s, members: ra.round_to_bf16(s / np.count_nonzero(members))
    _patch(monkeypatch, "ivf_build", lambda K, n, it: _kmeans(K, n, it, update=mean))
    assert _fails(pins.test_ivf_build_two_directions_is_a_fixed_point, 1)


def test_ivf_empty_cluster_zeroed_is_caught(monkeypatch):
    zero = lambda c: np.zeros_like(c)
    _patch(monkeypatch, "ivf_build", lambda K, n, it: _kmeans(K, n, it, empty=zero))
    assert _fails(pins.test_ivf_build_empty_cluster_keeps_its_centroid)


def test_ivf_start_from_the_first_keys_is_caught(monkeypatch):
    first = lambda N, nlist: list(range(nlist))
    _patch(monkeypatch, "ivf_build", lambda K, n, it: _kmeans(K, n, it, init=first))
    assert _fails(pins.test_ivf_build_two_directions_is_a_fixed_point, 0)
