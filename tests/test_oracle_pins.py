"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute the same way: exact
rational arithmetic, a closed form, an independent library routine (torch's
scaled-dot-product attention in float64), brute-force enumeration on tiny inputs, or an
identity the slides state.  A plausible mistake (wrong scale, dropped term, transposed
operand, wrong sort direction or tie rule, W and Omega overlapping, a missing rescale in
the merge) fails at least one of them.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from synth import gen

RNG = np.random.default_rng(1234)


def rand_bf16(shape, scale=1.0, rng=RNG):
    return gen.f64_to_bf16_bits(rng.standard_normal(shape) * scale)


# ---------------------------------------------------------------- bf16 decode


def test_bf16_decode_known_patterns():
    bits = np.array([0x3F80, 0xBF80, 0x4000, 0x3F00, 0x0000, 0x8000, 0x4049, 0x7F7F],
                    dtype=np.uint16)
    want = [1.0, -1.0, 2.0, 0.5, 0.0, -0.0, 3.140625, 3.3895313892515355e38]
    got = oracle.bf16_to_f64(bits)
    assert list(got) == want


# ---------------------------------------------------------------- Eq. (1) scores


@pytest.mark.parametrize("d", [64, 128])
def test_scores_match_exact_rationals(d):
    """z_i = q k_i / sqrt(d): the dot product of bf16 values is a dyadic rational that
    Fraction computes exactly; the oracle must agree to fp64 rounding."""
    q = rand_bf16(d)
    K = rand_bf16((17, d))
    z = oracle.scores(oracle.bf16_to_f64(q), oracle.bf16_to_f64(K))
    qf = [Fraction(float(x)) for x in oracle.bf16_to_f64(q)]
    for i in range(K.shape[0]):
        kf = [Fraction(float(x)) for x in oracle.bf16_to_f64(K[i])]
        dot = sum(a * b for a, b in zip(qf, kf))
        if d == 64:
            exact = float(dot / 8)          # sqrt(64) = 8 exactly
            assert abs(z[i] - exact) <= 4e-16 * max(1.0, abs(exact)) * d
        else:
            exact = float(dot) / math.sqrt(d)
            assert abs(z[i] - exact) <= 1e-14 * max(1.0, abs(exact))


def test_scores_unit_query_reads_one_channel():
    d = 128
    K = rand_bf16((9, d))
    Kf = oracle.bf16_to_f64(K)
    for j in (0, 5, 127):
        q = np.zeros(d)
        q[j] = 2.0
        z = oracle.scores(q, Kf)
        assert np.array_equal(z, 2.0 * Kf[:, j] / math.sqrt(d))


# ---------------------------------------------------------------- static set W


def test_static_set_and_candidates():
    W = oracle.static_set(1000, 4, 64)
    assert list(W) == list(range(4)) + list(range(936, 1000))
    C = oracle.candidate_set(1000, 4, 64)
    assert list(C) == list(range(4, 936))
    # overlap: N < n_sink + n_window -> W is everything, C empty
    assert list(oracle.static_set(50, 32, 32)) == list(range(50))
    assert oracle.candidate_set(50, 32, 32).size == 0
    # no static set at all
    assert oracle.static_set(10, 0, 0).size == 0
    assert list(oracle.candidate_set(10, 0, 0)) == list(range(10))
    # N smaller than the sink count
    assert list(oracle.static_set(3, 128, 0)) == [0, 1, 2]


# ---------------------------------------------------------------- selection


def _dominates(za, a, zb, b):
    return za > zb or (za == zb and a < b)


@pytest.mark.parametrize("trial", range(40))
def test_topk_brute_force_with_ties(trial):
    """For N <= 12 enumerate every k-subset of C; exactly one dominates all the rest
    pairwise (higher z, ties to the lower position): it must be the oracle's Omega."""
    rng = np.random.default_rng(trial)
    N = int(rng.integers(1, 13))
    n_sink = int(rng.integers(0, 3))
    n_window = int(rng.integers(0, 3))
    z = rng.integers(-3, 4, size=N).astype(np.float64) * 0.5   # many exact ties
    C = oracle.candidate_set(N, n_sink, n_window)
    for k in range(0, C.size + 2):
        om = oracle.select_topk(z, C, k)
        k_eff = min(k, C.size)
        winners = []
        for S in itertools.combinations(C.tolist(), k_eff):
            rest = [b for b in C.tolist() if b not in S]
            if all(_dominates(z[a], a, z[b], b) for a in S for b in rest):
                winners.append(set(S))
        assert len(winners) == 1
        assert set(om.tolist()) == winners[0]
        assert om.size == k_eff
        assert not set(om.tolist()) & set(oracle.static_set(N, n_sink, n_window).tolist())


def test_topk_order_is_by_score_then_position():
    z = np.array([1.0, 3.0, 3.0, 2.0, 3.0, -1.0])
    om = oracle.select_topk(z, np.arange(6), 4)
    assert list(om) == [1, 2, 4, 3]


def test_eq2_threshold_set_is_a_topk_set():
    """Eq. (2): I_eps = {i : a_i > eps}.  Softmax is monotone, so I_eps is the top-|I_eps|
    set of z (no static set, distinct scores)."""
    rng = np.random.default_rng(7)
    for _ in range(20):
        z = rng.standard_normal(300) * 2.0
        C = np.arange(300)
        for eps in (1e-1, 1e-2, 3e-3, 1e-3, 1e-4):
            I = oracle.threshold_set(z, eps)
            om = oracle.select_topk(z, C, I.size)
            assert set(I.tolist()) == set(om.tolist())


def test_topk_permutation_equivariant():
    rng = np.random.default_rng(3)
    N, d = 200, 64
    q = rand_bf16(d, rng=rng)
    K = rand_bf16((N, d), rng=rng)
    V = rand_bf16((N, d), rng=rng)
    o1, om1, _ = oracle.decode_head(q, K, V, 20, 4, 8)
    perm = np.arange(N)
    mid = rng.permutation(np.arange(4, N - 8))
    perm[4:N - 8] = mid
    o2, om2, _ = oracle.decode_head(q, K[perm], V[perm], 20, 4, 8)
    assert set(perm[om2].tolist()) == set(om1.tolist())
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)


def test_planted_needles_are_retrieved():
    """Needles whose score clears every other candidate by 1 must all be in Omega."""
    rng = np.random.default_rng(11)
    N, d, G = 4096, 128, 4
    q = rand_bf16((G, d), rng=rng)
    K = rand_bf16((N, d), rng=rng)
    V = rand_bf16((N, d), rng=rng)
    Kf = oracle.bf16_to_f64(K)
    n_sink, n_window, k = 16, 64, 40
    pos = rng.choice(np.arange(n_sink, N - n_window), size=8 * G, replace=False)
    for h in range(G):
        qf = oracle.bf16_to_f64(q[h])
        top = np.max(Kf @ qf / math.sqrt(d))
        lam = (top + 1.0) * math.sqrt(d) / np.linalg.norm(qf) * 1.05
        for j in range(8):
            K[pos[h * 8 + j]] = gen.needle_row(q[h], lam)
    for h in range(G):
        _, om, _ = oracle.decode_head(q[h], K, V, k, n_sink, n_window)
        mine = set(pos[h * 8:(h + 1) * 8].tolist())
        assert mine <= set(om.tolist())


# ---------------------------------------------------------------- attention


def _sdpa(z_q, K, V):
    """torch scaled_dot_product_attention in float64: an independent softmax attention."""
    q = torch.from_numpy(z_q)[None, None, None, :]
    k = torch.from_numpy(K)[None, None]
    v = torch.from_numpy(V)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0, 0].numpy()


@pytest.mark.parametrize("N,d", [(1, 64), (7, 128), (640, 128), (4097, 64)])
def test_dense_matches_torch_sdpa_fp64(N, d):
    rng = np.random.default_rng(N)
    q = rand_bf16(d, rng=rng)
    K = rand_bf16((N, d), 2.0, rng=rng)
    V = rand_bf16((N, d), rng=rng)
    o = oracle.dense_head(q, K, V)
    ref = _sdpa(oracle.bf16_to_f64(q), oracle.bf16_to_f64(K), oracle.bf16_to_f64(V))
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_sparse_union_matches_torch_sdpa_on_the_selected_rows():
    rng = np.random.default_rng(5)
    N, d = 3000, 128
    q = rand_bf16(d, rng=rng)
    K = rand_bf16((N, d), 2.0, rng=rng)
    V = rand_bf16((N, d), rng=rng)
    o, om, _ = oracle.decode_head(q, K, V, 100, 4, 64)
    U = np.concatenate([oracle.static_set(N, 4, 64), om])
    ref = _sdpa(oracle.bf16_to_f64(q), oracle.bf16_to_f64(K)[U], oracle.bf16_to_f64(V)[U])
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_two_keys_closed_form_logistic():
    """Two keys: o = v2 + sigmoid(z1 - z2) (v1 - v2)."""
    rng = np.random.default_rng(9)
    for _ in range(20):
        z = rng.standard_normal(2) * 3
        V = rng.standard_normal((2, 16))
        o = oracle.attend(z, V, np.array([0, 1]))
        ref = V[1] + expit(z[0] - z[1]) * (V[0] - V[1])
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-14)


def test_attention_is_a_convex_combination():
    rng = np.random.default_rng(10)
    z = rng.standard_normal(50) * 4
    U = np.arange(50)
    V = np.tile(rng.standard_normal(8), (50, 1))
    np.testing.assert_allclose(oracle.attend(z, V, U), V[0], rtol=0, atol=1e-14)
    # affine equivariance in V
    V = rng.standard_normal((50, 8))
    A = rng.standard_normal((8, 8))
    c = rng.standard_normal(8)
    np.testing.assert_allclose(oracle.attend(z, V @ A + c, U), oracle.attend(z, V, U) @ A + c,
                               rtol=0, atol=1e-12)
    # shift of every score (equivalently one vector added to every key) changes nothing
    np.testing.assert_allclose(oracle.attend(z + 123.25, V, U), oracle.attend(z, V, U),
                               rtol=0, atol=1e-13)


def test_identical_keys_give_the_mean_of_values():
    rng = np.random.default_rng(12)
    N, d = 33, 64
    q = rand_bf16(d, rng=rng)
    K = np.tile(rand_bf16(d, rng=rng), (N, 1))
    V = rand_bf16((N, d), rng=rng)
    o = oracle.dense_head(q, K, V)
    np.testing.assert_allclose(o, oracle.bf16_to_f64(V).mean(axis=0), rtol=0, atol=1e-14)


def test_one_dominant_key_limit():
    """A score gap g bounds |o - v_top| by (N-1) e^{-g} max|v - v_top|."""
    rng = np.random.default_rng(13)
    z = rng.standard_normal(100)
    z[17] = 40.0
    V = rng.standard_normal((100, 4))
    o = oracle.attend(z, V, np.arange(100))
    gap = 40.0 - np.max(np.delete(z, 17))
    bound = 99 * math.exp(-gap) * np.max(np.abs(V - V[17]))
    assert np.max(np.abs(o - V[17])) <= bound


# ---------------------------------------------------------------- merge (Eqs. 3-5)


@pytest.mark.parametrize("parts", [2, 3, 7])
def test_merge_of_disjoint_parts_equals_union_softmax(parts):
    """The slides' identity: merging partial states of disjoint subsets with gamma_S is the
    exact softmax over their union."""
    rng = np.random.default_rng(parts)
    z = rng.standard_normal(400) * 5 + 30     # large scores: needs the max subtraction
    V = rng.standard_normal((400, 16))
    U = rng.permutation(400)[:257]
    cuts = np.sort(rng.choice(np.arange(1, U.size), size=parts - 1, replace=False))
    subsets = np.split(U, cuts)
    states = [oracle.partial_state(z, V, S) for S in subsets]
    np.testing.assert_allclose(oracle.merge_partials(states), oracle.attend(z, V, U),
                               rtol=0, atol=1e-12)


def test_merge_of_static_and_dynamic_parts():
    rng = np.random.default_rng(21)
    N, d = 2000, 64
    q = rand_bf16(d, rng=rng)
    K = rand_bf16((N, d), 2.0, rng=rng)
    V = rand_bf16((N, d), rng=rng)
    o, om, z = oracle.decode_head(q, K, V, 50, 8, 32)
    W = oracle.static_set(N, 8, 32)
    Vf = oracle.bf16_to_f64(V)
    merged = oracle.merge_partials([oracle.partial_state(z, Vf, W),
                                    oracle.partial_state(z, Vf, om)])
    np.testing.assert_allclose(merged, o, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- decode-step invariants


@pytest.mark.parametrize("N,n_sink,n_window", [(500, 4, 64), (70, 64, 64), (33, 0, 0)])
def test_k_at_least_candidates_equals_dense(N, n_sink, n_window):
    """k >= |C| selects every candidate, so the step is full attention."""
    rng = np.random.default_rng(N)
    q = rand_bf16((1, 2, 64), rng=rng)
    K = rand_bf16((1, 1, N, 64), 2.0, rng=rng)
    V = rand_bf16((1, 1, N, 64), rng=rng)
    out, _ = oracle.decode_step(q, K, V, N, n_sink, n_window)
    dense = oracle.dense_decode(q, K, V)
    np.testing.assert_allclose(out, dense, rtol=0, atol=1e-13)


def test_k_zero_is_static_attention_only():
    """k = 0: the step attends to W only (the sink-plus-window special case)."""
    rng = np.random.default_rng(4)
    N, d = 300, 64
    q = rand_bf16(d, rng=rng)
    K = rand_bf16((N, d), rng=rng)
    V = rand_bf16((N, d), rng=rng)
    o, om, _ = oracle.decode_head(q, K, V, 0, 4, 16)
    assert om.size == 0
    W = oracle.static_set(N, 4, 16)
    ref = _sdpa(oracle.bf16_to_f64(q), oracle.bf16_to_f64(K)[W], oracle.bf16_to_f64(V)[W])
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-13)


def test_gqa_heads_select_separately_but_share_kv():
    rng = np.random.default_rng(8)
    B, Hq, Hkv, N, d = 2, 4, 2, 256, 64
    q = rand_bf16((B, Hq, d), rng=rng)
    K = rand_bf16((B, Hkv, N, d), rng=rng)
    V = rand_bf16((B, Hkv, N, d), rng=rng)
    out, oms = oracle.decode_step(q, K, V, 10, 2, 4)
    for b in range(B):
        for h in range(Hq):
            o, om, _ = oracle.decode_head(q[b, h], K[b, h // 2], V[b, h // 2], 10, 2, 4)
            np.testing.assert_array_equal(out[b, h], o)
            assert set(om.tolist()) == set(oms[b][h].tolist())
    # heads of one group generally pick different sets
    assert set(oms[0][0].tolist()) != set(oms[0][1].tolist())


def test_empty_cache_is_an_error():
    with pytest.raises(ValueError):
        oracle.decode_head(np.zeros(64, np.uint16), np.zeros((0, 64), np.uint16),
                           np.zeros((0, 64), np.uint16), 1, 0, 0)


# ---------------------------------------------------------------- attention-mass statistic


def test_topk_maximises_recovered_mass():
    """Fig. 2's statistic: the top-k set recovers at least the mass of any k-subset."""
    rng = np.random.default_rng(14)
    z = rng.standard_normal(9) * 2
    C = np.arange(9)
    assert abs(oracle.attention_mass(z, C) - 1.0) < 1e-15
    for k in range(1, 9):
        best = oracle.attention_mass(z, oracle.select_topk(z, C, k))
        for S in itertools.combinations(range(9), k):
            assert oracle.attention_mass(z, np.array(S)) <= best + 1e-15


# ---------------------------------------------------------------- sizes (Table 1)


def test_kv_capacity_table1():
    """Bytes per token of a Llama-3-8B cache (2 x 32 layers x 8 KV heads x 128 x 2 B) against
    the printed Table 1 capacities, whose prompt labels count thousands of tokens
    (1M = 1024 thousand) and whose unit is 2^30 bytes."""
    per_token = 2 * 32 * 8 * 128 * 2
    assert per_token == 131072
    w = gen.workload("l8b_1m_32layer")
    assert w.kv_bytes() == per_token * (1 << 20)
    path = os.path.join(os.path.dirname(__file__), "golden", "kv_capacity_table1.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    thousands = {"128K": 128, "256K": 256, "512K": 512, "1M": 1024}
    for label, gb in rows:
        cap = thousands[label] * 1000 * per_token / 2**30
        assert abs(cap - float(gb)) <= 0.06, (label, cap, gb)


# ---------------------------------------------------------------- prefill queries' top-k


def test_prefill_score_matrix_matches_exact_rationals():
    """Z = Q K^T / sqrt(d) for a batch of queries: every entry against Fraction arithmetic
    (d = 64, so the scale 1/8 is exact), catching a transposed operand or wrong scale."""
    d = 64
    Q = rand_bf16((5, d))
    K = rand_bf16((7, d))
    Z = oracle.prefill_score_matrix(Q, K)
    Qf = oracle.bf16_to_f64(Q)
    Kf = oracle.bf16_to_f64(K)
    for m in range(5):
        for i in range(7):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(Qf[m], Kf[i])) / 8
            assert abs(Z[m, i] - float(exact)) <= 4e-16 * d * max(1.0, abs(float(exact)))


@pytest.mark.parametrize("trial", range(12))
def test_prefill_topk_brute_force(trial):
    """Every query row of a tiny batch: the returned set is the unique k-subset of C that
    dominates the rest pairwise under exactly computed scores (ties to the lower position),
    with query head h reading KV head h // G."""
    rng = np.random.default_rng(100 + trial)
    B, Hkv, G, M, N, d = 1, 2, 2, 3, int(rng.integers(2, 11)), 64
    n_sink, n_window = int(rng.integers(0, 2)), int(rng.integers(0, 2))
    # few distinct values so that exact score ties occur
    Q = gen.f64_to_bf16_bits(rng.integers(-2, 3, size=(B, Hkv * G, M, d)).astype(np.float64))
    K = gen.f64_to_bf16_bits(rng.integers(-1, 2, size=(B, Hkv, N, d)).astype(np.float64))
    C = oracle.candidate_set(N, n_sink, n_window).tolist()
    for k in (0, 1, 2, 5):
        om = oracle.prefill_topk(Q, K, k, n_sink, n_window)
        k_eff = min(k, len(C))
        for h in range(Hkv * G):
            Kf = oracle.bf16_to_f64(K[0, h // G])
            for m in range(M):
                qf = oracle.bf16_to_f64(Q[0, h, m])
                z = {i: sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(qf, Kf[i]))
                     for i in C}
                winners = [set(S) for S in itertools.combinations(C, k_eff)
                           if all(_dominates(z[a], a, z[b], b)
                                  for a in S for b in C if b not in S)]
                assert len(winners) == 1
                assert set(om[0][h][m].tolist()) == winners[0]


def test_prefill_topk_rows_are_decode_selections():
    """A prefill query's selection is the decode step's selection for that query alone (the
    decode oracle scores by a matrix-vector product, the prefill oracle by a matrix product)."""
    B, Hq, Hkv, M, N, d = 2, 4, 2, 6, 300, 128
    Q = rand_bf16((B, Hq, M, d))
    K = rand_bf16((B, Hkv, N, d))
    V = rand_bf16((B, Hkv, N, d))
    om = oracle.prefill_topk(Q, K, 20, 4, 16)
    for m in range(M):
        _, dec = oracle.decode_step(np.ascontiguousarray(Q[:, :, m]), K, V, 20, 4, 16)
        for b in range(B):
            for h in range(Hq):
                assert np.array_equal(np.sort(om[b][h][m]), np.sort(dec[b][h]))


# ---------------------------------------------------------------- threshold budget (Eq. 2)


def test_threshold_two_keys_logistic_closed_form():
    """Two keys with z = (x, 0): a_0 = sigma(x) (the logistic function); key 0 passes a
    threshold eps exactly when sigma(x) > eps (no static set, generous k)."""
    for x in (-3.0, -0.5, 0.0, 0.7, 2.5):
        z = np.array([x, 0.0])
        for eps in (0.05, 0.3, 0.5, 0.8):
            om = set(oracle.select_threshold(z, np.arange(2), 5, eps).tolist())
            assert (0 in om) == (expit(x) > eps)
            assert (1 in om) == (expit(-x) > eps)


def test_threshold_set_is_eq2_set_and_top_k_cap():
    rng = np.random.default_rng(5)
    z = rng.standard_normal(400) * 2.0
    C = oracle.candidate_set(400, 3, 20)
    for eps in (1e-4, 1e-3, 1e-2):
        I = set(oracle.threshold_set(z, eps).tolist()) & set(C.tolist())   # Eq. (2) within C
        assert set(oracle.select_threshold(z, C, 10**6, eps).tolist()) == I
        om = oracle.select_threshold(z, C, 5, eps)
        assert om.size == min(5, len(I))
        assert set(om.tolist()) <= I
        if len(I) > 5:   # the cap keeps the largest scores
            assert min(z[om]) >= max(z[list(I - set(om.tolist()))])
    # a vanishing threshold is the plain top-k; no two keys can both exceed one half
    assert np.array_equal(np.sort(oracle.select_threshold(z, C, 30, 1e-300)),
                          np.sort(oracle.select_topk(z, C, 30)))
    assert oracle.select_threshold(z, C, 30, 0.5).size <= 1


def test_threshold_weights_use_the_full_softmax():
    """The weights are Eq. (1)'s over all N positions, sinks and window included: raising a
    window key's score lowers every candidate's weight."""
    z = np.array([1.0, 1.0, 1.0, 1.0, 0.0])
    C = oracle.candidate_set(5, 0, 1)                 # the window is position 4
    a_before = 1.0 / (4.0 + math.exp(-1.0))          # weight of each of the four candidates
    eps = a_before * 0.999
    assert oracle.select_threshold(z, C, 10, eps).size == 4
    z2 = z.copy()
    z2[4] = 5.0                                       # the window key takes most of the mass
    assert oracle.select_threshold(z2, C, 10, eps).size == 0


def test_pyramid_budgets_shape():
    for L, km, r in ((32, 2621, 0.25), (7, 100, 0.5), (5, 3, 1.0), (1, 9, 0.3), (80, 20971, 0.1)):
        b = oracle.pyramid_budgets(L, km, r)
        assert b.size == L and int(b.sum()) == L * km
        assert np.all(np.diff(b) <= 0)                        # shrinks with depth
        k_max = 2.0 * km / (1.0 + r)
        if L > 1:
            assert abs(b[0] - k_max) <= 1 and abs(b[-1] - r * k_max) <= 1
    assert list(oracle.pyramid_budgets(6, 11, 1.0)) == [11] * 6


# ---------------------------------------------------------------- paged layout


def test_gather_paged_inverts_a_scatter_by_the_definition():
    """Scatter dense caches of ragged lengths into a shuffled page pool following the layout
    (token i of sequence b in row i % 128 of page table[b][i // 128]); the gather must return
    them exactly, for every sequence and KV head."""
    rng = np.random.default_rng(9)
    B, Hkv, d, P = 3, 2, 8, 128
    lens = [1, 300, 129]
    pages_needed = [(n + P - 1) // P for n in lens]
    num_pages = sum(pages_needed) + 2
    order = rng.permutation(num_pages)
    table = np.full((B, 4), -1, dtype=np.int64)
    pool = rng.integers(0, 2**16, size=(num_pages, Hkv, P, d)).astype(np.uint16)
    dense = []
    j = 0
    for b, n in enumerate(lens):
        X = rng.integers(0, 2**16, size=(Hkv, n, d)).astype(np.uint16)
        dense.append(X)
        for pg in range(pages_needed[b]):
            table[b, pg] = order[j]
            j += 1
        for i in range(n):
            pool[table[b, i // P], :, i % P, :] = X[:, i, :]
    got = oracle.gather_paged(pool, table, lens)
    for b in range(B):
        assert np.array_equal(got[b], dense[b])


# ---------------------------------------------------------------- IVF retrieval


def test_ivf_probing_every_cluster_is_exact_retrieval():
    """With every cluster probed, IVF retrieval is the exact top-k step, for any partition of
    the keys into clusters (the index only restricts the candidates)."""
    rng = np.random.default_rng(21)
    N, d, nlist, k = 500, 64, 7, 40
    q, K, V = rand_bf16(d), rand_bf16((N, d)), rand_bf16((N, d))
    assign = rng.integers(0, nlist, size=N)
    pos = np.argsort(assign, kind="stable")
    offsets = np.concatenate([[0], np.cumsum(np.bincount(assign, minlength=nlist))])
    cent = rand_bf16((nlist, d))
    o_ivf, om_ivf, _, probe = oracle.ivf_decode_head(q, K, V, pos, offsets, cent, k, nlist, 4, 32)
    o, om, _ = oracle.decode_head(q, K, V, k, 4, 32)
    assert sorted(probe.tolist()) == list(range(nlist))
    assert np.array_equal(np.sort(om_ivf), np.sort(om))
    assert np.allclose(o_ivf, o, rtol=0, atol=1e-12)


def test_ivf_candidates_are_the_probed_clusters():
    """Keys of unprobed clusters are never retrieved; the probe is the top-nprobe centroids by
    q . c with ties to the lower index."""
    d, N = 64, 300
    q = gen.f64_to_bf16_bits(np.eye(d)[0] * 1.0)                     # q = e_0
    cent = gen.f64_to_bf16_bits(np.array([np.eye(d)[i % d] * (1.0 if i != 3 else 2.0)
                                          for i in range(6)]))        # c_3 scores 0, c_0 1
    cent[2] = cent[0]                                                 # c_0 and c_2 tie
    probe = oracle.ivf_probe(oracle.bf16_to_f64(q), oracle.bf16_to_f64(cent), 2)
    assert list(probe) == [0, 2]
    rng = np.random.default_rng(3)
    K, V = rand_bf16((N, d)), rand_bf16((N, d))
    assign = np.arange(N) % 6
    pos = np.argsort(assign, kind="stable")
    offsets = np.concatenate([[0], np.cumsum(np.bincount(assign, minlength=6))])
    _, om, _, _ = oracle.ivf_decode_head(q, K, V, pos, offsets, cent, 1000, 2, 0, 0)
    assert set(om.tolist()) == {i for i in range(N) if i % 6 in (0, 2)}


# ---------------------------------------------------------------- IVF index construction


def test_round_to_bf16_known_values():
    """Round to nearest even, from hand-worked float32 patterns: 0.6 = 0x3F19999A and 0.8 =
    0x3F4CCCCD round up (low halves above 0x8000); 1 + 2^-8 and 1 + 3 * 2^-8 sit exactly
    between two bf16 values and go to the even one; 12/13 = 0x3F6C4EC5 rounds down."""
    x = np.array([0.6, 0.8, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 12 / 13, -0.6, 0.0, 1.0])
    want = [0x3F1A, 0x3F4D, 0x3F80, 0x3F82, 0x3F6C, 0xBF1A, 0x0000, 0x3F80]
    assert oracle.round_to_bf16(x).tolist() == want


def _two_direction_keys():
    """40 keys in 64 channels: positions 0-19 are multiples of (3, 4) in channels 0-1,
    positions 20-39 multiples of (5, 12) in channels 2-3 (all exact in bf16)."""
    K = np.zeros((40, 64))
    for i in range(20):
        K[i, :2] = (1 + i % 3) * np.array([3.0, 4.0])
        K[20 + i, 2:4] = (1 + i % 3) * np.array([5.0, 12.0])
    return gen.f64_to_bf16_bits(K)


@pytest.mark.parametrize("iters", [0, 1, 3])
def test_ivf_build_two_directions_is_a_fixed_point(iters):
    """Two orthogonal groups of parallel keys: the evenly spaced start (positions 0 and 20)
    already points along each group, and the unit direction of a group's sum is that same
    direction, bf16 (3, 4) / 5 = (0x3F1A, 0x3F4D) and (5, 12) / 13 = (0x3EC5, 0x3F6C)
    (worked by hand, see test_round_to_bf16_known_values)."""
    cent, assign, pos, offsets = oracle.ivf_build(_two_direction_keys(), 2, iters)
    want = np.zeros((2, 64), np.uint16)
    want[0, :2] = [0x3F1A, 0x3F4D]
    want[1, 2:4] = [0x3EC5, 0x3F6C]
    assert np.array_equal(cent, want)
    assert assign.tolist() == [0] * 20 + [1] * 20
    assert pos.tolist() == list(range(40)) and offsets.tolist() == [0, 20, 40]


def test_ivf_build_ties_go_to_the_lower_centroid():
    """Keys e_0, e_1 (the two starting centroids) and e_0 + e_1, which scores 1 against both:
    it joins centroid 0.  One iteration later centroid 0 is the unit direction of (2, 1),
    bf16 (0x3F65, 0x3EE5), and the assignment is unchanged."""
    K = np.zeros((3, 64))
    K[0, 0] = K[1, 1] = 1.0
    K[2, :2] = 1.0
    bits = gen.f64_to_bf16_bits(K)
    cent, assign, _, _ = oracle.ivf_build(bits, 2, 0)
    assert assign.tolist() == [0, 1, 0]
    cent, assign, pos, offsets = oracle.ivf_build(bits, 2, 1)
    assert cent[0, :2].tolist() == [0x3F65, 0x3EE5] and cent[1, :2].tolist() == [0, 0x3F80]
    assert assign.tolist() == [0, 1, 0]
    assert pos.tolist() == [0, 2, 1] and offsets.tolist() == [0, 2, 3]


def test_ivf_build_empty_cluster_keeps_its_centroid():
    """Positions 0 and 2 hold the same key e_0, so both centroids start equal; every key ties
    and joins centroid 0, leaving cluster 1 empty: it keeps e_0 while centroid 0 moves to the
    unit direction of the sum (5, 2), bf16 (0x3F6E, 0x3EBE).  The final assignment then sends
    the two e_0 keys to centroid 1 (score 1 against 5 / sqrt(29) = 0.93)."""
    K = np.zeros((4, 64))
    K[0, 0] = K[2, 0] = 1.0
    K[1, :2] = (1.0, 1.0)
    K[3, :2] = (2.0, 1.0)
    cent, assign, pos, offsets = oracle.ivf_build(gen.f64_to_bf16_bits(K), 2, 1)
    assert cent[0, :2].tolist() == [0x3F6E, 0x3EBE] and np.all(cent[0, 2:] == 0)
    assert cent[1, :2].tolist() == [0x3F80, 0] and np.all(cent[1, 2:] == 0)
    assert assign.tolist() == [1, 0, 1, 0]
    assert pos.tolist() == [1, 3, 0, 2] and offsets.tolist() == [0, 2, 4]


def _bf16_rne_exact(x):
    """Nearest bf16 (ties to even) of an exact rational x, by comparing it with the two
    float32-truncated neighbours as Fractions (struct packing, no numpy)."""
    import struct
    xf = float(x)
    b = struct.unpack(">I", struct.pack(">f", xf))[0]
    s, lo = b >> 31, (b & 0x7FFFFFFF) >> 16

    def val(m):
        return Fraction(struct.unpack(">f", struct.pack(">I", (s << 31) | (m << 16)))[0])

    dl, dh = abs(x - val(lo)), abs(x - val(lo + 1))
    m = lo + 1 if (dh < dl or (dh == dl and lo & 1)) else lo
    return (s << 15) | m


def _unit_bf16_exact(v):
    from decimal import Decimal, getcontext
    getcontext().prec = 80
    n2 = sum(a * a for a in v)
    if n2 == 0:
        return [0] * len(v)
    n = (Decimal(n2.numerator) / Decimal(n2.denominator)).sqrt()
    return [_bf16_rne_exact(Fraction(Decimal(a.numerator) / Decimal(a.denominator) / n)) for a in v]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_ivf_build_matches_brute_force_on_tiny_inputs(seed):
    """Spherical k-means written out with exact rationals (scores, sums), an 80-digit square
    root and the nearest-even rounding above, on 11 keys of 4 channels into 3 clusters."""
    rng = np.random.default_rng(100 + seed)
    N, d, nlist, iters = 11, 4, 3, 2
    bits = rand_bf16((N, d), rng=rng)
    Kq = [[Fraction(float(x)) for x in row] for row in oracle.bf16_to_f64(bits)]
    cent = [_unit_bf16_exact(Kq[(j * N) // nlist]) for j in range(nlist)]
    for it in range(iters + 1):
        Cq = [[Fraction(float(x)) for x in oracle.bf16_to_f64(np.array(c, np.uint16))] for c in cent]
        assign = []
        for k in Kq:
            sc = [sum(a * b for a, b in zip(k, c)) for c in Cq]
            assign.append(max(range(nlist), key=lambda j: (sc[j], -j)))
        if it == iters:
            break
        for j in range(nlist):
            mem = [Kq[i] for i in range(N) if assign[i] == j]
            if mem:
                s = [sum(col) for col in zip(*mem)]
                if any(x != 0 for x in s):
                    cent[j] = _unit_bf16_exact(s)
    got_c, got_a, got_p, got_o = oracle.ivf_build(bits, nlist, iters)
    assert got_c.tolist() == cent
    assert got_a.tolist() == assign
    listing = [i for j in range(nlist) for i in range(N) if assign[i] == j]
    assert got_p.tolist() == listing
    assert got_o.tolist() == [0] + list(np.cumsum([assign.count(j) for j in range(nlist)]))
