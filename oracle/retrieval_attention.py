"""Oracle for one decode step of RetrievalAttention with exact top-k retrieval (fp64, CPU).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.  The
product (``top_retrieval_attention_b200``) never imports it and has no CPU fallback.

It is a plain, slow restatement of what the method computes, written from the slides
"RetrievalAttention: Accelerating Long-Context LLM Inference via Vector Retrieval"
(arXiv 2409.10516v3 paper discussion).  Library primitives used as single steps: a
matrix-vector product, a lexicographic sort, ``exp``.  No blocking, fusion or reordering.

Notation follows the slides: query q_t, keys k_i, values v_i, head dimension d, scores
z_i, static set W (first sink tokens plus the last window), dynamic set Omega (the
retrieved top-k), partial softmax state (m_S, Z_S, N_S, o_S) and merge weights gamma_S.

Inputs are bf16 bit patterns (uint16 arrays), decoded exactly to float64.
  q : [B, Hq, d]        K, V : [B, Hkv, N, d]        query head h reads KV head h // G.

Readings of points the slides leave open (each is listed with its reason in the design
notes of the repository):
  * W and Omega are disjoint ("The GPU keeps 640 fixed positions": "W and Omega are
    disjoint"), so the top-k runs over the candidates C = [0, N) minus W only.
  * Ties in z go to the lower position; k larger than |C| is clamped to |C|.
  * W = [0, min(n_sink, N)) union [max(0, N - n_window), N); the two may overlap.
  * The output is the exact softmax over U = W union Omega in fp64 ("Two local softmax
    outputs need global weights": the merge equals softmax over the selected union).
"""
from __future__ import annotations

import math

import numpy as np


# ------------------------------------------------------------------------------------
# inputs


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit pattern -> float64 (exact: bf16 is the top half of an IEEE float)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ------------------------------------------------------------------------------------
# Eq. (1): scaled dot-product scores and the softmax over the history


def scores(q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """z_i = q_t k_i^T / sqrt(d) for every cached key (slide "Sparse attention
    renormalizes selected tokens", Eq. (1)).  q [d] float64, K [N, d] float64."""
    d = q.shape[-1]
    return (K @ q) / math.sqrt(d)


def softmax_weights(z: np.ndarray) -> np.ndarray:
    """a_{t,i} = e^{z_i} / sum_j e^{z_j} over the whole history (Eq. (1)), computed with
    the max subtracted (the identity e^{z-m}/sum e^{z-m} = e^z/sum e^z)."""
    m = np.max(z)
    e = np.exp(z - m)
    return e / np.sum(e)


def threshold_set(z: np.ndarray, eps: float) -> np.ndarray:
    """I_{t,eps} = {i : a_{t,i} > eps} (Eq. (2)), ascending positions."""
    return np.nonzero(softmax_weights(z) > eps)[0]


def attention_mass(z: np.ndarray, U: np.ndarray) -> float:
    """Share of the full softmax mass that the positions U recover (the statistic of
    slide "The active tokens are sparse and dynamic", Fig. 2)."""
    return float(np.sum(softmax_weights(z)[np.asarray(U, dtype=np.int64)]))


# ------------------------------------------------------------------------------------
# the static set W and the candidates C ("The GPU keeps 640 fixed positions")


def static_set(N: int, n_sink: int, n_window: int) -> np.ndarray:
    """W: the first n_sink tokens plus the last n_window tokens, ascending, no repeats."""
    sink = np.arange(0, min(n_sink, N), dtype=np.int64)
    window = np.arange(max(0, N - n_window), N, dtype=np.int64)
    return np.union1d(sink, window)


def candidate_set(N: int, n_sink: int, n_window: int) -> np.ndarray:
    """C = [0, N) minus W: the positions the dynamic retrieval may return."""
    return np.setdiff1d(np.arange(N, dtype=np.int64), static_set(N, n_sink, n_window))


def select_topk(z: np.ndarray, C: np.ndarray, k: int) -> np.ndarray:
    """Omega: the min(k, |C|) candidates with the largest z (slide "Sparse attention
    renormalizes selected tokens": a fixed top-k budget rather than a threshold).
    Full sort by (z descending, position ascending), then take the head of the order."""
    C = np.asarray(C, dtype=np.int64)
    k_eff = min(max(k, 0), C.size)
    order = np.lexsort((C, -z[C]))
    return C[order[:k_eff]]


# ------------------------------------------------------------------------------------
# softmax over a selected set, partial states and their merge
# (slide "Two local softmax outputs need global weights", Eqs. (3)-(5), and the
#  slide "Backup: the normalization identity", Appendix B)


def attend(z: np.ndarray, V: np.ndarray, U: np.ndarray) -> np.ndarray:
    """o = sum_{i in U} e^{z_i} v_i / sum_{j in U} e^{z_j} (Eq. (2)'s renormalised sum
    over the selected set), evaluated with the max over U subtracted."""
    U = np.asarray(U, dtype=np.int64)
    zu = z[U]
    m = np.max(zu)
    w = np.exp(zu - m)
    return (w @ V[U]) / np.sum(w)


def partial_state(z: np.ndarray, V: np.ndarray, S: np.ndarray):
    """(m_S, Z_S, N_S) of one subset S: m_S = max z, Z_S = sum e^{z-m_S},
    N_S = sum e^{z-m_S} v (slide "Backup: the normalization identity", Appendix B).  o_S = N_S / Z_S."""
    S = np.asarray(S, dtype=np.int64)
    zs = z[S]
    m = float(np.max(zs))
    w = np.exp(zs - m)
    return m, float(np.sum(w)), w @ V[S]


def merge_partials(parts) -> np.ndarray:
    """o = sum_S gamma_S o_S with gamma_S = e^{m_S-m} Z_S / sum_T e^{m_T-m} Z_T and
    m = max_S m_S (Eqs. (3)-(5), generalised from the two parts W, Omega to any number of
    disjoint parts)."""
    m = max(p[0] for p in parts)
    den = sum(math.exp(mS - m) * ZS for mS, ZS, _ in parts)
    o = 0.0
    for mS, ZS, NS in parts:
        gamma = math.exp(mS - m) * ZS / den
        o = o + gamma * (NS / ZS)
    return np.asarray(o, dtype=np.float64)


# ------------------------------------------------------------------------------------
# the decode step


def decode_head(q_bits: np.ndarray, K_bits: np.ndarray, V_bits: np.ndarray, k: int,
                n_sink: int, n_window: int):
    """One query head: returns (o [d], Omega, z).  q [d], K/V [N, d] as bf16 bits."""
    q = bf16_to_f64(q_bits)
    K = bf16_to_f64(K_bits)
    V = bf16_to_f64(V_bits)
    N = K.shape[0]
    if N == 0:
        raise ValueError("empty cache")
    z = scores(q, K)
    W = static_set(N, n_sink, n_window)
    C = candidate_set(N, n_sink, n_window)
    omega = select_topk(z, C, k)
    U = np.concatenate([W, omega])
    if U.size == 0:
        raise ValueError("empty selected union")
    return attend(z, V, U), omega, z


def decode_step(q_bits: np.ndarray, K_bits: np.ndarray, V_bits: np.ndarray, k: int,
                n_sink: int, n_window: int):
    """All (b, h): out [B, Hq, d] float64 and Omega per (b, h) (list of lists).

    GQA: query head h reads KV head h // G with its own selection (slide "The GPU keeps
    640 fixed positions": GQA heads get separate indices but share KV storage)."""
    B, Hq, d = q_bits.shape
    Hkv = K_bits.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d), dtype=np.float64)
    omegas = [[None] * Hq for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            o, om, _ = decode_head(q_bits[b, h], K_bits[b, h // G], V_bits[b, h // G], k,
                                   n_sink, n_window)
            out[b, h] = o
            omegas[b][h] = om
    return out, omegas


def dense_head(q_bits: np.ndarray, K_bits: np.ndarray, V_bits: np.ndarray) -> np.ndarray:
    """Full attention of one query head over all N cached tokens (Eq. (1))."""
    q = bf16_to_f64(q_bits)
    K = bf16_to_f64(K_bits)
    V = bf16_to_f64(V_bits)
    z = scores(q, K)
    return attend(z, V, np.arange(K.shape[0]))


def dense_decode(q_bits: np.ndarray, K_bits: np.ndarray, V_bits: np.ndarray) -> np.ndarray:
    B, Hq, d = q_bits.shape
    G = Hq // K_bits.shape[1]
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            out[b, h] = dense_head(q_bits[b, h], K_bits[b, h // G], V_bits[b, h // G])
    return out


# ------------------------------------------------------------------------------------
# exact top-k of the prefill queries (slide "Prefill queries teach the key graph what
# matters": the prefill queries' exact top-k keys are the links the index is built from)


def prefill_score_matrix(Q_bits: np.ndarray, K_bits: np.ndarray) -> np.ndarray:
    """Z[m, i] = q_m k_i^T / sqrt(d) for the M queries of one head against its N keys
    (Eq. (1) for every query at once: one matrix product, exact on bf16 inputs in fp64)."""
    Q = bf16_to_f64(Q_bits)
    K = bf16_to_f64(K_bits)
    return (Q @ K.T) / math.sqrt(K.shape[1])


def prefill_topk(Q_bits: np.ndarray, K_bits: np.ndarray, k: int, n_sink: int,
                 n_window: int):
    """Omega for every prefill query: Q [B, Hq, M, d], K [B, Hkv, N, d] (bf16 bits).
    Query row (b, h, m) scores the keys of KV head h // G and keeps the min(k, |C|) largest
    over the same candidates C as the decode step (ties to the lower position).
    Returns a [B][Hq][M] nested list of position arrays."""
    B, Hq, M, _ = Q_bits.shape
    Hkv, N = K_bits.shape[1], K_bits.shape[2]
    G = Hq // Hkv
    C = candidate_set(N, n_sink, n_window)
    out = [[[None] * M for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            Z = prefill_score_matrix(Q_bits[b, h], K_bits[b, h // G])
            for m in range(M):
                out[b][h][m] = select_topk(Z[m], C, k)
    return out


# ------------------------------------------------------------------------------------
# threshold budget (Eq. (2): I_{t,eps} = {i : a_{t,i} > eps}, slide "Sparse attention
# renormalizes selected tokens")


def select_threshold(z: np.ndarray, C: np.ndarray, k: int, eps: float) -> np.ndarray:
    """Omega under a threshold: the candidates whose full softmax weight a_i (over all N
    positions, Eq. (1)) exceeds eps, cut to the k largest by (z descending, position ascending)
    when more than k pass."""
    a = softmax_weights(z)
    C = np.asarray(C, dtype=np.int64)
    passing = C[a[C] > eps]
    return select_topk(z, passing, k)


def decode_head_eps(q_bits: np.ndarray, K_bits: np.ndarray, V_bits: np.ndarray, k: int,
                    eps: float, n_sink: int, n_window: int):
    """One query head under the threshold budget: returns (o [d], Omega, z)."""
    q = bf16_to_f64(q_bits)
    K = bf16_to_f64(K_bits)
    V = bf16_to_f64(V_bits)
    N = K.shape[0]
    z = scores(q, K)
    W = static_set(N, n_sink, n_window)
    omega = select_threshold(z, candidate_set(N, n_sink, n_window), k, eps)
    U = np.concatenate([W, omega])
    if U.size == 0:
        raise ValueError("empty selected union")
    return attend(z, V, U), omega, z


def pyramid_budgets(L: int, k_mean: int, ratio: float) -> np.ndarray:
    """Per-layer budgets in the PyramidKV style (slide "Extra experiments show where budget
    matters": a layer budget that shrinks with depth): an arithmetic progression from k_max at
    layer 0 to ratio * k_max at layer L - 1 whose mean is k_mean, rounded down, with the
    remainder given one each to the lowest layers so that the total is exactly L * k_mean."""
    if L == 1:
        return np.array([k_mean], dtype=np.int64)
    k_max = 2.0 * k_mean / (1.0 + ratio)
    exact = [k_max * (1.0 - (1.0 - ratio) * l / (L - 1)) for l in range(L)]
    base = np.array([math.floor(x) for x in exact], dtype=np.int64)
    rem = L * k_mean - int(base.sum())
    base[:rem] += 1
    return base


# ------------------------------------------------------------------------------------
# paged caches (the serving layout): token i of sequence b, KV head g, is row i % P of page
# table[b][i // P] of the pool [num_pages, Hkv, P, d]


def gather_paged(pool: np.ndarray, table: np.ndarray, lens) -> list:
    """The dense [Hkv, N_b, d] cache of every sequence b, read out of a paged pool."""
    P = pool.shape[2]
    out = []
    for b, n in enumerate(lens):
        rows = [pool[table[b][i // P], :, i % P, :] for i in range(int(n))]
        out.append(np.stack(rows, axis=1) if rows else pool[:0, :, 0, :].transpose(1, 0, 2))
    return out


# ------------------------------------------------------------------------------------
# IVF retrieval (the pages' IVF baseline over the keys, slide "Available GPU memory changes
# the comparison"): given an index (keys grouped by cluster, unit-norm centroids), probe the
# nprobe clusters whose centroids score highest and take the exact top-k of their keys


def ivf_probe(q: np.ndarray, centroids: np.ndarray, nprobe: int) -> np.ndarray:
    """The nprobe clusters with the largest q . c (ties to the lower cluster index)."""
    zc = centroids @ q
    order = np.lexsort((np.arange(zc.size), -zc))
    return order[:nprobe]


def ivf_decode_head(q_bits: np.ndarray, K_bits: np.ndarray, V_bits: np.ndarray,
                    pos: np.ndarray, offsets: np.ndarray, cent_bits: np.ndarray, k: int,
                    nprobe: int, n_sink: int, n_window: int):
    """One query head through an IVF index of its KV head: returns (o [d], Omega, z, probe).
    pos [N_ix] are the cache positions grouped by cluster, offsets [nlist + 1] the groups."""
    q = bf16_to_f64(q_bits)
    K = bf16_to_f64(K_bits)
    V = bf16_to_f64(V_bits)
    N = K.shape[0]
    z = scores(q, K)
    probe = ivf_probe(q, bf16_to_f64(cent_bits), nprobe)
    cand = np.concatenate([pos[offsets[c]:offsets[c + 1]] for c in probe]).astype(np.int64)
    C = np.intersect1d(cand, candidate_set(N, n_sink, n_window))
    omega = select_topk(z, C, k)
    U = np.concatenate([static_set(N, n_sink, n_window), omega])
    return attend(z, V, U), omega, z, probe


# ------------------------------------------------------------------------------------
# IVF index construction (the pages name IVF over the keys as a baseline without fixing a
# construction; read as spherical k-means): centroids are unit vectors stored in bf16, keys go
# to the centroid of largest inner product, Lloyd iterations move each centroid to the unit
# direction of its keys' sum, and the index lists the keys cluster by cluster


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of the float64 values x, rounded to nearest with ties to
    even.  The two bf16 neighbours of x are found from a float32 copy truncated to its top 16
    bits and the next magnitude up, and the nearer one (exact float64 distances) is kept."""
    x = np.asarray(x, dtype=np.float64)
    t = x.astype(np.float32).view(np.uint32)
    sign = t & np.uint32(0x80000000)
    lo_bits = (t & np.uint32(0x7FFFFFFF)) >> np.uint32(16)
    hi_bits = lo_bits + np.uint32(1)
    lo = ((lo_bits << np.uint32(16)) | sign).view(np.float32).astype(np.float64)
    hi = ((hi_bits << np.uint32(16)) | sign).view(np.float32).astype(np.float64)
    dlo, dhi = np.abs(x - lo), np.abs(x - hi)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((lo_bits & np.uint32(1)) == 1))
    mag = np.where(pick_hi, hi_bits, lo_bits)
    return (mag | (sign >> np.uint32(16))).astype(np.uint16)


def unit_bf16(v: np.ndarray) -> np.ndarray:
    """bf16 bits of v / ||v|| (a zero vector stays zero)."""
    n = math.sqrt(float(np.sum(v * v)))
    return round_to_bf16(v / n if n > 0 else np.zeros_like(v))


def ivf_build(K_bits: np.ndarray, nlist: int, iters: int):
    """Spherical k-means index of one KV head's keys K [N, d] (bf16 bits).

    Centroid j starts as the unit key at position floor(j * N / nlist); each of `iters` Lloyd
    iterations assigns every key to the centroid of largest k . c (ties to the lower centroid)
    and moves every non-empty cluster's centroid to the unit direction of its keys' sum (an
    empty cluster keeps its centroid); a final assignment fixes the clusters.  Centroids are
    held as bf16.  Returns (centroid bits [nlist, d], assignment [N], the positions grouped by
    cluster in increasing position order [N], cluster offsets [nlist + 1])."""
    K = bf16_to_f64(K_bits)
    N = K.shape[0]
    cent = np.stack([unit_bf16(K[(j * N) // nlist]) for j in range(nlist)])
    for it in range(iters + 1):
        S = K @ bf16_to_f64(cent).T
        assign = np.argmax(S, axis=1)            # the first maximum: ties to the lower centroid
        if it == iters:
            break
        for j in range(nlist):
            members = assign == j
            if np.any(members):
                s = np.sum(K[members], axis=0)
                if np.sum(s * s) > 0:
                    cent[j] = unit_bf16(s)
    pos = np.argsort(assign, kind="stable")
    offsets = np.concatenate([[0], np.cumsum(np.bincount(assign, minlength=nlist))])
    return cent, assign, pos, offsets
