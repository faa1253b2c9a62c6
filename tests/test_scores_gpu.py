"""The decode scan's fp32 scores against the oracle's fp64 scores (Eq. (1), slide "Sparse
attention renormalizes selected tokens"), element by element, read back from the step's
workspace (GPU only).

Bound: the scan sums bf16 x bf16 products in fp32, so each score may differ from the exact
value by at most d * 2^-24 * sum_c |q_c k_c| / sqrt(d); the tests allow 1e-5 * sum_c |q_c k_c| /
sqrt(d) + 1e-6 (about 10x that at d = 128, and far inside the selection's 1e-4 tie tolerance).
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import top_retrieval_attention_b200 as ra
from gpu_util import cache_from_host, cache_from_workload, to_dev_bf16
from synth import gen

pytestmark = pytest.mark.gpu


def _align(x):
    return (x + 255) // 256 * 256


def _scores_in_workspace(ws, R, N):
    """The fp32 score rows of a decode workspace (layout: digit-1 histograms [R, 2048] u32,
    counters [R, 8] u32, then scores [R, round4(N)] fp32, each section 256-byte aligned)."""
    off = _align(R * 2048 * 4) + _align(R * 8 * 4)
    ldS = (N + 3) // 4 * 4
    return ws[off:off + R * ldS * 4].view(torch.float32).view(R, ldS)[:, :N].cpu().numpy()


def _check_row(got, q_bits, K_bits, what):
    q = oracle.bf16_to_f64(q_bits)
    K = oracle.bf16_to_f64(K_bits)
    z = oracle.scores(q, K)
    bound = 1e-5 * (np.abs(K) @ np.abs(q)) / math.sqrt(q.size) + 1e-6
    err = np.abs(got.astype(np.float64) - z)
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, f"{what}: {bad.size} scores off, e.g. position {bad[0]}: {got[bad[0]]} vs {z[bad[0]]}"


def _host_case(seed, B, Hq, Hkv, N, d):
    q = gen.gen_q(seed, B, Hq, d)
    K = np.empty((B, Hkv, N, d), np.uint16)
    V = np.empty_like(K)
    for b in range(B):
        for g in range(Hkv):
            K[b, g] = gen.gen_k_rows(seed, 0, b, g, d, 0, N, True)
            V[b, g] = gen.gen_v_rows(seed, 0, b, g, d, 0, N)
    return q, K, V


SMALL = [
    # B, Hq, Hkv, N, d, k
    (1, 4, 1, 300, 128, 10),          # under three tiles, ragged end
    (2, 8, 4, 4097, 64, 50),          # d = 64 (256-key tiles), batch 2
    (1, 16, 2, 9000, 128, 700),       # G = 8
    (3, 4, 4, 5000, 64, 257),         # G = 1, batch 3
    (1, 32, 8, 20000, 128, 200),      # Llama-3-8B heads
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,k", SMALL)
def test_every_score_of_small_shapes(B, Hq, Hkv, N, d, k):
    q, K, V = _host_case(3000 + N + d, B, Hq, Hkv, N, d)
    cache = cache_from_host(K, V, cap=N + 1)
    ws = ra.decode_workspace(cache, Hq, k, 4, 64)
    ra.decode_step(cache, to_dev_bf16(q), k, 4, 64, ws=ws)
    torch.cuda.synchronize()
    S = _scores_in_workspace(ws, B * Hq, N)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            _check_row(S[b * Hq + h], q[b, h], K[b, h // G], f"b {b} h {h}")


@pytest.mark.parametrize("N", [4096, 4097, 5000])
def test_scores_with_the_token_appended_inside_the_scan(N):
    """The fused step writes the new token's key into the staged tile before scoring it: the
    appended position's score (and every other) matches the oracle's over the grown cache."""
    B, Hq, Hkv, d, k = 1, 8, 2, 128, 40
    q, K, V = _host_case(8800 + N, B, Hq, Hkv, N, d)
    cache = cache_from_host(K[:, :, :N - 1], V[:, :, :N - 1], cap=N)
    ws = torch.zeros(ra.ra_decode_workspace_bytes(B, Hq, N, d, k, 4, 64), dtype=torch.uint8,
                     device="cuda")
    ra.decode_step_append(cache, to_dev_bf16(q), to_dev_bf16(K[:, :, N - 1:]),
                          to_dev_bf16(V[:, :, N - 1:]), k, 4, 64, ws=ws)
    torch.cuda.synchronize()
    assert cache.N == N
    S = _scores_in_workspace(ws, B * Hq, N)
    for h in range(Hq):
        _check_row(S[h], q[0, h], K[0, h // (Hq // Hkv)], f"h {h}")


def _sampled_workload(name, heads, layer=0):
    w = gen.workload(name)
    cache, q, nd = cache_from_workload(w, layer)
    ws = ra.decode_workspace(cache, w.Hq, w.k, w.n_sink, w.n_window)
    ra.decode_step(cache, q, w.k, w.n_sink, w.n_window, ws=ws)
    torch.cuda.synchronize()
    qh = gen.gen_q(w.seed, w.B, w.Hq, w.d)
    R, ldS = w.B * w.Hq, (w.N + 3) // 4 * 4
    off = _align(R * 2048 * 4) + _align(R * 8 * 4)
    for (b, h) in heads:
        r = b * w.Hq + h
        row = ws[off + r * ldS * 4: off + r * ldS * 4 + w.N * 4].view(torch.float32).cpu().numpy()
        Kh, _ = gen.host_head(w, layer, b, h // w.G, w.N, nd)
        _check_row(row, qh[b, h], Kh, f"{name} b {b} h {h}")
    del cache, ws
    torch.cuda.empty_cache()


def test_sampled_heads_of_the_128k_layer():
    _sampled_workload("l8b_128k_k1pct", [(0, 5), (0, 30)])


def test_sampled_head_of_the_1m_layer():
    _sampled_workload("l8b_1m_32layer", [(0, 3)], layer=17)


# ---- the scan's digit-1 histogram
#
# The selection's first radix digit is a bin of the score: with a the bits [17, 31) of the fp32
# score's pattern (exponent and top 6 mantissa bits of |z|) and m = clamp(a - A0, 0, 1023),
# A0 = 119 * 64 - 1 (so m = 1 starts at |z| = 2^-8), the bin is 1024 + m for z >= +0 and
# 1023 - m for z < 0.  Restated here from that definition, on the scores the scan returned.
A0 = 119 * 64 - 1


def _bins(S):
    u = np.ascontiguousarray(S, dtype=np.float32).view(np.uint32)
    m = np.clip(((u >> 17) & 0x3FFF).astype(np.int64) - A0, 0, 1023)
    return np.where((u >> 31) == 1, 1023 - m, 1024 + m)


def test_bin_rule_on_known_scores():
    # -250 and 250: |z| = 2^7 (1 + 61/64 + ...), the last window step (m = 1022)
    z = np.array([-1e30, -256.0, -250.0, -1.0, -2 ** -8, -0.003, 0.0, 0.003, 2 ** -8, 1.0, 250.0,
                  256.0, 1e30], np.float32)
    assert _bins(z).tolist() == [0, 0, 1, 510, 1022, 1023, 1024, 1024, 1025, 1537, 2046, 2047, 2047]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,k", [(1, 8, 2, 5000, 128, 40), (2, 8, 8, 3000, 64, 100),
                                            (1, 32, 4, 20000, 128, 300)])
def test_scan_histogram_counts_every_candidate_in_its_bin(B, Hq, Hkv, N, d, k):
    """The scan alone (no selection behind it, which would clear the histograms): each row's
    2048 counts equal the bins of its candidate scores [n_sink, N - n_window), and no score is
    a negative zero."""
    q, K, V = _host_case(4100 + N + d, B, Hq, Hkv, N, d)
    cache = cache_from_host(K, V, cap=N + 1)
    n_sink, n_window = 4, 64
    R = B * Hq
    nb = ra.ra_decode_workspace_bytes(B, Hq, N, d, k, n_sink, n_window)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    qd = to_dev_bf16(q)
    sp = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ra.check(ra.ra_score_gqa(cache.kv, qd.data_ptr(), Hq, k, n_sink, n_window, ws.data_ptr(), nb,
                             sp), "score_gqa")
    torch.cuda.synchronize()
    hist = ws[:R * 2048 * 4].view(torch.int32).view(R, 2048).cpu().numpy()
    S = _scores_in_workspace(ws, R, N)
    assert not np.any((S == 0) & np.signbit(S))
    for r in range(R):
        want = np.bincount(_bins(S[r, n_sink:N - n_window]), minlength=2048)
        assert np.array_equal(hist[r], want), f"row {r}"


def _scaled_case(N, d, zs, seed):
    """One KV head whose scores against q = (s, 0, ..., 0) are (nearly) the given values: key i
    is (zs[i] * sqrt(d) / s, small noise) in bf16."""
    rng = np.random.default_rng(seed)
    s = 8.0
    X = np.zeros((N, d))
    X[:, 0] = zs * math.sqrt(d) / s
    X[:, 1:] = 1e-3 * rng.standard_normal((N, d - 1))
    K = gen.f64_to_bf16_bits(X)[None, None]
    V = gen.f64_to_bf16_bits(rng.standard_normal((N, d)))[None, None]
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = s
    return gen.f64_to_bf16_bits(q), K, V


@pytest.mark.parametrize("where,seed", [("above_256", 11), ("below_m256", 12), ("tiny_pos", 13),
                                        ("tiny_neg", 14), ("window_edge", 15),
                                        ("near_zero_wide", 16)])
def test_selection_when_the_threshold_is_in_a_catch_all_bin(where, seed):
    """Scores laid out so that the k-th largest candidate falls in each bin that shares no key
    prefix (z >= 256, z <= -256, 0 <= z < 2^-8, -2^-8 < z < 0, the last from two ranges), and in
    the first window bin just above 2^-8 with the bin below it crowded and about 270 keys equal
    to the k-th score (bf16 keys leave some 20 distinct scores): Omega and out against the
    oracle, and Omega against the exact top-k of the scan's own scores."""
    from parity import check_head
    N, d, k = 6000, 128, 300
    rng = np.random.default_rng(seed)
    if where == "above_256":
        zs = rng.uniform(200.0, 400.0, N)
    elif where == "below_m256":
        zs = rng.uniform(-600.0, -250.0, N)
    elif where == "tiny_pos":
        zs = rng.uniform(-0.01, 0.0042, N)
    elif where == "tiny_neg":
        zs = rng.uniform(-0.0045, 0.00005, N)
    elif where == "window_edge":
        zs = rng.uniform(0.0035, 0.00395, N)
    else:
        zs = rng.uniform(-0.1, 2 ** -8 * 1.05, N)
    q, K, V = _scaled_case(N, d, zs, 77)
    cache = cache_from_host(K, V, cap=N + 1)
    ws = ra.decode_workspace(cache, 1, k, 4, 64)
    out, idx = ra.decode_step(cache, to_dev_bf16(q), k, 4, 64, ws=ws)
    torch.cuda.synchronize()
    got = idx[0, 0].cpu().numpy()
    check_head(q[0, 0], K[0, 0], V[0, 0], k, 4, 64, out[0, 0].cpu().numpy(), got)
    # exactly the top-k of the scan's own fp32 scores, equal scores to the lower position
    S = _scores_in_workspace(ws, 1, N)[0].astype(np.float64)
    C = np.arange(4, N - 64)
    want = C[np.lexsort((C, -S[C]))[:k]]
    assert set(got[:k].tolist()) == set(want.tolist())
