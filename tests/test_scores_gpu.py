"""The decode scan's fp32 scores against the oracle's fp64 scores (Eq. (1), slide "Sparse
attention renormalizes selected tokens"), element by element, read back from the step's
workspace (GPU only).

Bound: the scan sums bf16 x bf16 products in fp32, so each score may differ from the exact
value by at most d * 2^-24 * sum_c |q_c k_c| / sqrt(d); the tests allow 1e-5 * sum_c |q_c k_c| /
sqrt(d) + 1e-6 (about 10x that at d = 128, and far inside the selection's 1e-4 tie tolerance).
"""
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
