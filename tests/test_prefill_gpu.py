"""Exact top-k of prefill queries (tcgen05 score GEMM + cluster selection) against the fp64
oracle, through the C ABI (GPU only).

Every query row's selection is checked with the decode rules (exact set up to near ties);
the tensor-core scores themselves are compared with the oracle's score matrix on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import top_retrieval_attention_b200 as ra
from gpu_util import cache_from_host, to_dev_bf16
from parity import check_omega
from synth import gen

pytestmark = pytest.mark.gpu


def _case(seed, B, Hq, Hkv, M, N, d):
    Q = np.empty((B, Hq, M, d), np.uint16)
    for b in range(B):
        Q[b] = gen.gen_q(seed + 17 * b, Hq, M, d).reshape(Hq, M, d)
    K = np.empty((B, Hkv, N, d), np.uint16)
    V = np.empty_like(K)
    for b in range(B):
        for g in range(Hkv):
            K[b, g] = gen.gen_k_rows(seed, 0, b, g, d, 0, N, True)
            V[b, g] = gen.gen_v_rows(seed, 0, b, g, d, 0, N)
    return Q, K, V


def _align(x):
    return (x + 255) // 256 * 256


def _scores_in_workspace(ws, B, Hq, M, N):
    """The fp32 score rows the prefill kernel left in the workspace (layout: digit-1
    histograms [R, 2048] u32, counters [R, 8] u32, then scores [R, round4(N)] fp32)."""
    R = B * Hq * M
    off = _align(R * 2048 * 4) + _align(R * 8 * 4)
    ldS = (N + 3) // 4 * 4
    return ws[off:off + R * ldS * 4].view(torch.float32).view(R, ldS)[:, :N]


CASES = [
    # B, Hq, Hkv, M, N, d, k, n_sink, n_window
    (1, 4, 1, 32, 300, 128, 10, 4, 16),          # one tile each way, ragged keys
    (1, 8, 2, 37, 5000, 128, 100, 128, 512),     # 148 rows per KV head: two row blocks
    (2, 4, 4, 130, 3000, 64, 50, 0, 64),         # d = 64, G = 1, batch 2
    (1, 16, 2, 40, 2048, 128, 3000, 8, 8),       # G = 8, k >= |C|: every candidate
    (1, 4, 1, 20, 1000, 128, 0, 4, 4),           # k = 0
    (1, 32, 8, 16, 20000, 128, 200, 128, 512),   # Llama-3-8B heads, several clusters per row
]


@pytest.mark.parametrize("B,Hq,Hkv,M,N,d,k,n_sink,n_window", CASES)
def test_prefill_topk_every_query(B, Hq, Hkv, M, N, d, k, n_sink, n_window):
    Q, K, V = _case(7000 + N + M + d, B, Hq, Hkv, M, N, d)
    cache = cache_from_host(K, V, cap=N + 3)
    qd = to_dev_bf16(Q)
    n = ra.ra_prefill_workspace_bytes(B, Hq, M, N, d, k, n_sink, n_window)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    idx = ra.prefill_topk(cache, qd, k, n_sink, n_window, ws=ws)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    S = _scores_in_workspace(ws, B, Hq, M, N).cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            Z = oracle.prefill_score_matrix(Q[b, h], K[b, h // G])
            # tensor-core scores: fp32 accumulation of exact bf16 products
            Qf = oracle.bf16_to_f64(Q[b, h])
            Kf = oracle.bf16_to_f64(K[b, h // G])
            bound = 1e-5 * (np.abs(Qf) @ np.abs(Kf).T) / np.sqrt(d) + 1e-6
            rows = S[(b * Hq + h) * M:(b * Hq + h + 1) * M]
            assert np.all(np.abs(rows - Z) <= bound), float(np.max(np.abs(rows - Z) - bound))
            for m in range(M):
                if k == 0:
                    continue
                check_omega(idx[b, h, m], Z[m], N, n_sink, n_window, k)


def test_prefill_phases_equal_the_call():
    B, Hq, Hkv, M, N, d, k = 1, 8, 2, 50, 4000, 128, 64
    Q, K, V = _case(91, B, Hq, Hkv, M, N, d)
    cache = cache_from_host(K, V)
    qd = to_dev_bf16(Q)
    idx1 = ra.prefill_topk(cache, qd, k, 16, 64)
    n = ra.ra_prefill_workspace_bytes(B, Hq, M, N, d, k, 16, 64)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    idx2 = torch.empty((B, Hq, M, k), dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert ra.ra_prefill_score(cache.kv, qd.data_ptr(), Hq, M, k, 16, 64, ws.data_ptr(), n, s) == 0
    assert ra.ra_prefill_select(cache.kv, Hq, M, k, 16, 64, idx2.data_ptr(), ws.data_ptr(), n, s) == 0
    torch.cuda.synchronize()
    a = np.sort(idx1.cpu().numpy(), -1)
    b = np.sort(idx2.cpu().numpy(), -1)
    assert np.array_equal(a, b)


def test_prefill_of_one_query_equals_the_decode_selection():
    B, Hq, Hkv, N, d, k = 1, 8, 2, 6000, 128, 77
    Q, K, V = _case(93, B, Hq, Hkv, 1, N, d)
    cache = cache_from_host(K, V)
    idx_p = ra.prefill_topk(cache, to_dev_bf16(Q), k, 4, 64)
    _, idx_d = ra.decode_step(cache, to_dev_bf16(np.ascontiguousarray(Q[:, :, 0])), k, 4, 64)
    torch.cuda.synchronize()
    assert np.array_equal(np.sort(idx_p.cpu().numpy()[:, :, 0], -1), np.sort(idx_d.cpu().numpy(), -1))
