"""CUDA path against the fp64 oracle, element by element, through the C ABI (GPU only).

Small cases compare every query head; the full-size workloads (device-filled caches with the
same bits as the host generator) compare sampled heads, which the oracle recomputes from the
regenerated head data.
"""
import numpy as np
import pytest
import torch

import oracle
import top_retrieval_attention_b200 as ra
from gpu_util import cache_from_host, cache_from_workload, from_dev_bits, run_decode, to_dev_bf16
from parity import check_dense_head, check_head, check_out
from synth import device as sdev
from synth import gen

pytestmark = pytest.mark.gpu


def _host_case(seed, B, Hq, Hkv, N, d, offset=True):
    q = gen.gen_q(seed, B, Hq, d)
    K = np.empty((B, Hkv, N, d), np.uint16)
    V = np.empty_like(K)
    for b in range(B):
        for g in range(Hkv):
            K[b, g] = gen.gen_k_rows(seed, 0, b, g, d, 0, N, offset)
            V[b, g] = gen.gen_v_rows(seed, 0, b, g, d, 0, N)
    return q, K, V


def _check_all_heads(q, K, V, k, n_sink, n_window, out, idx):
    B, Hq, _ = q.shape
    G = Hq // K.shape[1]
    for b in range(B):
        for h in range(Hq):
            check_head(q[b, h], K[b, h // G], V[b, h // G], k, n_sink, n_window, out[b, h],
                       idx[b, h])


def test_device_generator_matches_host_bits():
    w = gen.Workload("t", 2, 8, 2, 128, 1000, 10, 4, 16, n_needle=3, seed=77)
    c, q, nd = cache_from_workload(w, layer=5, cap=1024)
    torch.cuda.synchronize()
    qh = gen.gen_q(77, 2, 8, 128)
    assert np.array_equal(from_dev_bits(q), qh)
    for b in range(2):
        for g in range(2):
            Kh, Vh = gen.host_head(w, 5, b, g, 1000, nd)
            assert np.array_equal(from_dev_bits(c.K[b, g, :1000]), Kh)
            assert np.array_equal(from_dev_bits(c.V[b, g, :1000]), Vh)
    for d in (64, 128):
        K = torch.empty((1, 1, 300, d), dtype=torch.bfloat16, device="cuda")
        V = torch.empty_like(K)
        sdev.fill_kv(K, V, 100, 150, 9, 2, with_offset=False)
        torch.cuda.synchronize()
        assert np.array_equal(from_dev_bits(K[0, 0, 100:250]), gen.gen_k_rows(9, 2, 0, 0, d, 100, 150, False))


SMALL = [
    # B, Hq, Hkv, N, d, k, n_sink, n_window
    (1, 4, 1, 1, 128, 1, 0, 0),
    (1, 4, 1, 7, 128, 3, 1, 2),
    (1, 2, 2, 640, 64, 10, 128, 512),      # C empty: W only
    (1, 2, 2, 641, 64, 10, 128, 512),      # one candidate
    (1, 8, 1, 4097, 128, 100, 4, 64),
    (2, 8, 4, 4097, 64, 50, 3, 17),
    (1, 8, 8, 3000, 128, 0, 16, 32),       # k = 0: static set only
    (1, 4, 1, 3000, 128, 1, 0, 0),         # k = 1, no static set
    (1, 4, 2, 2500, 128, 5000, 8, 8),      # k >= |C|: full attention
    (1, 16, 2, 9000, 128, 700, 128, 512),  # G = 8
    (3, 4, 4, 5000, 64, 257, 0, 64),       # G = 1, batch 3
    (1, 4, 1, 70000, 128, 900, 128, 512),  # a 16-CTA cluster per head, ragged chunks
    (1, 4, 1, 70000, 128, 40000, 128, 512),  # keys above b1 overflow a CTA's list: re-read path
    (2, 16, 2, 150000, 64, 3000, 3, 100),  # batch 2, G = 8, unaligned sink end
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,k,n_sink,n_window", SMALL)
def test_small_shapes_every_head(B, Hq, Hkv, N, d, k, n_sink, n_window):
    seed = 1000 + N + d + k
    q, K, V = _host_case(seed, B, Hq, Hkv, N, d)
    cache = cache_from_host(K, V, cap=N + 5)
    out, idx = run_decode(cache, to_dev_bf16(q), k, n_sink, n_window)
    _check_all_heads(q, K, V, k, n_sink, n_window, out, idx)
    dense = ra.dense_decode(cache, to_dev_bf16(q)).cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            check_dense_head(q[b, h], K[b, h // G], V[b, h // G], dense[b, h])


def test_k_at_least_candidates_equals_dense_on_gpu():
    q, K, V = _host_case(5, 1, 8, 2, 3333, 128)
    cache = cache_from_host(K, V)
    out, _ = run_decode(cache, to_dev_bf16(q), 3333, 4, 64)
    dense = ra.dense_decode(cache, to_dev_bf16(q)).cpu().numpy()
    np.testing.assert_allclose(out, dense, rtol=0, atol=2e-5)


def test_exact_ties_go_to_the_lower_position():
    rng = np.random.default_rng(3)
    N, d = 6000, 128
    q, K, V = _host_case(11, 1, 4, 1, N, d)
    # 40 copies of one strong key at random candidate positions: all tie exactly
    row = gen.needle_row(q[0, 0], 20.0)
    pos = rng.choice(np.arange(100, N - 100), size=40, replace=False)
    K[0, 0, pos] = row
    cache = cache_from_host(K, V)
    out, idx = run_decode(cache, to_dev_bf16(q), 25, 16, 16)
    _check_all_heads(q, K, V, 25, 16, 16, out, idx)
    assert set(idx[0, 0, :25].tolist()) == set(np.sort(pos)[:25].tolist())


def test_all_scores_equal_takes_the_lowest_positions():
    """Every key identical: one radix bucket holds all candidates (more than fit in shared
    memory), and the selection must be the k lowest candidate positions."""
    N, d = 20000, 64
    q, K, V = _host_case(12, 1, 2, 1, N, d)
    K[0, 0, :] = K[0, 0, 0]
    cache = cache_from_host(K, V)
    out, idx = run_decode(cache, to_dev_bf16(q), 5000, 4, 8)
    for h in range(2):
        assert set(idx[0, h].tolist()) == set(range(4, 5004))
    _check_all_heads(q, K, V, 5000, 4, 8, out, idx)


def test_phases_equal_the_step():
    q, K, V = _host_case(21, 1, 8, 2, 5000, 128)
    cache = cache_from_host(K, V)
    qd = to_dev_bf16(q)
    out1, idx1 = ra.decode_step(cache, qd, 77, 4, 64)
    ws = ra.decode_workspace(cache, 8, 77, 4, 64)
    out2 = torch.empty_like(out1)
    idx2 = torch.empty((1, 8, 77), dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert ra.ra_score_gqa(cache.kv, qd.data_ptr(), 8, 77, 4, 64, ws.data_ptr(), ws.numel(), s) == 0
    assert ra.ra_topk_select(cache.kv, 8, 77, 4, 64, idx2.data_ptr(), ws.data_ptr(), ws.numel(), s) == 0
    assert ra.ra_sparse_attn(cache.kv, 8, 77, 4, 64, idx2.data_ptr(), out2.data_ptr(),
                             ws.data_ptr(), ws.numel(), s) == 0
    out3 = torch.empty_like(out1)
    idx3 = torch.empty((1, 8, 77), dtype=torch.int32, device="cuda")
    assert ra.ra_score_gqa(cache.kv, qd.data_ptr(), 8, 77, 4, 64, ws.data_ptr(), ws.numel(), s) == 0
    assert ra.ra_select_attend(cache.kv, 8, 77, 4, 64, idx3.data_ptr(), out3.data_ptr(),
                               ws.data_ptr(), ws.numel(), s) == 0
    torch.cuda.synchronize()
    # Omega's order in idx (shared-memory list appends) decides the attention split, so sums
    # may round differently
    np.testing.assert_allclose(out1.cpu().numpy(), out2.cpu().numpy(), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(out1.cpu().numpy(), out3.cpu().numpy(), rtol=1e-5, atol=1e-6)
    assert np.array_equal(np.sort(idx1.cpu().numpy(), -1), np.sort(idx2.cpu().numpy(), -1))
    assert np.array_equal(np.sort(idx1.cpu().numpy(), -1), np.sort(idx3.cpu().numpy(), -1))


def test_append_then_decode_equals_decode_of_the_full_cache():
    q, K, V = _host_case(31, 2, 4, 2, 3001, 128)
    full = cache_from_host(K, V)
    out_full, idx_full = run_decode(full, to_dev_bf16(q), 60, 4, 32)
    grow = cache_from_host(K[:, :, :2990], V[:, :, :2990], cap=3001)
    ra.append_kv(grow, to_dev_bf16(K[:, :, 2990:]), to_dev_bf16(V[:, :, 2990:]))
    assert grow.N == 3001
    out_g, idx_g = run_decode(grow, to_dev_bf16(q), 60, 4, 32)
    np.testing.assert_allclose(out_g, out_full, rtol=1e-5, atol=1e-6)
    assert np.array_equal(np.sort(idx_g, -1), np.sort(idx_full, -1))


def test_repeated_calls_reuse_the_workspace():
    q, K, V = _host_case(41, 1, 8, 2, 7000, 128)
    cache = cache_from_host(K, V)
    qd = to_dev_bf16(q)
    ws = ra.decode_workspace(cache, 8, 300, 16, 64)
    first = None
    for _ in range(3):
        out, idx = ra.decode_step(cache, qd, 300, 16, 64, ws=ws)
        torch.cuda.synchronize()
        cur = (out.cpu().numpy(), np.sort(idx.cpu().numpy(), -1))
        if first is None:
            first = cur
        np.testing.assert_allclose(cur[0], first[0], rtol=1e-5, atol=1e-6)
        assert np.array_equal(cur[1], first[1])


# ------------------------------------------------------------------ named workloads


def _sampled(w: gen.Workload, heads, layer=0):
    cache, q, nd = cache_from_workload(w, layer)
    out, idx = run_decode(cache, q, w.k, w.n_sink, w.n_window)
    dense = ra.dense_decode(cache, q).cpu().numpy()
    qh = gen.gen_q(w.seed, w.B, w.Hq, w.d)
    hits = []
    for (b, h) in heads:
        g = h // w.G
        Kh, Vh = gen.host_head(w, layer, b, g, w.N, nd)
        check_head(qh[b, h], Kh, Vh, w.k, w.n_sink, w.n_window, out[b, h], idx[b, h])
        check_dense_head(qh[b, h], Kh, Vh, dense[b, h])
        if nd is not None:
            mine = nd.pos[b, g][nd.head[b, g] == h]
            hits.append(np.isin(mine, idx[b, h]).mean())
    del cache
    torch.cuda.empty_cache()
    return hits


def test_tiny_single_group_every_head():
    w = gen.workload("tiny")
    cache, q, nd = cache_from_workload(w)
    out, idx = run_decode(cache, q, w.k, w.n_sink, w.n_window)
    qh, K, V, nd_h = gen.host_layer(w)
    assert np.array_equal(from_dev_bits(cache.K[:, :, :w.N]), K)
    _check_all_heads(qh, K, V, w.k, w.n_sink, w.n_window, out, idx)


@pytest.mark.parametrize("name", ["l8b_128k_k100", "l8b_128k_k1pct"])
def test_llama8b_layer_128k(name):
    w = gen.workload(name)
    _sampled(w, [(0, 0), (0, 5), (0, 18), (0, 31)])


def test_llama8b_layer_1m_top2pct():
    w = gen.workload("l8b_1m_32layer")
    _sampled(w, [(0, 3), (0, 30)], layer=17)


def test_batch16_256k():
    w = gen.workload("l8b_b16_256k")
    _sampled(w, [(0, 0), (7, 13), (15, 31)])


@pytest.mark.parametrize("name", gen.sweep_names())
def test_sweep_point(name):
    w = gen.workload(name)
    _sampled(w, [(0, 9)])
