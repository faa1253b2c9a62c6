"""The threshold budget (Eq. (2): keep the candidates whose full softmax weight exceeds eps, at
most k of them) against the fp64 oracle, through the C ABI (GPU only)."""
import numpy as np
import pytest
import torch

import oracle
import top_retrieval_attention_b200 as ra
from gpu_util import cache_from_host, cache_from_workload, to_dev_bf16
from parity import check_omega_eps, check_out
from synth import gen

pytestmark = pytest.mark.gpu


def _host_case(seed, B, Hq, Hkv, N, d):
    q = gen.gen_q(seed, B, Hq, d)
    K = np.empty((B, Hkv, N, d), np.uint16)
    V = np.empty_like(K)
    for b in range(B):
        for g in range(Hkv):
            K[b, g] = gen.gen_k_rows(seed, 0, b, g, d, 0, N, True)
            V[b, g] = gen.gen_v_rows(seed, 0, b, g, d, 0, N)
    return q, K, V


def _check_head(q_bits, K_bits, V_bits, k, eps, n_sink, n_window, out_gpu, idx_gpu):
    z = oracle.scores(oracle.bf16_to_f64(q_bits), oracle.bf16_to_f64(K_bits))
    N = K_bits.shape[0]
    om_gpu = check_omega_eps(idx_gpu, z, N, n_sink, n_window, k, eps)
    U = np.concatenate([oracle.static_set(N, n_sink, n_window), om_gpu])
    check_out(out_gpu, oracle.attend(z, oracle.bf16_to_f64(V_bits), U))
    return om_gpu.size


CASES = [
    # B, Hq, Hkv, N, d, k, eps, n_sink, n_window
    (1, 8, 2, 5000, 128, 100, 1e-3, 4, 64),
    (1, 8, 2, 5000, 128, 100, 1e-5, 4, 64),     # the cap binds
    (2, 4, 4, 3000, 64, 2000, 1e-4, 0, 16),     # d = 64, G = 1
    (1, 16, 2, 9000, 128, 700, 2e-4, 128, 512), # G = 8
    (1, 4, 1, 70000, 128, 40000, 1e-6, 128, 512),  # large k: split attention, list overflow
    (1, 4, 1, 3000, 128, 50, 0.5, 8, 8),        # nothing passes: static set only
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,k,eps,n_sink,n_window", CASES)
def test_threshold_every_head(B, Hq, Hkv, N, d, k, eps, n_sink, n_window):
    q, K, V = _host_case(3000 + N + k, B, Hq, Hkv, N, d)
    cache = cache_from_host(K, V)
    out, idx = ra.decode_step_eps(cache, to_dev_bf16(q), k, eps, n_sink, n_window)
    torch.cuda.synchronize()
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            _check_head(q[b, h], K[b, h // G], V[b, h // G], k, eps, n_sink, n_window,
                        out[b, h], idx[b, h])


@pytest.mark.parametrize("eps", [1e-4, 2e-5, 4e-6])   # the mean weight is 1 / N = 7.6e-6
def test_threshold_llama8b_layer_128k(eps):
    w = gen.workload("l8b_128k_k1pct")
    cache, qd, nd = cache_from_workload(w)
    out, idx = ra.decode_step_eps(cache, qd, w.k, eps, w.n_sink, w.n_window)
    torch.cuda.synchronize()
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    qh = gen.gen_q(w.seed, w.B, w.Hq, w.d)
    kept = []
    for h in (0, 7, 21, 31):
        Kh, Vh = gen.host_head(w, 0, 0, h // w.G, w.N, nd)
        kept.append(_check_head(qh[0, h], Kh, Vh, w.k, eps, w.n_sink, w.n_window, out[0, h],
                                idx[0, h]))
    if eps < 1e-5:
        assert max(kept) > 0   # below the mean weight some candidates pass


def test_vanishing_threshold_equals_the_top_k_step():
    q, K, V = _host_case(77, 1, 8, 2, 6000, 128)
    cache = cache_from_host(K, V)
    qd = to_dev_bf16(q)
    out_e, idx_e = ra.decode_step_eps(cache, qd, 90, 1e-30, 4, 64)
    out_k, idx_k = ra.decode_step(cache, qd, 90, 4, 64)
    torch.cuda.synchronize()
    assert np.array_equal(np.sort(idx_e.cpu().numpy(), -1), np.sort(idx_k.cpu().numpy(), -1))
    np.testing.assert_allclose(out_e.cpu().numpy(), out_k.cpu().numpy(), rtol=1e-5, atol=1e-6)
