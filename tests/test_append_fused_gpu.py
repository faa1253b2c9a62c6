"""The decode step with the token's append fused into the scan (ra_decode_step_append) through
the C ABI: it must give what ra_append_kv followed by ra_decode_step gives (the same cache rows
and retrieved set, the output up to fp32 summation order), and match the fp64 oracle over the
grown cache.  The new
token lands on the first, a middle and the last row of a score tile, in an empty cache, and
(with no window) as a candidate that the selection must rank (GPU only)."""
import numpy as np
import pytest
import torch

import oracle
import top_retrieval_attention_b200 as ra
from gpu_util import cache_from_host, from_dev_bits, to_dev_bf16
from parity import check_head
from synth import gen

pytestmark = pytest.mark.gpu


def _rows(seed, B, Hkv, N, d):
    K = np.empty((B, Hkv, N, d), np.uint16)
    V = np.empty_like(K)
    for b in range(B):
        for g in range(Hkv):
            K[b, g] = gen.gen_k_rows(seed, 0, b, g, d, 0, N, True)
            V[b, g] = gen.gen_v_rows(seed, 0, b, g, d, 0, N)
    return K, V


def _both_paths(q, K, V, k, n_sink, n_window):
    """(out, idx, K rows, V rows) of the separate and the fused path, caches of N - 1 tokens
    plus the token at N - 1."""
    B, Hkv, N, d = K.shape
    res = []
    for fused in (False, True):
        cache = cache_from_host(K[:, :, :N - 1], V[:, :, :N - 1], cap=N + 3)
        kn, vn = to_dev_bf16(K[:, :, N - 1:N]), to_dev_bf16(V[:, :, N - 1:N])
        qd = to_dev_bf16(q)
        if fused:
            out, idx = ra.decode_step_append(cache, qd, kn, vn, k, n_sink, n_window)
        else:
            ra.append_kv(cache, kn, vn)
            out, idx = ra.decode_step(cache, qd, k, n_sink, n_window)
        torch.cuda.synchronize()
        assert cache.N == N
        res.append((out.cpu().numpy(), idx.cpu().numpy(), from_dev_bits(cache.K[:, :, :N]),
                    from_dev_bits(cache.V[:, :, :N])))
    return res


@pytest.mark.parametrize("N,d,k,n_sink,n_window", [
    (129, 128, 20, 4, 16),      # the token is row 0 of the second tile
    (256, 128, 30, 4, 16),      # row 127 of the second tile
    (5000, 64, 100, 16, 64),    # a middle row, d = 64
    (1, 128, 5, 4, 16),         # an empty cache: the token is the whole step
    (4097, 128, 300, 8, 0),     # no window: the token is a candidate
    (256, 64, 20, 4, 16),       # d = 64 scans 256-key tiles: row 255 of the first tile
    (257, 64, 20, 4, 16),       # row 0 of the second 256-key tile
])
def test_fused_append_equals_append_then_decode_and_the_oracle(N, d, k, n_sink, n_window):
    B, Hq, Hkv = 2, 8, 2
    q = gen.gen_q(41 + N, B, Hq, d)
    K, V = _rows(43 + N, B, Hkv, N, d)
    (o1, i1, K1, V1), (o2, i2, K2, V2) = _both_paths(q, K, V, k, n_sink, n_window)
    assert np.array_equal(K1, K) and np.array_equal(V1, V)
    assert np.array_equal(K2, K) and np.array_equal(V2, V)
    # the same set and the same output up to the summation order (idx is a set filled by
    # atomics, so the attention may add its entries in another order)
    assert np.array_equal(np.sort(i1, -1), np.sort(i2, -1))
    np.testing.assert_allclose(o2, o1, rtol=1e-5, atol=1e-6)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            check_head(q[b, h], K[b, h // G], V[b, h // G], k, n_sink, n_window, o2[b, h], i2[b, h])


def test_appended_needle_is_scored_from_the_patched_tile():
    # the new key points along query head 0's direction with a score far above every other
    # candidate: with no window it is a candidate, and query head 0 must retrieve it
    B, Hq, Hkv, N, d, k = 1, 4, 1, 3000, 128, 10
    q = gen.gen_q(77, B, Hq, d)
    K, V = _rows(79, B, Hkv, N, d)
    qh = oracle.bf16_to_f64(q[0, 0])
    z_max = (oracle.bf16_to_f64(K[0, 0, :N - 1]) @ qh).max()
    lam = (z_max + 8.0 * np.sqrt(d)) / np.linalg.norm(qh)
    K[0, 0, N - 1] = gen.f64_to_bf16_bits(lam * qh / np.linalg.norm(qh))
    cache = cache_from_host(K[:, :, :N - 1], V[:, :, :N - 1], cap=N)
    out, idx = ra.decode_step_append(cache, to_dev_bf16(q), to_dev_bf16(K[:, :, N - 1:N]),
                                     to_dev_bf16(V[:, :, N - 1:N]), k, 2, 0)
    torch.cuda.synchronize()
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    assert N - 1 in set(idx[0, 0].tolist())
    for h in range(Hq):
        check_head(q[0, h], K[0, 0], V[0, 0], k, 2, 0, out[0, h], idx[0, h])
