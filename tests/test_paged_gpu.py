"""The decode step on paged caches with ragged sequence lengths, against the fp64 oracle on the
gathered per-sequence caches, through the C ABI (GPU only)."""
import numpy as np
import pytest
import torch

import oracle
import top_retrieval_attention_b200 as ra
from gpu_util import from_dev_bits, to_dev_bf16
from parity import check_head
from synth import gen

pytestmark = pytest.mark.gpu
PAGE = 128


def _paged_case(seed, lens, Hq, Hkv, d, spare_pages=3, extra_tokens=0):
    """Ragged sequences scattered into a shuffled page pool (with room for extra_tokens more
    per sequence).  Returns (cache, q bits, pool K bits, pool V bits, table)."""
    rng = np.random.default_rng(seed)
    B = len(lens)
    need = [(n + extra_tokens + PAGE - 1) // PAGE for n in lens]
    num_pages = sum(need) + spare_pages
    max_pages = max(need)
    order = rng.permutation(num_pages)
    table = np.zeros((B, max_pages), dtype=np.int32)
    j = 0
    for b in range(B):
        for p in range(need[b]):
            table[b, p] = order[j]
            j += 1
    Kp = gen.f64_to_bf16_bits(rng.standard_normal((num_pages, Hkv, PAGE, d)))
    Vp = gen.f64_to_bf16_bits(rng.standard_normal((num_pages, Hkv, PAGE, d)))
    # give each sequence a per-channel key offset, as the workloads do
    for b in range(B):
        off = 1.4 * rng.standard_normal((Hkv, 1, d))
        for p in range(need[b]):
            Kp[table[b, p]] = gen.f64_to_bf16_bits(oracle.bf16_to_f64(Kp[table[b, p]]) + off)
    cache = ra.PagedKVCache(B, Hkv, d, num_pages, max_pages)
    cache.K.copy_(to_dev_bf16(Kp))
    cache.V.copy_(to_dev_bf16(Vp))
    cache.block_table.copy_(torch.from_numpy(table))
    cache.set_lengths(lens)
    q = gen.gen_q(seed, B, Hq, d)
    return cache, q, Kp, Vp, table


CASES = [
    # lens, Hq, Hkv, d, k, n_sink, n_window
    ([300, 5000, 1, 129, 2048], 8, 2, 128, 100, 4, 64),
    ([7000, 3000], 32, 8, 128, 500, 128, 512),
    ([128, 256, 1000, 4097], 4, 4, 64, 50, 0, 16),
    ([640, 641, 9000], 16, 2, 128, 700, 128, 512),   # C empty, one candidate, G = 8
    ([70000, 20000], 4, 1, 128, 40000, 128, 512),    # large k: list overflow, split attention
]


@pytest.mark.parametrize("lens,Hq,Hkv,d,k,n_sink,n_window", CASES)
def test_paged_decode_every_head(lens, Hq, Hkv, d, k, n_sink, n_window):
    cache, q, Kp, Vp, table = _paged_case(500 + sum(lens) + k, lens, Hq, Hkv, d)
    out, idx = ra.paged_decode_step(cache, to_dev_bf16(q), k, n_sink, n_window)
    torch.cuda.synchronize()
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    Ks = oracle.gather_paged(Kp, table, lens)
    Vs = oracle.gather_paged(Vp, table, lens)
    G = Hq // Hkv
    for b in range(len(lens)):
        for h in range(Hq):
            check_head(q[b, h], Ks[b][h // G], Vs[b][h // G], k, n_sink, n_window, out[b, h],
                       idx[b, h])


def test_paged_append_then_decode():
    lens = [1000, 2500, 130]
    Hq, Hkv, d, k = 8, 2, 128, 60
    cache, q, Kp, Vp, table = _paged_case(77, lens, Hq, Hkv, d, extra_tokens=3)
    rng = np.random.default_rng(78)
    T = 3
    kn = gen.f64_to_bf16_bits(rng.standard_normal((len(lens), Hkv, T, d)))
    vn = gen.f64_to_bf16_bits(rng.standard_normal((len(lens), Hkv, T, d)))
    ra.paged_append_kv(cache, to_dev_bf16(kn), to_dev_bf16(vn))
    assert cache.seq_len == [n + T for n in lens]
    out, idx = ra.paged_decode_step(cache, to_dev_bf16(q), k, 4, 32)
    torch.cuda.synchronize()
    # the host copy of the pool with the appended rows written by the layout's definition
    Kh = from_dev_bits(cache.K)
    Vh = from_dev_bits(cache.V)
    for b, n in enumerate(lens):
        for t in range(T):
            pos = n + t
            assert np.array_equal(Kh[table[b, pos // PAGE], :, pos % PAGE], kn[b, :, t])
            assert np.array_equal(Vh[table[b, pos // PAGE], :, pos % PAGE], vn[b, :, t])
    lens2 = cache.seq_len
    Ks = oracle.gather_paged(Kh, table, lens2)
    Vs = oracle.gather_paged(Vh, table, lens2)
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    for b in range(len(lens)):
        for h in range(Hq):
            check_head(q[b, h], Ks[b][h // (Hq // Hkv)], Vs[b][h // (Hq // Hkv)], k, 4, 32,
                       out[b, h], idx[b, h])


def test_paged_equals_dense_when_lengths_agree():
    """Equal lengths: the paged step equals the dense step on the gathered cache."""
    lens = [3000, 3000]
    Hq, Hkv, d, k = 8, 2, 128, 80
    cache, q, Kp, Vp, table = _paged_case(91, lens, Hq, Hkv, d)
    out_p, idx_p = ra.paged_decode_step(cache, to_dev_bf16(q), k, 4, 64)
    Ks = oracle.gather_paged(Kp, table, lens)
    Vs = oracle.gather_paged(Vp, table, lens)
    dense = ra.KVCache(2, Hkv, d, 3000)
    dense.K.copy_(to_dev_bf16(np.stack(Ks)))
    dense.V.copy_(to_dev_bf16(np.stack(Vs)))
    dense.N = 3000
    out_d, idx_d = ra.decode_step(dense, to_dev_bf16(q), k, 4, 64)
    torch.cuda.synchronize()
    assert np.array_equal(np.sort(idx_p.cpu().numpy(), -1), np.sort(idx_d.cpu().numpy(), -1))
    np.testing.assert_allclose(out_p.cpu().numpy(), out_d.cpu().numpy(), rtol=1e-5, atol=1e-6)
