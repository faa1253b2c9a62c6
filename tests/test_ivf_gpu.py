"""IVF retrieval on the device: the index the GPU builds (checked for structure and for the
spherical k-means assignment rule in fp64) and the decode step through it (checked against the
fp64 oracle given that index), through the C ABI (GPU only)."""
import numpy as np
import pytest
import torch

import oracle
import top_retrieval_attention_b200 as ra
from gpu_util import cache_from_host, from_dev_bits, to_dev_bf16
from parity import TIE_REL, check_out
from synth import gen

pytestmark = pytest.mark.gpu


def _case(seed, B, Hq, Hkv, N, d):
    q = gen.gen_q(seed, B, Hq, d)
    K = np.empty((B, Hkv, N, d), np.uint16)
    V = np.empty_like(K)
    for b in range(B):
        for g in range(Hkv):
            K[b, g] = gen.gen_k_rows(seed, 0, b, g, d, 0, N, True)
            V[b, g] = gen.gen_v_rows(seed, 0, b, g, d, 0, N)
    return q, K, V


def _index_host(ix):
    return (from_dev_bits(ix.Ksorted), ix.pos.cpu().numpy(), ix.offsets.cpu().numpy(),
            from_dev_bits(ix.centroids))


@pytest.mark.parametrize("N,d,nlist,iters", [(5000, 128, 32, 3), (3000, 64, 16, 0), (20000, 128, 100, 4)])
def test_ivf_build_structure_and_assignment(N, d, nlist, iters):
    q, K, V = _case(N + nlist, 2, 4, 2, N, d)
    cache = cache_from_host(K, V, cap=N + 7)
    ix = ra.ivf_build(cache, nlist, iters)
    torch.cuda.synchronize()
    Ks, pos, offs, cent = _index_host(ix)
    for b in range(2):
        for g in range(2):
            o = offs[b, g]
            assert o[0] == 0 and o[-1] == N and np.all(np.diff(o) >= 0)
            assert np.array_equal(np.sort(pos[b, g]), np.arange(N))      # a permutation
            assert np.array_equal(Ks[b, g], K[b, g][pos[b, g]])         # the keys, regrouped
            C = oracle.bf16_to_f64(cent[b, g])
            norms = np.linalg.norm(C, axis=1)
            assert np.all(np.abs(norms - 1.0) < 2e-2)                   # unit norm (bf16)
            Kf = oracle.bf16_to_f64(K[b, g])
            S = Kf @ C.T                                                # exact key-centroid scores
            cl = np.repeat(np.arange(nlist), np.diff(o))                # cluster of each sorted key
            got = S[pos[b, g], cl]
            best = S[pos[b, g]].max(axis=1)
            # each key sits in a centroid of (near) largest inner product (fp32 products)
            tol = 1e-5 * (np.abs(Kf[pos[b, g]]) @ np.abs(C).T).max(axis=1) + 1e-6
            assert np.all(got >= best - tol)


def _check_ivf_head(qh, Kh, Vh, pos, offs, cent, k, nprobe, n_sink, n_window, out, idx_row):
    o_ref, om, z, probe = oracle.ivf_decode_head(qh, Kh, Vh, pos, offs, cent, k, nprobe,
                                                 n_sink, n_window)
    N = Kh.shape[0]
    got = idx_row[idx_row >= 0]
    assert np.unique(got).size == got.size
    assert np.all(np.isin(got, oracle.candidate_set(N, n_sink, n_window)))
    # the probe boundary may tie in fp32: then only membership in the probed clusters is checked
    zc = oracle.bf16_to_f64(cent) @ oracle.bf16_to_f64(qh)
    srt = np.sort(zc)[::-1]
    ambiguous = nprobe < zc.size and abs(srt[nprobe - 1] - srt[nprobe]) <= TIE_REL * max(1.0, abs(srt[nprobe - 1]))
    if not ambiguous:
        diff = set(got.tolist()) ^ set(om.tolist())
        if diff:
            s_k = z[om[-1]]
            bad = [a for a in diff if abs(z[a] - s_k) > TIE_REL * max(1.0, abs(s_k))]
            assert not bad, bad[:5]
    U = np.concatenate([oracle.static_set(N, n_sink, n_window), got])
    check_out(out, oracle.attend(z, oracle.bf16_to_f64(Vh), U))
    return om, got


@pytest.mark.parametrize("N,d,nlist,nprobe,k", [(6000, 128, 48, 8, 100), (4000, 64, 20, 5, 300)])
def test_ivf_decode_against_the_oracle(N, d, nlist, nprobe, k):
    B, Hq, Hkv = 1, 8, 2
    q, K, V = _case(17 + N, B, Hq, Hkv, N, d)
    cache = cache_from_host(K, V)
    ix = ra.ivf_build(cache, nlist, 3)
    out, idx = ra.ivf_decode_step(cache, ix, to_dev_bf16(q), k, nprobe, 16, 64)
    torch.cuda.synchronize()
    Ks, pos, offs, cent = _index_host(ix)
    out, idx = out.cpu().numpy(), idx.cpu().numpy()
    for h in range(Hq):
        g = h // (Hq // Hkv)
        _check_ivf_head(q[0, h], K[0, g], V[0, g], pos[0, g], offs[0, g], cent[0, g], k, nprobe,
                        16, 64, out[0, h], idx[0, h])


def test_ivf_probing_every_cluster_equals_the_exact_step():
    B, Hq, Hkv, N, d, nlist, k = 1, 8, 2, 5000, 128, 24, 150
    q, K, V = _case(555, B, Hq, Hkv, N, d)
    cache = cache_from_host(K, V)
    ix = ra.ivf_build(cache, nlist, 2)
    out_i, idx_i = ra.ivf_decode_step(cache, ix, to_dev_bf16(q), k, nlist, 8, 32)
    out_e, idx_e = ra.decode_step(cache, to_dev_bf16(q), k, 8, 32)
    torch.cuda.synchronize()
    assert np.array_equal(np.sort(idx_i.cpu().numpy(), -1), np.sort(idx_e.cpu().numpy(), -1))
    np.testing.assert_allclose(out_i.cpu().numpy(), out_e.cpu().numpy(), rtol=1e-5, atol=1e-6)


def test_ivf_covers_tokens_appended_after_the_build_through_the_window():
    B, Hq, Hkv, N, d, k = 1, 4, 1, 3000, 128, 50
    q, K, V = _case(777, B, Hq, Hkv, N + 5, d)
    cache = cache_from_host(K[:, :, :N], V[:, :, :N], cap=N + 5)
    ix = ra.ivf_build(cache, 16, 2)
    ra.append_kv(cache, to_dev_bf16(K[:, :, N:]), to_dev_bf16(V[:, :, N:]))
    out, idx = ra.ivf_decode_step(cache, ix, to_dev_bf16(q), k, 4, 4, 32)
    torch.cuda.synchronize()
    Ks, pos, offs, cent = _index_host(ix)
    _check_ivf_head(q[0, 0], K[0, 0], V[0, 0], pos[0, 0], offs[0, 0], cent[0, 0], k, 4, 4, 32,
                    out.cpu().numpy()[0, 0], idx.cpu().numpy()[0, 0])
