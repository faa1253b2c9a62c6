"""IVF retrieval on the device, through the C ABI (GPU only): the index the GPU builds against
the fp64 oracle's spherical k-means (oracle.ivf_build), its determinism and structure, and the
decode step through it against the fp64 oracle given that index."""
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


def _separated_keys(seed, Hkv, N, d, nlist):
    """Keys of nlist well-separated directions, block j of positions [j N / nlist, (j+1) N /
    nlist) along direction u_j with magnitudes in [1, 3) and a little noise: the evenly spaced
    starting keys fall one in each block and no key is near a tie between two centroids."""
    rng = np.random.default_rng(seed)
    K = np.empty((1, Hkv, N, d), np.uint16)
    for g in range(Hkv):
        U = rng.standard_normal((nlist, d))
        U /= np.linalg.norm(U, axis=1, keepdims=True)
        blk = (np.arange(N) * nlist) // N
        X = U[blk] * rng.uniform(1.0, 3.0, (N, 1)) + 0.03 * rng.standard_normal((N, d))
        K[0, g] = gen.f64_to_bf16_bits(X)
    return K


def _centroid_bits_close(got, want, exact):
    """Centroid bits equal, except an element whose exact unit value lies within 1e-5 relative
    of the midpoint between two bf16 values: fp32 arithmetic may round it either way (one ulp)."""
    diff = got.astype(np.int32) - want.astype(np.int32)
    if not np.any(diff):
        return
    lo = oracle.bf16_to_f64(np.minimum(got, want))
    hi = oracle.bf16_to_f64(np.maximum(got, want))
    mid = (lo + hi) / 2
    near = np.abs(exact - mid) <= 1e-5 * np.maximum(np.abs(exact), 1e-30)
    assert np.all((diff == 0) | ((np.abs(diff) == 1) & near)), np.argwhere((diff != 0) & ~near)[:5]


def _exact_units(K_bits, assign, cent_bits, nlist):
    """The fp64 unit direction each centroid was rounded from (its cluster's key sum, or the
    centroid itself when the cluster is empty)."""
    K = oracle.bf16_to_f64(K_bits)
    out = oracle.bf16_to_f64(cent_bits).copy()
    for j in range(nlist):
        m = assign == j
        if np.any(m):
            s = K[m].sum(axis=0)
            out[j] = s / np.linalg.norm(s)
    return out


@pytest.mark.parametrize("N,d,nlist,iters", [(4096, 128, 16, 3), (3000, 64, 12, 2), (9000, 128, 40, 4)])
def test_ivf_build_matches_the_oracle_on_separated_clusters(N, d, nlist, iters):
    Hkv = 2
    K = _separated_keys(N + d + nlist, Hkv, N, d, nlist)
    cache = cache_from_host(K, K.copy(), cap=N + 3)
    ix = ra.ivf_build(cache, nlist, iters)
    torch.cuda.synchronize()
    Ks, pos, offs, cent = _index_host(ix)
    for g in range(Hkv):
        c_o, a_o, p_o, o_o = oracle.ivf_build(K[0, g], nlist, iters)
        assert np.array_equal(offs[0, g], o_o)
        assert np.array_equal(pos[0, g], p_o)
        assert np.array_equal(Ks[0, g], K[0, g][p_o])
        # the last update ran with the previous assignment, which on these keys is the final one
        _centroid_bits_close(cent[0, g], c_o, _exact_units(K[0, g], a_o, c_o, nlist))


def test_ivf_build_matches_the_oracle_at_the_start():
    """The decode workload's own keys (offset channels, no planted structure), no iteration: the
    starting centroids are the unit keys at evenly spaced positions, and every key joins the
    oracle's centroid except where two centroid scores tie within the fp32 tolerance."""
    N, d, nlist = 6000, 128, 48
    _, K, V = _case(4242, 1, 4, 2, N, d)
    cache = cache_from_host(K, V)
    ix = ra.ivf_build(cache, nlist, 0)
    torch.cuda.synchronize()
    Ks, pos, offs, cent = _index_host(ix)
    for g in range(2):
        c_o, a_o, _, _ = oracle.ivf_build(K[0, g], nlist, 0)
        Kf = oracle.bf16_to_f64(K[0, g])
        starts = Kf[(np.arange(nlist) * N) // nlist]
        _centroid_bits_close(cent[0, g], c_o, starts / np.linalg.norm(starts, axis=1, keepdims=True))
        C = oracle.bf16_to_f64(cent[0, g])
        S = Kf @ C.T
        a_gpu = np.repeat(np.arange(nlist), np.diff(offs[0, g]))[np.argsort(pos[0, g])]
        tol = 1e-5 * (np.abs(Kf) @ np.abs(C).T).max(axis=1) + 1e-6
        differ = np.nonzero(a_gpu != a_o)[0]
        for i in differ:   # only near-ties may go either way
            assert S[i, a_gpu[i]] >= S[i, a_o[i]] - tol[i], (i, a_gpu[i], a_o[i])
        assert differ.size <= N // 100
        # listing: by cluster, increasing position inside a cluster
        for c in range(nlist):
            seg = pos[0, g][offs[0, g][c]:offs[0, g][c + 1]]
            assert np.all(np.diff(seg) > 0) and np.all(a_gpu[seg] == c)


def test_ivf_build_is_deterministic():
    N, d, nlist = 20000, 128, 100
    _, K, V = _case(99, 1, 8, 2, N, d)
    cache = cache_from_host(K, V)
    a = _index_host(ra.ivf_build(cache, nlist, 3))
    b = _index_host(ra.ivf_build(cache, nlist, 3))
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


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
            for c in range(nlist):                                      # position order inside
                assert np.all(np.diff(pos[b, g][o[c]:o[c + 1]]) > 0)


def _check_ivf_head(qh, Kh, Vh, pos, offs, cent, k, nprobe, n_sink, n_window, out, idx_row):
    o_ref, om, z, probe = oracle.ivf_decode_head(qh, Kh, Vh, pos, offs, cent, k, nprobe,
                                                 n_sink, n_window)
    N = Kh.shape[0]
    C = oracle.candidate_set(N, n_sink, n_window)
    got = idx_row[idx_row >= 0]
    assert np.unique(got).size == got.size
    assert np.all(np.isin(got, C))
    zc = oracle.bf16_to_f64(cent) @ oracle.bf16_to_f64(qh)
    srt = np.sort(zc)[::-1]
    thr = srt[nprobe - 1]
    tol = TIE_REL * max(1.0, abs(thr))
    ambiguous = nprobe < zc.size and abs(thr - srt[nprobe]) <= tol
    if not ambiguous:
        diff = set(got.tolist()) ^ set(om.tolist())
        if diff:
            s_k = z[om[-1]]
            bad = [a for a in diff if abs(z[a] - s_k) > TIE_REL * max(1.0, abs(s_k))]
            assert not bad, bad[:5]
    else:
        # the probe boundary ties in fp32: the GPU probed every cluster scoring clearly above
        # the nprobe-th best ("sure") and then some of those within the tie tolerance of it.
        # Its keys come from the widened set, its Omega holds every key that is in the exact
        # top-k of the widened candidates and belongs to a sure cluster, and it is full.
        def keys_of(cl):
            return np.intersect1d(np.concatenate([pos[offs[c]:offs[c + 1]] for c in cl] or [[]]), C)
        wide = keys_of(np.nonzero(zc >= thr - tol)[0])
        sure = keys_of(np.nonzero(zc > thr + tol)[0])
        assert np.all(np.isin(got, wide)), np.setdiff1d(got, wide)[:5]
        top_wide = oracle.select_topk(z, wide, k)
        s_k = z[top_wide[-1]] if top_wide.size else 0.0
        must = [a for a in np.intersect1d(top_wide, sure)
                if z[a] > s_k + TIE_REL * max(1.0, abs(s_k))]
        assert np.all(np.isin(must, got)), np.setdiff1d(must, got)[:5]
        assert got.size >= min(k, sure.size)
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
