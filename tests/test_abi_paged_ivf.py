"""Host-side validation of the paged and IVF entry points (CPU only, no launch).

Every call here is one the library must refuse before enqueuing anything, so the pointers are
placeholders that are never dereferenced; the checks cover the status each wrong argument maps
to and that the caller's structs are left unchanged.
"""
import ctypes

import pytest

import top_retrieval_attention_b200 as ra

FAKE = 1 << 20   # a 16-byte aligned non-null address; never dereferenced on these paths
BIG = 1 << 40


def _paged(lens, Hkv=2, d=128, max_pages=4, num_pages=16):
    arr = (ctypes.c_int32 * len(lens))(*lens)
    kv = ra.ra_paged_kv(FAKE, FAKE, FAKE, arr, len(lens), Hkv, d, max_pages, num_pages)
    return kv, arr


def test_paged_append_checks_capacity_and_arguments():
    L = ra.lib()
    kv, arr = _paged([500, 512])                       # 512 = max_pages * 128: full
    assert L.ra_paged_append_kv(ctypes.byref(kv), FAKE, FAKE, 1, None) == ra.RA_ERR_CAPACITY
    assert L.ra_paged_append_kv(ctypes.byref(kv), FAKE, FAKE, -1, None) == ra.RA_ERR_ARG
    assert L.ra_paged_append_kv(ctypes.byref(kv), 0, FAKE, 1, None) == ra.RA_ERR_ARG
    assert list(arr) == [500, 512]                     # lengths untouched on every error


def test_paged_decode_rejects_bad_shapes_and_workspaces():
    L = ra.lib()
    args = (FAKE, 8, 10, 4, 16, FAKE, FAKE, FAKE)      # q, Hq, k, sinks, window, out, idx, ws
    kv, _ = _paged([300, 0])                           # an empty sequence cannot decode
    assert L.ra_paged_decode_step(ctypes.byref(kv), *args, BIG, None) == ra.RA_ERR_EMPTY
    kv, _ = _paged([300, 600])                         # longer than max_pages * 128
    assert L.ra_paged_decode_step(ctypes.byref(kv), *args, BIG, None) == ra.RA_ERR_SHAPE
    kv, _ = _paged([128] * 257)                        # more sequences than a call carries
    assert L.ra_paged_decode_step(ctypes.byref(kv), *args, BIG, None) == ra.RA_ERR_SHAPE
    kv, _ = _paged([300, 200], d=96)
    assert L.ra_paged_decode_step(ctypes.byref(kv), *args, BIG, None) == ra.RA_ERR_SHAPE
    kv, _ = _paged([300, 200])
    need = L.ra_paged_workspace_bytes(2, 8, 300, 128, 10, 4, 16)
    assert need > 0
    assert L.ra_paged_decode_step(ctypes.byref(kv), *args, need - 1, None) == ra.RA_ERR_WORKSPACE
    assert L.ra_paged_decode_step(ctypes.byref(kv), FAKE, 3, 10, 4, 16, FAKE, FAKE, FAKE, BIG,
                                  None) == ra.RA_ERR_SHAPE            # Hq % Hkv != 0
    assert L.ra_paged_workspace_bytes(2, 8, 300, 96, 10, 4, 16) == 0


def _ivf(B=1, Hkv=2, d=128, nlist=64, N=1000):
    return ra.ra_ivf(FAKE, FAKE, FAKE, FAKE, B, Hkv, d, nlist, N)


def test_ivf_build_checks_before_launch():
    L = ra.lib()
    kv = ra.ra_kv(FAKE, FAKE, 1, 2, 128, 2000, 1000)
    need = L.ra_ivf_build_workspace_bytes(1, 2, 1000, 128, 64)
    assert need > 0
    assert L.ra_ivf_build_workspace_bytes(1, 2, 1000, 96, 64) == 0        # d
    assert L.ra_ivf_build_workspace_bytes(1, 2, 1000, 128, 5000) == 0     # nlist > 4096
    ix = _ivf()
    assert L.ra_ivf_build(ctypes.byref(kv), ctypes.byref(ix), -1, FAKE, BIG, None) == ra.RA_ERR_ARG
    assert L.ra_ivf_build(ctypes.byref(kv), None, 2, FAKE, BIG, None) == ra.RA_ERR_ARG
    assert L.ra_ivf_build(ctypes.byref(kv), ctypes.byref(_ivf(N=1001)), 2, FAKE, BIG,
                          None) == ra.RA_ERR_SHAPE                       # more keys than cached
    assert L.ra_ivf_build(ctypes.byref(kv), ctypes.byref(_ivf(Hkv=4)), 2, FAKE, BIG,
                          None) == ra.RA_ERR_SHAPE
    assert L.ra_ivf_build(ctypes.byref(kv), ctypes.byref(_ivf(nlist=5000)), 2, FAKE, BIG,
                          None) == ra.RA_ERR_SHAPE
    assert L.ra_ivf_build(ctypes.byref(kv), ctypes.byref(ix), 2, FAKE, need - 1,
                          None) == ra.RA_ERR_WORKSPACE


def test_ivf_decode_checks_before_launch():
    L = ra.lib()
    kv = ra.ra_kv(FAKE, FAKE, 1, 2, 128, 2000, 1010)
    ix = _ivf(N=1000)
    need = L.ra_ivf_search_workspace_bytes(1, 8, 1010, 128, 50, 16)
    assert need > 0
    assert L.ra_ivf_search_workspace_bytes(1, 8, 1010, 128, 50, 65) == 0  # nprobe > 64

    def call(ix_, nprobe, n_window=32, ws_bytes=BIG, Hq=8):
        return L.ra_ivf_decode_step(ctypes.byref(kv), ctypes.byref(ix_), FAKE, Hq, 50, nprobe,
                                    4, n_window, FAKE, FAKE, FAKE, ws_bytes, None)

    assert call(ix, 0) == ra.RA_ERR_ARG
    assert call(ix, 65) == ra.RA_ERR_ARG
    assert call(_ivf(nlist=8), 16) == ra.RA_ERR_ARG              # nprobe > nlist
    assert call(ix, 16, n_window=5) == ra.RA_ERR_ARG             # appended keys past the window
    assert call(_ivf(N=1011), 16) == ra.RA_ERR_ARG               # index longer than the cache
    assert call(_ivf(Hkv=4), 16) == ra.RA_ERR_SHAPE
    assert call(ix, 16, Hq=7) == ra.RA_ERR_SHAPE                 # Hq % Hkv != 0
    assert call(ix, 16, ws_bytes=need - 1) == ra.RA_ERR_WORKSPACE
    assert kv.N == 1010


def _ivf_build_bound(B, Hkv, N, nlist):
    """The build workspace the header states: a key-centroid score block of at most 256 MB (or
    one 128-key tile's scores when a tile alone is larger), the assignments and the per-1024-key
    cluster counts, each section 256-byte aligned."""
    BH = B * Hkv
    ld = (nlist + 3) // 4 * 4
    block = max(256 << 20, BH * ld * 4 * 128)
    return block + 4 * BH * (N + nlist * ((N + 1023) // 1024)) + 4 * 256


@pytest.mark.parametrize("B,Hkv,N,d,nlist", [(1, 8, 1 << 20, 128, 1024), (1, 8, 131071, 128, 1024),
                                             (2, 8, 262144, 64, 256), (64, 8, 4096, 128, 4096)])
def test_ivf_build_workspace_is_bounded(B, Hkv, N, d, nlist):
    need = ra.lib().ra_ivf_build_workspace_bytes(B, Hkv, N, d, nlist)
    assert 4 * B * Hkv * N < need <= _ivf_build_bound(B, Hkv, N, nlist)
    # far below the whole key-centroid score matrix once N is large
    if N >= 1 << 20:
        assert need < B * Hkv * N * nlist * 4 // 50
