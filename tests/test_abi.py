"""The C ABI without a GPU: the libraries load, export what the headers declare, and reject
bad arguments on the host before anything is enqueued."""
import ctypes
import math
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import top_retrieval_attention_b200 as ra  # noqa: E402
from synth import device as sdev  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def built():
    from top_retrieval_attention_b200 import build
    build.build_all()


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:ra|synth)_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared("ra.h")
    assert set(names) == set(ra.EXPORTS)
    L = ctypes.CDLL(ra.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    S = ctypes.CDLL(sdev.LIB_PATH)
    for n in _declared("ra_synth.h"):
        assert hasattr(S, n), n


def test_library_needs_no_driver_at_load_time():
    out = subprocess.run(["ldd", ra.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out
    assert "libtorch" not in out


def test_status_strings_and_version():
    assert ra.ra_status_str(ra.RA_OK) == "RA_OK"
    assert ra.ra_status_str(ra.RA_ERR_WORKSPACE) == "RA_ERR_WORKSPACE"
    assert "sm_100a" in ra.ra_version()


FAKE = 1 << 20   # a 16-byte aligned non-null address; never dereferenced on these paths


def _kv(B=1, Hkv=2, d=128, cap=100, N=50, K=FAKE, V=FAKE):
    return ra.ra_kv(K, V, B, Hkv, d, cap, N)


def test_workspace_bytes():
    n = ra.ra_decode_workspace_bytes(1, 32, 131072, 128, 1310, 128, 512)
    # scores (32 x 131072 fp32) + digit-1 histograms (32 x 2048) + counters
    assert n >= 32 * 131072 * 4 + 32 * 2048 * 4 + 32 * 8 * 4
    assert n % 256 == 0
    assert ra.ra_decode_workspace_bytes(1, 32, 131072, 96, 10, 0, 0) == 0     # d
    assert ra.ra_decode_workspace_bytes(0, 32, 131072, 128, 10, 0, 0) == 0    # B
    assert ra.ra_decode_workspace_bytes(1, 32, 131072, 128, -1, 0, 0) == 0    # k
    assert ra.ra_dense_workspace_bytes(1, 32, 131072, 128) > 0
    assert ra.ra_dense_workspace_bytes(1, 32, 131072, 80) == 0


@pytest.mark.parametrize("mut,status", [
    (dict(K=0), ra.RA_ERR_ARG),
    (dict(V=FAKE + 8), ra.RA_ERR_ARG),
    (dict(d=96), ra.RA_ERR_SHAPE),
    (dict(N=101), ra.RA_ERR_SHAPE),
    (dict(B=0), ra.RA_ERR_ARG),
    (dict(N=0), ra.RA_ERR_EMPTY),
])
def test_decode_rejects_bad_cache(mut, status):
    kv = _kv(**mut)
    ws_bytes = 1 << 30
    s = ra.ra_decode_step(kv, FAKE, 4, 10, 4, 8, FAKE, FAKE, FAKE, ws_bytes, None)
    assert s == status


def test_decode_rejects_bad_arguments():
    kv = _kv()
    big = 1 << 30
    assert ra.ra_decode_step(kv, FAKE, 3, 10, 4, 8, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_SHAPE
    assert ra.ra_decode_step(kv, FAKE, 18, 10, 4, 8, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_SHAPE
    assert ra.ra_decode_step(kv, FAKE, 4, -1, 4, 8, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_decode_step(kv, FAKE, 4, 10, -4, 8, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_decode_step(kv, 0, 4, 10, 4, 8, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_decode_step(kv, FAKE, 4, 10, 4, 8, 0, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_decode_step(kv, FAKE, 4, 10, 4, 8, FAKE, 0, FAKE, big, None) == ra.RA_ERR_ARG
    # workspace: null, misaligned, too small
    assert ra.ra_decode_step(kv, FAKE, 4, 10, 4, 8, FAKE, FAKE, 0, big, None) == ra.RA_ERR_WORKSPACE
    assert ra.ra_decode_step(kv, FAKE, 4, 10, 4, 8, FAKE, FAKE, FAKE + 16, big, None) == ra.RA_ERR_WORKSPACE
    need = ra.ra_decode_workspace_bytes(1, 4, 50, 128, 10, 4, 8)
    assert ra.ra_decode_step(kv, FAKE, 4, 10, 4, 8, FAKE, FAKE, FAKE, need - 1, None) == ra.RA_ERR_WORKSPACE
    # empty selected union: no static set and k = 0
    assert ra.ra_decode_step(kv, FAKE, 4, 0, 0, 0, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_EMPTY


def test_phases_validate_like_the_step():
    kv = _kv()
    big = 1 << 30
    assert ra.ra_score_gqa(kv, 0, 4, 10, 4, 8, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_topk_select(kv, 4, 10, 4, 8, 0, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_sparse_attn(kv, 4, 10, 4, 8, FAKE, 0, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_sparse_attn(kv, 4, 10, 4, 8, FAKE, FAKE, FAKE, 10, None) == ra.RA_ERR_WORKSPACE
    assert ra.ra_select_attend(kv, 4, 10, 4, 8, 0, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_select_attend(kv, 4, 10, 4, 8, FAKE, 0, FAKE, big, None) == ra.RA_ERR_ARG
    assert ra.ra_select_attend(kv, 4, 10, 4, 8, FAKE, FAKE, FAKE, 10, None) == ra.RA_ERR_WORKSPACE


def test_dense_rejects_bad_arguments():
    kv = _kv()
    big = 1 << 30
    assert ra.ra_dense_decode(kv, FAKE, 3, FAKE, FAKE, big, None) == ra.RA_ERR_SHAPE
    assert ra.ra_dense_decode(_kv(N=0), FAKE, 4, FAKE, FAKE, big, None) == ra.RA_ERR_EMPTY
    assert ra.ra_dense_decode(kv, FAKE, 4, FAKE, FAKE, 16, None) == ra.RA_ERR_WORKSPACE


def test_append_capacity_and_arguments():
    kv = _kv(cap=100, N=98)
    assert ra.ra_append_kv(kv, FAKE, FAKE, 3, None) == ra.RA_ERR_CAPACITY
    assert kv.N == 98
    assert ra.ra_append_kv(kv, FAKE, FAKE, -1, None) == ra.RA_ERR_ARG
    assert ra.ra_append_kv(kv, 0, FAKE, 1, None) == ra.RA_ERR_ARG
    assert ra.ra_append_kv(kv, FAKE, FAKE, 0, None) == ra.RA_OK
    assert kv.N == 98


def test_fused_append_step_validates_before_launch():
    big = 1 << 30
    args = (FAKE, 4, 10, 4, 8, FAKE, FAKE, FAKE, big, None)   # Hq, k, sinks, window, out, idx, ws
    kv = _kv(cap=100, N=100)
    assert ra.ra_decode_step_append(kv, FAKE, FAKE, FAKE, *args[1:]) == ra.RA_ERR_CAPACITY
    assert ra.ra_score_gqa_append(kv, FAKE, FAKE, FAKE, 4, 10, 4, 8, FAKE, big, None) == ra.RA_ERR_CAPACITY
    kv = _kv(cap=100, N=50)
    assert ra.ra_decode_step_append(kv, FAKE, 0, FAKE, *args[1:]) == ra.RA_ERR_ARG
    assert ra.ra_decode_step_append(kv, FAKE, FAKE, FAKE + 8, *args[1:]) == ra.RA_ERR_ARG
    assert ra.ra_decode_step_append(kv, FAKE, FAKE, FAKE, 3, 10, 4, 8, FAKE, FAKE, FAKE, big,
                                    None) == ra.RA_ERR_SHAPE
    assert ra.ra_decode_step_append(kv, FAKE, FAKE, FAKE, 4, 10, 4, 8, FAKE, FAKE, FAKE, 16,
                                    None) == ra.RA_ERR_WORKSPACE
    assert ra.ra_decode_step_append(kv, 0, FAKE, FAKE, *args[1:]) == ra.RA_ERR_ARG
    assert kv.N == 50   # no error grows the cache


def test_launch_count_query():
    n = ra.lib().ra_decode_step_launches(1, 32, 8, 131072, 128, 1310, 128, 512)
    assert n in (2, 3)
    assert ra.lib().ra_decode_step_launches(1, 32, 8, 131072, 96, 1310, 128, 512) == -1   # d
    assert ra.lib().ra_decode_step_launches(1, 30, 8, 131072, 128, 1310, 128, 512) == -1  # Hq % Hkv
    assert ra.lib().ra_decode_step_launches(1, 32, 8, 0, 128, 10, 4, 8) == -1             # N == 0


def test_synth_constants_match_host_generator():
    from synth import gen
    a, b = sdev.constants()
    assert a == gen.IH_SCALE == math.sqrt(3) / 65536
    assert b == gen.OFF_STD == math.sqrt(2)


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "top_retrieval_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, re.M), f
                assert "oracle/" not in text, f



def test_pyramid_budgets_match_the_oracle_and_reject_bad_arguments():
    import oracle
    for L in (1, 2, 3, 7, 32, 80):
        for km in (0, 1, 7, 100, 1310, 20971):
            for r in (0.1, 0.25, 0.5, 0.9, 1.0):
                assert ra.pyramid_budgets(L, km, r) == list(oracle.pyramid_budgets(L, km, r))
    out = (ctypes.c_int32 * 4)()
    assert ra.lib().ra_pyramid_budgets(0, 10, 0.5, out) == ra.RA_ERR_ARG
    assert ra.lib().ra_pyramid_budgets(4, 10, 0.0, out) == ra.RA_ERR_ARG
    assert ra.lib().ra_pyramid_budgets(4, 10, 1.5, out) == ra.RA_ERR_ARG


def test_threshold_step_rejects_bad_arguments():
    kv = _kv()
    big = 1 << 30
    f = ra.lib().ra_decode_step_eps
    assert f(ctypes.byref(kv), FAKE, 4, 10, 0.0, 4, 8, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert f(ctypes.byref(kv), FAKE, 4, 10, 1.0, 4, 8, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert f(ctypes.byref(kv), FAKE, 4, 10, 1e-3, 0, 0, FAKE, FAKE, FAKE, big, None) == ra.RA_ERR_EMPTY
    assert f(ctypes.byref(kv), FAKE, 4, 10, 1e-3, 4, 8, FAKE, FAKE, FAKE, 10, None) == ra.RA_ERR_WORKSPACE


def test_prefill_rejects_bad_arguments():
    kv = _kv()
    big = 1 << 30
    L = ra.lib()
    assert L.ra_prefill_topk(ctypes.byref(kv), 0, 4, 8, 10, 4, 8, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert L.ra_prefill_topk(ctypes.byref(kv), FAKE, 4, 0, 10, 4, 8, FAKE, FAKE, big, None) == ra.RA_ERR_ARG
    assert L.ra_prefill_topk(ctypes.byref(kv), FAKE, 3, 8, 10, 4, 8, FAKE, FAKE, big, None) == ra.RA_ERR_SHAPE
    assert L.ra_prefill_topk(ctypes.byref(kv), FAKE, 4, 8, 10, 4, 8, FAKE, FAKE, 10, None) == ra.RA_ERR_WORKSPACE
    assert ra.ra_prefill_workspace_bytes(1, 4, 8, 100, 128, 10, 4, 8) > 4 * 8 * 100 * 4
    assert ra.ra_prefill_workspace_bytes(1, 4, 0, 100, 128, 10, 4, 8) == 0


def test_host_buffer_step_refuses_before_enqueuing():
    """ra_decode_step_append_host checks everything ra_decode_step_append checks, plus its
    host pointers, before the first copy: with a full cache or a null host buffer it returns an
    error and leaves kv unchanged."""
    H = (ctypes.c_uint16 * 4096)()
    O = (ctypes.c_float * 4096)()
    I = (ctypes.c_int32 * 4096)()
    dev = ra.ra_step_io(FAKE, FAKE, FAKE, FAKE, FAKE)
    ws_ok = 1 << 30
    ws = FAKE << 8   # 256-byte aligned
    full = _kv(N=100)   # N == cap: no room for the token
    st = ra.ra_decode_step_append_host(full, H, H, H, 4, 8, 4, 16, O, I, dev, ws, ws_ok, None)
    assert st == ra.RA_ERR_CAPACITY and full.N == 100
    kv = _kv(N=50)
    st = ra.ra_decode_step_append_host(kv, None, H, H, 4, 8, 4, 16, O, I, dev, ws, ws_ok, None)
    assert st == ra.RA_ERR_ARG and kv.N == 50
    st = ra.ra_decode_step_append_host(kv, H, H, H, 4, 8, 4, 16, O, None, dev, ws, ws_ok, None)
    assert st == ra.RA_ERR_ARG and kv.N == 50
    bad = ra.ra_step_io(FAKE, FAKE + 8, FAKE, FAKE, FAKE)          # misaligned device k_new
    st = ra.ra_decode_step_append_host(kv, H, H, H, 4, 8, 4, 16, O, I, bad, ws, ws_ok, None)
    assert st == ra.RA_ERR_ARG and kv.N == 50
    st = ra.ra_decode_step_append_host(kv, H, H, H, 4, 8, 4, 16, O, I, dev, ws, 256, None)
    assert st == ra.RA_ERR_WORKSPACE and kv.N == 50
