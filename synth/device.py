"""Device-side materialisation of the synthetic workloads (same bits as synth/gen.py).

Caches are filled in HBM by libra_synth.so; needles (a few rows, computed on the host by
synth/gen.py) are uploaded and written with torch indexing.  Input generation only.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_int32, c_int64, c_uint64, c_void_p

import numpy as np

from . import gen

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libra_synth.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libra_synth.so is not built ({LIB_PATH}); run "
                               "`python -m top_retrieval_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.synth_fill_kv.restype = c_int32
        L.synth_fill_kv.argtypes = [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_int32,
                                    c_int64, c_int64, c_uint64, c_int32, c_int32, c_void_p]
        L.synth_fill_q.restype = c_int32
        L.synth_fill_q.argtypes = [c_void_p, c_int32, c_int32, c_int32, c_uint64, c_void_p]
        L.synth_constants.restype = None
        L.synth_constants.argtypes = [ctypes.POINTER(ctypes.c_double)]
        _lib = L
    return _lib


def constants() -> tuple[float, float]:
    arr = (ctypes.c_double * 2)()
    lib().synth_constants(arr)
    return float(arr[0]), float(arr[1])


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return c_void_p(s.cuda_stream)


def fill_kv(K, V, row0: int, nrows: int, seed: int, layer: int, with_offset: bool = True,
            stream=None) -> None:
    B, Hkv, cap, d = K.shape
    r = lib().synth_fill_kv(K.data_ptr(), V.data_ptr(), B, Hkv, cap, d, row0, nrows, seed, layer,
                            int(with_offset), _stream(stream))
    if r != 0:
        raise RuntimeError(f"synth_fill_kv failed: {r}")


def fill_q(q, seed: int, stream=None) -> None:
    B, Hq, d = q.shape
    r = lib().synth_fill_q(q.data_ptr(), B, Hq, d, seed, _stream(stream))
    if r != 0:
        raise RuntimeError(f"synth_fill_q failed: {r}")


def plant_needles(K, nd: gen.Needles) -> None:
    import torch
    B, Hkv, n = nd.pos.shape
    if n == 0:
        return
    bi = torch.arange(B).repeat_interleave(Hkv * n)
    gi = torch.arange(Hkv).repeat_interleave(n).repeat(B)
    pi = torch.from_numpy(nd.pos.reshape(-1))
    rows = torch.from_numpy(nd.rows.reshape(-1, nd.rows.shape[-1]).view(np.int16))
    dev = K.device
    K.view(torch.int16)[bi.to(dev), gi.to(dev), pi.to(dev)] = rows.to(dev)


def device_layer(w: gen.Workload, layer: int, K, V, q=None, N: int | None = None,
                 needles: bool = True, stream=None):
    """Fill rows [0, N) of one layer's caches (and q if given); returns the host Needles."""
    N = w.N if N is None else N
    fill_kv(K, V, 0, N, w.seed, layer, True, stream)
    q_host = gen.gen_q(w.seed, w.B, w.Hq, w.d)
    if q is not None:
        fill_q(q, w.seed, stream)
    nd = None
    if needles and w.n_needle:
        nd = gen.gen_needles(w.seed, layer, q_host, w.Hkv, w.n_needle, N, w.n_sink, w.n_window,
                             w.needle_scale)
        plant_needles(K, nd)
    return nd
