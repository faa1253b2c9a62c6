"""ctypes binding of libra (include/ra.h): argument marshalling only.

The raw entry points keep the C names (``ra_decode_step`` ...) and take integer device
pointers; the small helpers below them (``KVCache``, ``decode_step`` ...) allocate outputs and
workspaces with torch and pass tensor pointers and the current torch stream.  Every step of the
computation runs in libra's CUDA kernels; there is no other implementation behind this module.
Loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_char_p, c_int32, c_int64, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libra.so")

RA_OK, RA_ERR_ARG, RA_ERR_SHAPE, RA_ERR_CAPACITY, RA_ERR_WORKSPACE, RA_ERR_CUDA, RA_ERR_EMPTY = range(7)

#: every symbol include/ra.h declares
EXPORTS = ("ra_status_str", "ra_version", "ra_last_error", "ra_append_kv",
           "ra_decode_workspace_bytes", "ra_decode_step", "ra_score_gqa", "ra_topk_select",
           "ra_sparse_attn", "ra_select_attend", "ra_dense_workspace_bytes", "ra_dense_decode",
           "ra_decode_step_static", "ra_prefill_workspace_bytes", "ra_prefill_topk",
           "ra_prefill_score", "ra_prefill_select", "ra_decode_step_eps", "ra_pyramid_budgets",
           "ra_paged_append_kv", "ra_paged_workspace_bytes", "ra_paged_decode_step",
           "ra_ivf_build_workspace_bytes", "ra_ivf_build", "ra_ivf_search_workspace_bytes",
           "ra_ivf_decode_step", "ra_decode_step_append", "ra_score_gqa_append",
           "ra_decode_step_launches", "ra_decode_step_append_host")


class ra_kv(ctypes.Structure):
    _fields_ = [("K", c_void_p), ("V", c_void_p), ("B", c_int32), ("Hkv", c_int32),
                ("d", c_int32), ("cap", c_int32), ("N", c_int64)]


class ra_paged_kv(ctypes.Structure):
    _fields_ = [("K", c_void_p), ("V", c_void_p), ("block_table", c_void_p),
                ("seq_len", ctypes.POINTER(c_int32)), ("B", c_int32), ("Hkv", c_int32),
                ("d", c_int32), ("max_pages", c_int32), ("num_pages", c_int32)]


class ra_step_io(ctypes.Structure):
    _fields_ = [("q", c_void_p), ("k_new", c_void_p), ("v_new", c_void_p), ("out", c_void_p),
                ("idx", c_void_p)]


class ra_ivf(ctypes.Structure):
    _fields_ = [("Ksorted", c_void_p), ("pos", c_void_p), ("offsets", c_void_p),
                ("centroids", c_void_p), ("B", c_int32), ("Hkv", c_int32), ("d", c_int32),
                ("nlist", c_int32), ("N", c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libra.so is not built ({LIB_PATH}); run "
                               "`python -m top_retrieval_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(ra_kv)
        sig = {
            "ra_status_str": (c_char_p, [c_int32]),
            "ra_version": (c_char_p, []),
            "ra_last_error": (c_char_p, []),
            "ra_append_kv": (c_int32, [P, c_void_p, c_void_p, c_int32, c_void_p]),
            "ra_decode_workspace_bytes": (c_size_t, [c_int32, c_int32, c_int64, c_int32, c_int32,
                                                     c_int32, c_int32]),
            "ra_decode_step": (c_int32, [P, c_void_p, c_int32, c_int32, c_int32, c_int32,
                                         c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
            "ra_score_gqa": (c_int32, [P, c_void_p, c_int32, c_int32, c_int32, c_int32, c_void_p,
                                       c_size_t, c_void_p]),
            "ra_topk_select": (c_int32, [P, c_int32, c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                         c_size_t, c_void_p]),
            "ra_sparse_attn": (c_int32, [P, c_int32, c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                         c_void_p, c_size_t, c_void_p]),
            "ra_select_attend": (c_int32, [P, c_int32, c_int32, c_int32, c_int32, c_void_p,
                                           c_void_p, c_void_p, c_size_t, c_void_p]),
            "ra_dense_workspace_bytes": (c_size_t, [c_int32, c_int32, c_int64, c_int32]),
            "ra_dense_decode": (c_int32, [P, c_void_p, c_int32, c_void_p, c_void_p, c_size_t,
                                          c_void_p]),
            "ra_paged_append_kv": (c_int32, [ctypes.POINTER(ra_paged_kv), c_void_p, c_void_p,
                                             c_int32, c_void_p]),
            "ra_paged_workspace_bytes": (c_size_t, [c_int32, c_int32, c_int64, c_int32, c_int32,
                                                    c_int32, c_int32]),
            "ra_paged_decode_step": (c_int32, [ctypes.POINTER(ra_paged_kv), c_void_p, c_int32, c_int32,
                                               c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                               c_size_t, c_void_p]),
            "ra_ivf_build_workspace_bytes": (c_size_t, [c_int32, c_int32, c_int64, c_int32, c_int32]),
            "ra_ivf_build": (c_int32, [P, ctypes.POINTER(ra_ivf), c_int32, c_void_p, c_size_t,
                                       c_void_p]),
            "ra_ivf_search_workspace_bytes": (c_size_t, [c_int32, c_int32, c_int64, c_int32,
                                                         c_int32, c_int32]),
            "ra_ivf_decode_step": (c_int32, [P, ctypes.POINTER(ra_ivf), c_void_p, c_int32, c_int32,
                                             c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                             c_void_p, c_size_t, c_void_p]),
            "ra_pyramid_budgets": (c_int32, [c_int32, c_int32, ctypes.c_double,
                                             ctypes.POINTER(c_int32)]),
            "ra_decode_step_eps": (c_int32, [P, c_void_p, c_int32, c_int32, ctypes.c_float, c_int32,
                                             c_int32, c_void_p, c_void_p, c_void_p, c_size_t,
                                             c_void_p]),
            "ra_prefill_workspace_bytes": (c_size_t, [c_int32, c_int32, c_int32, c_int64, c_int32,
                                                      c_int32, c_int32, c_int32]),
            "ra_prefill_topk": (c_int32, [P, c_void_p, c_int32, c_int32, c_int32, c_int32, c_int32,
                                          c_void_p, c_void_p, c_size_t, c_void_p]),
            "ra_prefill_score": (c_int32, [P, c_void_p, c_int32, c_int32, c_int32, c_int32, c_int32,
                                           c_void_p, c_size_t, c_void_p]),
            "ra_prefill_select": (c_int32, [P, c_int32, c_int32, c_int32, c_int32, c_int32, c_void_p,
                                            c_void_p, c_size_t, c_void_p]),
            "ra_decode_step_static": (c_int32, [P, c_void_p, c_int32, c_int32, c_int32, c_int32,
                                                c_void_p, c_void_p, c_void_p]),
            "ra_decode_step_append": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                                c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                                c_size_t, c_void_p]),
            "ra_score_gqa_append": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                              c_int32, c_int32, c_void_p, c_size_t, c_void_p]),
            "ra_decode_step_launches": (c_int32, [c_int32, c_int32, c_int32, c_int64, c_int32,
                                                  c_int32, c_int32, c_int32]),
            "ra_decode_step_append_host": (c_int32, [P, c_void_p, c_void_p, c_void_p, c_int32,
                                                     c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                                     ctypes.POINTER(ra_step_io), c_void_p, c_size_t,
                                                     c_void_p]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


# ------------------------------------------------------------------ raw entry points


def ra_status_str(s: int) -> str:
    return lib().ra_status_str(s).decode()


def ra_version() -> str:
    return lib().ra_version().decode()


def ra_last_error() -> str:
    return lib().ra_last_error().decode()


def ra_append_kv(kv, k_new, v_new, T, stream):
    return lib().ra_append_kv(ctypes.byref(kv), k_new, v_new, T, stream)


def ra_decode_workspace_bytes(B, Hq, N, d, k, n_sink, n_window) -> int:
    return lib().ra_decode_workspace_bytes(B, Hq, N, d, k, n_sink, n_window)


def ra_decode_step(kv, q, Hq, k, n_sink, n_window, out, idx, ws, ws_bytes, stream):
    return lib().ra_decode_step(ctypes.byref(kv), q, Hq, k, n_sink, n_window, out, idx, ws,
                                ws_bytes, stream)


def ra_score_gqa(kv, q, Hq, k, n_sink, n_window, ws, ws_bytes, stream):
    return lib().ra_score_gqa(ctypes.byref(kv), q, Hq, k, n_sink, n_window, ws, ws_bytes, stream)


def ra_topk_select(kv, Hq, k, n_sink, n_window, idx, ws, ws_bytes, stream):
    return lib().ra_topk_select(ctypes.byref(kv), Hq, k, n_sink, n_window, idx, ws, ws_bytes,
                                stream)


def ra_sparse_attn(kv, Hq, k, n_sink, n_window, idx, out, ws, ws_bytes, stream):
    return lib().ra_sparse_attn(ctypes.byref(kv), Hq, k, n_sink, n_window, idx, out, ws,
                                ws_bytes, stream)


def ra_select_attend(kv, Hq, k, n_sink, n_window, idx, out, ws, ws_bytes, stream):
    return lib().ra_select_attend(ctypes.byref(kv), Hq, k, n_sink, n_window, idx, out, ws,
                                  ws_bytes, stream)


def ra_decode_step_static(kv, q, Hq, k, n_sink, n_window, out, idx, stream):
    """ra_decode_step on libra's built-in 64 MiB scratch: for callers that cannot allocate."""
    return lib().ra_decode_step_static(ctypes.byref(kv), q, Hq, k, n_sink, n_window, out, idx,
                                       stream)


def ra_dense_workspace_bytes(B, Hq, N, d) -> int:
    return lib().ra_dense_workspace_bytes(B, Hq, N, d)


def ra_dense_decode(kv, q, Hq, out, ws, ws_bytes, stream):
    return lib().ra_dense_decode(ctypes.byref(kv), q, Hq, out, ws, ws_bytes, stream)


# ------------------------------------------------------------------ torch-facing helpers


class RaError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {ra_status_str(status)}"
        if status == RA_ERR_CUDA:
            msg += f" ({ra_last_error()})"
        super().__init__(msg)
        self.status = status


def check(status: int, where: str) -> None:
    if status != RA_OK:
        raise RaError(status, where)


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return c_void_p(s.cuda_stream)


class KVCache:
    """A layer's K and V caches ([B, Hkv, cap, d] bf16 torch tensors) and their ra_kv."""

    def __init__(self, B: int, Hkv: int, d: int, cap: int, device="cuda", K=None, V=None):
        import torch
        shape = (B, Hkv, cap, d)
        self.K = torch.empty(shape, dtype=torch.bfloat16, device=device) if K is None else K
        self.V = torch.empty(shape, dtype=torch.bfloat16, device=device) if V is None else V
        assert tuple(self.K.shape) == shape and self.K.is_contiguous() and self.V.is_contiguous()
        self.kv = ra_kv(self.K.data_ptr(), self.V.data_ptr(), B, Hkv, d, cap, 0)

    @property
    def N(self) -> int:
        return int(self.kv.N)

    @N.setter
    def N(self, n: int) -> None:
        self.kv.N = n

    B = property(lambda self: self.kv.B)
    Hkv = property(lambda self: self.kv.Hkv)
    d = property(lambda self: self.kv.d)
    cap = property(lambda self: self.kv.cap)


def append_kv(cache: KVCache, k_new, v_new, stream=None) -> None:
    T = int(k_new.shape[2])
    check(ra_append_kv(cache.kv, k_new.data_ptr(), v_new.data_ptr(), T, _stream(stream)),
          "ra_append_kv")


def decode_workspace(cache: KVCache, Hq: int, k: int, n_sink: int, n_window: int):
    import torch
    n = ra_decode_workspace_bytes(cache.B, Hq, cache.N, cache.d, k, n_sink, n_window)
    if n == 0:
        raise RaError(RA_ERR_SHAPE, "ra_decode_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=cache.K.device)


def decode_step(cache: KVCache, q, k: int, n_sink: int, n_window: int, out=None, idx=None,
                ws=None, stream=None):
    """Exact top-k retrieval attention for one decode step.  Returns (out fp32, idx int32)."""
    import torch
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hq, max(k, 1)), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = decode_workspace(cache, Hq, k, n_sink, n_window)
    check(ra_decode_step(cache.kv, q.data_ptr(), Hq, k, n_sink, n_window, out.data_ptr(),
                         idx.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)),
          "ra_decode_step")
    return out, idx[..., :k]


def ra_decode_step_append(kv, q, k_new, v_new, Hq, k, n_sink, n_window, out, idx, ws, ws_bytes,
                          stream):
    return lib().ra_decode_step_append(ctypes.byref(kv), q, k_new, v_new, Hq, k, n_sink, n_window,
                                       out, idx, ws, ws_bytes, stream)


def ra_decode_step_append_host(kv, q_host, k_new_host, v_new_host, Hq, k, n_sink, n_window,
                               out_host, idx_host, dev, ws, ws_bytes, stream):
    return lib().ra_decode_step_append_host(ctypes.byref(kv), q_host, k_new_host, v_new_host, Hq,
                                            k, n_sink, n_window, out_host, idx_host,
                                            ctypes.byref(dev), ws, ws_bytes, stream)


def ra_score_gqa_append(kv, q, k_new, v_new, Hq, k, n_sink, n_window, ws, ws_bytes, stream):
    return lib().ra_score_gqa_append(ctypes.byref(kv), q, k_new, v_new, Hq, k, n_sink, n_window,
                                     ws, ws_bytes, stream)


def decode_step_append(cache: KVCache, q, k_new, v_new, k: int, n_sink: int, n_window: int,
                       out=None, idx=None, ws=None, stream=None):
    """Append one token (k_new, v_new: bf16 [B, Hkv, 1, d]) and decode over the grown cache,
    the append done inside the scan.  Returns (out fp32, idx int32); cache.N grows by one."""
    import torch
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hq, max(k, 1)), dtype=torch.int32, device=q.device)
    if ws is None:
        n = ra_decode_workspace_bytes(B, Hq, cache.N + 1, d, k, n_sink, n_window)
        if n == 0:
            raise RaError(RA_ERR_SHAPE, "ra_decode_workspace_bytes")
        ws = torch.zeros(n, dtype=torch.uint8, device=q.device)
    check(ra_decode_step_append(cache.kv, q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), Hq, k,
                                n_sink, n_window, out.data_ptr(), idx.data_ptr(), ws.data_ptr(),
                                ws.numel(), _stream(stream)), "ra_decode_step_append")
    return out, idx[..., :k]


def ra_prefill_workspace_bytes(B, Hq, M, N, d, k, n_sink, n_window) -> int:
    return lib().ra_prefill_workspace_bytes(B, Hq, M, N, d, k, n_sink, n_window)


def ra_prefill_topk(kv, q, Hq, M, k, n_sink, n_window, idx, ws, ws_bytes, stream):
    return lib().ra_prefill_topk(ctypes.byref(kv), q, Hq, M, k, n_sink, n_window, idx, ws,
                                 ws_bytes, stream)


def ra_prefill_score(kv, q, Hq, M, k, n_sink, n_window, ws, ws_bytes, stream):
    return lib().ra_prefill_score(ctypes.byref(kv), q, Hq, M, k, n_sink, n_window, ws, ws_bytes,
                                  stream)


def ra_prefill_select(kv, Hq, M, k, n_sink, n_window, idx, ws, ws_bytes, stream):
    return lib().ra_prefill_select(ctypes.byref(kv), Hq, M, k, n_sink, n_window, idx, ws,
                                   ws_bytes, stream)


def prefill_topk(cache: KVCache, q, k: int, n_sink: int, n_window: int, idx=None, ws=None,
                 stream=None):
    """Exact top-k keys of every prefill query q [B, Hq, M, d].  Returns idx int32 [B, Hq, M, k]."""
    import torch
    B, Hq, M, d = q.shape
    if idx is None:
        idx = torch.empty((B, Hq, M, max(k, 1)), dtype=torch.int32, device=q.device)
    if ws is None:
        n = ra_prefill_workspace_bytes(B, Hq, M, cache.N, d, k, n_sink, n_window)
        if n == 0:
            raise RaError(RA_ERR_SHAPE, "ra_prefill_workspace_bytes")
        ws = torch.empty(n, dtype=torch.uint8, device=q.device)
    check(ra_prefill_topk(cache.kv, q.data_ptr(), Hq, M, k, n_sink, n_window, idx.data_ptr(),
                          ws.data_ptr(), ws.numel(), _stream(stream)), "ra_prefill_topk")
    return idx[..., :k]


def pyramid_budgets(L: int, k_mean: int, ratio: float) -> list[int]:
    """Per-layer budgets (ra_pyramid_budgets): a linear fall from layer 0 to layer L - 1 with
    mean k_mean, summing to exactly L * k_mean."""
    out = (c_int32 * L)()
    check(lib().ra_pyramid_budgets(L, k_mean, ratio, out), "ra_pyramid_budgets")
    return list(out)


def ra_decode_step_eps(kv, q, Hq, k, eps, n_sink, n_window, out, idx, ws, ws_bytes, stream):
    return lib().ra_decode_step_eps(ctypes.byref(kv), q, Hq, k, eps, n_sink, n_window, out, idx,
                                    ws, ws_bytes, stream)


def decode_step_eps(cache: KVCache, q, k: int, eps: float, n_sink: int, n_window: int, out=None,
                    idx=None, ws=None, stream=None):
    """Decode step keeping the candidates whose full softmax weight exceeds eps (at most k).
    Returns (out fp32, idx int32 with -1 past the kept keys)."""
    import torch
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hq, max(k, 1)), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = decode_workspace(cache, Hq, k, n_sink, n_window)
    check(ra_decode_step_eps(cache.kv, q.data_ptr(), Hq, k, eps, n_sink, n_window, out.data_ptr(),
                             idx.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)),
          "ra_decode_step_eps")
    return out, idx[..., :k]


PAGE = 128


class PagedKVCache:
    """A paged layer cache: torch-allocated page pools [num_pages, Hkv, 128, d] (bf16), a device
    block table [B, max_pages] (int32) and host lengths; `kv` is the C struct over them."""

    def __init__(self, B: int, Hkv: int, d: int, num_pages: int, max_pages: int, device="cuda"):
        import torch
        self.B, self.Hkv, self.d = B, Hkv, d
        self.num_pages, self.max_pages = num_pages, max_pages
        self.K = torch.empty((num_pages, Hkv, PAGE, d), dtype=torch.bfloat16, device=device)
        self.V = torch.empty_like(self.K)
        self.block_table = torch.zeros((B, max_pages), dtype=torch.int32, device=device)
        self._lens = (c_int32 * B)()
        self.kv = ra_paged_kv(self.K.data_ptr(), self.V.data_ptr(), self.block_table.data_ptr(),
                              self._lens, B, Hkv, d, max_pages, num_pages)

    @property
    def seq_len(self) -> list[int]:
        return list(self._lens)

    def set_lengths(self, lens) -> None:
        for b, n in enumerate(lens):
            self._lens[b] = int(n)


def paged_append_kv(cache: PagedKVCache, k_new, v_new, stream=None) -> None:
    """Append T tokens per sequence (k_new / v_new bf16 [B, Hkv, T, d])."""
    check(lib().ra_paged_append_kv(ctypes.byref(cache.kv), k_new.data_ptr(), v_new.data_ptr(),
                                   k_new.shape[2], _stream(stream)), "ra_paged_append_kv")


def paged_workspace(cache: PagedKVCache, Hq: int, k: int, n_sink: int, n_window: int):
    import torch
    n = lib().ra_paged_workspace_bytes(cache.B, Hq, max(cache.seq_len), cache.d, k, n_sink, n_window)
    if n == 0:
        raise RaError(RA_ERR_SHAPE, "ra_paged_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=cache.K.device)


def paged_decode_step(cache: PagedKVCache, q, k: int, n_sink: int, n_window: int, out=None,
                      idx=None, ws=None, stream=None):
    """The decode step on a paged cache with per-sequence lengths.  Returns (out, idx)."""
    import torch
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hq, max(k, 1)), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = paged_workspace(cache, Hq, k, n_sink, n_window)
    check(lib().ra_paged_decode_step(ctypes.byref(cache.kv), q.data_ptr(), Hq, k, n_sink, n_window,
                                     out.data_ptr(), idx.data_ptr(), ws.data_ptr(), ws.numel(),
                                     _stream(stream)), "ra_paged_decode_step")
    return out, idx[..., :k]


class IvfIndex:
    """An IVF index of a layer cache's first N keys: torch-allocated sorted keys, positions,
    offsets and centroids; `ix` is the C struct over them."""

    def __init__(self, cache: KVCache, nlist: int, N: int | None = None):
        import torch
        self.N = cache.N if N is None else N
        dev = cache.K.device
        B, Hkv, d = cache.B, cache.Hkv, cache.d
        self.nlist = nlist
        self.Ksorted = torch.empty((B, Hkv, self.N, d), dtype=torch.bfloat16, device=dev)
        self.pos = torch.empty((B, Hkv, self.N), dtype=torch.int32, device=dev)
        self.offsets = torch.empty((B, Hkv, nlist + 1), dtype=torch.int32, device=dev)
        self.centroids = torch.empty((B, Hkv, nlist, d), dtype=torch.bfloat16, device=dev)
        self.ix = ra_ivf(self.Ksorted.data_ptr(), self.pos.data_ptr(), self.offsets.data_ptr(),
                         self.centroids.data_ptr(), B, Hkv, d, nlist, self.N)


def ivf_build(cache: KVCache, nlist: int, iters: int = 4, N: int | None = None, stream=None):
    """Spherical k-means IVF index of the cache's first N keys (all by default)."""
    import torch
    ix = IvfIndex(cache, nlist, N)
    n = lib().ra_ivf_build_workspace_bytes(cache.B, cache.Hkv, ix.N, cache.d, nlist)
    if n == 0:
        raise RaError(RA_ERR_SHAPE, "ra_ivf_build_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=cache.K.device)
    check(lib().ra_ivf_build(ctypes.byref(cache.kv), ctypes.byref(ix.ix), iters, ws.data_ptr(), n,
                             _stream(stream)), "ra_ivf_build")
    return ix


def ivf_decode_step(cache: KVCache, ix: IvfIndex, q, k: int, nprobe: int, n_sink: int,
                    n_window: int, out=None, idx=None, ws=None, stream=None):
    """Decode step retrieving through the IVF index.  Returns (out fp32, idx int32)."""
    import torch
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hq, max(k, 1)), dtype=torch.int32, device=q.device)
    if ws is None:
        n = lib().ra_ivf_search_workspace_bytes(B, Hq, cache.N, d, k, nprobe)
        if n == 0:
            raise RaError(RA_ERR_SHAPE, "ra_ivf_search_workspace_bytes")
        ws = torch.zeros(n, dtype=torch.uint8, device=q.device)
    check(lib().ra_ivf_decode_step(ctypes.byref(cache.kv), ctypes.byref(ix.ix), q.data_ptr(), Hq, k,
                                   nprobe, n_sink, n_window, out.data_ptr(), idx.data_ptr(),
                                   ws.data_ptr(), ws.numel(), _stream(stream)),
          "ra_ivf_decode_step")
    return out, idx[..., :k]


def dense_workspace(cache: KVCache, Hq: int):
    import torch
    n = ra_dense_workspace_bytes(cache.B, Hq, cache.N, cache.d)
    if n == 0:
        raise RaError(RA_ERR_SHAPE, "ra_dense_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=cache.K.device)


def dense_decode(cache: KVCache, q, out=None, ws=None, stream=None):
    """Full attention over all N cached tokens.  Returns out fp32 [B, Hq, d]."""
    import torch
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = dense_workspace(cache, Hq)
    check(ra_dense_decode(cache.kv, q.data_ptr(), Hq, out.data_ptr(), ws.data_ptr(), ws.numel(),
                          _stream(stream)), "ra_dense_decode")
    return out
