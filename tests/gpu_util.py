"""Helpers of the GPU tests: moving generator output to the device and running the path."""
from __future__ import annotations

import numpy as np
import torch

import top_retrieval_attention_b200 as ra
from synth import device as sdev
from synth import gen


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def cache_from_host(K_bits: np.ndarray, V_bits: np.ndarray, cap: int | None = None) -> ra.KVCache:
    B, Hkv, N, d = K_bits.shape
    cap = N if cap is None else cap
    c = ra.KVCache(B, Hkv, d, max(cap, 1))
    c.K.zero_()
    c.V.zero_()
    if N:
        c.K[:, :, :N] = to_dev_bf16(K_bits)
        c.V[:, :, :N] = to_dev_bf16(V_bits)
    c.N = N
    return c


def cache_from_workload(w: gen.Workload, layer: int = 0, cap: int | None = None):
    """Device-filled cache of one layer plus the device query; returns (cache, q, needles)."""
    cap = w.N if cap is None else cap
    c = ra.KVCache(w.B, w.Hkv, w.d, cap)
    q = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    nd = sdev.device_layer(w, layer, c.K, c.V, q)
    c.N = w.N
    return c, q, nd


def run_decode(cache: ra.KVCache, q: torch.Tensor, k: int, n_sink: int, n_window: int):
    out, idx = ra.decode_step(cache, q, k, n_sink, n_window)
    torch.cuda.synchronize()
    return out.cpu().numpy(), idx.cpu().numpy()
