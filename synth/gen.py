"""Seeded synthetic decode workloads: the only code shared by the oracle's tests and the CUDA path.

This module draws inputs; it holds none of the attention method's arithmetic (no score,
no selection, no softmax).  Both sides consume exactly the same bf16 bit patterns:

* the host side (this file, numpy) produces any slice of any tensor on demand, so the
  oracle can regenerate one head of a 137 GB cache without the GPU;
* the device side (``synth/csrc/synth.cu``, loaded by ``synth.device``) fills caches
  in HBM with the same bits, computed from the same published definition below.

Generator (counter based, so any element is addressable independently):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014): state advances by gamma = 0x9E3779B97F4A7C15 and every output is the
  64-bit finaliser mix64(z) = z3 with z1 = (z ^ z >> 30) * 0xBF58476D1CE4E5B9,
  z2 = (z1 ^ z1 >> 27) * 0x94D049BB133111EB, z3 = z2 ^ z2 >> 31 (all mod 2^64).
* A stream is named by (seed, kind, layer, b, head); its key is
  mix64(seed * gamma + tag) with tag = kind<<56 | layer<<44 | b<<28 | head<<12, and its
  element i is mix64(key + (i + 1) * gamma), i.e. the (i+1)-th SplitMix64 output.
* A unit normal deviate is approximated by the Irwin-Hall sum of the four 16-bit fields
  h_j of one output: x = (h_0 + h_1 + h_2 + h_3 - 131070) * sqrt(3) / 65536 (mean 0,
  variance 1 - 2^-32, support +-3.46).  Only integer operations and correctly rounded
  IEEE double operations are used, so host and device agree bit for bit.
* A value is stored as bf16: double -> float (round to nearest even) -> bf16 (round to
  nearest even on the float's bit pattern).

Workload recipe (the decode problem of RetrievalAttention, "Sparse attention renormalizes
selected tokens" and "The GPU keeps 640 fixed positions" slides):

* q[b, h, :]        ~ N(0, 1)                    kind Q, stream (seed, Q, 0, b, h)
* K[l, b, g, i, :]  ~ N(0, 1) + off[l, b, g, :]  kind K, element i*d + c
* off[l, b, g, c]   = sqrt(2) * N(0, 1)          kind KOFF (variance 2: queries are out of
                                                 distribution w.r.t. keys, Fig. 3)
* V[l, b, g, i, :]  ~ N(0, 1)                    kind V, element i*d + c
* needles: per KV head, ``n_needle`` distinct positions drawn uniformly from the
  candidate range [n_sink, N - n_window); needle j targets query head g*G + (j mod G)
  and its key row is bf16(lam * q_h / ||q_h||) (no offset); V is left as drawn.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1

#: sqrt(3) / 65536 and sqrt(2), correctly rounded doubles (the device side uses the same
#: values as hexadecimal literals; a CPU test compares them with the library's copy).
IH_SCALE = math.sqrt(3.0) / 65536.0
OFF_STD = math.sqrt(2.0)

KIND_Q, KIND_K, KIND_KOFF, KIND_V, KIND_NEEDLE = 1, 2, 3, 4, 5


def _mix64_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= np.uint64(MIX1)
        z ^= z >> np.uint64(27)
        z *= np.uint64(MIX2)
        z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, kind: int, layer: int, b: int, head: int) -> int:
    tag = ((kind & 0xFF) << 56) | ((layer & 0xFFF) << 44) | ((b & 0xFFFF) << 28) \
        | ((head & 0xFFFF) << 12)
    return _mix64_int(((seed * GAMMA) & MASK64) + tag)


def raw_u64(key: int, start: int, count: int) -> np.ndarray:
    """Elements start .. start+count-1 of the stream with the given key (uint64)."""
    i = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + i * np.uint64(GAMMA)
    return _mix64(z)


def normal_f64(key: int, start: int, count: int) -> np.ndarray:
    u = raw_u64(key, start, count)
    m = np.uint64(0xFFFF)
    s = (u & m) + ((u >> np.uint64(16)) & m) + ((u >> np.uint64(32)) & m) \
        + ((u >> np.uint64(48)) & m)
    return (s.astype(np.int64) - 131070).astype(np.float64) * IH_SCALE


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """double -> float (RNE) -> bf16 bits (RNE); inputs are finite."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    r = (bits + np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (used only to build needle rows and for display)."""
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------------------
# tensors of the decode workload


def gen_q(seed: int, B: int, Hq: int, d: int) -> np.ndarray:
    out = np.empty((B, Hq, d), dtype=np.uint16)
    for b in range(B):
        for h in range(Hq):
            out[b, h] = f64_to_bf16_bits(normal_f64(stream_key(seed, KIND_Q, 0, b, h), 0, d))
    return out


def key_offset(seed: int, layer: int, b: int, g: int, d: int) -> np.ndarray:
    return OFF_STD * normal_f64(stream_key(seed, KIND_KOFF, layer, b, g), 0, d)


def gen_k_rows(seed: int, layer: int, b: int, g: int, d: int, row0: int, nrows: int,
               offset: bool = True) -> np.ndarray:
    x = normal_f64(stream_key(seed, KIND_K, layer, b, g), row0 * d, nrows * d).reshape(nrows, d)
    if offset:
        x = x + key_offset(seed, layer, b, g, d)[None, :]
    return f64_to_bf16_bits(x)


def gen_v_rows(seed: int, layer: int, b: int, g: int, d: int, row0: int, nrows: int) -> np.ndarray:
    x = normal_f64(stream_key(seed, KIND_V, layer, b, g), row0 * d, nrows * d).reshape(nrows, d)
    return f64_to_bf16_bits(x)


@dataclass
class Needles:
    """Planted needle keys of one layer: pos[b, g, j], target head, and the key rows."""
    pos: np.ndarray      # int64 [B, Hkv, n]
    head: np.ndarray     # int64 [B, Hkv, n]  query head (global index) each needle targets
    rows: np.ndarray     # uint16 [B, Hkv, n, d]


def needle_positions(seed: int, layer: int, b: int, g: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n distinct positions uniform in [lo, hi), by rejection on the stream's outputs."""
    span = hi - lo
    if n > span:
        raise ValueError(f"cannot place {n} needles in {span} candidate positions")
    key = stream_key(seed, KIND_NEEDLE, layer, b, g)
    got: list[int] = []
    seen: set[int] = set()
    i = 0
    while len(got) < n:
        u = int(raw_u64(key, i, 1)[0])
        i += 1
        p = lo + (u % span)
        if p not in seen:
            seen.add(p)
            got.append(p)
    return np.array(got, dtype=np.int64)


def needle_row(q_bits: np.ndarray, lam: float) -> np.ndarray:
    qf = bf16_bits_to_f32(q_bits).astype(np.float64)
    norm = math.sqrt(float(np.dot(qf, qf)))
    return f64_to_bf16_bits(lam * qf / norm)


def gen_needles(seed: int, layer: int, q_bits: np.ndarray, Hkv: int, n: int, N: int,
                n_sink: int, n_window: int, lam: float = 4.0) -> Needles:
    B, Hq, d = q_bits.shape
    G = Hq // Hkv
    lo, hi = min(n_sink, N), max(min(n_sink, N), N - n_window)
    pos = np.zeros((B, Hkv, n), dtype=np.int64)
    head = np.zeros((B, Hkv, n), dtype=np.int64)
    rows = np.zeros((B, Hkv, n, d), dtype=np.uint16)
    for b in range(B):
        for g in range(Hkv):
            if n:
                pos[b, g] = needle_positions(seed, layer, b, g, n, lo, hi)
            for j in range(n):
                h = g * G + (j % G)
                head[b, g, j] = h
                rows[b, g, j] = needle_row(q_bits[b, h], lam)
    return Needles(pos, head, rows)


def plant(K_bits: np.ndarray, needles: Needles) -> None:
    """Write needle rows into a host cache [B, Hkv, N, d] (in place)."""
    B, Hkv, n = needles.pos.shape
    for b in range(B):
        for g in range(Hkv):
            for j in range(n):
                K_bits[b, g, needles.pos[b, g, j]] = needles.rows[b, g, j]


# --------------------------------------------------------------------------------------
# named workloads (the five decode configurations, plus small parity cases)


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int
    k: int
    n_sink: int
    n_window: int
    layers: int = 1
    n_needle: int = 0           # per KV head
    needle_scale: float = 4.0
    seed: int = 0x5A00
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def kv_bytes(self) -> int:
        """bf16 K plus V bytes of all layers (2 * L * Hkv * d * 2 B per token per sequence)."""
        return 2 * self.layers * self.B * self.Hkv * self.N * self.d * 2


def pct_k(p: float, N: int) -> int:
    """Budget given as a fraction of the context: floor(p * N)."""
    return int(math.floor(p * N + 1e-9))


def workload(name: str) -> Workload:
    """The decode workloads of the benchmark suite, by name."""
    W = {
        # tiny single group: N=8192, 1 KV / 4 Q heads, d=128, 8 needles, k=100, sink 4, window 64
        "tiny": Workload("tiny", 1, 4, 1, 128, 8192, 100, 4, 64, n_needle=8, seed=0x5A01),
        # one Llama-3-8B-shaped layer at 128K, top-100 and top-1%
        "l8b_128k_k100": Workload("l8b_128k_k100", 1, 32, 8, 128, 131072, 100, 128, 512,
                                  n_needle=64, seed=0x5A02),
        "l8b_128k_k1pct": Workload("l8b_128k_k1pct", 1, 32, 8, 128, 131072,
                                   pct_k(0.01, 131072), 128, 512, n_needle=64, seed=0x5A02),
        # full 32-layer cache at 1M, top-2%
        "l8b_1m_32layer": Workload("l8b_1m_32layer", 1, 32, 8, 128, 1 << 20,
                                   pct_k(0.02, 1 << 20), 128, 512, layers=32, n_needle=64,
                                   seed=0x5A03),
        # batch 16 x 256K, top-1%
        "l8b_b16_256k": Workload("l8b_b16_256k", 16, 32, 8, 128, 262144,
                                 pct_k(0.01, 262144), 128, 512, n_needle=64, seed=0x5A04),
    }
    if name in W:
        return W[name]
    # sweep points at 512K: "sweep_k{100|1pct|5pct}_g{1|4|8}_d{64|128}"
    if name.startswith("sweep_"):
        _, kk, gg, dd = name.split("_")
        N = 1 << 19
        k = {"k100": 100, "k1pct": pct_k(0.01, N), "k5pct": pct_k(0.05, N)}[kk]
        G = int(gg[1:])
        d = int(dd[1:])
        return Workload(name, 1, 32, 32 // G, d, N, k, 128, 512, n_needle=64, seed=0x5A05)
    raise KeyError(name)


def sweep_names() -> list[str]:
    return [f"sweep_{k}_g{g}_d{d}" for k in ("k100", "k1pct", "k5pct") for g in (1, 4, 8)
            for d in (64, 128)]


def host_layer(w: Workload, layer: int = 0, N: int | None = None, with_needles: bool = True):
    """Whole layer on the host: (q, K, V, needles) as bf16 bits; K [B, Hkv, N, d]."""
    N = w.N if N is None else N
    q = gen_q(w.seed, w.B, w.Hq, w.d)
    K = np.empty((w.B, w.Hkv, N, w.d), dtype=np.uint16)
    V = np.empty_like(K)
    for b in range(w.B):
        for g in range(w.Hkv):
            K[b, g] = gen_k_rows(w.seed, layer, b, g, w.d, 0, N)
            V[b, g] = gen_v_rows(w.seed, layer, b, g, w.d, 0, N)
    nd = None
    if with_needles and w.n_needle:
        nd = gen_needles(w.seed, layer, q, w.Hkv, w.n_needle, N, w.n_sink, w.n_window,
                         w.needle_scale)
        plant(K, nd)
    return q, K, V, nd


def host_head(w: Workload, layer: int, b: int, g: int, N: int | None = None,
              needles: Needles | None = None):
    """One KV head's K and V rows [N, d] (bf16 bits), needles planted if given."""
    N = w.N if N is None else N
    K = gen_k_rows(w.seed, layer, b, g, w.d, 0, N)
    V = gen_v_rows(w.seed, layer, b, g, w.d, 0, N)
    if needles is not None:
        for j in range(needles.pos.shape[2]):
            K[needles.pos[b, g, j]] = needles.rows[b, g, j]
    return K, V
