"""Comparison rules between the CUDA path and the oracle (shared by the GPU tests and bench).

* Omega: exactly min(k, |C|) distinct positions of C, padded with -1; it must equal the
  oracle's set except for positions whose oracle score is within 1e-4 * max(1, |s_k|) of the
  oracle's k-th largest candidate score s_k (near ties, where fp32 and fp64 may order
  differently).
* out: max |gpu - ref| <= 2e-3 and sum |gpu - ref| / sum |ref| <= 1e-3, where ref is the
  oracle's softmax over the union the GPU selected (identical to the oracle's own union
  whenever the sets agree).
"""
from __future__ import annotations

import math

import numpy as np

import oracle

TIE_REL = 1e-4
MAX_ABS = 2e-3
MEAN_REL = 1e-3


def check_omega(got_row: np.ndarray, z: np.ndarray, N: int, n_sink: int, n_window: int, k: int):
    """Returns the GPU's Omega (as an int64 array) after validating it against the oracle."""
    C = oracle.candidate_set(N, n_sink, n_window)
    k_eff = min(k, C.size)
    got_row = np.asarray(got_row, dtype=np.int64)
    assert got_row.shape[0] >= k, (got_row.shape, k)
    om_gpu = got_row[:k_eff]
    assert np.all(got_row[k_eff:k] == -1), "entries past k_eff must be -1"
    assert np.unique(om_gpu).size == k_eff, "duplicate positions"
    if k_eff:
        assert np.all(np.isin(om_gpu, C)), "position outside the candidates"
    om = oracle.select_topk(z, C, k)
    diff = set(om_gpu.tolist()) ^ set(om.tolist())
    if diff:
        s_k = z[om[-1]]
        bad = [a for a in diff if abs(z[a] - s_k) > TIE_REL * max(1.0, abs(s_k))]
        assert not bad, f"{len(bad)} positions differ beyond the tie tolerance, e.g. {bad[:5]}"
    return om_gpu


def check_out(got: np.ndarray, ref: np.ndarray, what: str = "out"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    mean_rel = float(err.sum() / max(np.abs(ref).sum(), 1e-300))
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert mean_rel <= MEAN_REL, f"{what}: mean-rel {mean_rel:.3e} > {MEAN_REL}"
    return max_abs, mean_rel


def check_head(q_bits, K_bits, V_bits, k, n_sink, n_window, out_gpu, idx_gpu):
    """Full check of one query head: Omega and the sparse output."""
    q = oracle.bf16_to_f64(q_bits)
    K = oracle.bf16_to_f64(K_bits)
    V = oracle.bf16_to_f64(V_bits)
    N = K.shape[0]
    z = oracle.scores(q, K)
    om_gpu = check_omega(idx_gpu, z, N, n_sink, n_window, k)
    U = np.concatenate([oracle.static_set(N, n_sink, n_window), om_gpu])
    ref = oracle.attend(z, V, U)
    return check_out(out_gpu, ref)


def check_dense_head(q_bits, K_bits, V_bits, out_gpu):
    return check_out(out_gpu, oracle.dense_head(q_bits, K_bits, V_bits), "dense")


def check_omega_eps(got_row: np.ndarray, z: np.ndarray, N: int, n_sink: int, n_window: int,
                    k: int, eps: float):
    """The threshold budget's Omega: the oracle's set except near the threshold (scores within
    TIE_REL of T = ln eps + logsumexp(z), where fp32 and fp64 may decide differently) or near
    the cap's k-th score; entries past the GPU's count must be -1."""
    C = oracle.candidate_set(N, n_sink, n_window)
    got_row = np.asarray(got_row, dtype=np.int64)
    n_gpu = int(np.sum(got_row[:k] >= 0))
    om_gpu = got_row[:n_gpu]
    assert np.all(got_row[n_gpu:k] == -1), "kept keys must come first, then -1"
    assert np.unique(om_gpu).size == n_gpu, "duplicate positions"
    assert np.all(np.isin(om_gpu, C)), "position outside the candidates"
    om = oracle.select_threshold(z, C, k, eps)
    zmax = z.max()
    T = math.log(eps) + zmax + math.log(np.exp(z - zmax).sum())
    near = lambda a, ref: abs(z[a] - ref) <= TIE_REL * max(1.0, abs(ref))
    s_k = z[om[-1]] if om.size == k else None
    diff = set(om_gpu.tolist()) ^ set(om.tolist())
    bad = [a for a in diff if not (near(a, T) or (s_k is not None and near(a, s_k)))]
    assert not bad, f"{len(bad)} positions differ beyond the tolerance, e.g. {bad[:5]}"
    return om_gpu
