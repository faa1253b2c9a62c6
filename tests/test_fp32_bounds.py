"""The parity tolerances against fp32 arithmetic (CPU only).

The CUDA path scores in fp32 (bf16 products, which fp32 holds exactly, summed in fp32) and
attends in fp32; the fp64 oracle is the reference.  These tests redo the tiny decode workload
with numpy float32 arithmetic of that kind (a plain restatement, not the CUDA code) and check
that fp32 rounding alone stays inside the bounds the GPU is held to:

* every score is within the textbook bound for a sum of d terms in precision u = 2^-24,
  |fl(sum) - sum| <= d u sum|terms| (sequential summation), and an order of magnitude below
  the 1e-4 relative tie tolerance used for the selected set;
* the attention output over the oracle's union meets max-abs 2e-3 and mean-rel 1e-3 with a
  wide margin.
"""
import numpy as np

import oracle
from parity import MAX_ABS, MEAN_REL, TIE_REL
from synth import gen

U32 = 2.0 ** -24


def _f32(bits):
    return oracle.bf16_to_f64(bits).astype(np.float32)


def _scores_f32(q32, K32):
    """z = q . k / sqrt(d), every product and partial sum rounded to fp32, channel by channel."""
    acc = np.zeros(K32.shape[0], dtype=np.float32)
    for c in range(K32.shape[1]):
        acc = (acc + q32[c] * K32[:, c]).astype(np.float32)
    return (acc / np.float32(np.sqrt(K32.shape[1]))).astype(np.float32)


def _workload():
    w = gen.workload("tiny")
    q, K, V, _ = gen.host_layer(w)
    return w, q, K, V


def test_fp32_scores_stay_within_the_summation_bound():
    w, q, K, V = _workload()
    d = w.d
    for h in range(w.Hq):
        g = h // w.G
        z64 = oracle.scores(oracle.bf16_to_f64(q[0, h]), oracle.bf16_to_f64(K[0, g]))
        z32 = _scores_f32(_f32(q[0, h]), _f32(K[0, g])).astype(np.float64)
        mag = np.abs(oracle.bf16_to_f64(K[0, g])) @ np.abs(oracle.bf16_to_f64(q[0, h]))
        bound = (d + 2) * U32 * mag / np.sqrt(d) + U32 * np.abs(z64)   # sum, then the scaling
        err = np.abs(z32 - z64)
        assert np.all(err <= bound), float((err - bound).max())
        assert float((err / np.maximum(1.0, np.abs(z64))).max()) < TIE_REL / 10


def test_fp32_attention_meets_the_output_tolerances_with_margin():
    w, q, K, V = _workload()
    for h in range(w.Hq):
        g = h // w.G
        V64 = oracle.bf16_to_f64(V[0, g])
        z64 = oracle.scores(oracle.bf16_to_f64(q[0, h]), oracle.bf16_to_f64(K[0, g]))
        C = oracle.candidate_set(w.N, w.n_sink, w.n_window)
        U = np.concatenate([oracle.static_set(w.N, w.n_sink, w.n_window),
                            oracle.select_topk(z64, C, w.k)])
        ref = oracle.attend(z64, V64, U)
        # fp32: scores, max, exponentials, normaliser and weighted sum of V rows
        z32 = _scores_f32(_f32(q[0, h]), _f32(K[0, g]))[U]
        m = z32.max()
        e = np.exp((z32 - m).astype(np.float32)).astype(np.float32)
        num = np.zeros(w.d, dtype=np.float32)
        for i, pos in enumerate(U):
            num = (num + e[i] * V64[pos].astype(np.float32)).astype(np.float32)
        out = (num / np.float32(e.sum(dtype=np.float32))).astype(np.float64)
        err = np.abs(out - ref)
        assert err.max() <= MAX_ABS / 10
        assert err.sum() / np.abs(ref).sum() <= MEAN_REL / 10
