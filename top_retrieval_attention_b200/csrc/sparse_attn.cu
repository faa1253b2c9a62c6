// Sparse attention over U = W u Omega (RetrievalAttention slides: "Sparse attention
// renormalizes selected tokens", Eq. (2) with the selected set; "Two local softmax outputs
// need global weights", Eqs. (3)-(5), and its backup slide, Appendix B).
//
// Two kinds of CTA, each covering a range of the selected set, 64 entries at a time:
//   * static CTAs (one set per KV head and quad of its query heads): rows of W = sinks +
//     window, shared by the G query heads of the KV head (slide "The GPU keeps 640 fixed
//     positions"): each V row is gathered once and weighted for up to four heads;
//   * retrieved CTAs (one set per query head): rows of Omega, that head's top-k.
// A warp takes 16 entries: their positions, scores z (already computed; K is never read
// again) and V rows are loaded together, the warp reduces its own max m, sum Z and
// N = sum e^{z - m} v with shuffles, and the CTA combines its four warps into one partial
// state (m_S, Z_S, N_S).  The last CTA to finish a query head merges that head's partial states
// with the weights e^{m_S - m}, m = max_S m_S: the exact softmax over U.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "merge.cuh"

namespace ra {

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kRowsPerWarp = kAttnRange / kAttnWarps;   // 16
constexpr int kStaticHeads = 4;   // query heads served by one static CTA (a KV head's quad)

// One warp: 16 entries (rows) at positions pos (lane j < 16 holds entry j, -1 when absent),
// the scores of nh heads (z[h], lane j), V rows gathered 4 (d=128) or 2 (d=64) channels per
// lane.  Produces per head the warp's max m, sum Z (lane-uniform) and acc (this lane's
// channels).
template <int D, int NH>
__device__ __forceinline__ void warp_rows(const __nv_bfloat16 *Vh, int pos, const float (&z)[NH],
                                          int nh, float (&m)[NH], float (&Zs)[NH],
                                          float (&acc)[NH][D / 32]) {
  constexpr int CPL = D / 32;
  const int lane = threadIdx.x & 31;
  // V rows first: their loads overlap the reductions below
  uint32_t w[kRowsPerWarp][CPL / 2];
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) {
    const int pj = __shfl_sync(0xffffffffu, pos, j);
    if (pj >= 0) {
      const __nv_bfloat16 *row = Vh + static_cast<long long>(pj) * D;
      if constexpr (CPL == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(row) + lane);
        w[j][0] = v.x;
        w[j][1] = v.y;
      } else {
        w[j][0] = __ldg(reinterpret_cast<const uint32_t *>(row) + lane);
      }
    } else {
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) w[j][c] = 0u;
    }
  }
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    if (h >= nh) continue;
    const float zz = (lane < kRowsPerWarp && pos >= 0) ? z[h] : -INFINITY;
    float mh = zz;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) mh = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, o));
    mh = __shfl_sync(0xffffffffu, mh, 0);
    const float pe = (lane < kRowsPerWarp && pos >= 0) ? expf(zz - mh) : 0.f;
    float zs = pe;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
    m[h] = mh;
    Zs[h] = __shfl_sync(0xffffffffu, zs, 0);
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[h][c] = 0.f;
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
      const float pj = __shfl_sync(0xffffffffu, pe, j);
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) {
        acc[h][2 * c] += pj * bf16_lo(w[j][c]);
        acc[h][2 * c + 1] += pj * bf16_hi(w[j][c]);
      }
    }
  }
}

// Combines the four warps' states of one head (smem: m[4], Z[4], acc[4][D]) into a partial
// state in global memory.
template <int D>
__device__ __forceinline__ void cta_combine(const float *wm, const float *wz, const float *wacc,
                                            float *part) {
  const float M = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
  float e[kAttnWarps];
#pragma unroll
  for (int i = 0; i < kAttnWarps; ++i) e[i] = wm[i] == -INFINITY ? 0.f : expf(wm[i] - M);
  for (int c = threadIdx.x; c < D; c += kAttnThreads) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kAttnWarps; ++i) s += e[i] * wacc[i * D + c];
    part[kPartPad + c] = s;
  }
  if (threadIdx.x == 0) {
    float zt = 0.f;
#pragma unroll
    for (int i = 0; i < kAttnWarps; ++i) zt += e[i] * wz[i];
    part[0] = M;
    part[1] = zt;
  }
}

// Shared memory of one CTA: per-warp states of up to kStaticHeads heads, then the merge buffer.
template <int D>
struct AttnSmem {
  float m[kStaticHeads][kAttnWarps];
  float z[kStaticHeads][kAttnWarps];
  __align__(16) float acc[kStaticHeads * kAttnWarps * D + (D == 64 ? 256 : 0)];
  float red[kAttnWarps];
  int last[kStaticHeads];
};

// Running per-warp state of NH heads, merged group by group (online softmax):
//   m' = max(m, m_g), Z' = Z e^{m - m'} + Z_g e^{m_g - m'}, acc' likewise.
template <int D, int NH>
__device__ __forceinline__ void fold(float (&m)[NH], float (&Zs)[NH], float (&acc)[NH][D / 32],
                                     const float (&mg)[NH], const float (&Zg)[NH],
                                     const float (&ag)[NH][D / 32], int nh) {
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    if (h >= nh || mg[h] == -INFINITY) continue;
    const float mn = fmaxf(m[h], mg[h]);
    const float a = m[h] == -INFINITY ? 0.f : expf(m[h] - mn);
    const float bsc = expf(mg[h] - mn);
    Zs[h] = Zs[h] * a + Zg[h] * bsc;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) acc[h][c] = acc[h][c] * a + ag[h][c] * bsc;
    m[h] = mn;
  }
}

// The body for CTAs covering NH heads (NH = kMaxGroup for static CTAs, of which the first
// nrows are real; NH = 1 for retrieved CTAs), all array indices compile-time.  The CTA's
// entries [e_lo, e_hi) are taken 64 at a time; entry(e) gives the position and the scores.
template <int D, int NH, typename Entry>
__device__ __forceinline__ void attn_cta(const AttnParams &p, AttnSmem<D> &sm, int row0, int nrows,
                                         int split, const __nv_bfloat16 *Vh, long long e_lo,
                                         long long e_hi, Entry entry) {
  constexpr int CPL = D / 32;
  constexpr int PS = D + kPartPad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float m[NH], Zs[NH], acc[NH][CPL];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    m[h] = -INFINITY;
    Zs[h] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[h][c] = 0.f;
  }
  for (long long g0 = e_lo; g0 < e_hi; g0 += kAttnRange) {
    const long long e = g0 + warp * kRowsPerWarp + lane;
    int pos = -1;
    float z[NH];
    entry(lane < kRowsPerWarp && e < e_hi ? e : -1, pos, z);
    float mg[NH], Zg[NH], ag[NH][CPL];
    warp_rows<D, NH>(Vh, pos, z, nrows, mg, Zg, ag);
    fold<D, NH>(m, Zs, acc, mg, Zg, ag, nrows);
  }
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    if (h < nrows) {
      if (lane == 0) {
        sm.m[h][warp] = m[h];
        sm.z[h][warp] = Zs[h];
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) sm.acc[(h * kAttnWarps + warp) * D + lane * CPL + c] = acc[h][c];
    }
  }
  __syncthreads();
  for (int h = 0; h < nrows; ++h)
    cta_combine<D>(sm.m[h], sm.z[h], sm.acc + h * kAttnWarps * D,
                   p.part + (static_cast<long long>(row0 + h) * p.nsplit + split) * PS);

  // last-CTA hand-off per query head: the barrier orders this CTA's partial-state stores
  // before the release fence and counter update; a CTA that completes a head merges it
  __syncthreads();
  if (tid < nrows) {
    __threadfence();
    const uint32_t prev = atomicAdd(p.meta + (row0 + tid) * kMetaWords + kDone, 1u);
    sm.last[tid] = prev == static_cast<uint32_t>(p.nsplit - 1);
    if (sm.last[tid]) __threadfence();
  }
  __syncthreads();
  for (int h = 0; h < nrows; ++h) {
    if (!sm.last[h]) continue;   // uniform: shared flag
    const int row = row0 + h;
    merge_states<D, kAttnThreads>(p.part + static_cast<long long>(row) * p.nsplit * PS, p.nsplit,
                                  p.out + static_cast<long long>(row) * D, sm.red, sm.acc);
    if (tid == 0) p.meta[row * kMetaWords + kDone] = 0u;
  }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 6) sparse_attn_kernel(const AttnParams p) {
  __shared__ AttnSmem<D> sm;
  pdl_trigger();
  pdl_wait();
  const int n_quads = (p.G + kStaticHeads - 1) / kStaticHeads;   // head quads per KV head
  const long long n_static_ctas = static_cast<long long>(p.B) * p.Hkv * n_quads * p.nWsplit;
  if (blockIdx.x < n_static_ctas) {
    // (KV head, quad of its query heads, range of W)
    const long long gq = blockIdx.x / p.nWsplit;
    const int s = static_cast<int>(blockIdx.x - gq * p.nWsplit);
    const int grp = static_cast<int>(gq / n_quads);                  // b * Hkv + g
    const int quad = static_cast<int>(gq - static_cast<long long>(grp) * n_quads);
    const int b = grp / p.Hkv, g = grp - b * p.Hkv;
    const int row0 = b * p.Hq + g * p.G + quad * kStaticHeads;
    const int nrows = min(kStaticHeads, p.G - quad * kStaticHeads);
    const long long e_lo = static_cast<long long>(s) * p.wrange;
    const long long e_hi = min(e_lo + p.wrange, p.nW);
    auto entry = [&](long long e, int &pos, float (&z)[kStaticHeads]) {
      pos = e < 0 ? -1 : static_cast<int>(e < p.s1 ? e : p.w0 + (e - p.s1));
#pragma unroll
      for (int h = 0; h < kStaticHeads; ++h)
        z[h] = (h < nrows && pos >= 0) ? __ldcg(p.S + (row0 + h) * p.ldS + pos) : -INFINITY;
    };
    attn_cta<D, kStaticHeads>(p, sm, row0, nrows, s,
                              p.V + static_cast<long long>(grp) * p.cap * D, e_lo, e_hi, entry);
  } else {
    const long long id = blockIdx.x - n_static_ctas;
    const int row = static_cast<int>(id / p.nOsplit);
    const int s = static_cast<int>(id - static_cast<long long>(row) * p.nOsplit);
    const int b = row / p.Hq, h = row - b * p.Hq;
    const long long e_lo = static_cast<long long>(s) * p.orange;
    const long long e_hi = min(e_lo + p.orange, p.k_eff);
    const int32_t *irow = p.idx + static_cast<long long>(row) * p.k;
    const float *srow = p.S + row * p.ldS;
    auto entry = [&](long long e, int &pos, float (&z)[1]) {
      pos = e < 0 ? -1 : __ldg(irow + e);
      if (pos >= p.N) pos = -1;   // never for a completed selection
      z[0] = pos >= 0 ? __ldcg(srow + pos) : -INFINITY;
    };
    attn_cta<D, 1>(p, sm, row, 1, p.nWsplit + s,
                   p.V + (static_cast<long long>(b) * p.Hkv + h / p.G) * p.cap * D, e_lo, e_hi,
                   entry);
  }
}

cudaError_t launch_sparse_attn(const AttnParams &p, int d, cudaStream_t s) {
  const long long ctas = static_cast<long long>(p.B) * p.Hkv * ((p.G + 3) / 4) * p.nWsplit +
                         static_cast<long long>(p.R) * p.nOsplit;
  const dim3 grid(static_cast<unsigned>(ctas));
  return d == 128 ? launch_pdl(sparse_attn_kernel<128>, grid, dim3(kAttnThreads), 0, s, p)
                  : launch_pdl(sparse_attn_kernel<64>, grid, dim3(kAttnThreads), 0, s, p);
}

}  // namespace ra
