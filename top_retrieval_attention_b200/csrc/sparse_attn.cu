// Sparse attention over U = W u Omega (RetrievalAttention slides: "Sparse attention
// renormalizes selected tokens", Eq. (2) with the selected set; "Two local softmax outputs
// need global weights", Eqs. (3)-(5), and its backup slide, Appendix B).
//
// U is the virtual list [sinks, window, Omega].  It is cut into ranges of at most kMaxRange
// entries, one CTA per (range, query head).  A CTA reads the already computed scores z of its
// range (never K again), takes their max m_S, and gathers the V rows in sub-chunks of 64
// entries, accumulating N_S = sum e^{z - m_S} v and Z_S = sum e^{z - m_S} in fp32.  The last
// CTA of a head merges the partial states with the weights e^{m_S - m}, m = max_S m_S: the
// exact softmax over U.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "merge.cuh"

namespace ra {

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kSub = 64;                // entries per gather sub-chunk (16 rows per warp)

template <int D>
__global__ void __launch_bounds__(kAttnThreads) sparse_attn_kernel(const AttnParams p) {
  constexpr int CPL = D / 32;                 // channels per lane in the gather
  constexpr int RPW = kSub / kAttnWarps;      // rows per warp per sub-chunk
  constexpr int PS = D + kPartPad;            // partial-state stride (floats)
  const int split = blockIdx.x;
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = row / p.Hq;
  const int h = row - b * p.Hq;
  const int g = h / p.G;
  const __nv_bfloat16 *Vh = p.V + (static_cast<long long>(b) * p.Hkv + g) * p.cap * D;
  const float *srow = p.S + static_cast<long long>(row) * p.ldS;
  const int32_t *irow = p.idx + static_cast<long long>(row) * p.k;

  __shared__ int s_pos[kMaxRange];
  __shared__ float s_p[kMaxRange];
  __shared__ float s_red[kAttnWarps];
  __shared__ __align__(16) float s_acc[4 * kAttnThreads];   // per-warp sums, then merge buffer
  __shared__ bool s_last;

  pdl_trigger();
  pdl_wait();
  const long long nU = p.nW + p.k_eff;
  const long long e0 = static_cast<long long>(split) * p.range;
  const int n = static_cast<int>(min(static_cast<long long>(p.range), nU - e0));

  // positions and scores of this range; the range max
  float mloc = -INFINITY;
  for (int t = tid; t < n; t += kAttnThreads) {
    const long long e = e0 + t;
    int pos;
    if (e < p.s1)
      pos = static_cast<int>(e);
    else if (e < p.nW)
      pos = static_cast<int>(p.w0 + (e - p.s1));
    else
      pos = __ldg(irow + (e - p.nW));
    if (pos < 0 || pos >= p.N) pos = -1;   // never for a completed selection
    const float z = pos >= 0 ? __ldcg(srow + pos) : -INFINITY;
    s_pos[t] = pos;
    s_p[t] = z;
    mloc = fmaxf(mloc, z);
  }
  const float m = block_max<kAttnThreads>(mloc, s_red);   // barrier: s_pos / s_p complete
  float zsum = 0.f;
  for (int t = tid; t < n; t += kAttnThreads) {
    const float pe = s_pos[t] >= 0 ? expf(s_p[t] - m) : 0.f;
    s_p[t] = pe;
    zsum += pe;
  }
  const float Z = block_sum<kAttnThreads>(zsum, s_red);   // barrier: s_p holds the weights

  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
#pragma unroll 1
  for (int sc = 0; sc < n; sc += kSub) {
    if constexpr (CPL == 4) {
      uint2 w[RPW];
#pragma unroll
      for (int j = 0; j < RPW; ++j) {
        const int t = sc + warp + kAttnWarps * j;
        const int ps = t < n ? s_pos[t] : -1;
        w[j] = ps >= 0 ? __ldg(reinterpret_cast<const uint2 *>(Vh + static_cast<long long>(ps) * D) + lane)
                       : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int j = 0; j < RPW; ++j) {
        const int t = sc + warp + kAttnWarps * j;
        const float pw = t < n ? s_p[t] : 0.f;
        acc[0] += pw * bf16_lo(w[j].x);
        acc[1] += pw * bf16_hi(w[j].x);
        acc[2] += pw * bf16_lo(w[j].y);
        acc[3] += pw * bf16_hi(w[j].y);
      }
    } else {
      uint32_t w[RPW];
#pragma unroll
      for (int j = 0; j < RPW; ++j) {
        const int t = sc + warp + kAttnWarps * j;
        const int ps = t < n ? s_pos[t] : -1;
        w[j] = ps >= 0 ? __ldg(reinterpret_cast<const uint32_t *>(Vh + static_cast<long long>(ps) * D) + lane)
                       : 0u;
      }
#pragma unroll
      for (int j = 0; j < RPW; ++j) {
        const int t = sc + warp + kAttnWarps * j;
        const float pw = t < n ? s_p[t] : 0.f;
        acc[0] += pw * bf16_lo(w[j]);
        acc[1] += pw * bf16_hi(w[j]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < CPL; ++c) s_acc[warp * D + lane * CPL + c] = acc[c];
  __syncthreads();

  float *part = p.part + (static_cast<long long>(row) * p.nsplit + split) * PS;
  for (int c = tid; c < D; c += kAttnThreads)
    part[kPartPad + c] = (s_acc[c] + s_acc[D + c]) + (s_acc[2 * D + c] + s_acc[3 * D + c]);
  if (tid == 0) {
    part[0] = m;
    part[1] = Z;
  }
  // last-CTA hand-off: the barrier orders this CTA's partial-state stores before thread 0's
  // release fence and counter update; the CTA that sees the final count acquires and merges
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(p.meta + row * kMetaWords + kDone, 1u);
    s_last = prev == static_cast<uint32_t>(p.nsplit - 1);
    if (s_last) __threadfence();
  }
  __syncthreads();
  if (!s_last) return;

  // merge the partial states of all ranges of this query head (Eqs. (3)-(5))
  merge_states<D, kAttnThreads>(p.part + static_cast<long long>(row) * p.nsplit * PS, p.nsplit,
                                p.out + static_cast<long long>(row) * D, s_red, s_acc);
  if (tid == 0) p.meta[row * kMetaWords + kDone] = 0u;
}

cudaError_t launch_sparse_attn(const AttnParams &p, int d, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(p.nsplit), static_cast<unsigned>(p.R));
  return d == 128 ? launch_pdl(sparse_attn_kernel<128>, grid, dim3(kAttnThreads), 0, s, p)
                  : launch_pdl(sparse_attn_kernel<64>, grid, dim3(kAttnThreads), 0, s, p);
}

}  // namespace ra
