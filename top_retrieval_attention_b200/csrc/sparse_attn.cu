// Sparse attention over U = W u Omega (RetrievalAttention slides: "Sparse attention
// renormalizes selected tokens", Eq. (2) with the selected set; "Two local softmax outputs
// need global weights", Eqs. (3)-(5), and its backup slide, Appendix B).
//
// U is split into chunks of kAttnChunk entries.  Each CTA reads the already computed scores
// z (never K again) and gathers the V rows of its chunk, producing the partial state
// (m_S, Z_S, N_S) of its subset; the last CTA of a query head merges all partial states with
// the weights e^{m_S - m} (m = max_S m_S), which is the exact softmax over U.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace ra {

constexpr int kAttnThreads = 128;

__device__ __forceinline__ float block_reduce_max(float v, float *red) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kAttnThreads / 32; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}
__device__ __forceinline__ float block_reduce_sum(float v, float *red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < kAttnThreads / 32; ++w) r += red[w];
  __syncthreads();
  return r;
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads) sparse_attn_kernel(const AttnParams p) {
  constexpr int CH = kAttnChunk;
  constexpr int kWarps = kAttnThreads / 32;
  constexpr int CPL = D / 32;                 // channels per lane
  constexpr int RPW = CH / kWarps;            // rows per warp
  const int split = blockIdx.x;
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = row / p.Hq;
  const int h = row - b * p.Hq;
  const int g = h / p.G;
  const __nv_bfloat16 *Vh = p.V + (static_cast<long long>(b) * p.Hkv + g) * p.cap * D;
  const float *srow = p.S + static_cast<long long>(row) * p.ldS;

  __shared__ int s_pos[CH];
  __shared__ float s_p[CH];
  __shared__ float s_red[kWarps];
  __shared__ float s_acc[kWarps][D];
  __shared__ bool s_last;

  const long long nU = p.nW + p.k_eff;
  const long long e0 = static_cast<long long>(split) * CH;
  int pos = -1;
  float z = -INFINITY;
  if (tid < CH) {
    const long long e = e0 + tid;
    if (e < nU) {
      if (e < p.s1)
        pos = static_cast<int>(e);
      else if (e < p.nW)
        pos = static_cast<int>(p.w0 + (e - p.s1));
      else
        pos = __ldg(p.idx + static_cast<long long>(row) * p.k + (e - p.nW));
      if (pos < 0 || pos >= p.N) pos = -1;   // never for a completed selection
      if (pos >= 0) z = __ldcg(srow + pos);
    }
    s_pos[tid] = pos;
  }
  const float m = block_reduce_max(z, s_red);
  const float pe = pos >= 0 ? expf(z - m) : 0.f;
  if (tid < CH) s_p[tid] = pe;
  const float Z = block_reduce_sum(pe, s_red);   // contains a barrier: s_pos/s_p visible

  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
  if constexpr (CPL == 4) {
    uint2 w[RPW];
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
      const int ps = s_pos[warp + kWarps * j];
      w[j] = ps >= 0 ? __ldg(reinterpret_cast<const uint2 *>(Vh + static_cast<long long>(ps) * D) + lane)
                     : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
      const float pw = s_p[warp + kWarps * j];
      acc[0] += pw * bf16_lo(w[j].x);
      acc[1] += pw * bf16_hi(w[j].x);
      acc[2] += pw * bf16_lo(w[j].y);
      acc[3] += pw * bf16_hi(w[j].y);
    }
  } else {
    uint32_t w[RPW];
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
      const int ps = s_pos[warp + kWarps * j];
      w[j] = ps >= 0 ? __ldg(reinterpret_cast<const uint32_t *>(Vh + static_cast<long long>(ps) * D) + lane)
                     : 0u;
    }
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
      const float pw = s_p[warp + kWarps * j];
      acc[0] += pw * bf16_lo(w[j]);
      acc[1] += pw * bf16_hi(w[j]);
    }
  }
#pragma unroll
  for (int c = 0; c < CPL; ++c) s_acc[warp][lane * CPL + c] = acc[c];
  __syncthreads();

  float *part = p.part + (static_cast<long long>(row) * p.nsplit + split) * (D + 2);
  for (int c = tid; c < D; c += kAttnThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += s_acc[w][c];
    part[2 + c] = s;
  }
  if (tid == 0) {
    part[0] = m;
    part[1] = Z;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(p.meta + row * kMetaWords + kDone, 1u);
    s_last = prev == static_cast<uint32_t>(p.nsplit - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // merge the partial states of all splits of this query head (Eqs. (3)-(5))
  const float *prow = p.part + static_cast<long long>(row) * p.nsplit * (D + 2);
  float M = -INFINITY;
  for (int j = 0; j < p.nsplit; ++j) M = fmaxf(M, __ldcg(prow + j * (D + 2)));
  for (int c = tid; c < D; c += kAttnThreads) {
    float num = 0.f, den = 0.f;
    for (int j = 0; j < p.nsplit; ++j) {
      const float wj = expf(__ldcg(prow + j * (D + 2)) - M);
      den += wj * __ldcg(prow + j * (D + 2) + 1);
      num += wj * __ldcg(prow + j * (D + 2) + 2 + c);
    }
    p.out[static_cast<long long>(row) * D + c] = num / den;
  }
  if (tid == 0) p.meta[row * kMetaWords + kDone] = 0u;
}

cudaError_t launch_sparse_attn(const AttnParams &p, int d, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(p.nsplit), static_cast<unsigned>(p.R));
  if (d == 128)
    sparse_attn_kernel<128><<<grid, kAttnThreads, 0, s>>>(p);
  else
    sparse_attn_kernel<64><<<grid, kAttnThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ra
