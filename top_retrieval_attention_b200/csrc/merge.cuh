// Merge of split partial softmax states, shared by the sparse and dense attention kernels.
//
// A partial state of subset S is (m_S, Z_S, N_S) with m_S = max z, Z_S = sum e^{z - m_S} and
// N_S = sum e^{z - m_S} v (RetrievalAttention slides, slide "Backup: the normalization
// identity", Appendix B).  Disjoint subsets merge to the exact softmax over their union:
//   o = sum_S e^{m_S - m} N_S / sum_S e^{m_S - m} Z_S,  m = max_S m_S      (Eqs. (3)-(5)).
// Layout of one state: [m, Z, pad, pad, N[0..D)], stride D + kPartPad floats (16-byte rows).
#pragma once

#include <math.h>

#include "common.cuh"

namespace ra {

constexpr int kPartPad = 4;

template <int kThreads>
__device__ __forceinline__ float block_max(float v, float *red) {
  v = warp_max(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

template <int kThreads>
__device__ __forceinline__ float block_sum(float v, float *red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) r += red[w];
  __syncthreads();
  return r;
}

// Merges the nsplit states at prow (stride D + kPartPad) into out[0..D) with the whole block.
// Two dependent L2 round trips: (m_S, Z_S) in one pass with a running max, then N_S with the
// loads spread over (channel quad, split group).  red: kThreads / 32 floats; buf: 4 * kThreads floats (16-byte aligned).
template <int D, int kThreads>
__device__ __forceinline__ void merge_states(const float *prow, int nsplit, float *out, float *red,
                                             float *buf) {
  constexpr int PS = D + kPartPad;
  constexpr int kQuads = D / 4;
  constexpr int kGroups = kThreads / kQuads;
  const int tid = threadIdx.x;
  // one pass over (m_S, Z_S): each thread keeps a running (max, normaliser) of its states
  float mt = -INFINITY, zt = 0.f;
  for (int j = tid; j < nsplit; j += kThreads) {
    const float m = __ldcg(prow + j * PS), z = __ldcg(prow + j * PS + 1);
    if (m == -INFINITY) continue;   // an empty state contributes nothing
    if (m > mt) {
      zt = zt * expf(mt - m) + z;
      mt = m;
    } else {
      zt += z * expf(m - mt);
    }
  }
  const float M = block_max<kThreads>(mt, red);
  const float den = block_sum<kThreads>(mt == -INFINITY ? 0.f : zt * expf(mt - M), red);
  const int cq = tid % kQuads, sg = tid / kQuads;
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int j = sg; j < nsplit; j += kGroups) {
    const float wj = expf(__ldcg(prow + j * PS) - M);
    const float4 nv = __ldcg(reinterpret_cast<const float4 *>(prow + j * PS + kPartPad) + cq);
    num.x += wj * nv.x;
    num.y += wj * nv.y;
    num.z += wj * nv.z;
    num.w += wj * nv.w;
  }
  reinterpret_cast<float4 *>(buf + sg * D)[cq] = num;
  __syncthreads();
  for (int c = tid; c < D; c += kThreads) {
    float s = 0.f;
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) s += buf[gi * D + c];
    out[c] = s / den;
  }
  __syncthreads();
}

}  // namespace ra
