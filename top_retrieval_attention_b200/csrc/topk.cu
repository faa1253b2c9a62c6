// Exact per-query-head top-k over the candidate positions C = [0, N) \ W (RetrievalAttention
// slides, "The GPU keeps 640 fixed positions": W and Omega are disjoint, one index per query
// head; "Sparse attention renormalizes selected tokens": a fixed top-k budget).
//
// Keys are compared as 64-bit composites (order_key(z) << 32 | ~position), so every key is
// distinct, larger z wins and equal z goes to the lower position.  The selection is a radix
// select:
//   1. (score kernel) histogram of the top 11 bits of order_key(z) per query head;
//   2. collect: every CTA of a head finds the threshold bin b* from that histogram; positions
//      whose bin is above b* are selected outright, those in b* become candidates;
//   3. finish (one CTA per head): further 8-bit digits of the composite narrow the threshold
//      bucket until it is taken whole or holds at most 64 keys, which one warp sorts with a
//      bitonic network; the top remainder is emitted.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace ra {

constexpr int kCollectThreads = 256;
constexpr int kFinishThreads = 512;
constexpr int kFinishCache = 8192;   // candidates cached in shared memory (64 KB)
constexpr int kBitonic = 64;

__device__ __forceinline__ uint64_t composite(const float *srow, uint32_t pos) {
  return (static_cast<uint64_t>(order_key(srow[pos])) << 32) | (0xFFFFFFFFu - pos);
}
__device__ __forceinline__ uint32_t comp_pos(uint64_t x) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(x);
}

// Inclusive prefix sum over the threads of a block of kThreads (multiple of 32).
template <int kThreads>
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t *warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kThreads / 32 ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < kThreads / 32) warp_tot[lane] = w;
  }
  __syncthreads();
  return v + (warp > 0 ? warp_tot[warp - 1] : 0u);
}

__global__ void __launch_bounds__(kCollectThreads) topk_collect_kernel(const TopkParams p) {
  const int row = blockIdx.y;
  const int tid = threadIdx.x;
  __shared__ uint32_t warp_tot[kCollectThreads / 32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  if (p.k_eff == 0) return;
  const bool take_all = p.k_eff >= p.nC;
  int bstar = -1;
  if (!take_all) {
    // thread t owns bins [2048 - 8(t+1), 2048 - 8t): thread 0 holds the highest bins
    constexpr int kPer = kHistBins / kCollectThreads;
    const uint32_t *h = p.hist + static_cast<long long>(row) * kHistBins;
    uint32_t loc[kPer];
    uint32_t s = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      loc[i] = h[kHistBins - kPer * (tid + 1) + (kPer - 1 - i)];   // i = 0 is the highest bin
      s += loc[i];
    }
    const uint32_t incl = block_incl_scan<kCollectThreads>(s, warp_tot);
    const uint32_t excl = incl - s;
    const uint32_t kk = static_cast<uint32_t>(p.k_eff);
    if (excl < kk && kk <= incl) {
      uint32_t cum = excl;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (cum + loc[i] >= kk) {
          s_bin = kHistBins - kPer * (tid + 1) + (kPer - 1 - i);
          s_above = cum;
          break;
        }
        cum += loc[i];
      }
    }
    __syncthreads();
    bstar = s_bin;
    if (blockIdx.x == 0 && tid == 0) {
      p.meta[row * kMetaWords + kThreshBin] = static_cast<uint32_t>(bstar);
      p.meta[row * kMetaWords + kAbove] = s_above;
    }
  }

  const float *srow = p.S + static_cast<long long>(row) * p.ldS;
  int32_t *irow = p.idx + static_cast<long long>(row) * p.k;
  uint32_t *crow = p.cand + static_cast<long long>(row) * p.ldC;
  uint32_t *sel_ctr = p.meta + row * kMetaWords + kSelCount;
  uint32_t *cand_ctr = p.meta + row * kMetaWords + kCandCount;
  long long lo = static_cast<long long>(blockIdx.x) * p.chunk;
  long long hi = lo + p.chunk;
  if (lo < p.cand_lo) lo = p.cand_lo;
  if (hi > p.cand_hi) hi = p.cand_hi;
  if (lo >= hi) return;
  const long long base = lo & ~3LL;
#pragma unroll 1
  for (long long i0 = base; i0 < hi; i0 += 4 * kCollectThreads) {
    const long long i = i0 + 4 * tid;
    float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < hi) z4 = __ldcg(reinterpret_cast<const float4 *>(srow + i));
    const float zz[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const long long pos = i + e;
      const bool valid = pos >= lo && pos < hi;
      const int bin = static_cast<int>(order_key(zz[e]) >> (32 - kHistBits));
      bool ok;
      const uint32_t s1 = warp_append(valid && bin > bstar, sel_ctr, ok);
      if (ok && s1 < p.k_eff) irow[s1] = static_cast<int32_t>(pos);
      const uint32_t s2 = warp_append(valid && !take_all && bin == bstar, cand_ctr, ok);
      if (ok && s2 < p.ldC) crow[s2] = static_cast<uint32_t>(pos);
    }
  }
}

__global__ void __launch_bounds__(kFinishThreads) topk_finish_kernel(const TopkParams p) {
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int32_t *irow = p.idx + static_cast<long long>(row) * p.k;
  for (long long i = p.k_eff + tid; i < p.k; i += kFinishThreads) irow[i] = -1;

  // read this row's counters, then leave the counter block zero for the next call
  uint32_t *meta_w = p.meta + row * kMetaWords;
  const uint32_t above = meta_w[kAbove];
  const uint32_t n_cand = meta_w[kCandCount];
  const uint32_t bstar = meta_w[kThreshBin];
  __syncthreads();
  if (tid < kError) meta_w[tid] = 0u;
  {
    uint32_t *h = const_cast<uint32_t *>(p.hist) + static_cast<long long>(row) * kHistBins;
    for (int i = tid; i < kHistBins; i += kFinishThreads) h[i] = 0u;
  }
  if (p.k_eff == 0 || p.k_eff >= p.nC) return;

  extern __shared__ __align__(16) uint64_t cache[];
  __shared__ uint32_t h256[256];
  __shared__ uint32_t s_out;
  __shared__ int s_digit;
  __shared__ uint32_t s_cum, s_cnt, s_nb;
  __shared__ uint64_t bs[kBitonic];

  uint32_t rr = static_cast<uint32_t>(p.k_eff) - above;    // 1 <= rr <= n_cand
  const float *srow = p.S + static_cast<long long>(row) * p.ldS;
  const uint32_t *crow = p.cand + static_cast<long long>(row) * p.ldC;
  if (n_cand > p.nC || above >= p.k_eff) return;   // counters not from this call
  const bool cached = n_cand <= static_cast<uint32_t>(kFinishCache);
  if (tid == 0) s_out = above;
  if (cached)
    for (uint32_t i = tid; i < n_cand; i += kFinishThreads) cache[i] = composite(srow, __ldcg(crow + i));
  __syncthreads();
  auto get = [&](uint32_t i) -> uint64_t {
    return cached ? cache[i] : composite(srow, __ldcg(crow + i));
  };

  uint64_t prefix = bstar;    // the top (64 - shift) bits shared by the remaining keys
  int shift = 64 - kHistBits;
  uint32_t cnt = n_cand;
  if (tid == 0) s_digit = 0;
  // at most ceil(53 / 8) + 1 rounds: every round fixes 8 more bits of a unique 64-bit key
#pragma unroll 1
  for (int round = 0; round < 9; ++round) {
    if (cnt == rr) {   // the whole bucket is taken
      for (uint32_t i = tid; i < n_cand; i += kFinishThreads) {
        const uint64_t x = get(i);
        if ((x >> shift) == prefix) {
          const uint32_t o = atomicAdd(&s_out, 1u);
          if (o < p.k_eff) irow[o] = static_cast<int32_t>(comp_pos(x));
        }
      }
      return;
    }
    if (cnt <= kBitonic) {   // bitonic finish of the threshold bucket
      if (tid < kBitonic) bs[tid] = 0;
      if (tid == 0) s_nb = 0;
      __syncthreads();
      for (uint32_t i = tid; i < n_cand; i += kFinishThreads) {
        const uint64_t x = get(i);
        if ((x >> shift) == prefix) bs[atomicAdd(&s_nb, 1u)] = x;
      }
      __syncthreads();
      if (warp == 0) {
#pragma unroll 1
        for (int size = 2; size <= kBitonic; size <<= 1) {
#pragma unroll 1
          for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const int i = 2 * stride * (lane / stride) + (lane % stride);
            const int j = i + stride;
            const uint64_t a = bs[i], b = bs[j];
            const bool desc = (i & size) == 0;
            if (desc ? (a < b) : (a > b)) {
              bs[i] = b;
              bs[j] = a;
            }
            __syncwarp();
          }
        }
        for (uint32_t i = lane; i < rr && s_out + i < p.k_eff; i += 32)
          irow[s_out + i] = static_cast<int32_t>(comp_pos(bs[i]));
      }
      return;
    }
    // one more radix digit of the composite
    const int nshift = shift > 8 ? shift - 8 : 0;
    const int nb = shift - nshift;
    const uint64_t dmask = (1ull << nb) - 1;
    if (tid < 256) h256[tid] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < n_cand; i += kFinishThreads) {
      const uint64_t x = get(i);
      if ((x >> shift) == prefix) atomicAdd(&h256[(x >> nshift) & dmask], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits [256 - 8(l+1), 256 - 8l), highest first
      uint32_t loc[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        loc[i] = h256[255 - 8 * lane - i];
        s += loc[i];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      const uint32_t excl = incl - s;
      if (excl < rr && rr <= incl) {
        uint32_t cum = excl;
        for (int i = 0; i < 8; ++i) {
          if (cum + loc[i] >= rr) {
            s_digit = 255 - 8 * lane - i;
            s_cum = cum;
            s_cnt = loc[i];
            break;
          }
          cum += loc[i];
        }
      }
    }
    __syncthreads();
    const uint64_t v = static_cast<uint64_t>(s_digit);
    const uint32_t cum = s_cum;
    // keys of this bucket with a larger digit are selected
    for (uint32_t i = tid; i < n_cand; i += kFinishThreads) {
      const uint64_t x = get(i);
      if ((x >> shift) == prefix && ((x >> nshift) & dmask) > v) {
        const uint32_t o = atomicAdd(&s_out, 1u);
        if (o < p.k_eff) irow[o] = static_cast<int32_t>(comp_pos(x));
      }
    }
    rr -= cum;
    cnt = s_cnt;
    prefix = (prefix << nb) | v;
    shift = nshift;
    __syncthreads();
  }
  if (tid == 0) p.meta[row * kMetaWords + kError] = 1u;   // unreachable for unique keys
}

cudaError_t launch_topk(const TopkParams &p, cudaStream_t s) {
  if (p.k_eff > 0) {
    const long long chunks = (p.N + p.chunk - 1) / p.chunk;
    dim3 grid(static_cast<unsigned>(chunks), static_cast<unsigned>(p.R));
    topk_collect_kernel<<<grid, kCollectThreads, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.k > 0) {
    const size_t smem = static_cast<size_t>(kFinishCache) * sizeof(uint64_t);
    static bool done[64] = {};
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(topk_finish_kernel),
                                            static_cast<int>(smem), done);
    if (e != cudaSuccess) return e;
    topk_finish_kernel<<<p.R, kFinishThreads, smem, s>>>(p);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace ra
