// Exact per-query-head top-k over the candidate positions C = [0, N) \ W (RetrievalAttention
// slides, "The GPU keeps 640 fixed positions": W and Omega are disjoint, one index per query
// head; "Sparse attention renormalizes selected tokens": a fixed top-k budget).
//
// Keys are compared as 64-bit composites (order_key(z) << 32 | ~position), so every key is
// distinct, larger z wins and equal z goes to the lower position.  The selection is a radix
// select over digits of the composite, in two kernels:
//   * collect, (head, chunk) CTAs: digit 1 = the top 11 bits of order_key(z), histogrammed
//     by the score kernel; every CTA finds the threshold bin b1 (the bin holding the k-th
//     largest key), writes out the keys above b1 and lists the keys in b1 (position and
//     key), placing them with one block scan and one reservation atomic per list, and
//     histograms digit 2 (the next 11 bits) of the listed keys;
//   * refine, (head, part) CTAs over the list: the digit-2 threshold bin b2; listed keys
//     above (b1, b2) are written out and those in (b1, b2) moved to a bucket; the last CTA
//     of a head narrows the bucket with further 8-bit digits until it is taken whole or
//     holds at most 64 keys, which one warp sorts with a bitonic network.
// A digit-1 bin is a range of z (order_key is monotone), so the per-key test is a pair of
// float comparisons.  Histograms and counters are left zero for the next call.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace ra {

constexpr int kTkThreads = 256;
constexpr int kBucketCap = kTopkBucket;   // bucket entries kept per head (32 KB in the tail)
constexpr int kBitonic = 64;
constexpr int kDigit2Shift = 10;     // digit 2 = bits [10, 21) of the order key
constexpr int kRefineParts = 16;     // refine CTAs per query head
constexpr int kPerThread = kTopkChunk / kTkThreads;   // 32 keys per thread
constexpr int kVec = kPerThread / 4;                  // float4 loads per thread


__device__ __forceinline__ uint64_t make_composite(uint32_t key, uint32_t pos) {
  return (static_cast<uint64_t>(key) << 32) | (0xFFFFFFFFu - pos);
}
__device__ __forceinline__ uint32_t comp_pos(uint64_t x) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(x);
}

// Inclusive prefix sum over the threads of a block of kThreads (multiple of 32, <= 1024).
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
  const uint32_t r = v + (warp > 0 ? warp_tot[warp - 1] : 0u);
  __syncthreads();   // warp_tot may be reused by the caller
  return r;
}

// Threshold bin of a 2048-bin histogram h (global, read through L2): the bin holding the
// `want`-th largest element, the count above it and its own count.  Whole block, one result
// in shared memory (valid after the call).
struct Thresh {
  int bin;
  uint32_t above, cnt;
};
template <int kThreads>
__device__ __forceinline__ Thresh find_threshold(const uint32_t *h, uint32_t want,
                                                 uint32_t *warp_tot, Thresh *out) {
  constexpr int kPer = kHistBins / kThreads;
  uint32_t loc[kPer];   // loc[0] = highest bin of this thread; thread 0 owns the highest bins
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    loc[i] = __ldcg(h + kHistBins - kPer * (threadIdx.x + 1) + (kPer - 1 - i));
    s += loc[i];
  }
  const uint32_t incl = block_incl_scan<kThreads>(s, warp_tot);
  const uint32_t excl = incl - s;
  if (excl < want && want <= incl) {
    uint32_t cum = excl;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (cum + loc[i] >= want) {
        out->bin = kHistBins - kPer * (static_cast<int>(threadIdx.x) + 1) + (kPer - 1 - i);
        out->above = cum;
        out->cnt = loc[i];
        break;
      }
      cum += loc[i];
    }
  }
  __syncthreads();
  return *out;
}

// The float whose order key is `key` (order_key is a bijection on bit patterns and monotone,
// so key(z) >= key  <=>  z >= key_float(key) for the finite keys used as thresholds here).
__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// This CTA's chunk of z (kPerThread values per thread, all loads in flight).  Element j of a
// thread is chunk offset off(j) = 4 * ((j / 4) * kTkThreads + tid) + j % 4.
__device__ __forceinline__ void load_chunk(const float *src, int l0, int l1, float (&z)[kPerThread]) {
#pragma unroll
  for (int u = 0; u < kVec; ++u) {
    const int i = 4 * (u * kTkThreads + static_cast<int>(threadIdx.x));
    const float4 v = (i + 3 >= l0 && i < l1) ? __ldcg(reinterpret_cast<const float4 *>(src + i))
                                             : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    z[4 * u] = v.x;
    z[4 * u + 1] = v.y;
    z[4 * u + 2] = v.z;
    z[4 * u + 3] = v.w;
  }
}
__device__ __forceinline__ int chunk_off(int j) {
  return 4 * ((j / 4) * kTkThreads + static_cast<int>(threadIdx.x)) + (j & 3);
}

// Last-CTA hand-off per head: after this CTA's global writes, count it in; true for the CTA
// that completes the head (it then sees every other CTA's writes).
__device__ __forceinline__ bool last_of_row(uint32_t *counter, uint32_t total, bool *s_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(counter, 1u);
    *s_flag = prev == total - 1;
    if (*s_flag) {
      __threadfence();
      *counter = 0u;   // left zero for the next kernel that counts with it
    }
  }
  __syncthreads();
  return *s_flag;
}

// ---- one pass per (head, chunk): keys above the digit-1 threshold bin b1 are emitted, keys
//      in b1 are listed with their order keys; the head's last CTA selects the rest from
//      that list and leaves the histogram and counters zero
__global__ void __launch_bounds__(kTkThreads, 4) topk_collect_kernel(const TopkParams p) {
  __shared__ uint32_t warp_tot[kTkThreads / 32];
  __shared__ Thresh s_t;
  __shared__ uint32_t h2[kHistBins];      // digit-2 histogram of this CTA's listed keys
  __shared__ uint32_t s_ns, s_nc, s_bs, s_bc;
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.y;
  const int tid = threadIdx.x;
  int32_t *irow = p.idx + static_cast<long long>(row) * p.k;
  if (blockIdx.x == 0)
    for (long long i = p.k_eff + tid; i < p.k; i += kTkThreads) irow[i] = -1;
  if (p.k_eff == 0) return;
  const long long c0 = static_cast<long long>(blockIdx.x) * kTopkChunk;
  const int l0 = static_cast<int>(max(c0, p.cand_lo) - c0);
  const int l1 = static_cast<int>(min(c0 + kTopkChunk, p.cand_hi) - c0);
  if (l0 >= l1) return;
  const bool take_all = p.k_eff >= p.nC;
  // the chunk's loads go out first and are in flight while the threshold is found
  float z[kPerThread];
  load_chunk(p.S + static_cast<long long>(row) * p.ldS + c0, l0, l1, z);
  uint32_t *meta = p.meta + row * kMetaWords;
  uint32_t *h1g = p.hist + static_cast<long long>(row) * kHistBins;
  int b1 = -1;
  uint32_t above1 = 0;
  float zlo = -INFINITY, zhi = -INFINITY;   // emit z >= zhi; list zlo <= z < zhi
  if (!take_all) {
    const Thresh t1 = find_threshold<kTkThreads>(h1g, static_cast<uint32_t>(p.k_eff), warp_tot, &s_t);
    b1 = t1.bin;
    above1 = t1.above;
    zlo = key_float(static_cast<uint32_t>(b1) << (32 - kHistBits));
    zhi = b1 + 1 < kHistBins ? key_float(static_cast<uint32_t>(b1 + 1) << (32 - kHistBits)) : INFINITY;
  }
  for (int i = tid; i < kHistBins; i += kTkThreads) h2[i] = 0;
  const bool edge = l0 > 0 || l1 < kTopkChunk;
  uint2 *crow = p.cand + static_cast<long long>(row) * p.ldC;
  // count this thread's selected (z >= zhi) and listed (zlo <= z < zhi) keys ...
  uint32_t ns = 0, nc = 0;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    bool in = true;
    if (edge) in = chunk_off(j) >= l0 && chunk_off(j) < l1;
    ns += (in && z[j] >= zhi) ? 1u : 0u;
    nc += (in && z[j] >= zlo && z[j] < zhi) ? 1u : 0u;
  }
  // ... place them with one block scan and one global reservation per list ...
  const uint32_t packed = ns | (nc << 16);   // at most kPerThread each
  const uint32_t incl = block_incl_scan<kTkThreads>(packed, warp_tot);
  if (tid == kTkThreads - 1) {
    s_ns = incl & 0xFFFFu;
    s_nc = incl >> 16;
    s_bs = s_ns ? atomicAdd(meta + kSelCount, s_ns) : 0u;
    s_bc = s_nc ? atomicAdd(meta + kCandCount, s_nc) : 0u;
  }
  __syncthreads();
  uint32_t os = s_bs + ((incl - packed) & 0xFFFFu);
  uint32_t oc = s_bc + ((incl - packed) >> 16);
  // ... and write them
  bool any_cand = false;
  if (ns | nc) {
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      bool in = true;
      if (edge) in = chunk_off(j) >= l0 && chunk_off(j) < l1;
      const uint32_t pos = static_cast<uint32_t>(c0 + chunk_off(j));
      if (in && z[j] >= zhi) {
        if (os < p.k_eff) irow[os] = static_cast<int32_t>(pos);
        ++os;
      } else if (in && z[j] >= zlo) {
        const uint32_t key = order_key(z[j]);
        if (oc < p.ldC) crow[oc] = make_uint2(pos, key);
        ++oc;
        atomicAdd(&h2[(key >> kDigit2Shift) & (kHistBins - 1)], 1u);
        any_cand = true;
      }
    }
  }
  uint32_t *h2g = p.hist2 + static_cast<long long>(row) * kHistBins;
  if (__syncthreads_or(any_cand))
    for (int i = tid; i < kHistBins; i += kTkThreads)
      if (h2[i]) atomicAdd(h2g + i, h2[i]);

  if (!take_all && blockIdx.x == p.cand_lo / kTopkChunk && tid == 0) {
    meta[kThresh1] = static_cast<uint32_t>(b1);
    meta[kAbove1] = above1;   // the keys above b1, all written out by this kernel
  }
}

// ---- refine, (head, part) CTAs over the head's list of bin-b1 keys: the digit-2 threshold
//      bin b2, the listed keys above (b1, b2) written out, those in (b1, b2) moved to the
//      head's bucket; the head's last CTA selects the rest from the bucket and leaves the
//      histograms and counters zero
__global__ void __launch_bounds__(kTkThreads) topk_refine_kernel(const TopkParams p) {
  __shared__ __align__(16) uint64_t bucket[kBucketCap];
  __shared__ uint32_t warp_tot[kTkThreads / 32];
  __shared__ Thresh s_t;
  __shared__ uint32_t h256[256];
  __shared__ uint64_t bs[kBitonic];
  __shared__ uint32_t s_bs, s_out, s_cnt, s_cum, s_nb;
  __shared__ int s_digit;
  __shared__ bool s_last;
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (p.k_eff == 0) return;
  const bool take_all = p.k_eff >= p.nC;
  uint32_t *meta = p.meta + row * kMetaWords;
  uint32_t *h1g = p.hist + static_cast<long long>(row) * kHistBins;
  uint32_t *h2g = p.hist2 + static_cast<long long>(row) * kHistBins;
  int32_t *irow = p.idx + static_cast<long long>(row) * p.k;
  const uint2 *crow = p.cand + static_cast<long long>(row) * p.ldC;        // bin-b1 list
  uint2 *brow = p.bucket + static_cast<long long>(row) * kBucketCap;       // (b1, b2) bucket
  const uint32_t above1 = __ldcg(meta + kAbove1);    // keys above b1, written by collect
  const uint32_t n_list = min(__ldcg(meta + kCandCount), static_cast<uint32_t>(p.ldC));
  const uint32_t b1 = __ldcg(meta + kThresh1);
  const uint32_t wbase = static_cast<uint32_t>(tid - lane);
  uint32_t rr = static_cast<uint32_t>(p.k_eff) - min(above1, static_cast<uint32_t>(p.k_eff));
  const bool active = !take_all && rr > 0 && n_list > 0;
  uint32_t b2 = 0, above2 = 0;
  if (active) {
    const Thresh t2 = find_threshold<kTkThreads>(h2g, rr, warp_tot, &s_t);
    b2 = static_cast<uint32_t>(t2.bin);
    above2 = t2.above;
    // this CTA's part of the list: keys above (b1, b2) counted, placed and written; keys in
    // (b1, b2) appended to the bucket
    const uint32_t per = (n_list + gridDim.x - 1) / gridDim.x;
    const uint32_t i_lo = blockIdx.x * per, i_hi = min(n_list, i_lo + per);
    constexpr int kBatch = 8;
    for (uint32_t i0 = i_lo; i0 < i_hi; i0 += kBatch * kTkThreads) {
      uint2 cb[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const uint32_t i = i0 + u * kTkThreads + tid;
        cb[u] = i < i_hi ? __ldcg(&crow[i]) : make_uint2(0u, 0u);
      }
      uint32_t n_up = 0;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const uint32_t i = i0 + u * kTkThreads + tid;
        const uint32_t d2 = (cb[u].y >> kDigit2Shift) & (kHistBins - 1);
        n_up += (i < i_hi && d2 > b2) ? 1u : 0u;
        if (i < i_hi && d2 == b2) {   // a handful per head
          const uint32_t o = atomicAdd(meta + kBuckCount, 1u);
          if (o < static_cast<uint32_t>(kBucketCap)) brow[o] = cb[u];
        }
      }
      const uint32_t incl = block_incl_scan<kTkThreads>(n_up, warp_tot);
      if (tid == kTkThreads - 1) s_bs = incl ? atomicAdd(meta + kSelCount, incl) : 0u;
      __syncthreads();
      uint32_t o = s_bs + incl - n_up;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const uint32_t i = i0 + u * kTkThreads + tid;
        const uint32_t d2 = (cb[u].y >> kDigit2Shift) & (kHistBins - 1);
        if (i < i_hi && d2 > b2) {
          if (o < p.k_eff) irow[o] = static_cast<int32_t>(cb[u].x);
          ++o;
        }
      }
      __syncthreads();
    }
  }

  if (!last_of_row(meta + kDone, gridDim.x, &s_last)) return;
  // ---- the head's last CTA
  const uint32_t n_bk = __ldcg(meta + kBuckCount);
  __syncthreads();
  if (tid < kError) meta[tid] = 0u;
  if (!take_all)
    for (int i = tid; i < kHistBins; i += kTkThreads) {
      h1g[i] = 0u;
      h2g[i] = 0u;
    }
  if (!active) return;
  uint32_t rr2 = rr - above2;                    // 1 <= rr2 <= size of the bucket
  // a bucket of at most kBucketCap keys is complete in brow and goes to shared memory; a larger
  // one (only with massive ties) is read from the whole list, filtered by its digits
  const bool in_smem = n_bk <= static_cast<uint32_t>(kBucketCap);
  const uint32_t n_buck = in_smem ? n_bk : n_list;
  if (in_smem)
    for (uint32_t i = tid; i < n_buck; i += kTkThreads) {
      const uint2 c = __ldcg(&brow[i]);
      bucket[i] = make_composite(c.y, c.x);
    }
  if (tid == 0) s_out = above1 + above2;
  __syncthreads();
  auto get = [&](uint32_t i) -> uint64_t {
    if (in_smem) return bucket[i];
    const uint2 c = __ldcg(&crow[i]);
    return make_composite(c.y, c.x);
  };
  auto emit = [&](bool pred, uint32_t pos) {
    bool ok;
    const uint32_t o = warp_append(pred, &s_out, ok);
    if (ok && o < p.k_eff) irow[o] = static_cast<int32_t>(pos);
  };
  uint64_t prefix = (static_cast<uint64_t>(b1) << kHistBits) | b2;
  int shift = 64 - 2 * kHistBits;
  uint32_t cnt = n_bk;
  // every round fixes 8 more bits of a unique 64-bit key: at most ceil(42 / 8) + 1 rounds
#pragma unroll 1
  for (int round = 0; round < 8; ++round) {
    if (cnt == rr2) {   // the whole bucket is taken
      for (uint32_t i0 = wbase; i0 < n_buck; i0 += kTkThreads) {
        const uint32_t i = i0 + lane;
        const uint64_t x = i < n_buck ? get(i) : 0ull;
        emit(i < n_buck && (x >> shift) == prefix, comp_pos(x));
      }
      return;
    }
    if (cnt <= kBitonic) {   // bitonic finish of the threshold bucket
      if (tid < kBitonic) bs[tid] = 0;
      if (tid == 0) s_nb = 0;
      __syncthreads();
      for (uint32_t i = tid; i < n_buck; i += kTkThreads) {
        const uint64_t x = get(i);
        if ((x >> shift) == prefix) {
          const uint32_t o = atomicAdd(&s_nb, 1u);
          if (o < kBitonic) bs[o] = x;
        }
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
        const uint32_t o0 = s_out;
        for (uint32_t i = lane; i < rr2 && o0 + i < p.k_eff; i += 32)
          irow[o0 + i] = static_cast<int32_t>(comp_pos(bs[i]));
      }
      return;
    }
    // one more 8-bit digit
    const int nshift = shift > 8 ? shift - 8 : 0;
    const int nb = shift - nshift;
    const uint64_t dmask = (1ull << nb) - 1;
    h256[tid] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < n_buck; i += kTkThreads) {
      const uint64_t x = get(i);
      if ((x >> shift) == prefix) atomicAdd(&h256[(x >> nshift) & dmask], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits [256 - 8(l+1), 256 - 8l), highest first
      uint32_t lc[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        lc[i] = h256[255 - 8 * lane - i];
        sum += lc[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t nn = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nn;
      }
      const uint32_t excl = incl - sum;
      if (excl < rr2 && rr2 <= incl) {
        uint32_t cum = excl;
        for (int i = 0; i < 8; ++i) {
          if (cum + lc[i] >= rr2) {
            s_digit = 255 - 8 * lane - i;
            s_cum = cum;
            s_cnt = lc[i];
            break;
          }
          cum += lc[i];
        }
      }
    }
    __syncthreads();
    const uint64_t v = static_cast<uint64_t>(s_digit);
    const uint32_t cum = s_cum;
    for (uint32_t i0 = wbase; i0 < n_buck; i0 += kTkThreads) {
      const uint32_t i = i0 + lane;
      const uint64_t x = i < n_buck ? get(i) : 0ull;
      emit(i < n_buck && (x >> shift) == prefix && ((x >> nshift) & dmask) > v, comp_pos(x));
    }
    rr2 -= cum;
    cnt = s_cnt;
    prefix = (prefix << nb) | v;
    shift = nshift;
    __syncthreads();
  }
  if (tid == 0) atomicOr(p.meta + kError, 4u);   // unreachable for unique keys
}

cudaError_t launch_topk(const TopkParams &p, cudaStream_t s) {
  if (p.k <= 0) return cudaSuccess;
  const long long chunks = (p.N + kTopkChunk - 1) / kTopkChunk;
  cudaError_t e = launch_pdl(topk_collect_kernel,
                             dim3(static_cast<unsigned>(chunks), static_cast<unsigned>(p.R)),
                             dim3(kTkThreads), 0, s, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_refine_kernel, dim3(kRefineParts, static_cast<unsigned>(p.R)),
                    dim3(kTkThreads), 0, s, p);
}

}  // namespace ra
