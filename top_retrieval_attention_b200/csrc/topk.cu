// Exact per-query-head top-k over the candidate positions C = [0, N) \ W (RetrievalAttention
// slides, "The GPU keeps 640 fixed positions": W and Omega are disjoint, one index per query
// head; "Sparse attention renormalizes selected tokens": a fixed top-k budget).
//
// Keys are compared as 64-bit composites (order_key(z) << 32 | ~position), so every key is
// distinct, larger z wins and equal z goes to the lower position.  The selection is a radix
// select over digits of the composite, done for each query head by one thread-block cluster
// of kSelCluster CTAs, each owning a contiguous slice of the positions:
//   1. digit 1 = the top 11 bits of order_key(z): its histogram comes from the score kernel;
//      every CTA finds the threshold bin b1 (the bin holding the k-th largest key);
//   2. every CTA reads its slice of z (keeping the keys in shared memory when they fit) and
//      histograms digit 2 (the next 11 bits) of its keys in bin b1; the CTAs add up the
//      cluster's histograms through distributed shared memory and find the bin b2;
//   3. keys above (b1, b2) are selected and written out in rounds, each round reserving its
//      output range with one atomic; keys in (b1, b2) go to a bucket in the shared memory of
//      the cluster's first CTA (or, if it overflows, to a global list);
//   4. the first CTA narrows the bucket with further 8-bit digits until it is taken whole or
//      holds at most 64 keys, which one warp sorts with a bitonic network.
#include <cooperative_groups.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace ra {

constexpr int kSelThreads = 512;
constexpr int kKeyCache = 16384;     // keys of a slice kept in shared memory (64 KB)
constexpr int kRound = 2048;         // positions per emission round
constexpr int kBucketCap = 4096;     // (b1, b2) bucket held in shared memory (32 KB)
constexpr int kBitonic = 64;
constexpr int kDigit2Shift = 10;     // digit 2 = bits [10, 21) of the order key

struct SelectSmem {
  uint32_t keys[kKeyCache];
  uint64_t bucket[kBucketCap];
  uint32_t h2[kHistBins];
  uint32_t list[kRound];
};

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

// Finds, in a histogram owned kPer bins per thread from the top (loc[0] = highest bin of this
// thread, thread 0 owns the highest bins), the bin holding the `want`-th largest element.
// Exactly one thread writes *bin_out, *above_out (elements in higher bins) and *cnt_out.
template <int kThreads, int kPer>
__device__ __forceinline__ void find_threshold(const uint32_t (&loc)[kPer], uint32_t want,
                                               uint32_t *warp_tot, int *bin_out,
                                               uint32_t *above_out, uint32_t *cnt_out) {
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) s += loc[i];
  const uint32_t incl = block_incl_scan<kThreads>(s, warp_tot);
  const uint32_t excl = incl - s;
  if (excl < want && want <= incl) {
    uint32_t cum = excl;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (cum + loc[i] >= want) {
        *bin_out = kHistBins - kPer * (static_cast<int>(threadIdx.x) + 1) + (kPer - 1 - i);
        *above_out = cum;
        *cnt_out = loc[i];
        break;
      }
      cum += loc[i];
    }
  }
}

__global__ void __cluster_dims__(kSelCluster, 1, 1) __launch_bounds__(kSelThreads)
    topk_select_kernel(const TopkParams p) {
  constexpr int kPer = kHistBins / kSelThreads;   // 4 histogram bins per thread
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SelectSmem &sm = *reinterpret_cast<SelectSmem *>(smem_raw);
  __shared__ uint32_t warp_tot[kSelThreads / 32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_cnt;
  __shared__ uint32_t s_nlist, s_base, s_bucket_n, s_out;
  __shared__ uint32_t h256[256];
  __shared__ uint64_t bs[kBitonic];

  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank();
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_trigger();
  pdl_wait();

  int32_t *irow = p.idx + static_cast<long long>(row) * p.k;
  uint32_t *meta = p.meta + row * kMetaWords;
  if (rank == 0)
    for (long long i = p.k_eff + tid; i < p.k; i += kSelThreads) irow[i] = -1;
  if (p.k_eff == 0) return;   // uniform over the cluster: no cluster barrier is reached

  // this CTA's slice of the candidates
  const long long part = ((p.N + kSelCluster - 1) / kSelCluster + 3) & ~3LL;
  long long lo = static_cast<long long>(rank) * part, hi = lo + part;
  if (lo < p.cand_lo) lo = p.cand_lo;
  if (hi > p.cand_hi) hi = p.cand_hi;
  const int n_my = hi > lo ? static_cast<int>(hi - lo) : 0;
  const bool cached = n_my <= kKeyCache;
  const float *srow = p.S + static_cast<long long>(row) * p.ldS + lo;
  const bool take_all = p.k_eff >= p.nC;

  // ---- 1. digit-1 threshold (every CTA, from the score kernel's histogram)
  int b1 = -1;
  uint32_t above1 = 0;
  if (!take_all) {
    const uint32_t *h = p.hist + static_cast<long long>(row) * kHistBins;
    uint32_t loc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) loc[i] = __ldcg(h + kHistBins - kPer * (tid + 1) + (kPer - 1 - i));
    find_threshold<kSelThreads, kPer>(loc, static_cast<uint32_t>(p.k_eff), warp_tot, &s_bin,
                                      &s_above, &s_cnt);
  }
  for (int i = tid; i < kHistBins; i += kSelThreads) sm.h2[i] = 0;
  if (tid == 0) {
    s_nlist = 0;
    s_bucket_n = 0;
  }
  __syncthreads();
  if (!take_all) {
    b1 = s_bin;
    above1 = s_above;
  }

  // ---- 2. keys of the slice (cached when they fit) and their digit-2 histogram in bin b1
  constexpr int kLd = 8;
  for (int i0 = 0; i0 < n_my; i0 += kLd * kSelThreads) {
    float zb[kLd];
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int i = i0 + u * kSelThreads + tid;
      zb[u] = i < n_my ? __ldcg(srow + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int i = i0 + u * kSelThreads + tid;
      if (i < n_my) {
        const uint32_t key = order_key(zb[u]);
        if (cached) sm.keys[i] = key;
        if (!take_all && static_cast<int>(key >> (32 - kHistBits)) == b1)
          atomicAdd(&sm.h2[(key >> kDigit2Shift) & (kHistBins - 1)], 1u);
      }
    }
  }
  cluster.sync();   // every slice's digit-2 histogram is complete; digit-1 histogram read

  // ---- digit-2 threshold over the cluster's summed histograms
  uint32_t b2 = 0, above2 = 0, cnt2 = 0, rr = 0;
  if (!take_all) {
    if (rank == 0)   // leave the digit-1 histogram zero for the next call
      for (int i = tid; i < kHistBins; i += kSelThreads)
        p.hist[static_cast<long long>(row) * kHistBins + i] = 0u;
    uint32_t loc2[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) loc2[i] = 0;
    for (int r = 0; r < kSelCluster; ++r) {
      const uint32_t *rh = cluster.map_shared_rank(sm.h2, r);
#pragma unroll
      for (int i = 0; i < kPer; ++i) loc2[i] += rh[kHistBins - kPer * (tid + 1) + (kPer - 1 - i)];
    }
    rr = static_cast<uint32_t>(p.k_eff) - above1;
    find_threshold<kSelThreads, kPer>(loc2, rr, warp_tot, &s_bin, &s_above, &s_cnt);
    __syncthreads();
    b2 = static_cast<uint32_t>(s_bin);
    above2 = s_above;
    cnt2 = s_cnt;
  }
  const bool bucket_in_smem = cnt2 <= static_cast<uint32_t>(kBucketCap);
  uint64_t *bucket0 = cluster.map_shared_rank(sm.bucket, 0);
  uint32_t *bucket0_n = cluster.map_shared_rank(&s_bucket_n, 0);

  // ---- 3. emit the keys above (b1, b2); route (b1, b2) keys to the bucket
  constexpr int kPerRound = kRound / kSelThreads;   // 4 positions per thread per round
  for (int r0 = 0; r0 < n_my; r0 += kRound) {
    uint32_t kb[kPerRound];
#pragma unroll
    for (int u = 0; u < kPerRound; ++u) {   // all loads of the round in flight together
      const int i = r0 + u * kSelThreads + tid;
      kb[u] = i < n_my ? (cached ? sm.keys[i] : order_key(__ldcg(srow + i))) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kPerRound; ++u) {
      const int i = r0 + u * kSelThreads + tid;   // warp-uniform trip count: lanes differ by 1
      const bool in = i < n_my;
      const uint32_t key = kb[u];
      const int bin = static_cast<int>(key >> (32 - kHistBits));
      const uint32_t d2 = (key >> kDigit2Shift) & (kHistBins - 1);
      const bool sel = in && (take_all || bin > b1 || (bin == b1 && d2 > b2));
      const bool buck = in && !take_all && bin == b1 && d2 == b2;
      bool ok;
      const uint32_t o = warp_append(sel, &s_nlist, ok);
      if (ok) sm.list[o] = static_cast<uint32_t>(lo + i);
      if (buck) {
        const uint32_t pos = static_cast<uint32_t>(lo + i);
        if (bucket_in_smem) {
          const uint32_t b = atomicAdd(bucket0_n, 1u);
          if (b < static_cast<uint32_t>(kBucketCap)) bucket0[b] = make_composite(key, pos);
        } else {
          const uint32_t b = atomicAdd(meta + kCandCount, 1u);
          if (b < p.ldC) p.cand[static_cast<long long>(row) * p.ldC + b] = make_uint2(pos, key);
        }
      }
    }
    __syncthreads();
    const uint32_t n = s_nlist;
    if (tid == 0 && n) s_base = atomicAdd(meta + kSelCount, n);
    __syncthreads();
    for (uint32_t i = tid; i < n; i += kSelThreads) {
      const uint32_t o = s_base + i;
      if (o < p.k_eff) irow[o] = static_cast<int32_t>(sm.list[i]);
    }
    __syncthreads();
    if (tid == 0) s_nlist = 0;
    __syncthreads();
  }
  cluster.sync();   // all emissions and bucket entries are in place
  if (rank != 0) return;
  if (tid == 0) meta[kSelCount] = 0u;
  if (take_all) return;

  // ---- 4. the first CTA selects the remaining rr2 keys from the (b1, b2) bucket
  uint32_t rr2 = rr - above2;                       // 1 <= rr2 <= cnt2
  const uint32_t out0 = static_cast<uint32_t>(p.k_eff) - rr2;
  const uint32_t n_list = bucket_in_smem ? cnt2 : min(cnt2, static_cast<uint32_t>(p.ldC));
  const uint2 *crow = p.cand + static_cast<long long>(row) * p.ldC;
  auto get = [&](uint32_t i) -> uint64_t {
    if (bucket_in_smem) return sm.bucket[i];
    const uint2 c = __ldcg(&crow[i]);
    return make_composite(c.y, c.x);
  };
  if (tid == 0) s_out = out0;
  __syncthreads();
  if (tid == 0) meta[kCandCount] = 0u;
  auto emit = [&](bool pred, uint32_t pos) {
    bool ok;
    const uint32_t o = warp_append(pred, &s_out, ok);
    if (ok && o < p.k_eff) irow[o] = static_cast<int32_t>(pos);
  };
  const uint32_t wbase = static_cast<uint32_t>(tid - lane);
  uint64_t prefix = (static_cast<uint64_t>(b1) << kHistBits) | b2;
  int shift = 64 - 2 * kHistBits;
  uint32_t cnt = cnt2;
  // every round fixes 8 more bits of a unique 64-bit key: at most ceil(42 / 8) + 1 rounds
#pragma unroll 1
  for (int round = 0; round < 8; ++round) {
    if (cnt == rr2) {   // the whole bucket is taken
      for (uint32_t i0 = wbase; i0 < n_list; i0 += kSelThreads) {
        const uint32_t i = i0 + lane;
        const uint64_t x = i < n_list ? get(i) : 0ull;
        emit(i < n_list && (x >> shift) == prefix, comp_pos(x));
      }
      return;
    }
    if (cnt <= kBitonic) {   // bitonic finish of the threshold bucket
      if (tid < kBitonic) bs[tid] = 0;
      if (tid == 0) s_bucket_n = 0;
      __syncthreads();
      for (uint32_t i = tid; i < n_list; i += kSelThreads) {
        const uint64_t x = get(i);
        if ((x >> shift) == prefix) {
          const uint32_t o = atomicAdd(&s_bucket_n, 1u);
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
    if (tid < 256) h256[tid] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < n_list; i += kSelThreads) {
      const uint64_t x = get(i);
      if ((x >> shift) == prefix) atomicAdd(&h256[(x >> nshift) & dmask], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits [256 - 8(l+1), 256 - 8l), highest first
      uint32_t lc[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        lc[i] = h256[255 - 8 * lane - i];
        s += lc[i];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      const uint32_t excl = incl - s;
      if (excl < rr2 && rr2 <= incl) {
        uint32_t cum = excl;
        for (int i = 0; i < 8; ++i) {
          if (cum + lc[i] >= rr2) {
            s_bin = 255 - 8 * lane - i;
            s_above = cum;
            s_cnt = lc[i];
            break;
          }
          cum += lc[i];
        }
      }
    }
    __syncthreads();
    const uint64_t v = static_cast<uint64_t>(s_bin);
    const uint32_t cum = s_above;
    for (uint32_t i0 = wbase; i0 < n_list; i0 += kSelThreads) {
      const uint32_t i = i0 + lane;
      const uint64_t x = i < n_list ? get(i) : 0ull;
      emit(i < n_list && (x >> shift) == prefix && ((x >> nshift) & dmask) > v, comp_pos(x));
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
  static bool done[64] = {};
  const size_t smem = sizeof(SelectSmem);
  const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(topk_select_kernel),
                                          static_cast<int>(smem), done);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_select_kernel, dim3(kSelCluster, static_cast<unsigned>(p.R)),
                    dim3(kSelThreads), smem, s, p);
}

}  // namespace ra
