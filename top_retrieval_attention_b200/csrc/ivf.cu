// Device-side approximate retrieval with an inverted-file (IVF) index of the keys, the pages'
// IVF baseline (slides "RetrievalAttention splits the work across CPU and GPU" / "Available GPU
// memory changes the comparison": IVF over the keys, probed with the decode query), built and
// searched on the GPU.
//
// Build, per KV head: spherical k-means (Lloyd iterations) of the N keys into nlist unit-norm
// bf16 centroids, deterministic from start to end.  The key-centroid scores are the tcgen05
// prefill score kernel with the keys as its query rows and the centroids as its keys, over
// chunks of keys (the score workspace is bounded whatever N is); one warp per key takes the
// argmax (ties to the lower centroid).  A stable counting sort then lists the keys cluster by
// cluster in increasing position (per-chunk counts, a scan into slots, one warp per chunk
// placing its keys in order), and one warp per cluster sums its keys in that order into the
// next centroid (the unit direction of the sum; an empty cluster keeps its centroid).  The
// final sort also copies the keys into the sorted copy.
// Search, per query head: the scores of the nlist centroids and the nprobe best, the exact
// scores of every key of the probed clusters (read contiguously from the sorted copy; static-set
// positions excluded) and of the static set; the cluster kernel then selects the exact top-k of
// the probed candidates (reporting their cache positions) and attends over W and Omega.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace ra {

// ---- build

// Centroid c of head bg starts as the unit-normalised key at position floor(c * N / nlist).
__global__ void __launch_bounds__(128) ivf_init_kernel(const IvfParams p) {
  const long long bg = blockIdx.y;
  const int c = blockIdx.x;
  const long long pos = static_cast<long long>(c) * p.N / p.nlist;
  const __nv_bfloat16 *k = p.K + (bg * p.cap + pos) * p.d;
  float v = 0.f, ss = 0.f;
  if (threadIdx.x < p.d) {
    v = __bfloat162float(k[threadIdx.x]);
    ss = v * v;
  }
  __shared__ float red[4];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  const float norm = sqrtf(red[0] + red[1] + red[2] + red[3]);
  if (threadIdx.x < p.d)
    p.cent[(bg * p.nlist + c) * p.d + threadIdx.x] =
        __float2bfloat16_rn(norm > 0.f ? v / norm : 0.f);
}

// One warp per key of the chunk [c0, c0 + M): the argmax of its centroid scores (row of A, ties
// to the lower centroid) into assign.
__global__ void __launch_bounds__(256) ivf_assign_kernel(const IvfParams p) {
  const long long w = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(p.BH) * p.M;
  if (w >= rows) return;   // whole warps leave together
  const float *a = p.A + w * p.ldA;
  float best = -INFINITY;
  int bi = 0x7FFFFFFF;
  for (int c = lane; c < p.nlist; c += 32) {
    const float v = a[c];
    if (v > best || (v == best && c < bi)) {
      best = v;
      bi = c;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) {
      best = ov;
      bi = oi;
    }
  }
  if (lane == 0) {
    const long long bg = w / p.M;
    p.assign[bg * p.N + p.c0 + (w - bg * p.M)] = bi < p.nlist ? bi : 0;   // (a row of NaNs: 0)
  }
}

// The keys of each cluster in each sort chunk of kIvfSortChunk positions (one CTA per chunk).
__global__ void __launch_bounds__(256) ivf_chunk_count_kernel(const IvfParams p) {
  extern __shared__ uint32_t hc[];   // nlist counters
  const long long bg = blockIdx.y;
  const int ch = blockIdx.x;
  for (int c = threadIdx.x; c < p.nlist; c += 256) hc[c] = 0u;
  __syncthreads();
  const long long lo = static_cast<long long>(ch) * kIvfSortChunk;
  const long long hi = min(p.N, lo + kIvfSortChunk);
  for (long long i = lo + threadIdx.x; i < hi; i += 256) atomicAdd(&hc[p.assign[bg * p.N + i]], 1u);
  __syncthreads();
  uint32_t *out = p.chunk_cnt + (bg * p.nsort + ch) * p.nlist;
  for (int c = threadIdx.x; c < p.nlist; c += 256) out[c] = hc[c];
}

// One CTA per head: offsets (an exclusive scan of the cluster totals over the clusters) and,
// per sort chunk and cluster, the first slot of that chunk's keys of the cluster (the cluster's
// offset plus the counts of the earlier chunks), in place of the counts.
__global__ void __launch_bounds__(1024) ivf_slots_kernel(const IvfParams p) {
  const long long bg = blockIdx.x;
  uint32_t *cc = p.chunk_cnt + bg * p.nsort * p.nlist;
  int32_t *offs = p.offsets + bg * (p.nlist + 1);
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t carry;
  // earlier chunks' counts per cluster; the totals go to offs for the scan
  for (int c = threadIdx.x; c < p.nlist; c += 1024) {
    uint32_t run = 0;
    for (int ch = 0; ch < p.nsort; ++ch) {
      const uint32_t v = cc[static_cast<long long>(ch) * p.nlist + c];
      cc[static_cast<long long>(ch) * p.nlist + c] = run;
      run += v;
    }
    offs[c] = static_cast<int32_t>(run);
  }
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int c0 = 0; c0 < p.nlist; c0 += 1024) {
    const int c = c0 + threadIdx.x;
    const uint32_t v = c < p.nlist ? static_cast<uint32_t>(offs[c]) : 0u;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      uint32_t t = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[lane] = t;
    }
    __syncthreads();
    const uint32_t incl = carry + x + (warp > 0 ? warp_tot[warp - 1] : 0u);
    if (c < p.nlist) offs[c] = static_cast<int32_t>(incl - v);
    __syncthreads();
    if (threadIdx.x == 1023) carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) offs[p.nlist] = static_cast<int32_t>(carry);
  __syncthreads();
  for (int c = threadIdx.x; c < p.nlist; c += 1024) {
    const uint32_t base = static_cast<uint32_t>(offs[c]);
    for (int ch = 0; ch < p.nsort; ++ch) cc[static_cast<long long>(ch) * p.nlist + c] += base;
  }
}

// Stable scatter: one warp per sort chunk places the chunk's keys, 32 positions at a time in
// increasing order, at their clusters' next slots: lanes that share a cluster take consecutive
// slots in lane order and the group's first lane advances the chunk's slot counter (only this
// warp touches it).  With copy_rows the warp also copies the 32 keys into the sorted copy.
template <int D>
__global__ void __launch_bounds__(256) ivf_stable_scatter_kernel(const IvfParams p, int copy_rows) {
  const long long w = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(p.BH) * p.nsort) return;
  const long long bg = w / p.nsort;
  const int ch = static_cast<int>(w - bg * p.nsort);
  uint32_t *slots = p.chunk_cnt + (bg * p.nsort + ch) * p.nlist;
  const long long lo = static_cast<long long>(ch) * kIvfSortChunk;
  const long long hi = min(p.N, lo + kIvfSortChunk);
  for (long long base = lo; base < hi; base += 32) {
    const long long i = base + lane;
    const bool valid = i < hi;
    const int c = valid ? p.assign[bg * p.N + i] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, c);
    const int leader = __ffs(peers) - 1;
    const uint32_t rank = __popc(peers & lanemask_lt());
    uint32_t first = 0;
    if (valid && lane == leader) first = atomicAdd(slots + c, static_cast<uint32_t>(__popc(peers)));
    first = __shfl_sync(0xffffffffu, first, leader);
    const long long dst = bg * p.N + first + rank;
    if (valid) p.pos[dst] = static_cast<int32_t>(i);
    if (copy_rows) {
      constexpr int W = D / 64;   // 32-bit words of a row per lane
      for (int j = 0; j < 32 && base + j < hi; ++j) {
        const long long dj = __shfl_sync(0xffffffffu, dst, j);
        const uint32_t *src = reinterpret_cast<const uint32_t *>(p.K + (bg * p.cap + base + j) * D);
        uint32_t *out = reinterpret_cast<uint32_t *>(p.Ksorted + dj * D);
#pragma unroll
        for (int u = 0; u < W; ++u) out[lane + 32 * u] = src[lane + 32 * u];
      }
    }
  }
}

// Centroid c of head bg (one warp): the unit direction of the sum of its keys, added in
// increasing position (lane l keeps channels [l * D / 32, (l + 1) * D / 32)); an empty cluster,
// or a zero sum, keeps the centroid.
template <int D>
__global__ void __launch_bounds__(256) ivf_update_kernel(const IvfParams p) {
  constexpr int CPL = D / 32;
  const long long w = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(p.BH) * p.nlist) return;
  const long long bg = w / p.nlist;
  const int c = static_cast<int>(w - bg * p.nlist);
  const int32_t lo = p.offsets[bg * (p.nlist + 1) + c], hi = p.offsets[bg * (p.nlist + 1) + c + 1];
  float acc[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) acc[k] = 0.f;
  const __nv_bfloat16 *Kb = p.K + bg * p.cap * D + lane * CPL;
  const int32_t *pos = p.pos + bg * p.N;
  int32_t j = lo;
  for (; j + 4 <= hi; j += 4) {   // four rows' loads in flight, added in order
    float x[4][CPL];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const __nv_bfloat16 *row = Kb + static_cast<long long>(__ldg(pos + j + r)) * D;
#pragma unroll
      for (int k = 0; k < CPL; ++k) x[r][k] = __bfloat162float(row[k]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int k = 0; k < CPL; ++k) acc[k] += x[r][k];
  }
  for (; j < hi; ++j) {
    const __nv_bfloat16 *row = Kb + static_cast<long long>(__ldg(pos + j)) * D;
#pragma unroll
    for (int k = 0; k < CPL; ++k) acc[k] += __bfloat162float(row[k]);
  }
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < CPL; ++k) ss += acc[k] * acc[k];
  ss = warp_sum(ss);
  const float norm = sqrtf(ss);
  if (hi > lo && norm > 0.f) {
    __nv_bfloat16 *out = p.cent + (bg * p.nlist + c) * D + lane * CPL;
#pragma unroll
    for (int k = 0; k < CPL; ++k) out[k] = __float2bfloat16_rn(acc[k] / norm);
  }
}

// ---- search

constexpr int kIvfMaxList = 4096;    // clusters per head at most
constexpr int kProbeThreads = 512;
constexpr int kProbeCollect = 512;   // keys at or above the threshold bin ranked directly

// Exclusive prefix (from thread 0 up) of one value per thread of a kProbeThreads block, and the
// block total.  wsum holds kProbeThreads / 32 words.
__device__ __forceinline__ uint32_t probe_scan(uint32_t v, uint32_t *wsum, uint32_t &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  uint32_t before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kProbeThreads / 32; ++w) {
    const uint32_t t = wsum[w];
    before += w < warp ? t : 0u;
    total += t;
  }
  __syncthreads();
  return before + x - v;
}

// One CTA per query head row: the scores of its KV head's nlist centroids, the nprobe best
// (largest score first, ties to the lower cluster), their clusters' offsets in the row's
// candidate list.  The selection: an 11-bit histogram of the score keys gives the bin of the
// nprobe-th largest; the keys at or above it are gathered and each is ranked by counting the
// gathered keys above it.  Should that bin hold more keys than the gather takes, every key is
// sorted instead (bitonic, in shared memory).
template <int D>
__global__ void __launch_bounds__(kProbeThreads) ivf_probe_kernel(const IvfSearchParams p) {
  __shared__ unsigned long long keys[kIvfMaxList];
  __shared__ unsigned long long coll[kProbeCollect];
  __shared__ uint32_t hist[kHistBins];
  __shared__ float qs[128];
  __shared__ int32_t sel[64];
  __shared__ uint32_t wsum[kProbeThreads / 32];
  __shared__ int t_bin;
  __shared__ uint32_t n_coll;
  const int row = blockIdx.x, tid = threadIdx.x;
  const int b = row / p.Hq, h = row - b * p.Hq;
  const long long bg = static_cast<long long>(b) * p.Hkv + h / p.G;
  pdl_trigger();
  pdl_wait();   // the query and the cache may come from earlier kernels of the stream
  if (tid < D) qs[tid] = __bfloat162float(p.q[static_cast<long long>(row) * D + tid]);
  for (int i = tid; i < kHistBins; i += kProbeThreads) hist[i] = 0u;
  if (tid < 64) sel[tid] = 0;   // a valid cluster in every slot whatever happens below
  if (tid == 0) {
    t_bin = -1;
    n_coll = 0u;
  }
  __syncthreads();
  // a thread per centroid, its row read in 16-byte pieces (all in flight together)
  for (int c = tid; c < p.nlist; c += kProbeThreads) {
    const uint4 *cr = reinterpret_cast<const uint4 *>(p.cent + (bg * p.nlist + c) * D);
    uint4 row_v[D / 8];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) row_v[j] = __ldg(cr + j);
    float z = 0.f;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const uint4 v = row_v[j];
      const float *qq = qs + 8 * j;
      z += qq[0] * bf16_lo(v.x) + qq[1] * bf16_hi(v.x) + qq[2] * bf16_lo(v.y) +
           qq[3] * bf16_hi(v.y) + qq[4] * bf16_lo(v.z) + qq[5] * bf16_hi(v.z) +
           qq[6] * bf16_lo(v.w) + qq[7] * bf16_hi(v.w);
    }
    const uint32_t okey = order_key(canon_zero(z));
    keys[c] = (static_cast<unsigned long long>(okey) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(c));
    atomicAdd(&hist[okey >> (32 - kHistBits)], 1u);
  }
  __syncthreads();
  // the bin of the nprobe-th largest key: thread t owns bins [2048 - 4 (t + 1), 2048 - 4 t)
  {
    constexpr int per = kHistBins / kProbeThreads;
    uint32_t loc[per], s = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      loc[i] = hist[kHistBins - per * (tid + 1) + (per - 1 - i)];
      s += loc[i];
    }
    uint32_t total;
    const uint32_t before = probe_scan(s, wsum, total);
    const uint32_t want = static_cast<uint32_t>(p.nprobe);
    if (before < want && want <= before + s) {
      uint32_t cum = before;
#pragma unroll
      for (int i = 0; i < per; ++i) {
        if (cum + loc[i] >= want) {
          t_bin = kHistBins - per * (tid + 1) + (per - 1 - i);
          break;
        }
        cum += loc[i];
      }
    }
  }
  __syncthreads();
  const uint32_t tb = static_cast<uint32_t>(t_bin);   // found: nprobe <= nlist keys exist
  for (int c = tid; c < p.nlist; c += kProbeThreads) {
    const unsigned long long x = keys[c];
    if (static_cast<uint32_t>(x >> (64 - kHistBits)) >= tb) {
      const uint32_t slot = atomicAdd(&n_coll, 1u);
      if (slot < static_cast<uint32_t>(kProbeCollect)) coll[slot] = x;
    }
  }
  __syncthreads();
  const uint32_t m = n_coll;
  if (m <= static_cast<uint32_t>(kProbeCollect)) {
    for (uint32_t i = tid; i < m; i += kProbeThreads) {
      const unsigned long long x = coll[i];
      uint32_t r = 0;
      for (uint32_t j = 0; j < m; ++j) r += coll[j] > x ? 1u : 0u;
      if (r < static_cast<uint32_t>(p.nprobe))
        sel[r] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(x));
    }
  } else {   // a crowded bin: sort all keys, descending
    int np2 = 1;
    while (np2 < p.nlist) np2 <<= 1;
    for (int c = p.nlist + tid; c < np2; c += kProbeThreads) keys[c] = 0ull;   // below every key
    __syncthreads();
    for (int size = 2; size <= np2; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < np2 / 2; i += kProbeThreads) {
          const int lo = 2 * stride * (i / stride) + (i % stride);
          const int hi = lo + stride;
          const unsigned long long a = keys[lo], bb = keys[hi];
          const bool desc = (lo & size) == 0;
          if (desc ? (a < bb) : (a > bb)) {
            keys[lo] = bb;
            keys[hi] = a;
          }
        }
        __syncthreads();
      }
    }
    if (tid < p.nprobe) sel[tid] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(keys[tid]));
  }
  __syncthreads();
  // the probed clusters' sizes -> offsets in the candidate list (lane l: slots 2l and 2l + 1)
  if (tid < 32) {
    const int32_t *offs = p.offsets + bg * (p.nlist + 1);
    const int j0 = 2 * tid, j1 = j0 + 1;
    const int32_t s0 = j0 < p.nprobe ? offs[sel[j0] + 1] - offs[sel[j0]] : 0;
    const int32_t s1 = j1 < p.nprobe ? offs[sel[j1] + 1] - offs[sel[j1]] : 0;
    int32_t x = s0 + s1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (tid >= o) x += y;
    }
    const int32_t excl = x - s0 - s1;
    const int32_t total = __shfl_sync(0xffffffffu, x, 31);
    int32_t *probe = p.probe + static_cast<long long>(row) * p.nprobe;
    int32_t *off = p.cand_off + static_cast<long long>(row) * (p.nprobe + 1);
    if (j0 < p.nprobe) {
      probe[j0] = sel[j0];
      off[j0] = excl;
    }
    if (j1 < p.nprobe) {
      probe[j1] = sel[j1];
      off[j1] = excl + s0;
    }
    if (tid == 0) {
      off[p.nprobe] = total;
      p.n_cand[row] = total;
    }
  }
}

// Exact scores of the probed candidates (into S_cand, the candidate -> cache position map into
// pos_cand, and into the row's full score row at their positions) and of the static set (full
// score row).  Static-set keys among the candidates get -inf in S_cand and -1 in pos_cand (W is
// attended anyway).  Four lanes per key, each with a quarter of the channels in 16-byte loads;
// a warp scores eight keys at a time.
template <int D>
__global__ void __launch_bounds__(256) ivf_cand_kernel(const IvfSearchParams p) {
  constexpr int CPG = D / 4;    // channels per lane
  constexpr int NV = CPG / 8;   // 16-byte loads per lane
  __shared__ long long sbase[64];
  __shared__ int32_t soff[65];
  const int row = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane & 3, gi = lane >> 2;
  const int b = row / p.Hq, h = row - b * p.Hq;
  const long long bg = static_cast<long long>(b) * p.Hkv + h / p.G;
  pdl_trigger();
  pdl_wait();   // the probe's lists (and, before it, the appended keys)
  if (tid <= p.nprobe) {
    soff[tid] = p.cand_off[static_cast<long long>(row) * (p.nprobe + 1) + tid];
    if (tid < p.nprobe) {
      const int c = p.probe[static_cast<long long>(row) * p.nprobe + tid];
      sbase[tid] = bg * p.N + p.offsets[bg * (p.nlist + 1) + c];
    }
  }
  float qv[CPG];
  {
    const uint4 *qr = reinterpret_cast<const uint4 *>(p.q + static_cast<long long>(row) * D + sub * CPG);
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const uint4 w = __ldg(qr + v);
      qv[8 * v + 0] = bf16_lo(w.x); qv[8 * v + 1] = bf16_hi(w.x);
      qv[8 * v + 2] = bf16_lo(w.y); qv[8 * v + 3] = bf16_hi(w.y);
      qv[8 * v + 4] = bf16_lo(w.z); qv[8 * v + 5] = bf16_hi(w.z);
      qv[8 * v + 6] = bf16_lo(w.w); qv[8 * v + 7] = bf16_hi(w.w);
    }
  }
  __syncthreads();
  const long long n_cand = soff[p.nprobe];
  const long long total = n_cand + p.nW;
  float *srow = p.S + static_cast<long long>(row) * p.ldS;
  const long long step = static_cast<long long>(gridDim.x) * 64;
  for (long long e0 = (static_cast<long long>(blockIdx.x) * 8 + warp) * 8; e0 < total; e0 += step) {
    const long long e = e0 + gi;
    const bool valid = e < total;
    const __nv_bfloat16 *krow = nullptr;
    long long si = -1, pos = 0;
    if (valid) {
      if (e < n_cand) {
        int lo = 0, hi = p.nprobe - 1;   // the last probe slot starting at or before e
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (soff[mid] <= e) lo = mid;
          else hi = mid - 1;
        }
        si = sbase[lo] + (e - soff[lo]);
        krow = p.Ksorted + si * D;
        if (sub == 0) pos = __ldg(p.pos + si);   // in flight with the key's loads
      } else {
        const long long wi = e - n_cand;
        pos = wi < p.s1 ? wi : p.w0 + (wi - p.s1);
        krow = p.K + (bg * p.cap + pos) * D;
      }
    }
    float z = 0.f;
    if (valid) {
      const uint4 *kr = reinterpret_cast<const uint4 *>(krow + sub * CPG);
      uint4 kv[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) kv[v] = __ldg(kr + v);
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        z += qv[8 * v + 0] * bf16_lo(kv[v].x) + qv[8 * v + 1] * bf16_hi(kv[v].x) +
             qv[8 * v + 2] * bf16_lo(kv[v].y) + qv[8 * v + 3] * bf16_hi(kv[v].y) +
             qv[8 * v + 4] * bf16_lo(kv[v].z) + qv[8 * v + 5] * bf16_hi(kv[v].z) +
             qv[8 * v + 6] * bf16_lo(kv[v].w) + qv[8 * v + 7] * bf16_hi(kv[v].w);
      }
    }
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    if (valid && sub == 0) {
      z = canon_zero(z * p.scale);
      srow[pos] = z;
      if (e < n_cand) {
        const bool in_w = pos < p.s1 || pos >= p.w0;
        p.S_cand[static_cast<long long>(row) * p.ldC + e] = in_w ? -INFINITY : z;
        p.pos_cand[static_cast<long long>(row) * p.ldC + e] = in_w ? -1 : static_cast<int32_t>(pos);
      }
    }
  }
}

// ---- host

cudaError_t launch_ivf_init(const IvfParams &p, cudaStream_t s) {
  ivf_init_kernel<<<dim3(p.nlist, p.BH), 128, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_ivf_assign(const IvfParams &p, cudaStream_t s) {
  const long long warps = static_cast<long long>(p.BH) * p.M;
  ivf_assign_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_ivf_sort(const IvfParams &p, bool copy_rows, cudaStream_t s) {
  ivf_chunk_count_kernel<<<dim3(static_cast<unsigned>(p.nsort), static_cast<unsigned>(p.BH)), 256,
                           static_cast<size_t>(p.nlist) * 4, s>>>(p);
  ivf_slots_kernel<<<p.BH, 1024, 0, s>>>(p);
  const long long warps = static_cast<long long>(p.BH) * p.nsort;
  const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
  if (p.d == 128) ivf_stable_scatter_kernel<128><<<grid, 256, 0, s>>>(p, copy_rows ? 1 : 0);
  else ivf_stable_scatter_kernel<64><<<grid, 256, 0, s>>>(p, copy_rows ? 1 : 0);
  return cudaGetLastError();
}
cudaError_t launch_ivf_update(const IvfParams &p, cudaStream_t s) {
  const long long warps = static_cast<long long>(p.BH) * p.nlist;
  const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
  if (p.d == 128) ivf_update_kernel<128><<<grid, 256, 0, s>>>(p);
  else ivf_update_kernel<64><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_ivf_probe(const IvfSearchParams &p, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(p.R));
  if (p.d == 128) return launch_pdl(ivf_probe_kernel<128>, grid, dim3(kProbeThreads), 0, s, p);
  return launch_pdl(ivf_probe_kernel<64>, grid, dim3(kProbeThreads), 0, s, p);
}
cudaError_t launch_ivf_cand(const IvfSearchParams &p, int d, cudaStream_t s) {
  // CTAs per row from the expected candidate count (twice the mean cluster share), one key per
  // lane group at that count; the grid-stride loop covers any count
  const long long expect = 2 * p.N * p.nprobe / std::max(p.nlist, 1) + p.nW;
  const long long x = std::max<long long>(4, std::min<long long>(256, (expect + 255) / 256));
  const dim3 grid(static_cast<unsigned>(x), static_cast<unsigned>(p.R));
  if (d == 128) return launch_pdl(ivf_cand_kernel<128>, grid, dim3(256), 0, s, p);
  return launch_pdl(ivf_cand_kernel<64>, grid, dim3(256), 0, s, p);
}

}  // namespace ra
