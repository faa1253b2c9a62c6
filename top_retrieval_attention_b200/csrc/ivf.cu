// Device-side approximate retrieval with an inverted-file (IVF) index of the keys, the pages'
// IVF baseline (slides "RetrievalAttention splits the work across CPU and GPU" / "Available GPU
// memory changes the comparison": IVF over the keys, probed with the decode query), built and
// searched on the GPU.
//
// Build, per KV head: spherical k-means (Lloyd iterations) of the N keys into nlist unit-norm
// centroids.  The key-centroid scores of an iteration are the tcgen05 prefill score kernel with
// the keys as its query rows and the centroids as its keys; one warp per key takes the argmax
// (ties to the lower centroid) and adds the key into its centroid's fp32 sum; the sums are
// normalised into the next centroids.  A final assignment, a count per cluster, an exclusive
// scan and a scatter give the keys sorted by cluster (with their positions) and the cluster
// offsets.
// Search, per query head: the scores of the nlist centroids, the nprobe best (bitonic sort of
// (order key, id) in shared memory), the exact scores of every key of the probed clusters
// (read contiguously from the sorted copy; static-set positions excluded) and of the static
// set; the cluster kernel then selects the exact top-k of the probed candidates and attends.
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

// One warp per key: the argmax of its centroid scores (row of A, ties to the lower centroid),
// recorded in assign; with sums != nullptr the key is also added into its centroid's sum.
__global__ void __launch_bounds__(256) ivf_assign_kernel(const IvfParams p, int accumulate) {
  const long long w = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(p.BH) * p.N;
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
  const long long bg = w / p.N, pos = w - bg * p.N;
  if (lane == 0) {
    p.assign[w] = bi;
    atomicAdd(p.count + bg * p.nlist + bi, 1u);
  }
  if (accumulate) {
    const __nv_bfloat16 *k = p.K + (bg * p.cap + pos) * p.d;
    float *sum = p.sums + (bg * p.nlist + bi) * p.d;
    for (int c = lane; c < p.d; c += 32) atomicAdd(sum + c, __bfloat162float(k[c]));
  }
}

// Centroid c of head bg becomes its normalised sum (kept when the cluster is empty); the sums
// and counts are cleared for the next iteration.
__global__ void __launch_bounds__(128) ivf_update_kernel(const IvfParams p) {
  const long long bg = blockIdx.y;
  const int c = blockIdx.x;
  float *sum = p.sums + (bg * p.nlist + c) * p.d;
  float v = 0.f;
  if (threadIdx.x < p.d) v = sum[threadIdx.x];
  __shared__ float red[4];
  float ss = warp_sum(v * v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  const float norm = sqrtf(red[0] + red[1] + red[2] + red[3]);
  const uint32_t n = p.count[bg * p.nlist + c];
  if (threadIdx.x < p.d) {
    if (n > 0 && norm > 0.f)
      p.cent[(bg * p.nlist + c) * p.d + threadIdx.x] = __float2bfloat16_rn(v / norm);
    sum[threadIdx.x] = 0.f;
  }
  __syncthreads();
  if (threadIdx.x == 0) p.count[bg * p.nlist + c] = 0u;
}

// Exclusive scan of one head's cluster counts into offsets[0..nlist] (one CTA per head); the
// scatter cursors are cleared.
__global__ void __launch_bounds__(1024) ivf_offsets_kernel(const IvfParams p) {
  const long long bg = blockIdx.x;
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int c0 = 0; c0 < p.nlist; c0 += 1024) {
    const int c = c0 + threadIdx.x;
    const uint32_t v = c < p.nlist ? p.count[bg * p.nlist + c] : 0u;
    uint32_t x = v;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
    if (c < p.nlist) {
      p.offsets[bg * (p.nlist + 1) + c] = static_cast<int32_t>(incl - v);
      p.cursor[bg * p.nlist + c] = 0u;
    }
    __syncthreads();
    if (threadIdx.x == 1023) carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.offsets[bg * (p.nlist + 1) + p.nlist] = static_cast<int32_t>(carry);
}

// Every key to its cluster's next free slot of the sorted copy, with its position.
__global__ void __launch_bounds__(256) ivf_scatter_kernel(const IvfParams p) {
  const long long w = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(p.BH) * p.N;
  if (w >= rows) return;
  const long long bg = w / p.N, pos = w - bg * p.N;
  const int c = p.assign[w];
  uint32_t slot = 0;
  if (lane == 0) slot = atomicAdd(p.cursor + bg * p.nlist + c, 1u);
  slot = __shfl_sync(0xffffffffu, slot, 0);
  const long long dst = bg * p.N + p.offsets[bg * (p.nlist + 1) + c] + slot;
  if (lane == 0) p.pos[dst] = static_cast<int32_t>(pos);
  const uint32_t *src = reinterpret_cast<const uint32_t *>(p.K + (bg * p.cap + pos) * p.d);
  uint32_t *out = reinterpret_cast<uint32_t *>(p.Ksorted + dst * p.d);
  for (int c2 = lane; c2 < p.d / 2; c2 += 32) out[c2] = src[c2];
}

// ---- search

constexpr int kIvfMaxList = 4096;   // clusters per head at most (the probe sorts them in smem)

// One CTA per query head row: centroid scores, the nprobe best clusters, their candidate offsets.
__global__ void __launch_bounds__(256) ivf_probe_kernel(const IvfSearchParams p) {
  __shared__ unsigned long long keys[kIvfMaxList];
  __shared__ float qs[128];
  const int row = blockIdx.x, tid = threadIdx.x;
  const int b = row / p.Hq, h = row - b * p.Hq;
  const long long bg = static_cast<long long>(b) * p.Hkv + h / p.G;
  if (tid < p.d) qs[tid] = __bfloat162float(p.q[static_cast<long long>(row) * p.d + tid]);
  int np2 = 1;
  while (np2 < p.nlist) np2 <<= 1;
  __syncthreads();
  for (int c = tid; c < np2; c += 256) {
    unsigned long long key = 0ull;   // below every real key
    if (c < p.nlist) {
      const __nv_bfloat16 *cent = p.cent + (bg * p.nlist + c) * p.d;
      float z = 0.f;
      for (int j = 0; j < p.d; j += 2) {
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(cent + j);
        z += qs[j] * __low2float(v) + qs[j + 1] * __high2float(v);
      }
      key = (static_cast<unsigned long long>(order_key(canon_zero(z))) << 32) |
            (0xFFFFFFFFu - static_cast<uint32_t>(c));
    }
    keys[c] = key;
  }
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= np2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < np2 / 2; i += 256) {
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
  if (tid == 0) {
    int32_t *probe = p.probe + static_cast<long long>(row) * p.nprobe;
    int32_t *off = p.cand_off + static_cast<long long>(row) * (p.nprobe + 1);
    const int32_t *offs = p.offsets + bg * (p.nlist + 1);
    int32_t acc = 0;
    for (int j = 0; j < p.nprobe; ++j) {
      const int c = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(keys[j]));
      probe[j] = c;
      off[j] = acc;
      acc += offs[c + 1] - offs[c];
    }
    off[p.nprobe] = acc;
    p.n_cand[row] = acc;
  }
}

// Exact scores of the probed candidates (into S_cand, positions into pos_cand, and into the
// row's full score row at their positions) and of the static set (full score row).  Static-set
// positions among the candidates get -inf in S_cand (W is attended anyway).  One warp per key.
template <int D>
__global__ void __launch_bounds__(256) ivf_cand_kernel(const IvfSearchParams p) {
  constexpr int CPL = D / 32;
  const int row = blockIdx.y, lane = threadIdx.x & 31;
  const int b = row / p.Hq, h = row - b * p.Hq;
  const long long bg = static_cast<long long>(b) * p.Hkv + h / p.G;
  float qv[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c)
    qv[c] = __bfloat162float(p.q[static_cast<long long>(row) * D + lane * CPL + c]);
  const int32_t *off = p.cand_off + static_cast<long long>(row) * (p.nprobe + 1);
  const int32_t *probe = p.probe + static_cast<long long>(row) * p.nprobe;
  const int32_t *offs = p.offsets + bg * (p.nlist + 1);
  const long long n_cand = off[p.nprobe];
  const long long total = n_cand + p.nW;
  float *srow = p.S + static_cast<long long>(row) * p.ldS;
  const long long warps = static_cast<long long>(gridDim.x) * 8;
  for (long long e = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5); e < total; e += warps) {
    const __nv_bfloat16 *krow;
    long long pos;
    if (e < n_cand) {
      int j = 0;   // the probe slot holding candidate e
      while (j + 1 < p.nprobe && off[j + 1] <= e) ++j;
      const long long si = bg * p.N + offs[probe[j]] + (e - off[j]);
      pos = p.pos[si];
      krow = p.Ksorted + si * D;
    } else {
      const long long wi = e - n_cand;
      pos = wi < p.s1 ? wi : p.w0 + (wi - p.s1);
      krow = p.K + (bg * p.cap + pos) * D;
    }
    float z = 0.f;
    if constexpr (CPL == 4) {
      const uint2 v = *reinterpret_cast<const uint2 *>(krow + lane * 4);
      z = qv[0] * bf16_lo(v.x) + qv[1] * bf16_hi(v.x) + qv[2] * bf16_lo(v.y) + qv[3] * bf16_hi(v.y);
    } else {
      const uint32_t v = *reinterpret_cast<const uint32_t *>(krow + lane * 2);
      z = qv[0] * bf16_lo(v) + qv[1] * bf16_hi(v);
    }
    z = canon_zero(warp_sum(z) * p.scale);
    if (lane == 0) {
      srow[pos] = z;
      if (e < n_cand) {
        const bool in_w = pos < p.s1 || pos >= p.w0;
        p.S_cand[static_cast<long long>(row) * p.ldC + e] = in_w ? -INFINITY : z;
        p.pos_cand[static_cast<long long>(row) * p.ldC + e] = static_cast<int32_t>(pos);
      }
    }
  }
}

// Candidate indices chosen by the selection -> cache positions (-1 for none or a W key).
__global__ void __launch_bounds__(256) ivf_map_kernel(const IvfSearchParams p) {
  const long long n = static_cast<long long>(p.R) * p.k;
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n; i += static_cast<long long>(gridDim.x) * 256) {
    const long long row = i / p.k;
    const int32_t e = p.idx_cand[i];
    int32_t pos = -1;
    if (e >= 0 && e < p.n_cand[row] &&
        p.S_cand[row * p.ldC + e] != -INFINITY)
      pos = p.pos_cand[row * p.ldC + e];
    p.idx[i] = pos;
  }
}

// ---- host

cudaError_t launch_ivf_init(const IvfParams &p, cudaStream_t s) {
  ivf_init_kernel<<<dim3(p.nlist, p.BH), 128, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_ivf_assign(const IvfParams &p, bool accumulate, cudaStream_t s) {
  const long long warps = static_cast<long long>(p.BH) * p.N;
  ivf_assign_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(p, accumulate ? 1 : 0);
  return cudaGetLastError();
}
cudaError_t launch_ivf_update(const IvfParams &p, cudaStream_t s) {
  ivf_update_kernel<<<dim3(p.nlist, p.BH), 128, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_ivf_sort(const IvfParams &p, cudaStream_t s) {
  ivf_offsets_kernel<<<p.BH, 1024, 0, s>>>(p);
  const long long warps = static_cast<long long>(p.BH) * p.N;
  ivf_scatter_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_ivf_probe(const IvfSearchParams &p, cudaStream_t s) {
  ivf_probe_kernel<<<p.R, 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_ivf_cand(const IvfSearchParams &p, int d, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(std::max<long long>(1, std::min<long long>(64, (p.N + 2047) / 2048))),
                  static_cast<unsigned>(p.R));
  if (d == 128) ivf_cand_kernel<128><<<grid, 256, 0, s>>>(p);
  else ivf_cand_kernel<64><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_ivf_map(const IvfSearchParams &p, cudaStream_t s) {
  const long long n = static_cast<long long>(p.R) * p.k;
  ivf_map_kernel<<<static_cast<unsigned>(std::max<long long>(1, std::min<long long>(1024, (n + 255) / 256))), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ra
