// Dense flash-decode: full attention of every query head over all N cached tokens
// (RetrievalAttention slides, Eq. (1)), the comparison path of the sparse step.
//
// Grid: (split, KV head).  Each CTA streams a contiguous key range of one KV head in tiles of
// 128 keys (K and V staged by cp.async into swizzled shared memory, a ring of kStages
// tiles); the G query heads are scored against the tile on tensor cores (bf16 m16n8k16,
// fp32 accumulate), an online softmax keeps (m, l) per head, and P.V accumulates in fp32 on
// the CUDA cores.  The last CTA of a KV head merges the split partial states with the
// weights of Eqs. (3)-(5).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace ra {

template <int D>
struct DenseCfg {
  static constexpr int kThreads = 256;
  static constexpr int kWarps = 8;
  static constexpr int kTile = kDenseTile;
  static constexpr int kRowBytes = D * 2;
  static constexpr int kTileBytes = kTile * kRowBytes;         // one of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kChunksPerRow = kRowBytes / 16;
  static constexpr int kCopiesPerThread = kTile * kChunksPerRow / kThreads;
  static constexpr int kPairs = D / 2;                          // channel pairs
  static constexpr int kHeadSlots = kThreads / kPairs;          // 4 (d=128) / 8 (d=64)
  static constexpr int kHeadsPerThread = (kMaxGroup + kHeadSlots - 1) / kHeadSlots;
  static constexpr size_t smem_bytes() {
    return static_cast<size_t>(kStages) * kStageBytes + 2 * kMaxGroup * kTile * sizeof(float);
  }
};

template <int D>
__global__ void __launch_bounds__(256, 1) dense_decode_kernel(const DenseParams p) {
  using C = DenseCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  float *z_s = reinterpret_cast<float *>(smem + C::kStages * C::kStageBytes);   // [8][128]
  float *p_s = z_s + kMaxGroup * C::kTile;                                         // [8][128]
  __shared__ float alpha_s[kMaxGroup];
  __shared__ float m_s[kMaxGroup];
  __shared__ float l_s[kMaxGroup];
  __shared__ bool s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / p.Hkv;
  const int g = bg - b * p.Hkv;
  const long long rowbase = static_cast<long long>(b) * p.Hq + static_cast<long long>(g) * p.G;
  const __nv_bfloat16 *Kh = p.K + static_cast<long long>(bg) * p.cap * D;
  const __nv_bfloat16 *Vh = p.V + static_cast<long long>(bg) * p.cap * D;
  const long long k_begin = static_cast<long long>(split) * p.keys_per_split;
  long long k_end = k_begin + p.keys_per_split;
  if (k_end > p.N) k_end = p.N;
  const int n_tiles = static_cast<int>((k_end - k_begin + C::kTile - 1) / C::kTile);

  auto load_tile = [&](int t, int slot) {
    const long long key0 = k_begin + static_cast<long long>(t) * C::kTile;
    const uint32_t dk = smem_u32(smem + slot * C::kStageBytes);
    const uint32_t dv = dk + C::kTileBytes;
#pragma unroll
    for (int i = 0; i < C::kCopiesPerThread; ++i) {
      const int ci = i * C::kThreads + tid;
      const int r = ci / C::kChunksPerRow;
      const int c = ci % C::kChunksPerRow;
      const bool valid = key0 + r < k_end;
      const long long off = (key0 + r) * D + c * 8;
      cp_async16(dk + swz(r, c, C::kRowBytes), valid ? static_cast<const void *>(Kh + off) : p.K,
                 valid ? 16u : 0u);
      cp_async16(dv + swz(r, c, C::kRowBytes), valid ? static_cast<const void *>(Vh + off) : p.V,
                 valid ? 16u : 0u);
    }
  };

#pragma unroll 1
  for (int s = 0; s < C::kStages - 1; ++s) {
    if (s < n_tiles) load_tile(s, s);
    cp_async_commit();
  }

  // query fragments (B operand): head n = lane / 4
  const int g4 = lane >> 2, t4 = lane & 3;
  uint32_t bq[D / 16][2];
  {
    const uint32_t *qrow =
        reinterpret_cast<const uint32_t *>(p.q + (rowbase + (g4 < p.G ? g4 : 0)) * D);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      bq[kk][0] = g4 < p.G ? __ldg(qrow + kk * 8 + t4) : 0u;
      bq[kk][1] = g4 < p.G ? __ldg(qrow + kk * 8 + t4 + 4) : 0u;
    }
  }
  const int mat = lane >> 3;
  const int arow = warp * 16 + (lane & 7) + (mat & 1) * 8;

  // P.V ownership: channel pair cp, heads hs, hs + kHeadSlots, ...
  const int cp = tid % C::kPairs;
  const int hs = tid / C::kPairs;
  float acc[C::kHeadsPerThread][2];
#pragma unroll
  for (int j = 0; j < C::kHeadsPerThread; ++j) acc[j][0] = acc[j][1] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;   // meaningful in warp h < G for head h

#pragma unroll 1
  for (int t = 0; t < n_tiles; ++t) {
    cp_async_wait<C::kStages - 2>();
    __syncthreads();
    {
      const int tn = t + C::kStages - 1;
      if (tn < n_tiles) load_tile(tn, tn % C::kStages);
      cp_async_commit();
    }
    const int slot = t % C::kStages;
    const uint32_t kbase = smem_u32(smem + slot * C::kStageBytes);
    const uint8_t *vtile = smem + slot * C::kStageBytes + C::kTileBytes;
    const long long key0 = k_begin + static_cast<long long>(t) * C::kTile;

    // scores of 16 keys per warp for all heads
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < D / 16; kk += 2) {
      uint32_t a[4], a2[4];
      ldmatrix_x4(kbase + swz(arow, 2 * kk + (mat >> 1), C::kRowBytes), a[0], a[1], a[2], a[3]);
      ldmatrix_x4(kbase + swz(arow, 2 * kk + 2 + (mat >> 1), C::kRowBytes), a2[0], a2[1], a2[2],
                  a2[3]);
      mma_bf16_16816(a0, a, bq[kk][0], bq[kk][1]);
      mma_bf16_16816(a1, a2, bq[kk + 1][0], bq[kk + 1][1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h = 2 * t4 + (e & 1);
      const int kr = warp * 16 + g4 + (e >> 1) * 8;
      const bool valid = key0 + kr < k_end;
      z_s[h * C::kTile + kr] = valid ? (a0[e] + a1[e]) * p.scale : -INFINITY;
    }
    __syncthreads();

    // online softmax, one warp per head
    if (warp < p.G) {
      const float4 zv = *reinterpret_cast<const float4 *>(z_s + warp * C::kTile + lane * 4);
      const float tmax = warp_max(fmaxf(fmaxf(zv.x, zv.y), fmaxf(zv.z, zv.w)));
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = expf(m_run - m_new);
      float4 pv;
      pv.x = expf(zv.x - m_new);
      pv.y = expf(zv.y - m_new);
      pv.z = expf(zv.z - m_new);
      pv.w = expf(zv.w - m_new);
      *reinterpret_cast<float4 *>(p_s + warp * C::kTile + lane * 4) = pv;
      l_run = l_run * alpha + warp_sum(pv.x + pv.y + pv.z + pv.w);
      m_run = m_new;
      if (lane == 0) alpha_s[warp] = alpha;
    }
    __syncthreads();

    // P.V: acc[h][pair] = alpha_h * acc + sum_key p[h][key] * V[key][pair]
#pragma unroll
    for (int j = 0; j < C::kHeadsPerThread; ++j) {
      const int h = hs + j * C::kHeadSlots;
      if (h < p.G) {
        const float al = alpha_s[h];
        acc[j][0] *= al;
        acc[j][1] *= al;
      }
    }
    const int chunk = cp >> 2;            // 16-byte chunk holding this pair
    const int within = (cp & 3) * 4;      // byte offset of the pair inside the chunk
#pragma unroll 4
    for (int kr = 0; kr < C::kTile; kr += 4) {
      uint32_t vw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        vw[u] = *reinterpret_cast<const uint32_t *>(vtile + swz(kr + u, chunk, C::kRowBytes) + within);
#pragma unroll
      for (int j = 0; j < C::kHeadsPerThread; ++j) {
        const int h = hs + j * C::kHeadSlots;
        if (h < p.G) {
          const float4 pw = *reinterpret_cast<const float4 *>(p_s + h * C::kTile + kr);
          const float pu[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            acc[j][0] += pu[u] * bf16_lo(vw[u]);
            acc[j][1] += pu[u] * bf16_hi(vw[u]);
          }
        }
      }
    }
  }
  cp_async_wait<0>();

  if (warp < p.G && lane == 0) {
    m_s[warp] = m_run;
    l_s[warp] = l_run;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < C::kHeadsPerThread; ++j) {
    const int h = hs + j * C::kHeadSlots;
    if (h < p.G) {
      float *part = p.part + ((rowbase + h) * p.nsplit + split) * (D + 2);
      part[2 + 2 * cp] = acc[j][0];
      part[3 + 2 * cp] = acc[j][1];
      if (cp == 0) {
        part[0] = m_s[h];
        part[1] = l_s[h];
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(p.meta + rowbase * kMetaWords + kDenseDone, 1u);
    s_last = prev == static_cast<uint32_t>(p.nsplit - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = tid; i < p.G * D; i += C::kThreads) {
    const int h = i / D, c = i - h * D;
    const float *prow = p.part + (rowbase + h) * p.nsplit * (D + 2);
    float M = -INFINITY;
    for (int j = 0; j < p.nsplit; ++j) M = fmaxf(M, __ldcg(prow + j * (D + 2)));
    float num = 0.f, den = 0.f;
    for (int j = 0; j < p.nsplit; ++j) {
      const float wj = expf(__ldcg(prow + j * (D + 2)) - M);
      den += wj * __ldcg(prow + j * (D + 2) + 1);
      num += wj * __ldcg(prow + j * (D + 2) + 2 + c);
    }
    p.out[(rowbase + h) * D + c] = num / den;
  }
  if (tid == 0) p.meta[rowbase * kMetaWords + kDenseDone] = 0u;
}

template <int D>
static cudaError_t launch_dense_t(const DenseParams &p, cudaStream_t s) {
  using C = DenseCfg<D>;
  const size_t smem = C::smem_bytes();
  static bool done[64] = {};
  const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(dense_decode_kernel<D>),
                                          static_cast<int>(smem), done);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(p.nsplit), static_cast<unsigned>(p.B * p.Hkv));
  dense_decode_kernel<D><<<grid, C::kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_dense(const DenseParams &p, int d, cudaStream_t s) {
  return d == 128 ? launch_dense_t<128>(p, s) : launch_dense_t<64>(p, s);
}

}  // namespace ra
