// Dense flash-decode: full attention of every query head over all N cached tokens
// (RetrievalAttention slides, Eq. (1)), the comparison path of the sparse step.
//
// Grid: (split, KV head), one CTA per SM.  Each CTA streams a contiguous key range of one KV
// head in tiles of 128 keys.  One thread issues TMA loads of the K and V tiles (128-byte
// swizzled boxes) into a ring of kStages stages with one mbarrier each.  Per tile:
//   * scores of the G query heads: bf16 m16n8k16 tensor-core products (fp32 accumulate),
//     16 keys per warp, from ldmatrix fragments of the K tile;
//   * online softmax, one warp per head: running max m and sum l, rescale factor alpha, and the
//     weights p split into two bf16 parts p_hi + p_lo (p_hi = bf16(p), p_lo = bf16(p - p_hi)),
//     which keeps about 16 significant bits of p through the bf16 tensor-core product;
//   * P.V on tensor cores: A = the 16 x 16 weight tile (heads x keys, both parts), B = the V
//     tile read with ldmatrix.trans, fp32 accumulators rescaled by alpha per head.
// The last CTA of a KV head merges the split partial states with the weights of Eqs. (3)-(5).
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "merge.cuh"
#include "tma.cuh"

namespace ra {

template <int D>
struct DenseCfg {
  static constexpr int kThreads = 256;
  static constexpr int kWarps = 8;
  static constexpr int kTile = kDenseTile;                 // 128 keys
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = kTile * 128;            // 16 KB
  static constexpr int kTileBytes = kBoxes * kBoxBytes;    // K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kPBytes = 16 * kTile * 2;           // one 16 x 128 bf16 weight tile
  static constexpr int kNT = D / 64;                       // n8 tiles per warp in P.V
  static constexpr size_t smem_bytes() {
    return 1024 + static_cast<size_t>(kStages) * kStageBytes + 2 * kPBytes +
           static_cast<size_t>(kMaxGroup) * kTile * 4 + kStages * 8;
  }
};

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                                  uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t addr, uint32_t &r0, uint32_t &r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

// byte offset of logical 16-byte chunk c of row r in a 128-byte-swizzled tile of `rows` rows
__device__ __forceinline__ uint32_t tile_off(int r, int c, int box_bytes) {
  return static_cast<uint32_t>((c >> 3) * box_bytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}
// byte offset of chunk c of row r in a 16 x 128 bf16 weight tile (256-byte rows, XOR swizzle)
__device__ __forceinline__ uint32_t p_off(int r, int c) {
  return static_cast<uint32_t>(r * 256 + ((c ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(256, 1)
    dense_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DenseParams p) {
  using C = DenseCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t stages = (raw + 1023u) & ~1023u;
  uint8_t *base_ptr = smem_raw + (stages - raw);
  const uint32_t phi = stages + C::kStages * C::kStageBytes;     // weights, high parts
  const uint32_t plo = phi + C::kPBytes;                           // weights, low parts
  uint8_t *phi_ptr = base_ptr + C::kStages * C::kStageBytes;
  uint8_t *plo_ptr = phi_ptr + C::kPBytes;
  float *z_s = reinterpret_cast<float *>(plo_ptr + C::kPBytes);   // [8][128]
  const uint32_t bars = plo + C::kPBytes + kMaxGroup * C::kTile * 4;
  __shared__ float alpha_s[16];
  __shared__ float m_s[kMaxGroup];
  __shared__ float l_s[kMaxGroup];
  __shared__ bool s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int split = blockIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / p.Hkv;
  const int g = bg - b * p.Hkv;
  const long long rowbase = static_cast<long long>(b) * p.Hq + static_cast<long long>(g) * p.G;
  const long long k_begin = static_cast<long long>(split) * p.keys_per_split;
  long long k_end = k_begin + p.keys_per_split;
  if (k_end > p.N) k_end = p.N;
  const int n_tiles = static_cast<int>((k_end - k_begin + C::kTile - 1) / C::kTile);
  pdl_trigger();

  if (tid == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    for (int s = 0; s < C::kStages; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  // weight tiles: rows of absent heads stay zero for the whole kernel
  for (int i = tid; i < 2 * C::kPBytes / 16; i += C::kThreads)
    reinterpret_cast<uint4 *>(phi_ptr)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (tid < 16) alpha_s[tid] = 1.f;
  __syncthreads();
  pdl_wait();

  const uint64_t pol = policy_evict_first();
  auto issue = [&](int t, int slot) {
    const uint32_t bar = bars + 8 * slot;
    const int key0 = static_cast<int>(k_begin + static_cast<long long>(t) * C::kTile);
    mbar_arrive_expect_tx(bar, C::kStageBytes);
    const uint32_t dk = stages + slot * C::kStageBytes;
#pragma unroll
    for (int bx = 0; bx < C::kBoxes; ++bx) {
      tma_load_3d(dk + bx * C::kBoxBytes, &tmK, bx * 64, key0, bg, bar, pol);
      tma_load_3d(dk + C::kTileBytes + bx * C::kBoxBytes, &tmV, bx * 64, key0, bg, bar, pol);
    }
  };
  if (tid == 0)
    for (int s = 0; s < C::kStages - 1 && s < n_tiles; ++s) issue(s, s);

  // query fragments (B operand of the score product): head n = lane / 4
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
  const int arow = warp * 16 + (lane & 7) + (mat & 1) * 8;   // score ldmatrix row (key)
  const int prow = (lane & 7) + (mat & 1) * 8;               // weight ldmatrix row (head)

  float acc[C::kNT][4];
#pragma unroll
  for (int nt = 0; nt < C::kNT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;   // meaningful in warp h < G for head h

  int t = 0;
#pragma unroll 1
  for (; t < n_tiles; ++t) {
    const int slot = t % C::kStages;
    const bool landed = mbar_wait(bars + 8 * slot, static_cast<uint32_t>((t / C::kStages) & 1));
    if (!__syncthreads_and(landed)) break;
    if (tid == 0 && t + C::kStages - 1 < n_tiles)
      issue(t + C::kStages - 1, (t + C::kStages - 1) % C::kStages);
    const uint32_t kt = stages + slot * C::kStageBytes;
    const uint32_t vt = kt + C::kTileBytes;
    const long long key0 = k_begin + static_cast<long long>(t) * C::kTile;

    // scores: 16 keys per warp, all heads
    {
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < D / 16; kk += 2) {
        const int c0 = 2 * kk + (mat >> 1);
        uint32_t a[4], a2[4];
        ldmatrix_x4(kt + tile_off(arow, c0, C::kBoxBytes), a[0], a[1], a[2], a[3]);
        ldmatrix_x4(kt + tile_off(arow, c0 + 2, C::kBoxBytes), a2[0], a2[1], a2[2], a2[3]);
        mma_bf16_16816(a0, a, bq[kk][0], bq[kk][1]);
        mma_bf16_16816(a1, a2, bq[kk + 1][0], bq[kk + 1][1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = 2 * t4 + (e & 1);
        const int kr = warp * 16 + g4 + (e >> 1) * 8;
        z_s[h * C::kTile + kr] = key0 + kr < k_end ? (a0[e] + a1[e]) * p.scale : -INFINITY;
      }
    }
    __syncthreads();

    // online softmax, one warp per head; weights written as two bf16 parts
    if (warp < p.G) {
      const float4 zv = *reinterpret_cast<const float4 *>(z_s + warp * C::kTile + lane * 4);
      const float tmax = warp_max(fmaxf(fmaxf(zv.x, zv.y), fmaxf(zv.z, zv.w)));
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = expf(m_run - m_new);
      const float pv[4] = {expf(zv.x - m_new), expf(zv.y - m_new), expf(zv.z - m_new),
                           expf(zv.w - m_new)};
      uint32_t hi[2], lo[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(pv[2 * u], pv[2 * u + 1]);
        const float2 hf = __bfloat1622float2(h2);
        const __nv_bfloat162 l2 = __floats2bfloat162_rn(pv[2 * u] - hf.x, pv[2 * u + 1] - hf.y);
        hi[u] = *reinterpret_cast<const uint32_t *>(&h2);
        lo[u] = *reinterpret_cast<const uint32_t *>(&l2);
      }
      const uint32_t off = p_off(warp, lane >> 1) + (lane & 1) * 8;
      *reinterpret_cast<uint2 *>(phi_ptr + off) = make_uint2(hi[0], hi[1]);
      *reinterpret_cast<uint2 *>(plo_ptr + off) = make_uint2(lo[0], lo[1]);
      l_run = l_run * alpha + warp_sum((pv[0] + pv[1]) + (pv[2] + pv[3]));
      m_run = m_new;
      if (lane == 0) alpha_s[warp] = alpha;
    }
    __syncthreads();

    // P.V: warp w owns channels [w * D / 8, (w + 1) * D / 8)
    {
      const float al0 = alpha_s[g4], al1 = alpha_s[g4 + 8];
#pragma unroll
      for (int nt = 0; nt < C::kNT; ++nt) {
        acc[nt][0] *= al0;
        acc[nt][1] *= al0;
        acc[nt][2] *= al1;
        acc[nt][3] *= al1;
      }
#pragma unroll
      for (int kk = 0; kk < C::kTile / 16; ++kk) {
        uint32_t ah[4], alw[4];
        const int pc = 2 * kk + (mat >> 1);
        ldmatrix_x4(phi + p_off(prow, pc), ah[0], ah[1], ah[2], ah[3]);
        ldmatrix_x4(plo + p_off(prow, pc), alw[0], alw[1], alw[2], alw[3]);
        const int vkey = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        if constexpr (C::kNT == 2) {
          const int vc = 2 * warp + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(vt + tile_off(vkey, vc, C::kBoxBytes), b0, b1, b2, b3);
          mma_bf16_16816(acc[0], ah, b0, b1);
          mma_bf16_16816(acc[0], alw, b0, b1);
          mma_bf16_16816(acc[1], ah, b2, b3);
          mma_bf16_16816(acc[1], alw, b2, b3);
        } else {
          uint32_t b0, b1;
          ldmatrix_x2_trans(vt + tile_off(vkey, warp, C::kBoxBytes), b0, b1);
          mma_bf16_16816(acc[0], ah, b0, b1);
          mma_bf16_16816(acc[0], alw, b0, b1);
        }
      }
    }
  }

  if (t < n_tiles) {
    // a stage never completed: record it, wait (bounded) for the copies still in flight
    if (tid == 0) {
      atomicOr(p.err, kErrDenseWait);
      for (int tt = t; tt < n_tiles && tt < t + C::kStages - 1; ++tt)
        mbar_wait(bars + 8 * (tt % C::kStages), static_cast<uint32_t>((tt / C::kStages) & 1));
    }
    return;
  }

  if (warp < p.G && lane == 0) {
    m_s[warp] = m_run;
    l_s[warp] = l_run;
  }
  __syncthreads();
  // C fragment rows g4 (head g4) and g4 + 8 (absent: G <= 8); columns 2 t4, 2 t4 + 1
  if (g4 < p.G) {
    float *part = p.part + ((rowbase + g4) * p.nsplit + split) * (D + kPartPad);
#pragma unroll
    for (int nt = 0; nt < C::kNT; ++nt) {
      const int c = warp * (D / 8) + nt * 8 + 2 * t4;
      *reinterpret_cast<float2 *>(part + kPartPad + c) = make_float2(acc[nt][0], acc[nt][1]);
    }
    if (warp == 0 && t4 == 0) {
      part[0] = m_s[g4];
      part[1] = l_s[g4];
    }
  }
  // last-CTA hand-off: the barrier orders this CTA's partial-state stores before thread 0's
  // release fence and counter update; the CTA that sees the final count acquires and merges
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(p.meta + rowbase * kMetaWords + kDone, 1u);
    s_last = prev == static_cast<uint32_t>(p.nsplit - 1);
    if (s_last) __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  // merge the split states of the G query heads of this KV head (Eqs. (3)-(5))
  float *red = reinterpret_cast<float *>(base_ptr);   // the stage ring is free now
  float *buf = red + 64;                               // 16-byte aligned, 4 * 256 floats
  for (int h = 0; h < p.G; ++h)
    merge_states<D, C::kThreads>(p.part + (rowbase + h) * p.nsplit * (D + kPartPad), p.nsplit,
                                 p.out + (rowbase + h) * D, red, buf);
  if (tid == 0) p.meta[rowbase * kMetaWords + kDone] = 0u;
}

template <int D>
static cudaError_t launch_dense_t(const DenseParams &p, cudaStream_t s) {
  using C = DenseCfg<D>;
  const size_t smem = C::smem_bytes();
  static bool done[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(dense_decode_kernel<D>),
                                    static_cast<int>(smem), done);
  if (e != cudaSuccess) return e;
  CUtensorMap tk, tv;
  const uint64_t planes = static_cast<uint64_t>(p.B) * p.Hkv;
  if (!encode_rows_tmap(&tk, p.K, D, static_cast<uint64_t>(p.N), planes, C::kTile,
                        static_cast<uint64_t>(p.cap)) ||
      !encode_rows_tmap(&tv, p.V, D, static_cast<uint64_t>(p.N), planes, C::kTile,
                        static_cast<uint64_t>(p.cap)))
    return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(p.nsplit), static_cast<unsigned>(p.B * p.Hkv));
  return launch_pdl(dense_decode_kernel<D>, grid, dim3(C::kThreads), smem, s, tk, tv, p);
}

cudaError_t launch_dense(const DenseParams &p, int d, cudaStream_t s) {
  return d == 128 ? launch_dense_t<128>(p, s) : launch_dense_t<64>(p, s);
}

}  // namespace ra
