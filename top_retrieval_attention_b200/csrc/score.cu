// Score kernel: z[b, h, i] = q[b, h] . K[b, h / G, i] / sqrt(d) for every cached position i
// (RetrievalAttention slides, "Sparse attention renormalizes selected tokens", Eq. (1)),
// all G query heads of a KV head scored in one pass over that head's keys (slide "The GPU
// keeps 640 fixed positions": GQA heads share KV storage).
//
// Design (HBM bound: 2d bytes of K per position against 2Gd flops):
//   * persistent grid, one CTA per SM, each CTA streams a contiguous range of 128-key tiles;
//   * tiles are staged global -> shared by 16-byte cp.async into an XOR-swizzled ring of
//     kStages tiles, so several tiles are in flight per SM while one is computed;
//   * the G query vectors are the n = 8 operand of a bf16 m16n8k16 tensor-core product with
//     fp32 accumulation; each warp scores 16 keys of the tile from ldmatrix fragments;
//   * the epilogue scales, writes fp32 z, and builds the first radix digit's histogram
//     (top 11 bits of the order-preserving key) of the candidate positions in shared
//     memory, flushed to global once per KV head.
#include "common.cuh"
#include "kernels.h"

namespace ra {

template <int D>
struct ScoreCfg {
  static constexpr int kThreads = 256;
  static constexpr int kWarps = 8;
  static constexpr int kTile = kScoreTile;               // keys per tile (16 per warp)
  static constexpr int kRowBytes = D * 2;
  static constexpr int kTileBytes = kTile * kRowBytes;   // 32 KB (d=128) / 16 KB (d=64)
  static constexpr int kStages = D == 128 ? 4 : 6;
  static constexpr int kChunksPerRow = kRowBytes / 16;
  static constexpr int kCopiesPerThread = kTile * kChunksPerRow / kThreads;
  static constexpr size_t smem_bytes(int G) {
    return static_cast<size_t>(kStages) * kTileBytes + static_cast<size_t>(G) * kHistBins * 4;
  }
};

template <int D>
__global__ void __launch_bounds__(256, 1) score_gqa_kernel(const ScoreParams p) {
  using C = ScoreCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *tiles = smem;
  uint32_t *hist_s = reinterpret_cast<uint32_t *>(smem + C::kStages * C::kTileBytes);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const long long per = p.total_tiles / gridDim.x;
  const long long rem = p.total_tiles % gridDim.x;
  const long long t_begin = blockIdx.x * per + min(static_cast<long long>(blockIdx.x), rem);
  const int n_local = static_cast<int>(per + (blockIdx.x < rem ? 1 : 0));

  if (p.do_hist)
    for (int i = tid; i < p.G * kHistBins; i += C::kThreads) hist_s[i] = 0;

  auto load_tile = [&](long long t, int slot) {
    const long long bg = t / p.tiles_per_head;
    const long long key0 = (t - bg * p.tiles_per_head) * C::kTile;
    const __nv_bfloat16 *src0 = p.K + (bg * p.cap + key0) * D;
    const uint32_t dst0 = smem_u32(tiles + slot * C::kTileBytes);
#pragma unroll
    for (int i = 0; i < C::kCopiesPerThread; ++i) {
      const int ci = i * C::kThreads + tid;
      const int r = ci / C::kChunksPerRow;
      const int c = ci % C::kChunksPerRow;
      const bool valid = key0 + r < p.N;
      const void *src = valid ? static_cast<const void *>(src0 + static_cast<long long>(r) * D + c * 8)
                              : static_cast<const void *>(p.K);
      cp_async16(dst0 + swz(r, c, C::kRowBytes), src, valid ? 16u : 0u);
    }
  };

  auto flush_hist = [&](long long bg) {
    const long long b = bg / p.Hkv;
    const long long g = bg - b * p.Hkv;
    uint32_t *dst = p.hist + (b * p.Hq + g * p.G) * kHistBins;
    for (int i = tid; i < p.G * kHistBins; i += C::kThreads) {
      const uint32_t v = hist_s[i];
      if (v) {
        atomicAdd(dst + i, v);
        hist_s[i] = 0;
      }
    }
  };

#pragma unroll 1
  for (int s = 0; s < C::kStages - 1; ++s) {
    if (s < n_local) load_tile(t_begin + s, s);
    cp_async_commit();
  }

  long long cur_bg = -1;
  long long rowbase = 0;
  uint32_t bq[D / 16][2];
  const int mat = lane >> 3;
  const int arow = warp * 16 + (lane & 7) + (mat & 1) * 8;   // ldmatrix source row
  const int g4 = lane >> 2;
  const int t4 = lane & 3;

#pragma unroll 1
  for (int j = 0; j < n_local; ++j) {
    cp_async_wait<C::kStages - 2>();
    __syncthreads();
    {
      const int jn = j + C::kStages - 1;
      if (jn < n_local) load_tile(t_begin + jn, jn % C::kStages);
      cp_async_commit();
    }
    const long long t = t_begin + j;
    const long long bg = t / p.tiles_per_head;
    const long long key0 = (t - bg * p.tiles_per_head) * C::kTile;
    if (bg != cur_bg) {
      if (cur_bg >= 0 && p.do_hist) {
        flush_hist(cur_bg);
        __syncthreads();
      }
      cur_bg = bg;
      const long long b = bg / p.Hkv;
      const long long g = bg - b * p.Hkv;
      rowbase = b * p.Hq + g * p.G;
      // B operand (col-major k x n): element (k = channel, n = query head g4)
      const uint32_t *qrow =
          reinterpret_cast<const uint32_t *>(p.q + (rowbase + (g4 < p.G ? g4 : 0)) * D);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        bq[kk][0] = g4 < p.G ? __ldg(qrow + kk * 8 + t4) : 0u;
        bq[kk][1] = g4 < p.G ? __ldg(qrow + kk * 8 + t4 + 4) : 0u;
      }
    }

    const uint32_t tbase = smem_u32(tiles + (j % C::kStages) * C::kTileBytes);
    float acc0[4] = {0.f, 0.f, 0.f, 0.f};
    float acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < D / 16; kk += 2) {
      uint32_t a[4], a2[4];
      ldmatrix_x4(tbase + swz(arow, 2 * kk + (mat >> 1), C::kRowBytes), a[0], a[1], a[2], a[3]);
      ldmatrix_x4(tbase + swz(arow, 2 * kk + 2 + (mat >> 1), C::kRowBytes), a2[0], a2[1], a2[2],
                  a2[3]);
      mma_bf16_16816(acc0, a, bq[kk][0], bq[kk][1]);
      mma_bf16_16816(acc1, a2, bq[kk + 1][0], bq[kk + 1][1]);
    }

    // C fragment: e = 0,1 -> key g4, heads 2t4, 2t4+1; e = 2,3 -> key g4 + 8
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h = 2 * t4 + (e & 1);
      const long long key = key0 + warp * 16 + g4 + (e >> 1) * 8;
      if (h < p.G && key < p.N) {
        const float z = canon_zero((acc0[e] + acc1[e]) * p.scale);
        p.S[(rowbase + h) * p.ldS + key] = z;
        if (p.do_hist && key >= p.cand_lo && key < p.cand_hi)
          atomicAdd(&hist_s[h * kHistBins + (order_key(z) >> (32 - kHistBits))], 1u);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  if (cur_bg >= 0 && p.do_hist) flush_hist(cur_bg);
}

template <int D>
static cudaError_t launch_score_t(const ScoreParams &p, cudaStream_t s) {
  using C = ScoreCfg<D>;
  const size_t smem = C::smem_bytes(p.G);
  static bool done[64] = {};
  const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(score_gqa_kernel<D>),
                                          static_cast<int>(C::smem_bytes(kMaxGroup)), done);
  if (e != cudaSuccess) return e;
  long long grid = num_sms();
  if (grid > p.total_tiles) grid = p.total_tiles;
  if (grid < 1) grid = 1;
  score_gqa_kernel<D><<<static_cast<unsigned>(grid), C::kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_score(const ScoreParams &p, int d, cudaStream_t s) {
  return d == 128 ? launch_score_t<128>(p, s) : launch_score_t<64>(p, s);
}

}  // namespace ra
