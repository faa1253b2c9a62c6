// Score kernel: z[b, h, i] = q[b, h] . K[b, h / G, i] / sqrt(d) for every cached position i
// (RetrievalAttention slides, "Sparse attention renormalizes selected tokens", Eq. (1)),
// all G query heads of a KV head scored in one pass over that head's keys (slide "The GPU
// keeps 640 fixed positions": GQA heads share KV storage).
//
// Design (HBM bound: 2d bytes of K per position against 2Gd flops):
//   * persistent grid, one CTA per SM; each CTA streams a contiguous range of 128-key tiles
//     (the tile cursor advances incrementally, no per-tile division);
//   * one thread issues TMA bulk tensor loads (128-byte swizzled boxes of 128 keys x 64
//     channels, L2 evict-first) into a ring of kStages tiles, completion counted on one
//     mbarrier per stage; every thread waits on the stage barrier with a bounded poll;
//   * the G query vectors are the n = 8 operand of bf16 m16n8k16 tensor-core products with
//     fp32 accumulation; each warp scores 16 keys of the tile from ldmatrix fragments;
//   * the epilogue scales, writes fp32 z, and builds the first radix digit's histogram (top
//     11 bits of the order-preserving key) of the candidate positions in shared memory,
//     flushed to global once per KV head;
//   * optionally the step's append is fused in: the CTA whose tile holds the new token writes
//     its K and V rows to the cache and patches the key row into the staged tile.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace ra {

// ROWS keys per tile: 128 (d = 128, and every paged tile, which is one page) or 256 (dense
// d = 64, so that a tile carries as many bytes, and as much fixed per-tile work per byte, as a
// d = 128 tile).
template <int D, int ROWS>
struct ScoreCfg {
  static constexpr int kThreads = 256;
  static constexpr int kWarps = 8;
  static constexpr int kTile = ROWS;                       // keys per tile
  static constexpr int kGroups = ROWS / 128;               // 16-key MMA row groups per warp
  static constexpr int kBoxes = D / 64;                    // 64-channel boxes per tile
  static constexpr int kBoxBytes = kTile * 128;            // 16 KB per 128 rows
  static constexpr int kTileBytes = kBoxes * kBoxBytes;    // 32 KB (d=128 or 256 rows) / 16 KB
  static constexpr int kStages = kTileBytes == 32768 ? 5 : 8;
  static constexpr size_t smem_bytes(int G) {
    return 1024 + static_cast<size_t>(kStages) * kTileBytes +
           static_cast<size_t>(G) * kHistBins * 4 + kStages * 8;
  }
};

// ---- cache geometry: the dense [B, Hkv, cap, d] layout or 128-token pages (one tile each)

// Tokens of the (b, g) head bg.
__device__ __forceinline__ long long seq_n(const ScoreParams &p, const NoPaging &, long long) {
  return p.N;
}
__device__ __forceinline__ long long seq_n(const ScoreParams &p, const PagedInfo &pg, long long bg) {
  return pg.seq_len[bg / p.Hkv];
}
// The head and first key of flattened tile t (tiles ordered by head, then key; rows keys each).
__device__ __forceinline__ void tile_start(const ScoreParams &p, const NoPaging &, long long t,
                                           long long &bg, long long &key, int rows) {
  bg = t / p.tiles_per_head;
  key = (t - bg * p.tiles_per_head) * rows;
}
__device__ __forceinline__ void tile_start(const ScoreParams &p, const PagedInfo &pg, long long t,
                                           long long &bg, long long &key, int) {
  int b = 0;
  while (b + 1 < p.B && pg.tile_off[b + 1] <= t) ++b;   // once per CTA
  const long long per_head = (pg.seq_len[b] + kScoreTile - 1) / kScoreTile;
  const long long r = t - pg.tile_off[b];
  bg = static_cast<long long>(b) * p.Hkv + r / per_head;
  key = (r % per_head) * kScoreTile;
}
// TMA coordinates (rows, plane) of the tile at (bg, key).
__device__ __forceinline__ void tile_coords(const ScoreParams &, const NoPaging &, long long bg,
                                            long long key, int &y, int &z) {
  y = static_cast<int>(key);
  z = static_cast<int>(bg);
}
__device__ __forceinline__ void tile_coords(const ScoreParams &p, const PagedInfo &pg, long long bg,
                                            long long key, int &y, int &z) {
  const long long b = bg / p.Hkv, g = bg - b * p.Hkv;
  const int page = __ldg(pg.block_table + b * pg.max_pages + key / kPageSize);
  y = static_cast<int>(key % kPageSize);
  z = static_cast<int>(static_cast<long long>(page) * p.Hkv + g);
}
// The candidate range of head bg and whether its histogram is wanted.
__device__ __forceinline__ void cand_range(const ScoreParams &p, const NoPaging &, long long,
                                           long long &lo, long long &hi, bool &hist) {
  lo = p.cand_lo;
  hi = p.cand_hi;
  hist = p.do_hist != 0;
}
__device__ __forceinline__ void cand_range(const ScoreParams &p, const PagedInfo &pg, long long bg,
                                           long long &lo, long long &hi, bool &hist) {
  const long long N = pg.seq_len[bg / p.Hkv];
  lo = min(static_cast<long long>(pg.n_sink), N);
  hi = max(lo, N - pg.n_window);
  const long long k_eff = min(static_cast<long long>(pg.k), hi - lo);
  hist = p.do_hist != 0 && k_eff > 0 && k_eff < hi - lo;
}

template <int D, int ROWS, class Pg>
__global__ void __launch_bounds__(256, 1)
    score_gqa_kernel(const __grid_constant__ CUtensorMap tmK, const ScoreParams p, const Pg pg) {
  using C = ScoreCfg<D, ROWS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t tiles = (raw + 1023u) & ~1023u;          // swizzled boxes need 1024-byte alignment
  uint32_t *hist_s = reinterpret_cast<uint32_t *>(smem_raw + (tiles - raw) + C::kStages * C::kTileBytes);
  const uint32_t bars = tiles + C::kStages * C::kTileBytes + p.G * kHistBins * 4;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const long long per = p.total_tiles / gridDim.x;
  const long long rem = p.total_tiles % gridDim.x;
  const long long t_begin = blockIdx.x * per + min(static_cast<long long>(blockIdx.x), rem);
  const int n_local = static_cast<int>(per + (blockIdx.x < rem ? 1 : 0));
  pdl_trigger();
  if (n_local <= 0) return;

  if (tid == 0) {
    prefetch_tmap(&tmK);
    for (int s = 0; s < C::kStages; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  if (p.do_hist)
    for (int i = tid; i < p.G * kHistBins; i += C::kThreads) hist_s[i] = 0;
  __syncthreads();
  pdl_wait();   // K (appended rows) and the score / histogram buffers belong to the predecessor

  // load cursor (thread 0 only) and compute cursor (all threads)
  long long bg0, key0;
  tile_start(p, pg, t_begin, bg0, key0, C::kTile);
  long long l_bg = bg0, l_key = key0;
  long long c_bg = bg0, c_key = key0;
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int slot) {
    const uint32_t bar = bars + 8 * slot;
    mbar_arrive_expect_tx(bar, C::kTileBytes);
    int ty, tz;
    tile_coords(p, pg, l_bg, l_key, ty, tz);
#pragma unroll
    for (int bx = 0; bx < C::kBoxes; ++bx)
      tma_load_3d(tiles + slot * C::kTileBytes + bx * C::kBoxBytes, &tmK, bx * 64, ty, tz, bar, pol);
    l_key += C::kTile;
    if (l_key >= seq_n(p, pg, l_bg)) {
      l_key = 0;
      ++l_bg;
    }
  };
  if (tid == 0)
    for (int s = 0; s < C::kStages - 1 && s < n_local; ++s) issue(s);

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

  long long cur_bg = -1;
  long long rowbase = 0;
  long long cur_lo = 0, cur_hi = 0, cur_n = 0;
  bool cur_hist = false;
  uint32_t bq[D / 16][2];
  const int mat = lane >> 3;
  // ldmatrix source row of group gi: warp * (16 kGroups) + 16 gi + (lane & 7) + 8 (mat & 1)
  const int arow0 = warp * 16 * C::kGroups + (lane & 7) + (mat & 1) * 8;
  const int g4 = lane >> 2;
  const int t4 = lane & 3;
  int j = 0;

#pragma unroll 1
  for (; j < n_local; ++j) {
    const int slot = j % C::kStages;
    const bool landed = mbar_wait(bars + 8 * slot, static_cast<uint32_t>((j / C::kStages) & 1));
    if (!__syncthreads_and(landed)) break;     // uniform: every warp also finished tile j-1
    if (tid == 0 && j + C::kStages - 1 < n_local) issue((j + C::kStages - 1) % C::kStages);

    if (c_bg != cur_bg) {
      if (cur_bg >= 0 && cur_hist) {
        flush_hist(cur_bg);
        __syncthreads();
      }
      cur_bg = c_bg;
      cand_range(p, pg, cur_bg, cur_lo, cur_hi, cur_hist);
      cur_n = seq_n(p, pg, cur_bg);
      const long long b = c_bg / p.Hkv;
      const long long g = c_bg - b * p.Hkv;
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

    const uint32_t tbase = tiles + slot * C::kTileBytes;
    if (std::is_same<Pg, NoPaging>::value && p.k_new != nullptr && c_key <= p.N - 1 &&
        p.N - 1 < c_key + C::kTile) {
      // the tile holding the token this step appends (uniform over the CTA): its key row
      // replaces the stale row in the staged tile, and its K and V rows go to the cache
      const int r = static_cast<int>(p.N - 1 - c_key);
      constexpr int kChunks = D / 8;   // 16-byte chunks of a row
      const long long src = c_bg * D, dst = (c_bg * p.cap + p.N - 1) * D;
      if (tid < kChunks) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.k_new + src) + tid);
        st_shared_v4(tbase + (tid >> 3) * C::kBoxBytes + r * 128 + (((tid & 7) ^ (r & 7)) << 4), v);
        reinterpret_cast<uint4 *>(p.K_cache + dst)[tid] = v;
        fence_proxy_async_smem();   // before a later TMA load refills this stage
      } else if (tid >= 32 && tid < 32 + kChunks) {
        reinterpret_cast<uint4 *>(p.V_cache + dst)[tid - 32] =
            __ldg(reinterpret_cast<const uint4 *>(p.v_new + src) + (tid - 32));
      }
      __syncthreads();
    }
#pragma unroll
    for (int gi = 0; gi < C::kGroups; ++gi) {
      const int arow = arow0 + 16 * gi;
      float acc0[4] = {0.f, 0.f, 0.f, 0.f};
      float acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < D / 16; kk += 2) {
        // logical 16-byte chunk c of row r lives in box c / 8 at swizzled chunk (c % 8) ^ (r % 8)
        const int c0 = 2 * kk + (mat >> 1);
        const int c1 = c0 + 2;
        uint32_t a[4], a2[4];
        ldmatrix_x4(tbase + (c0 >> 3) * C::kBoxBytes + arow * 128 + (((c0 & 7) ^ (arow & 7)) << 4),
                    a[0], a[1], a[2], a[3]);
        ldmatrix_x4(tbase + (c1 >> 3) * C::kBoxBytes + arow * 128 + (((c1 & 7) ^ (arow & 7)) << 4),
                    a2[0], a2[1], a2[2], a2[3]);
        mma_bf16_16816(acc0, a, bq[kk][0], bq[kk][1]);
        mma_bf16_16816(acc1, a2, bq[kk + 1][0], bq[kk + 1][1]);
      }

      // C fragment: e = 0,1 -> key g4, heads 2t4, 2t4+1; e = 2,3 -> key g4 + 8
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = 2 * t4 + (e & 1);
        const long long key = c_key + warp * 16 * C::kGroups + 16 * gi + g4 + (e >> 1) * 8;
        if (h < p.G && key < cur_n) {
          const float z = canon_zero((acc0[e] + acc1[e]) * p.scale);
          p.S[(rowbase + h) * p.ldS + key] = z;
          if (cur_hist && key >= cur_lo && key < cur_hi)
            atomicAdd(&hist_s[h * kHistBins + (order_key(z) >> (32 - kHistBits))], 1u);
        }
      }
    }
    c_key += C::kTile;
    if (c_key >= cur_n) {
      c_key = 0;
      ++c_bg;
    }
  }

  if (j < n_local) {
    // a stage never completed: record it, wait (bounded) for the copies still in flight
    if (tid == 0) {
      atomicOr(p.err, kErrScoreWait);
      for (int jj = j; jj < n_local && jj < j + C::kStages - 1; ++jj)
        mbar_wait(bars + 8 * (jj % C::kStages), static_cast<uint32_t>((jj / C::kStages) & 1));
    }
    return;
  }
  __syncthreads();
  if (cur_bg >= 0 && cur_hist) flush_hist(cur_bg);
}

template <int D, int ROWS, class Pg>
static cudaError_t launch_score_t(const ScoreParams &p, const Pg &pg, long long num_pages,
                                  cudaStream_t s) {
  using C = ScoreCfg<D, ROWS>;
  static bool done[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(score_gqa_kernel<D, ROWS, Pg>),
                                    static_cast<int>(C::smem_bytes(kMaxGroup)), done);
  if (e != cudaSuccess) return e;
  CUtensorMap tm;
  const bool paged = num_pages > 0;
  // dense: [B * Hkv planes][N rows (cap apart)][d]; paged: [pages * Hkv planes][128 rows][d]
  if (!encode_rows_tmap(&tm, p.K, D, paged ? kPageSize : static_cast<uint64_t>(p.N),
                        paged ? static_cast<uint64_t>(num_pages) * p.Hkv
                              : static_cast<uint64_t>(p.B) * p.Hkv,
                        C::kTile, paged ? kPageSize : static_cast<uint64_t>(p.cap)))
    return cudaErrorInvalidValue;
  long long grid = num_sms();
  if (grid > p.total_tiles) grid = p.total_tiles;
  if (grid < 1) grid = 1;
  return launch_pdl(score_gqa_kernel<D, ROWS, Pg>, dim3(static_cast<unsigned>(grid)),
                    dim3(C::kThreads), C::smem_bytes(p.G), s, tm, p, pg);
}

int score_tile_rows(int d) { return d == 64 ? 256 : 128; }

cudaError_t launch_score(const ScoreParams &p, int d, cudaStream_t s) {
  const NoPaging pg{};
  // the tile count follows the tile size of this head dimension
  ScoreParams q = p;
  const int rows = score_tile_rows(d);
  q.tiles_per_head = (p.N + rows - 1) / rows;
  q.total_tiles = q.tiles_per_head * p.B * p.Hkv;
  return d == 128 ? launch_score_t<128, 128>(q, pg, 0, s) : launch_score_t<64, 256>(q, pg, 0, s);
}

cudaError_t launch_score_paged(const ScoreParams &p, const PagedInfo &pg, long long num_pages, int d,
                               cudaStream_t s) {
  return d == 128 ? launch_score_t<128, 128>(p, pg, num_pages, s)
                  : launch_score_t<64, 128>(p, pg, num_pages, s);
}

}  // namespace ra
