// Score kernel: z[b, h, i] = q[b, h] . K[b, h / G, i] / sqrt(d) for every cached position i
// (RetrievalAttention slides, "Sparse attention renormalizes selected tokens", Eq. (1)),
// all G query heads of a KV head scored in one pass over that head's keys (slide "The GPU
// keeps 640 fixed positions": GQA heads share KV storage).
//
// Design (HBM bound: 2d bytes of K per position against 2Gd flops):
//   * persistent grid, one CTA per SM; the tiles, ordered by KV head and then key, are dealt
//     out in runs of consecutive tiles, run r to CTA r mod grid: on long scans the runs are a
//     few tiles, so all CTAs sweep the heads in the same order and each head's scores are
//     complete long before the scan ends (short scans: one contiguous range per CTA); a CTA
//     done with a head publishes that on a per-head counter, which the selection kernel
//     (launched behind it and resident beside it) waits on to work on that head during the scan;
//   * warp-specialised pipeline: one producer warp issues TMA bulk tensor loads (128-byte
//     swizzled boxes of 128 keys x 64 channels, L2 evict-first) plus a bulk copy of the head
//     group's query vectors into a ring of stages (a full and an empty mbarrier per stage);
//     eight consumer warps each score their 16 keys of a staged tile and release the stage, with
//     no CTA-wide barrier per tile; every wait is bounded;
//   * the G query vectors are the n = 8 operand of bf16 m16n8k16 tensor-core products with
//     fp32 accumulation, read from the stage's query copy when the KV head changes;
//   * the epilogue scales, writes fp32 z, and builds the histogram of the selection's first
//     radix digit (digit1_bin_z, computed from the float) over the candidate positions in
//     shared memory (16-bit counts, two bins a word), flushed to global when the CTA moves to
//     another KV head; score-row and histogram pointers are set per head and key ranges are
//     checked per tile, since the consumer warps' issue rate bounds the scan at G = 4-8;
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
  static constexpr int kConsumers = 8;                     // warps scoring tiles
  static constexpr int kThreads = 32 * (kConsumers + 1);   // + the producer warp
  static constexpr int kTile = ROWS;                       // keys per tile
  static constexpr int kGroups = ROWS / 128;               // 16-key MMA row groups per warp
  static constexpr int kBoxes = D / 64;                    // 64-channel boxes per tile
  static constexpr int kBoxBytes = kTile * 128;            // 16 KB per 128 rows
  static constexpr int kTileBytes = kBoxes * kBoxBytes;    // 32 KB (d=128 or 256 rows) / 16 KB
  static constexpr int kMaxStages = kTileBytes == 32768 ? 5 : 8;
  static constexpr int kHistWords = kHistBins / 2;         // 16-bit bins, two per word
  // a flush before any 16-bit count can reach 65536 (a CTA scores at most kTile keys a tile)
  static constexpr int kFlushTiles = 65535 / kTile;
  static constexpr int q_bytes(int G) { return G * D * 2; }   // a multiple of 16
  // tiles (1024-byte aligned), query copies, histograms, full + empty barriers, abort flag
  static constexpr size_t smem_bytes(int G, int stages) {
    return 1024 + static_cast<size_t>(stages) * (kTileBytes + q_bytes(G)) +
           static_cast<size_t>(G) * kHistWords * 4 + 16 * stages + 16;
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
// Tiles are visited in increasing t, so the paged lookup walks its sequence index b forward.
__device__ __forceinline__ void tile_start(const ScoreParams &p, const NoPaging &, long long t,
                                           int &, long long &bg, long long &key, int rows) {
  bg = t / p.tiles_per_head;
  key = (t - bg * p.tiles_per_head) * rows;
}
__device__ __forceinline__ void tile_start(const ScoreParams &p, const PagedInfo &pg, long long t,
                                           int &b, long long &bg, long long &key, int) {
  while (b + 1 < p.B && pg.tile_off[b + 1] <= t) ++b;
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

// A CTA's walk over its tiles: runs of `chunk` consecutive tiles (in the order of heads, then
// keys), run r = blockIdx.x + m * gridDim.x.  Inside a run the head and key advance by
// addition; only the first tile of a run is located by division.
template <int ROWS>
struct TileWalk {
  long long t, bg, key, n;   // n: tokens of head bg
  int b, run;
  template <class Pg>
  __device__ __forceinline__ void locate(const ScoreParams &p, const Pg &pg) {
    if (t < p.total_tiles) {
      tile_start(p, pg, t, b, bg, key, ROWS);
      n = seq_n(p, pg, bg);
    }
  }
  template <class Pg>
  __device__ __forceinline__ void start(const ScoreParams &p, const Pg &pg, int chunk) {
    b = 0;
    run = 0;
    bg = key = n = 0;
    t = static_cast<long long>(blockIdx.x) * chunk;
    locate(p, pg);
  }
  template <class Pg>
  __device__ __forceinline__ void next(const ScoreParams &p, const Pg &pg, int chunk) {
    ++t;
    if (++run == chunk) {
      run = 0;
      t += static_cast<long long>(gridDim.x - 1) * chunk;
      locate(p, pg);
    } else {
      key += ROWS;
      if (key >= n) {   // the run crosses into the next head
        if constexpr (std::is_same<Pg, NoPaging>::value) {
          key = 0;
          ++bg;
        } else {
          locate(p, pg);
        }
      }
    }
  }
};

// At most 104 registers a thread: registers are allocated per SM sub-partition (16K each),
// which gets three of this kernel's nine warps, and a selection CTA (eight warps of at most 96
// registers, two a sub-partition) must still fit beside them: 3 * 104 + 2 * 96 <= 512 (x 32).
template <int D, int ROWS, class Pg>
__global__ void __maxnreg__(104)
    score_gqa_kernel(const __grid_constant__ CUtensorMap tmK, const ScoreParams p, const Pg pg,
                     const int stages, const int chunk) {
  using C = ScoreCfg<D, ROWS>;
  constexpr int kCons = 32 * C::kConsumers;   // consumer threads
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t tiles = (raw + 1023u) & ~1023u;          // swizzled boxes need 1024-byte alignment
  const int qb = C::q_bytes(p.G);
  const uint32_t qs = tiles + stages * C::kTileBytes;      // query copy of each stage
  uint8_t *base = smem_raw + (tiles - raw);
  uint32_t *hist_s = reinterpret_cast<uint32_t *>(base + stages * (C::kTileBytes + qb));
  const uint32_t full = qs + stages * qb + p.G * C::kHistWords * 4;
  const uint32_t empty = full + 8 * stages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(base + (empty + 8 * stages - tiles));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const long long BH = static_cast<long long>(p.B) * p.Hkv;

  // this CTA's tile count
  const long long n_runs = (p.total_tiles + chunk - 1) / chunk;
  const long long my_runs = n_runs > blockIdx.x ? (n_runs - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const long long last_run = blockIdx.x + (my_runs - 1) * static_cast<long long>(gridDim.x);
  const int n_local = my_runs == 0 ? 0
                                   : static_cast<int>((my_runs - 1) * chunk +
                                                      min(static_cast<long long>(chunk),
                                                          p.total_tiles - last_run * chunk));

  if (tid == 0) {
    prefetch_tmap(&tmK);
    for (int s = 0; s < stages; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, C::kConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (p.do_hist)
    for (int i = tid; i < p.G * C::kHistWords; i += C::kThreads) hist_s[i] = 0;
  __syncthreads();
  pdl_wait();   // K (appended rows), the score / histogram buffers and the counters belong to the
                // predecessor; the selection that waits on the counters is let in only now
  pdl_trigger();

  if (warp == C::kConsumers) {
    // ---------------------------------------------------------------- producer warp
    if (lane == 0) {
      TileWalk<ROWS> w;
      w.start(p, pg, chunk);
      const uint64_t pol = policy_evict_first();
      long long q_bg = -1;
      const __nv_bfloat16 *q_src = p.q;
      int slot = 0;
      uint32_t epar = 0;
      int j = 0;
      for (; j < n_local; ++j) {
        // the k-th reuse of a slot waits for the consumers' release of its (k-1)-th use
        if (j >= stages && !mbar_wait_or_abort(empty + 8 * slot, epar, abort_flag)) break;
        const uint32_t bar = full + 8 * slot;
        mbar_arrive_expect_tx(bar, C::kTileBytes + qb);
        int ty, tz;
        tile_coords(p, pg, w.bg, w.key, ty, tz);
#pragma unroll
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(tiles + slot * C::kTileBytes + bx * C::kBoxBytes, &tmK, bx * 64, ty, tz, bar, pol);
        if (w.bg != q_bg) {   // the group's query vectors: rows b * Hq + g * G .. + G
          q_bg = w.bg;
          const long long bq0 = w.bg / p.Hkv;
          q_src = p.q + (bq0 * p.Hq + (w.bg - bq0 * p.Hkv) * p.G) * D;
        }
        bulk_load(qs + slot * qb, q_src, qb, bar);
        if (++slot == stages) {
          slot = 0;
          if (j >= stages) epar ^= 1u;   // the next round of the ring waits one phase later
        }
        w.next(p, pg, chunk);
      }
      if (j < n_local) {
        // a stage was never released: stop, and wait (bounded) for the copies in flight
        atomicOr(p.err, kErrScoreWait);
        *abort_flag = 1;
        for (int jj = max(0, j - stages); jj < j; ++jj)
          mbar_wait(full + 8 * (jj % stages), static_cast<uint32_t>((jj / stages) & 1));
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumer warps
  // Heads [0, upto) are finished for this CTA: publish the ones not yet published.  Every CTA
  // publishes every head exactly once, so a head is complete when its counter reaches gridDim.x.
  long long published = 0;
  auto publish = [&](long long upto) {   // all consumer threads, after a consumer barrier
    if (p.ready != nullptr && tid == 0)
      for (long long g = published; g < upto; ++g) red_release_add1(p.ready + g * p.ready_stride);
    published = upto;
  };
  // Adds this CTA's counts of head bg to the global histograms and clears them.  Word i (bins
  // 2i and 2i + 1 of its head) belongs to thread i mod kCons, so a head's few busy words are
  // spread over many threads; a word's two 16-bit counts go out as one 64-bit add onto the two
  // adjacent 32-bit global bins (no carry crosses between them: a bin counts fewer than 2^31
  // keys).  Loads are issued eight at a time before any test.
  auto flush_hist = [&](long long bg) {
    constexpr int kPer = kMaxGroup * C::kHistWords / kCons;   // words a thread owns at G = 8
    constexpr int kBatch = 8;
    const int nw = p.G * C::kHistWords;
    const long long b = bg / p.Hkv;
    uint32_t *dst = p.hist + (b * p.Hq + (bg - b * p.Hkv) * p.G) * kHistBins;
#pragma unroll 1
    for (int u0 = 0; u0 < kPer; u0 += kBatch) {
      if (u0 * kCons >= nw) break;
      uint32_t v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = tid + (u0 + u) * kCons;
        v[u] = i < nw ? hist_s[i] : 0u;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (v[u] == 0u) continue;
        const int i = tid + (u0 + u) * kCons;
        hist_s[i] = 0u;
        // head i / kHistWords, bins 2 (i % kHistWords) and the next
        unsigned long long *pair = reinterpret_cast<unsigned long long *>(
            dst + (i / C::kHistWords) * kHistBins + 2 * (i % C::kHistWords));
        atomicAdd(pair, (static_cast<unsigned long long>(v[u] >> 16) << 32) | (v[u] & 0xFFFFu));
      }
    }
  };

  TileWalk<ROWS> w;
  w.start(p, pg, chunk);
  long long cur_bg = -1;
  long long cur_lo = 0, cur_hi = 0, cur_n = 0;
  // this lane's two query heads of the group (C fragment columns 2 t4 and 2 t4 + 1): their score
  // rows and shared histograms, set at each head change
  float *srow0 = nullptr, *srow1 = nullptr;
  uint32_t *hrow0 = hist_s, *hrow1 = hist_s;
  bool hv0 = false, hv1 = false;
  bool cur_hist = false;
  int since_flush = 0;
  uint32_t bq[D / 16][2];
  const int mat = lane >> 3;
  // ldmatrix source row of group gi: warp * (16 kGroups) + 16 gi + (lane & 7) + 8 (mat & 1)
  const int arow0 = warp * 16 * C::kGroups + (lane & 7) + (mat & 1) * 8;
  const int g4 = lane >> 2;
  const int t4 = lane & 3;
  int slot = 0;
  uint32_t fpar = 0;
  bool ok = true;

#pragma unroll 1
  for (int j = 0; j < n_local; ++j) {
    ok = ok && mbar_wait_or_abort(full + 8 * slot, fpar, abort_flag);
    if (!ok && lane == 0 && *abort_flag == 0) {
      atomicOr(p.err, kErrScoreWait);
      *abort_flag = 1;
    }
    // the same head changes in every consumer warp (a function of j only): consumer barriers
    if (w.bg != cur_bg || since_flush == C::kFlushTiles) {
      named_bar_sync(kCons);   // every consumer warp is done with the earlier tiles
      if (cur_bg >= 0 && cur_hist) flush_hist(cur_bg);
      named_bar_sync(kCons);   // the flush is complete before any warp counts again
      since_flush = 0;
      if (w.bg != cur_bg) {
        publish(w.bg);           // every head before this tile's is done for this CTA
        cur_bg = w.bg;
        cand_range(p, pg, cur_bg, cur_lo, cur_hi, cur_hist);
        cur_n = w.n;
        const long long b = cur_bg / p.Hkv;
        const long long g = cur_bg - b * p.Hkv;
        const long long rowbase = b * p.Hq + g * p.G;
        hv0 = 2 * t4 < p.G;
        hv1 = 2 * t4 + 1 < p.G;
        srow0 = p.S + (rowbase + (hv0 ? 2 * t4 : 0)) * p.ldS;
        srow1 = p.S + (rowbase + (hv1 ? 2 * t4 + 1 : 0)) * p.ldS;
        hrow0 = hist_s + (hv0 ? 2 * t4 : 0) * C::kHistWords;
        hrow1 = hist_s + (hv1 ? 2 * t4 + 1 : 0) * C::kHistWords;
        if (ok) {
          // B operand (col-major k x n): element (k = channel, n = query head g4), from the
          // stage's copy of the group's queries
          const uint32_t qrow = qs + slot * qb + (g4 < p.G ? g4 : 0) * D * 2;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t x0, x1;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x0) : "r"(qrow + (kk * 8 + t4) * 4));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x1) : "r"(qrow + (kk * 8 + t4 + 4) * 4));
            bq[kk][0] = g4 < p.G ? x0 : 0u;
            bq[kk][1] = g4 < p.G ? x1 : 0u;
          }
        }
      }
    }

    const uint32_t tbase = tiles + slot * C::kTileBytes;
    if (std::is_same<Pg, NoPaging>::value && p.k_new != nullptr && w.key <= p.N - 1 &&
        p.N - 1 < w.key + C::kTile) {
      // the tile holding the token this step appends (the same tile in every consumer warp):
      // its key row replaces the stale row in the staged tile, and its K and V rows go to the
      // cache
      const int r = static_cast<int>(p.N - 1 - w.key);
      constexpr int kChunks = D / 8;   // 16-byte chunks of a row
      const long long src = w.bg * D, dst = (w.bg * p.cap + p.N - 1) * D;
      if (ok && tid < kChunks) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.k_new + src) + tid);
        st_shared_v4(tbase + (tid >> 3) * C::kBoxBytes + r * 128 + (((tid & 7) ^ (r & 7)) << 4), v);
        reinterpret_cast<uint4 *>(p.K_cache + dst)[tid] = v;
        fence_proxy_async_smem();   // before a later TMA load refills this stage
      } else if (ok && tid >= 32 && tid < 32 + kChunks) {
        reinterpret_cast<uint4 *>(p.V_cache + dst)[tid - 32] =
            __ldg(reinterpret_cast<const uint4 *>(p.v_new + src) + (tid - 32));
      }
      named_bar_sync(kCons);   // the patched row is in place for every consumer warp
    }
    if (ok) {
      // the whole tile holds cached candidates: no per-key range checks
      const bool tile_in = w.key >= cur_lo && w.key + C::kTile <= cur_hi && w.key + C::kTile <= cur_n;
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
        // C fragment: e = 0,1 -> key g4, heads 2t4, 2t4+1; e = 2,3 -> key g4 + 8.  The
        // zero of a product is made +0 by the fused add of +0.
        const long long k0 = w.key + warp * 16 * C::kGroups + 16 * gi + g4;
        float *s0 = srow0 + k0, *s1 = srow1 + k0;
        if (tile_in) {   // every key of the tile is cached and a candidate
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool hv = (e & 1) ? hv1 : hv0;
            if (!hv) continue;
            const float z = fmaf(acc0[e] + acc1[e], p.scale, 0.0f);
            ((e & 1) ? s1 : s0)[(e >> 1) * 8] = z;
            if (cur_hist) {
              const uint32_t bin = digit1_bin_z(z);
              atomicAdd(((e & 1) ? hrow1 : hrow0) + (bin >> 1), 1u << ((bin & 1u) << 4));
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool hv = (e & 1) ? hv1 : hv0;
            const long long key = k0 + (e >> 1) * 8;
            if (!hv || key >= cur_n) continue;
            const float z = fmaf(acc0[e] + acc1[e], p.scale, 0.0f);
            ((e & 1) ? s1 : s0)[(e >> 1) * 8] = z;
            if (cur_hist && key >= cur_lo && key < cur_hi) {
              const uint32_t bin = digit1_bin_z(z);
              atomicAdd(((e & 1) ? hrow1 : hrow0) + (bin >> 1), 1u << ((bin & 1u) << 4));
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + 8 * slot);   // this warp is done with the stage
    ++since_flush;
    if (++slot == stages) {
      slot = 0;
      fpar ^= 1u;
    }
    w.next(p, pg, chunk);
  }
  named_bar_sync(kCons);
  if (cur_bg >= 0 && cur_hist) flush_hist(cur_bg);
  named_bar_sync(kCons);
  publish(BH);
}

// Run length of the tile hand-out.  A long scan (at least kSweepMinTiles tiles a CTA) is dealt
// in about kRounds rounds of one run per CTA, so the CTAs sweep the heads together (each head's
// scores are complete after the rounds that cover it) while a CTA changes head only a few tens
// of times (each change costs it a histogram flush).  A short scan (the 128K-token layer: 55
// tiles a CTA) gives each CTA one contiguous range: there the heads finishing last would have
// their selection after the scan anyway (measured on B200: 51 us contiguous against 57-59 us
// in runs of 8-16 tiles).
constexpr long long kSweepMinTiles = 128;
constexpr long long kRounds = 16;
static int score_chunk(long long total_tiles, int grid) {
  if (total_tiles / grid < kSweepMinTiles) return static_cast<int>((total_tiles + grid - 1) / grid);
  return static_cast<int>(total_tiles / (static_cast<long long>(grid) * kRounds));
}

// Ring depth: the deepest ring (at most kMaxStages) that leaves room on the SM for one
// selection CTA beside the score CTA, so the selection can run on finished heads during the scan.
template <int D, int ROWS>
static int score_stages(int G, int d) {
  using C = ScoreCfg<D, ROWS>;
  constexpr size_t kSmPerSm = 233472;   // 228 KB of shared memory per SM
  constexpr size_t kPerCta = 1024;      // reserved by the system per resident CTA
  const size_t sel = select_smem_bytes(d) + kPerCta;
  int s = C::kMaxStages;
  while (s > 2 && C::smem_bytes(G, s) + kPerCta + sel > kSmPerSm) --s;
  return s;
}

template <int D, int ROWS, class Pg>
static cudaError_t launch_score_t(const ScoreParams &p, const Pg &pg, long long num_pages,
                                  cudaStream_t s, int *grid_out) {
  using C = ScoreCfg<D, ROWS>;
  static bool done[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(score_gqa_kernel<D, ROWS, Pg>),
                                    static_cast<int>(C::smem_bytes(kMaxGroup, C::kMaxStages)), done);
  if (e != cudaSuccess) return e;
  CUtensorMap tm;
  const bool paged = num_pages > 0;
  // dense: [B * Hkv planes][N rows (cap apart)][d]; paged: [pages * Hkv planes][128 rows][d]
  if (!encode_rows_tmap(&tm, p.K, D, paged ? kPageSize : static_cast<uint64_t>(p.N),
                        paged ? static_cast<uint64_t>(num_pages) * p.Hkv
                              : static_cast<uint64_t>(p.B) * p.Hkv,
                        C::kTile, paged ? kPageSize : static_cast<uint64_t>(p.cap)))
    return cudaErrorInvalidValue;
  const int grid = score_grid(p.total_tiles);
  if (grid_out) *grid_out = grid;
  const int stages = score_stages<D, ROWS>(p.G, D);
  const int chunk = score_chunk(p.total_tiles, grid);
  return launch_pdl(score_gqa_kernel<D, ROWS, Pg>, dim3(static_cast<unsigned>(grid)),
                    dim3(C::kThreads), C::smem_bytes(p.G, stages), s, tm, p, pg, stages, chunk);
}

int score_grid(long long total_tiles) {
  long long grid = num_sms();
  if (grid > total_tiles) grid = total_tiles;
  if (grid < 1) grid = 1;
  return static_cast<int>(grid);
}

int score_tile_rows(int d) { return d == 64 ? 256 : 128; }

cudaError_t launch_score(const ScoreParams &p, int d, cudaStream_t s, int *grid) {
  const NoPaging pg{};
  // the tile count follows the tile size of this head dimension
  ScoreParams q = p;
  const int rows = score_tile_rows(d);
  q.tiles_per_head = (p.N + rows - 1) / rows;
  q.total_tiles = q.tiles_per_head * p.B * p.Hkv;
  return d == 128 ? launch_score_t<128, 128>(q, pg, 0, s, grid)
                  : launch_score_t<64, 256>(q, pg, 0, s, grid);
}

cudaError_t launch_score_paged(const ScoreParams &p, const PagedInfo &pg, long long num_pages, int d,
                               cudaStream_t s, int *grid) {
  return d == 128 ? launch_score_t<128, 128>(p, pg, num_pages, s, grid)
                  : launch_score_t<64, 128>(p, pg, num_pages, s, grid);
}

}  // namespace ra
