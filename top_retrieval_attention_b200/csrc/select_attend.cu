// Exact per-query-head top-k selection fused with the sparse attention over the selected set
// (RetrievalAttention slides: "The GPU keeps 640 fixed positions" -- W and Omega disjoint, one
// index set per query head; "Sparse attention renormalizes selected tokens" -- Eq. (2) over
// U = W u Omega; "Two local softmax outputs need global weights" -- Eqs. (3)-(5)).
//
// One thread-block cluster per query head (b, h); the cluster's CTAs split the head's
// candidate positions C = [s1, w0) into contiguous chunks.  During a decode step the kernel is
// launched behind the score kernel and starts on a head as soon as that head's scores are
// complete (a per-KV-head counter), so it runs beside the scan of the remaining heads.
//
// Selection, a radix select over the 64-bit composite x = order_key(z) << 32 | ~position (all
// keys distinct: larger z first, equal z to the lower position):
//   * digit 1 (digit1_bin of order_key: 64 bins per octave where thresholds lie, a 15-bit key
//     prefix each) was histogrammed by the score kernel; every CTA finds the threshold bin b1
//     (the bin of the k-th largest key) from it;
//   * one streaming pass over the CTA's chunk of scores keeps the positions of the keys above
//     b1 ("sure") in shared memory, keeps the composites of the keys in b1 (the "list") in
//     shared memory, past its capacity in the CTA's slice of a per-head list in the workspace,
//     and histograms digit 2 of the list;
//   * each later digit is settled across the cluster: every CTA sums one slice of the CTAs'
//     digit histograms through distributed shared memory, the threshold digit is found from
//     the slice totals, keys above it are written out at offsets from a cluster-wide prefix
//     of per-CTA counts, and the keys at it either are all taken, or (at most 64 of them) are
//     sent to the first CTA for a bitonic finish, or become the next round's domain;
//   * a CTA with more sure keys than its shared array holds (very large k) writes them out from
//     its chunk of the score row, re-read.
// Attention: the CTAs split U (W first, then Omega from idx) into ranges and stage their range's
// positions and scores in shared memory (W's scores from the score row, Omega's from the scores
// the selection wrote beside idx); a warp takes 16 entries at a time at d = 128 (32 at d = 64),
// gathers their V rows 16 bytes per lane with all loads in flight together, keeps an online
// softmax state, the CTA combines its warps, every CTA pushes its partial state (m_S, Z_S,
// N_S) into the first CTA's shared memory, and the first CTA merges them with weights
// e^{m_S - m} into the output.
//
// The same kernel selects from per-row candidate lists (IVF: row_n candidates per row, their
// cache positions in pos_map) and builds its own digit-1 histogram or applies Eq. (2)'s
// threshold when asked; those modes run a separate instantiation (kFull), so the decode step's
// launches carry none of their code.
#include <cooperative_groups.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "merge.cuh"

namespace cg = cooperative_groups;

namespace ra {

constexpr int kSaThreads = 256;
constexpr int kSaWarps = kSaThreads / 32;
constexpr int kSureCap = 4096;    // keys above b1 kept per CTA: positions
constexpr int kListSmem = 1536;   // keys in b1 kept in shared memory per CTA (the rest in the
                                  // CTA's slice of the workspace list)
constexpr int kFinish = 64;       // bitonic finish size (one warp)
constexpr int kStreamVec = 8;     // float4 score loads per thread in flight

// The first CTA's digit histogram doubles as the attention's exchange area: one D-float
// numerator per CTA of the cluster.
static_assert(kMaxCluster * 128 * sizeof(float) <= kHistBins * sizeof(uint32_t), "exchange area");

template <int D>
struct __align__(16) SaSmem {
  uint32_t sure[kSureCap];        // positions of the keys above b1
  unsigned long long list[kListSmem];   // composites of the first keys in b1
  float wacc[kSaWarps * D];       // attention: per-warp numerators
  uint32_t h[kHistBins];          // digit histogram of the current round (slice reduced in place)
  unsigned long long fin[kFinish];  // first CTA: keys of the final bucket
  float wm[kSaWarps], wz[kSaWarps];
  uint32_t x_a[kMaxCluster];      // per-rank exchange slots (written remotely before a barrier)
  uint32_t x_b[kMaxCluster];
  uint32_t x_tot[kMaxCluster];
  float x_m[kMaxCluster], x_s[kMaxCluster];   // per-rank (max, sum e^{z - max}): of a row's
                                              // scores, or of a CTA's attention partial state
  uint32_t warp_tot[2 * kSaWarps];
  uint32_t n_sure, n_list;
  int t_bin;
  uint32_t t_above, t_cnt;
  uint32_t x_ok;                  // the wait verdict, from the first CTA
};

// The index a selected entry e of row blockIdx.y is reported as in idx: its position in the
// score row, or, for a candidate list (pos_map set), the cache position the list maps it to (-1:
// a static-set key).  Read from the parameter block, so it costs the callers no registers.
template <bool kFull>
__device__ __forceinline__ int32_t idx_of(const SaParams &p, uint32_t e) {
  if constexpr (kFull) {
    if (p.pos_map) return __ldcg(p.pos_map + static_cast<long long>(blockIdx.y) * p.ldS + e);
  }
  return static_cast<int32_t>(e);
}

__device__ __forceinline__ unsigned long long composite(uint32_t key, uint32_t pos) {
  return (static_cast<unsigned long long>(key) << 32) | (0xFFFFFFFFu - pos);
}
__device__ __forceinline__ uint32_t composite_pos(unsigned long long x) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(x);
}
__device__ __forceinline__ float composite_z(unsigned long long x) {
  return key_float(static_cast<uint32_t>(x >> 32));
}

// Selected entry o of row blockIdx.y: its index into idx and, when the launch keeps them, its
// score into sel_z.
template <bool kFull>
__device__ __forceinline__ void put_sel(const SaParams &p, int32_t *irow, uint32_t o, uint32_t e,
                                        float z) {
  irow[o] = idx_of<kFull>(p, e);
  if (p.sel_z) p.sel_z[static_cast<long long>(blockIdx.y) * p.k + o] = z;
}

// Block-wide inclusive prefix sums of two counters at once; warp_tot holds 2 * kSaWarps words.
// Returns the inclusive sums; the block totals are left in tot_a / tot_b.
__device__ __forceinline__ uint2 block_scan2(uint32_t a, uint32_t b, uint32_t *warp_tot,
                                             uint32_t &tot_a, uint32_t &tot_b) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t na = __shfl_up_sync(0xffffffffu, a, o);
    const uint32_t nb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += na;
      b += nb;
    }
  }
  if (lane == 31) {
    warp_tot[warp] = a;
    warp_tot[kSaWarps + warp] = b;
  }
  __syncthreads();
  uint32_t pa = 0, pb = 0;
  tot_a = 0;
  tot_b = 0;
#pragma unroll
  for (int w = 0; w < kSaWarps; ++w) {
    const uint32_t ta = warp_tot[w], tb = warp_tot[kSaWarps + w];
    if (w < warp) {
      pa += ta;
      pb += tb;
    }
    tot_a += ta;
    tot_b += tb;
  }
  __syncthreads();   // warp_tot may be reused
  return make_uint2(a + pa, b + pb);
}

// Threshold in a histogram of nb bins (digit value ascending with the bin index): the bin that
// holds the want-th largest key, counting base_above keys as already above every bin here.
// Sets sm.t_bin (-1 if the bins hold fewer than want - base_above keys), sm.t_above (keys above
// the bin, base_above included) and sm.t_cnt.  src is global memory written by an earlier kernel
// (kGlobal, read through L2) or shared memory, possibly another CTA's.  Whole block; the result
// is valid after the call.
template <int D, bool kGlobal>
__device__ __forceinline__ void find_thresh(SaSmem<D> &sm, const uint32_t *src, int nb,
                                            uint32_t want, uint32_t base_above) {
  const int tid = threadIdx.x;
  const int per = (nb + kSaThreads - 1) / kSaThreads;   // <= 8 bins per thread
  uint32_t loc[8];
  uint32_t s = 0;
  // thread t owns bins [nb - per (t + 1), nb - per t): thread 0 the highest
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int bin = nb - per * (tid + 1) + (per - 1 - i);
    loc[i] = (i < per && bin >= 0 && bin < nb) ? (kGlobal ? __ldcg(src + bin) : src[bin]) : 0u;
    s += loc[i];
  }
  if (tid == 0) sm.t_bin = -1;
  uint32_t ta, tb;
  const uint2 incl = block_scan2(s, 0u, sm.warp_tot, ta, tb);
  const uint32_t excl = base_above + incl.x - s;
  if (excl < want && want <= excl + s) {
    uint32_t cum = excl;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < per && cum + loc[i] >= want) {
        sm.t_bin = nb - per * (tid + 1) + (per - 1 - i);
        sm.t_above = cum;
        sm.t_cnt = loc[i];
        break;
      }
      cum += loc[i];
    }
  }
  __syncthreads();
}

// The CTA's threshold-bin keys (composites): the first kListSmem in shared memory, the rest in
// the CTA's slice of the head's list in the workspace (read back through L2).
template <int D>
struct ListSrc {
  const SaSmem<D> *sm;
  const unsigned long long *spill;
  uint32_t n;
  template <class F>
  __device__ __forceinline__ void for_each(F f) const {
    for (uint32_t i = threadIdx.x; i < n; i += kSaThreads)
      f(i < static_cast<uint32_t>(kListSmem) ? sm->list[i] : __ldcg(spill + i));
  }
};

// The CTA's candidates [lo, hi), re-read from the score row (float4 units from the aligned
// chunk start a0).  Iteration order per thread is fixed, so a counting pass and a writing pass
// agree on every thread's running offsets.
struct ChunkSrc {
  const float *srow;
  long long a0, lo, hi;
  template <class F>
  __device__ __forceinline__ void for_each(F f) const {
    for (long long b = a0 + 4LL * threadIdx.x; b < hi; b += 4LL * kSaThreads) {
      if (b + 4 <= lo) continue;
      const float4 v = __ldcg(reinterpret_cast<const float4 *>(srow + b));
      const float zz[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const long long pos = b + e;
        if (pos >= lo && pos < hi) f(composite(order_key(zz[e]), static_cast<uint32_t>(pos)));
      }
    }
  }
};

// Sorts the kFinish keys at f into descending order.  One warp (all 32 lanes).
__device__ __forceinline__ void bitonic_desc64(unsigned long long *f) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int size = 2; size <= kFinish; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int i = 2 * stride * (lane / stride) + (lane % stride);
      const int j = i + stride;
      const unsigned long long a = f[i], b = f[j];
      const bool desc = (i & size) == 0;
      if (desc ? (a < b) : (a > b)) {
        f[i] = b;
        f[j] = a;
      }
      __syncwarp();
    }
  }
}

// Bitonic finish in the first CTA: the n <= kFinish keys in sm.fin, the `want` largest written
// to irow[o0 ..].  One warp.
template <int D, bool kFull>
__device__ __forceinline__ void bitonic_finish(const SaParams &p, SaSmem<D> &sm, uint32_t n,
                                               uint32_t want, int32_t *irow, uint32_t o0) {
  const int tid = threadIdx.x, lane = tid & 31;
  if (n <= 32) {   // one key per lane: a key is taken when fewer than `want` keys exceed it
    if (tid < 32) {
      const unsigned long long x = static_cast<uint32_t>(lane) < n ? sm.fin[lane] : 0ull;
      uint32_t above = 0;
      for (int j = 0; j < 32; ++j) above += __shfl_sync(0xffffffffu, x, j) > x ? 1u : 0u;
      if (static_cast<uint32_t>(lane) < n && above < want)
        put_sel<kFull>(p, irow, o0 + above, composite_pos(x), composite_z(x));
    }
    return;
  }
  for (uint32_t i = n + tid; i < kFinish; i += kSaThreads) sm.fin[i] = 0ull;   // below every key
  __syncthreads();
  if (tid < 32) {
    bitonic_desc64(sm.fin);
    for (uint32_t i = lane; i < want; i += 32)
      put_sel<kFull>(p, irow, o0 + i, composite_pos(sm.fin[i]), composite_z(sm.fin[i]));
  }
}

// The cluster-wide threshold of one digit: every CTA's sm.h holds its histogram of nb bins
// (nb >= ncl) and the cluster has synchronised since.  Each CTA sums its slice of the CTAs'
// histograms in place (through distributed shared memory) and sends the slice total to every
// CTA; after a barrier every CTA finds the slice holding the want-th largest key (highest
// slices first) and the bin inside it.  Returns the slice's first bin; sm.t_bin (relative to
// it, -1 if the counts are inconsistent), sm.t_above (keys above that bin, cluster-wide) and
// sm.t_cnt are set.  Other CTAs read this CTA's sm.h until the caller's next cluster barrier.
template <int D>
__device__ int cluster_thresh(SaSmem<D> &sm, cg::cluster_group &cl, int rank, int ncl, int nb,
                              uint32_t want) {
  const int tid = threadIdx.x;
  const int sz = nb / ncl;
  const int s0 = rank * sz;
  uint32_t part = 0;
  for (int bin = s0 + tid; bin < s0 + sz; bin += kSaThreads) {
    uint32_t s = 0;
    for (int c = 0; c < ncl; ++c) s += cl.map_shared_rank(sm.h, c)[bin];
    sm.h[bin] = s;
    part += s;
  }
  uint32_t tot, unused;
  block_scan2(part, 0u, sm.warp_tot, tot, unused);
  if (tid < ncl) cl.map_shared_rank(sm.x_tot, tid)[rank] = tot;
  cl.sync();   // slices summed, slice totals exchanged
  uint32_t above = 0;
  int rs = ncl - 1;
  for (; rs > 0; --rs) {
    if (above + sm.x_tot[rs] >= want) break;
    above += sm.x_tot[rs];
  }
  find_thresh<D, false>(sm, cl.map_shared_rank(sm.h, rs) + rs * sz, sz, want, above);
  return rs * sz;
}

// Rounds below digit 1 over the keys of bin b1 (src): digit 2 first, whose histogram is already
// complete in every CTA's sm.h with the cluster synchronised since, then further 11-bit digits
// of the composite.  `want` keys are still to be chosen; they go to irow[base ..).  Every CTA of
// the cluster runs the same rounds (all decisions come from cluster-wide totals).
template <int D, bool kFull, class Src>
__device__ void select_rounds(const SaParams &p, SaSmem<D> &sm, cg::cluster_group &cl, int rank,
                              int ncl, const Src &src, uint32_t b1, uint32_t want, uint32_t base,
                              int32_t *irow, uint32_t k_eff) {
  const int tid = threadIdx.x;
  // the composite bits the keys of b1 share (none for a catch-all bin) and the bits below them
  const int pbits = digit1_prefix_bits(b1);
  unsigned long long prefix = pbits ? digit1_floor(b1) >> (32 - pbits) : 0ull;
  int sh = 64 - pbits;
  const auto top = [&sh](unsigned long long x) { return sh >= 64 ? 0ull : x >> sh; };
  bool have_hist = true;
#pragma unroll 1
  for (int round = 0; round < 6 && sh > 0; ++round) {
    const int w = sh < kHistBits ? sh : kHistBits;
    const int nsh = sh - w;
    const uint32_t mask = (1u << w) - 1u;
    const int nb = 1 << w;
    if (!have_hist) {
      src.for_each([&](unsigned long long x) {
        if (top(x) == prefix) atomicAdd(&sm.h[static_cast<uint32_t>(x >> nsh) & mask], 1u);
      });
      __syncthreads();
      cl.sync();   // every CTA's digit histogram is complete
    }
    have_hist = false;
    const int base_bin = cluster_thresh(sm, cl, rank, ncl, nb, want);
    if (sm.t_bin < 0) {   // inconsistent counts (never for a score row and its own histogram)
      if (tid == 0 && rank == 0) atomicOr(p.err, kErrSelect);
      return;
    }
    const uint32_t t = static_cast<uint32_t>(base_bin + sm.t_bin);
    const uint32_t up = sm.t_above;   // keys of the prefix above digit t, cluster-wide
    const uint32_t eq = sm.t_cnt;     // keys of the prefix at digit t
    const uint32_t want2 = want - up; // 1 <= want2 <= eq
    const bool take_eq = want2 == eq;
    const bool fin = !take_eq && eq <= static_cast<uint32_t>(kFinish);
    uint32_t cu = 0, ce = 0;
    src.for_each([&](unsigned long long x) {
      if (top(x) == prefix) {
        const uint32_t dg = static_cast<uint32_t>(x >> nsh) & mask;
        cu += dg > t ? 1u : 0u;
        ce += dg == t ? 1u : 0u;
      }
    });
    uint32_t tu, te;
    const uint2 inc = block_scan2(cu, ce, sm.warp_tot, tu, te);
    if (tid < ncl) {
      cl.map_shared_rank(sm.x_a, tid)[rank] = tu;
      cl.map_shared_rank(sm.x_b, tid)[rank] = te;
    }
    cl.sync();   // per-CTA counts exchanged
    uint32_t off_u = 0, off_e = 0;
    for (int c = 0; c < rank; ++c) {
      off_u += sm.x_a[c];
      off_e += sm.x_b[c];
    }
    uint32_t ou = base + off_u + inc.x - cu;
    uint32_t oe = off_e + inc.y - ce;
    unsigned long long *fin0 = cl.map_shared_rank(sm.fin, 0);
    src.for_each([&](unsigned long long x) {
      if (top(x) != prefix) return;
      const uint32_t dg = static_cast<uint32_t>(x >> nsh) & mask;
      if (dg > t) {
        if (ou < k_eff) put_sel<kFull>(p, irow, ou, composite_pos(x), composite_z(x));
        ++ou;
      } else if (dg == t) {
        if (take_eq) {
          if (base + up + oe < k_eff)
            put_sel<kFull>(p, irow, base + up + oe, composite_pos(x), composite_z(x));
        } else if (fin && oe < static_cast<uint32_t>(kFinish)) {
          fin0[oe] = x;
        }
        ++oe;
      }
    });
    if (take_eq) return;
    if (fin) {
      cl.sync();   // the final bucket is complete in the first CTA
      if (rank == 0)
        bitonic_finish<D, kFull>(p, sm, eq, min(want2, k_eff - min(k_eff, base + up)), irow,
                                 base + up);
      return;
    }
    // next digit: every remote read of sm.h came before the last barrier
    for (int i = tid; i < kHistBins; i += kSaThreads) sm.h[i] = 0u;
    __syncthreads();
    prefix = (prefix << w) | t;
    sh = nsh;
    want = want2;
    base += up;
  }
  if (tid == 0 && rank == 0) atomicOr(p.err, kErrSelect);   // unreachable for distinct keys
}

// The score at bit j of a thread's hit masks: element j % 4 of its (j / 4)-th loaded vector,
// chosen from registers by a three-level select on the vector index (no dynamic indexing).
__device__ __forceinline__ float pick_score(const float4 (&v)[kStreamVec], int j) {
  static_assert(kStreamVec == 8, "three select levels");
  const int u = j >> 2, e = j & 3;
  const float4 a0 = (u & 1) ? v[1] : v[0], a1 = (u & 1) ? v[3] : v[2];
  const float4 a2 = (u & 1) ? v[5] : v[4], a3 = (u & 1) ? v[7] : v[6];
  const float4 b0 = (u & 2) ? a1 : a0, b1 = (u & 2) ? a3 : a2;
  const float4 c = (u & 4) ? b1 : b0;
  return e == 0 ? c.x : e == 1 ? c.y : e == 2 ? c.z : c.w;
}

// Inclusive warp prefix sums of two per-lane counts; the warp totals come back in lane 31.
__device__ __forceinline__ void warp_scan2(uint32_t &a, uint32_t &b) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t na = __shfl_up_sync(0xffffffffu, a, o);
    const uint32_t nb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += na;
      b += nb;
    }
  }
}

// One pass over the CTA's candidates [lo, hi) of the score row.  Keys above the digit-1
// threshold bin b1 (z >= zhi, the bottom of bin b1 + 1) go to sm.sure as positions, their
// scores to the top of `spill` (entry i at spill[hi - lo - 1 - i]); keys in b1
// (zlo <= z < zhi) go to sm.list as composites, past its capacity to `spill` (room for hi - lo
// entries: the two never meet, a candidate being one or the other), with their digit-2
// histogram in sm.h; the counters keep counting past the capacities.  Hits are a small
// fraction of the keys (about k / |C| plus the bin's share): each thread makes two bit masks
// with two compares per score, the warp reserves its slots with one shared atomic per list and
// iteration (offsets from a warp prefix scan of the per-lane counts), and every lane then walks
// its own set bits (the warp loops as often as its busiest lane has hits), the score of a key
// in b1 picked from its registers.
template <int D>
__device__ __forceinline__ void stream_chunk(SaSmem<D> &sm, const float *srow,
                                             unsigned long long *spill, long long a0, long long lo,
                                             long long hi, uint32_t b1) {
  constexpr long long kStep = 4LL * kSaThreads * kStreamVec;
  static_assert(4 * kStreamVec <= 32, "one mask bit per score");
  // b1 is [zlo, zhi) in score order; digit 2 is the 11 key bits below those its keys share
  const float zlo = b1 == 0u ? -INFINITY : key_float(static_cast<uint32_t>(digit1_floor(b1)));
  const float zhi = b1 + 1 < static_cast<uint32_t>(kHistBins)
                        ? key_float(static_cast<uint32_t>(digit1_floor(b1 + 1))) : INFINITY;
  const int d2sh = 32 - digit1_prefix_bits(b1) - kHistBits;   // digit 2 within the order key
  const int lane = threadIdx.x & 31;
  for (long long it = a0; it < hi; it += kStep) {
    const long long b0 = it + 4LL * threadIdx.x;
    float4 v[kStreamVec];
#pragma unroll
    for (int u = 0; u < kStreamVec; ++u) {
      const long long b = b0 + 4LL * kSaThreads * u;
      v[u] = (b < hi && b + 4 > lo) ? __ldcg(reinterpret_cast<const float4 *>(srow + b))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const bool interior = it >= lo && it + kStep <= hi;
    uint32_t ms = 0, me = 0;   // above b1, in b1
#pragma unroll
    for (int u = 0; u < kStreamVec; ++u) {
      const float zz[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t s4 = 0, e4 = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s4 |= (zz[e] >= zhi ? 1u : 0u) << e;
        e4 |= (zz[e] >= zlo && zz[e] < zhi ? 1u : 0u) << e;
      }
      if (!interior) {
        const long long b = b0 + 4LL * kSaThreads * u;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (b + e < lo || b + e >= hi) {
            s4 &= ~(1u << e);
            e4 &= ~(1u << e);
          }
      }
      ms |= s4 << (4 * u);
      me |= e4 << (4 * u);
    }
    if (!__any_sync(0xffffffffu, (ms | me) != 0u)) continue;
    const uint32_t ns = __popc(ms), ne = __popc(me);
    uint32_t ps = ns, pe = ne;
    warp_scan2(ps, pe);
    uint32_t bs = 0, be = 0;
    if (lane == 31) {
      if (ps) bs = atomicAdd(&sm.n_sure, ps);
      if (pe) be = atomicAdd(&sm.n_list, pe);
    }
    uint32_t os = __shfl_sync(0xffffffffu, bs, 31) + ps - ns;
    uint32_t oe = __shfl_sync(0xffffffffu, be, 31) + pe - ne;
    while (ms) {   // keys above b1: positions, their scores at the slice's top
      const int j = __ffs(ms) - 1;
      ms &= ms - 1;
      if (os < static_cast<uint32_t>(kSureCap)) {
        sm.sure[os] = static_cast<uint32_t>(b0 + 4LL * kSaThreads * (j >> 2) + (j & 3));
        spill[hi - lo - 1 - os] = __float_as_uint(pick_score(v, j));
      }
      ++os;
    }
    while (me) {   // keys in b1: composites and the digit-2 histogram
      const int j = __ffs(me) - 1;
      me &= me - 1;
      const uint32_t pos = static_cast<uint32_t>(b0 + 4LL * kSaThreads * (j >> 2) + (j & 3));
      const uint32_t key = order_key(pick_score(v, j));
      const unsigned long long x = composite(key, pos);
      if (oe < static_cast<uint32_t>(kListSmem)) sm.list[oe] = x;
      else spill[oe] = x;
      atomicAdd(&sm.h[(key >> d2sh) & (kHistBins - 1)], 1u);
      ++oe;
    }
  }
}

// The per-row geometry of the step: N, W = [0, s1) u [w0, N), C = [s1, w0), the budget k_eff
// and the cluster's chunking of C.  Dense caches share one geometry (from the parameters);
// paged caches derive it from the row's sequence length.
struct RowGeo {
  long long N, s1, w0, nW, nC, k_eff, cbase, cper;
};
template <bool kFull>
__device__ __forceinline__ RowGeo row_geo(const SaParams &p, const NoPaging &, int row, int ncl) {
  if (kFull && p.row_n) {   // a candidate list of its own length, no static set
    RowGeo g;
    g.N = p.row_n[row];
    g.s1 = 0;
    g.w0 = g.N;
    g.nW = 0;
    g.nC = g.N;
    g.k_eff = min(static_cast<long long>(p.k), g.N);
    g.cbase = 0;
    g.cper = ((max(g.N, 1LL) + ncl - 1) / ncl + 3) / 4 * 4;
    return g;
  }
  return RowGeo{p.N, p.s1, p.w0, p.nW, p.nC, p.k_eff, p.cbase, p.cper};
}
template <bool kFull>
__device__ __forceinline__ RowGeo row_geo(const SaParams &p, const PagedInfo &pg, int row, int ncl) {
  RowGeo g;
  g.N = pg.seq_len[row / p.Hq];
  g.s1 = min(static_cast<long long>(pg.n_sink), g.N);
  g.w0 = max(g.s1, g.N - pg.n_window);
  g.nW = g.s1 + (g.N - g.w0);
  g.nC = g.w0 - g.s1;
  g.k_eff = min(static_cast<long long>(pg.k), g.nC);
  g.cbase = g.s1 & ~3LL;
  const long long span = max(g.w0 - g.cbase, 1LL);
  g.cper = ((span + ncl - 1) / ncl + 3) / 4 * 4;
  return g;
}
// The geometry the attention uses: the row's own, except that a candidate list's Omega (the
// min(k, candidates) entries of idx) is attended together with the cache's static set.
template <bool kFull, class Pg>
__device__ __forceinline__ RowGeo attend_geo(const SaParams &p, const Pg &pg, int row, int ncl) {
  RowGeo g = row_geo<kFull>(p, pg, row, ncl);
  if (kFull && p.row_n) g = RowGeo{p.N, p.s1, p.w0, p.nW, p.nC, g.k_eff, p.cbase, p.cper};
  return g;
}
// Where token `pos` of sequence b, KV head gk, sits in V: v_base(...) + v_index(...) * d.
// Dense caches: the (b, gk) plane and the position; paged caches: the pool and the pool row
// of the token's page.
template <int D>
__device__ __forceinline__ const __nv_bfloat16 *v_base(const SaParams &p, const NoPaging &, int b,
                                                       int gk) {
  return p.V + (static_cast<long long>(b) * p.Hkv + gk) * p.cap * D;
}
template <int D>
__device__ __forceinline__ const __nv_bfloat16 *v_base(const SaParams &p, const PagedInfo &, int,
                                                       int) {
  return p.V;
}
__device__ __forceinline__ int v_index(const SaParams &, const NoPaging &, int, int, int pos) {
  return pos;
}
__device__ __forceinline__ int v_index(const SaParams &p, const PagedInfo &pg, int b, int gk, int pos) {
  const int page = __ldg(pg.block_table + static_cast<long long>(b) * pg.max_pages + pos / kPageSize);
  return (page * p.Hkv + gk) * kPageSize + pos % kPageSize;
}

// ln sum_{j < N} e^{z_j} of one score row (the log of Eq. (1)'s softmax normaliser), cluster-
// wide: each CTA folds its candidates [lo, hi) and its share of W into a running (max, sum),
// the CTAs exchange theirs through distributed shared memory and all merge them.
template <int D>
__device__ float row_logsumexp(const RowGeo &gm, SaSmem<D> &sm, cg::cluster_group &cl, int rank,
                               int ncl, const float *srow, long long lo, long long hi) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float m = -INFINITY, s = 0.f;
  auto add = [&](float z) {
    if (z > m) {
      s = s * expf(m - z) + 1.f;   // expf(-inf) = 0 for the first element
      m = z;
    } else {
      s += expf(z - m);
    }
  };
  for (long long i = lo + tid; i < hi; i += kSaThreads) add(__ldcg(srow + i));
  const long long wper = (gm.nW + ncl - 1) / ncl;
  const long long w_hi = min(gm.nW, (rank + 1) * wper);
  for (long long e = rank * wper + tid; e < w_hi; e += kSaThreads)
    add(__ldcg(srow + (e < gm.s1 ? e : gm.w0 + (e - gm.s1))));
  // merge (m, s) over the warp, then over the CTA's warps
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o), so = __shfl_xor_sync(0xffffffffu, s, o);
    const float mn = fmaxf(m, mo);
    s = (m == -INFINITY ? 0.f : s * expf(m - mn)) + (mo == -INFINITY ? 0.f : so * expf(mo - mn));
    m = mn;
  }
  if (lane == 0) {
    sm.wm[warp] = m;
    sm.wz[warp] = s;
  }
  __syncthreads();
  if (tid < ncl) {
    float M = -INFINITY, Z = 0.f;
    for (int w = 0; w < kSaWarps; ++w) M = fmaxf(M, sm.wm[w]);
    for (int w = 0; w < kSaWarps; ++w)
      if (sm.wm[w] != -INFINITY) Z += sm.wz[w] * expf(sm.wm[w] - M);
    cl.map_shared_rank(sm.x_m, tid)[rank] = M;
    cl.map_shared_rank(sm.x_s, tid)[rank] = Z;
  }
  cl.sync();   // every CTA's (max, sum) is in every CTA
  float M = -INFINITY, Z = 0.f;
  for (int c = 0; c < ncl; ++c) M = fmaxf(M, sm.x_m[c]);
  for (int c = 0; c < ncl; ++c)
    if (sm.x_m[c] != -INFINITY) Z += sm.x_s[c] * expf(sm.x_m[c] - M);
  return M + logf(Z);
}

// Omega of one query head into irow (cluster-wide; every CTA takes the same branches).
template <int D, bool kFull>
__device__ void select_phase(const SaParams &p, const RowGeo &gm, SaSmem<D> &sm,
                             cg::cluster_group &cl, int rank, int ncl, int row) {
  const int tid = threadIdx.x;
  int32_t *irow = p.idx + static_cast<long long>(row) * p.k;
  if (rank == 0)
    for (long long i = gm.k_eff + tid; i < p.k; i += kSaThreads) irow[i] = -1;
  if (gm.k_eff == 0) return;
  const long long a0 = gm.cbase + static_cast<long long>(rank) * gm.cper;
  const long long lo = max(a0, gm.s1), hi = min(a0 + gm.cper, gm.w0);
  const float *srow = p.S + static_cast<long long>(row) * p.ldS;
  uint32_t *h1 = p.hist + static_cast<long long>(row) * kHistBins;
  const ChunkSrc chunk{srow, a0, lo, hi};
  long long k_sel = gm.k_eff;   // keys to select (the budget; fewer under a threshold)
  for (int i = tid; i < kHistBins; i += kSaThreads) sm.h[i] = 0u;
  if (tid == 0) {
    sm.n_sure = 0u;
    sm.n_list = 0u;
  }
  const bool build = kFull && (p.mode & (kSaBuildHist | kSaEps)) != 0;
  int b1i = -1;
  if (kFull && (p.mode & kSaEps)) {
    // Eq. (2)'s threshold: a_i > eps  <=>  z_i > T = ln(eps) + ln sum_j e^{z_j} (all N)
    const float T = p.log_eps + row_logsumexp(gm, sm, cl, rank, ncl, srow, lo, hi);
    // this CTA's digit-1 histogram of its candidates and its count of z > T
    uint32_t cnt = 0;
    chunk.for_each([&](unsigned long long x) {
      atomicAdd(&sm.h[digit1_bin(static_cast<uint32_t>(x >> 32))], 1u);
      cnt += key_float(static_cast<uint32_t>(x >> 32)) > T ? 1u : 0u;
    });
    uint32_t tot, unused;
    block_scan2(cnt, 0u, sm.warp_tot, tot, unused);
    if (tid < ncl) cl.map_shared_rank(sm.x_b, tid)[rank] = tot;
    __syncthreads();
    cl.sync();   // histograms and counts complete
    long long above_t = 0;
    for (int c = 0; c < ncl; ++c) above_t += sm.x_b[c];
    k_sel = min(k_sel, above_t);
    if (rank == 0)
      for (long long i = k_sel + tid; i < gm.k_eff; i += kSaThreads) irow[i] = -1;
    if (k_sel == 0) return;
    if (k_sel < gm.nC) {
      b1i = cluster_thresh(sm, cl, rank, ncl, kHistBins, static_cast<uint32_t>(k_sel));
      b1i = sm.t_bin < 0 ? -1 : b1i + sm.t_bin;
    }
    cl.sync();   // every CTA has read the slices it needed: the histograms can be cleared
    for (int i = tid; i < kHistBins; i += kSaThreads) sm.h[i] = 0u;
    __syncthreads();
  }
  if (k_sel >= gm.nC) {   // every candidate is selected
    for (long long i = lo + tid; i < hi; i += kSaThreads)
      put_sel<kFull>(p, irow, static_cast<uint32_t>(i - gm.s1), static_cast<uint32_t>(i),
                     p.sel_z ? __ldcg(srow + i) : 0.f);
    return;
  }
  const uint32_t k_eff = static_cast<uint32_t>(k_sel);
  if (kFull && (p.mode & kSaEps)) {
    // b1 found above
  } else if (build) {
    // digit 1 from the scores themselves: this CTA's histogram, then the cluster's threshold
    __syncthreads();
    chunk.for_each([&](unsigned long long x) {
      atomicAdd(&sm.h[digit1_bin(static_cast<uint32_t>(x >> 32))], 1u);
    });
    __syncthreads();
    cl.sync();   // every CTA's digit-1 histogram is complete
    b1i = cluster_thresh(sm, cl, rank, ncl, kHistBins, k_eff);
    b1i = sm.t_bin < 0 ? -1 : b1i + sm.t_bin;
    cl.sync();   // every CTA has read the slices it needed: the histograms can be cleared
    for (int i = tid; i < kHistBins; i += kSaThreads) sm.h[i] = 0u;
    __syncthreads();
  } else {
    // digit 1: the threshold bin of the score kernel's candidate histogram
    find_thresh<D, true>(sm, h1, kHistBins, k_eff, 0u);
    b1i = sm.t_bin;
  }
  const uint32_t above1 = sm.t_above;
  const uint32_t b1 = b1i < 0 ? 0u : static_cast<uint32_t>(b1i);
  unsigned long long *spill = p.list + static_cast<long long>(row) * p.ldL + (lo - gm.s1);
  if (b1i >= 0) stream_chunk<D>(sm, srow, spill, a0, lo, hi, b1);
  __syncthreads();
  if (tid < ncl) cl.map_shared_rank(sm.x_a, tid)[rank] = sm.n_sure;
  cl.sync();   // lists, counts and digit-2 histograms complete; every CTA has read h1
  if (b1i < 0) {   // the histogram does not count k_eff candidates: not this row's scores
    if (tid == 0 && rank == 0) atomicOr(p.err, kErrSelect);
    return;
  }
  if (rank == 0 && !build)
    for (int i = tid; i < kHistBins; i += kSaThreads) h1[i] = 0u;   // left zero for the next call
  uint32_t off = 0;
  for (int c = 0; c < rank; ++c) off += sm.x_a[c];
  // the keys above b1 take idx slots [0, above1), CTA by CTA
  if (sm.n_sure <= static_cast<uint32_t>(kSureCap)) {
    // their scores sit at the top of the CTA's spill slice (stream_chunk)
    const unsigned long long *ztop = spill + (hi - lo - 1);
    for (uint32_t i = tid; i < sm.n_sure; i += kSaThreads)
      if (off + i < k_eff)
        put_sel<kFull>(p, irow, off + i, sm.sure[i], __uint_as_float(static_cast<uint32_t>(__ldcg(ztop - i))));
  } else {   // more sure keys than sm.sure holds: from the chunk again
    uint32_t cu = 0;
    chunk.for_each([&](unsigned long long x) {
      cu += digit1_bin(static_cast<uint32_t>(x >> 32)) > b1 ? 1u : 0u;
    });
    uint32_t tu, unused;
    const uint2 inc = block_scan2(cu, 0u, sm.warp_tot, tu, unused);
    uint32_t o = off + inc.x - cu;
    chunk.for_each([&](unsigned long long x) {
      if (digit1_bin(static_cast<uint32_t>(x >> 32)) > b1) {
        if (o < k_eff) put_sel<kFull>(p, irow, o, composite_pos(x), composite_z(x));
        ++o;
      }
    });
  }
  // the keys of b1, from the CTAs' lists
  select_rounds<D, kFull>(p, sm, cl, rank, ncl, ListSrc<D>{&sm, spill, sm.n_list}, b1, k_eff - above1,
                          above1, irow, k_eff);
}

constexpr int kStage = kSureCap / 2;   // entries staged at a time (the sure array is free here)

// The attention gathers V rows with 16-byte loads: a row of D bf16 is D / 8 lanes, so one load
// instruction of the warp fetches 256 / D rows (2 at d = 128, 4 at d = 64), and a warp takes
// kLoads instructions' worth of rows at a time (16 at d = 128, 32 at d = 64).  Lane l keeps the
// channels [8 (l mod D/8), + 8) of the rows of its lane group.
template <int D>
struct AttnCfg {
  static constexpr int kLanesPerRow = D / 8;
  static constexpr int kRowsPerLoad = 32 / kLanesPerRow;
  static constexpr int kLoads = 8;
  static constexpr int kRows = kLoads * kRowsPerLoad;
  static_assert(kRows <= 32, "one entry per lane");
};

// One warp's online-softmax update over up to AttnCfg<D>::kRows entries: lane j < kRows holds
// entry j's V row index vi (-1: no entry) and score z.  All the rows' loads are issued together,
// then folded into the warp's state (m, zs) and the lane's eight channel numerators acc.
template <int D>
__device__ __forceinline__ void attend_rows(const __nv_bfloat16 *Vb, int vi, float z, float &m,
                                            float &zs, float (&acc)[8]) {
  using A = AttnCfg<D>;
  const int lane = threadIdx.x & 31;
  const int grp = lane / A::kLanesPerRow;
  const int c0 = (lane % A::kLanesPerRow) * 8;
  if (vi < 0) z = -INFINITY;
  uint4 wv[A::kLoads];
#pragma unroll
  for (int i = 0; i < A::kLoads; ++i) {
    const int pj = __shfl_sync(0xffffffffu, vi, i * A::kRowsPerLoad + grp);
    wv[i] = pj >= 0 ? __ldcg(reinterpret_cast<const uint4 *>(Vb + static_cast<long long>(pj) * D + c0))
                    : make_uint4(0u, 0u, 0u, 0u);
  }
  float mg = lane < A::kRows ? z : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, o));
  if (mg == -INFINITY) return;   // warp-uniform: no entry in this group
  const float mn = fmaxf(m, mg);
  const float sc = expf(m - mn);   // 0 while m is -inf
  const float pe = (lane >= A::kRows || z == -INFINITY) ? 0.f : expf(z - mn);
  float ps = pe;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
  zs = zs * sc + ps;
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] *= sc;
#pragma unroll
  for (int i = 0; i < A::kLoads; ++i) {
    const float pj = __shfl_sync(0xffffffffu, pe, i * A::kRowsPerLoad + grp);
    const uint32_t w[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      acc[2 * c] += pj * bf16_lo(w[c]);
      acc[2 * c + 1] += pj * bf16_hi(w[c]);
    }
  }
  m = mn;
}

// The CTA's warps' states -> one partial state (m_S, Z_S, N_S), pushed into the first CTA's
// exchange slots (its digit histogram, free during the attention); after the cluster barrier the
// first CTA merges the cluster's states into the output, or, with several clusters per head
// (grid z), into this cluster's state for the head's last cluster to merge (Eqs. (3)-(5)).
template <int D>
__device__ void combine_and_merge(const SaParams &p, SaSmem<D> &sm, cg::cluster_group &cl,
                                  int rank, int ncl, int row, float m, float zs, float (&acc)[8]) {
  using A = AttnCfg<D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (lane == 0) {
    sm.wm[warp] = m;
    sm.wz[warp] = zs;
  }
  // the lane groups' numerators of the same channels add up
#pragma unroll
  for (int o = A::kLanesPerRow; o < 32; o <<= 1)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], o);
  if (lane < A::kLanesPerRow)
#pragma unroll
    for (int c = 0; c < 8; ++c) sm.wacc[warp * D + lane * 8 + c] = acc[c];
  __syncthreads();
  float M = sm.wm[0];
#pragma unroll
  for (int i = 1; i < kSaWarps; ++i) M = fmaxf(M, sm.wm[i]);
  float ew[kSaWarps];
#pragma unroll
  for (int i = 0; i < kSaWarps; ++i) ew[i] = sm.wm[i] == -INFINITY ? 0.f : expf(sm.wm[i] - M);
  float *xacc0 = reinterpret_cast<float *>(cl.map_shared_rank(sm.h, 0));
  for (int c = tid; c < D; c += kSaThreads) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kSaWarps; ++i) s += ew[i] * sm.wacc[i * D + c];
    xacc0[rank * D + c] = s;
  }
  if (tid == 0) {
    float zt = 0.f;
#pragma unroll
    for (int i = 0; i < kSaWarps; ++i) zt += ew[i] * sm.wz[i];
    cl.map_shared_rank(sm.x_m, 0)[rank] = M;
    cl.map_shared_rank(sm.x_s, 0)[rank] = zt;
  }
  cl.sync();   // every CTA's partial state is in the first CTA
  if (rank == 0) {
    const float *xacc = reinterpret_cast<const float *>(sm.h);
    float Mx = -INFINITY;
    for (int c = 0; c < ncl; ++c) Mx = fmaxf(Mx, sm.x_m[c]);
    float den = 0.f;
    for (int c = 0; c < ncl; ++c)
      if (sm.x_m[c] != -INFINITY) den += expf(sm.x_m[c] - Mx) * sm.x_s[c];
    // one cluster: the output; several: this cluster's state for the last one to merge
    constexpr int PS = D + kPartPad;
    float *prow = p.part + static_cast<long long>(row) * kMaxAttnSplit * PS;
    float *mine = prow + static_cast<long long>(blockIdx.z) * PS;
    for (int ch = tid; ch < D; ch += kSaThreads) {
      float num = 0.f;
      for (int c = 0; c < ncl; ++c)
        if (sm.x_m[c] != -INFINITY) num += expf(sm.x_m[c] - Mx) * xacc[c * D + ch];
      if (p.nsplit == 1) p.out[static_cast<long long>(row) * D + ch] = num / den;
      else mine[kPartPad + ch] = num;
    }
    if (p.nsplit > 1) {
      if (tid == 0) {
        mine[0] = Mx;
        mine[1] = den;
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(p.meta + static_cast<long long>(row) * kMetaWords + kDone, 1u);
        sm.t_bin = prev == static_cast<uint32_t>(p.nsplit - 1) ? 1 : 0;
        if (sm.t_bin) __threadfence();
      }
      __syncthreads();
      if (sm.t_bin) {   // the head's last cluster: merge the nsplit states
        merge_states<D, kSaThreads>(prow, p.nsplit, p.out + static_cast<long long>(row) * D,
                                    reinterpret_cast<float *>(sm.warp_tot),
                                    reinterpret_cast<float *>(sm.sure));
        if (tid == 0) p.meta[static_cast<long long>(row) * kMetaWords + kDone] = 0u;
      }
    }
  }
  // no CTA reads another's shared memory after the exchange barrier: all may leave
}

// Softmax attention of one query head over U = W u Omega (Omega read from idx), split across
// the nsplit clusters of the head (grid z) and the CTAs of each.  Each CTA stages its entries'
// positions and scores in shared memory (in blocks of kStage), then its warps gather V rows
// (attend_rows) and keep online-softmax states.
template <int D, bool kFull, class Pg>
__device__ void attend_phase(const SaParams &p, const RowGeo &gm, const Pg &pg, SaSmem<D> &sm,
                             cg::cluster_group &cl, int rank, int ncl, int row) {
  constexpr int kPer = kStage / kSaThreads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long nU = gm.nW + gm.k_eff;
  const long long parts = static_cast<long long>(ncl) * p.nsplit;
  const long long per = (nU + parts - 1) / parts;
  const long long e_lo = (static_cast<long long>(blockIdx.z) * ncl + rank) * per;
  const long long e_hi = min(nU, e_lo + per);
  const int b = row / p.Hq, h = row - b * p.Hq;
  const __nv_bfloat16 *Vb = v_base<D>(p, pg, b, h / p.G);
  const float *srow = ((kFull && p.S_att) ? p.S_att : p.S) + static_cast<long long>(row) * p.ldS;
  const int32_t *irow = p.idx + static_cast<long long>(row) * p.k;
  const float *zrow = p.sel_z ? p.sel_z + static_cast<long long>(row) * p.k : nullptr;
  int *spos = reinterpret_cast<int *>(sm.sure);   // staged: the entry's V row (-1: none)
  float *sz = reinterpret_cast<float *>(sm.sure + kStage);
  constexpr int kRows = AttnCfg<D>::kRows;
  float m = -INFINITY, zs = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  for (long long blk = e_lo; blk < e_hi; blk += kStage) {
    const int nb = static_cast<int>(min(static_cast<long long>(kStage), e_hi - blk));
    // positions (W computed, Omega from idx), then their scores: two rounds of loads in flight
    // positions (W computed, Omega from idx) and, for Omega, the scores the selection kept
    // beside idx, loaded together; the other scores from the score row
    int pp[kPer];
    float zk[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = tid + j * kSaThreads;
      const long long e = blk + i;
      long long pos = -1;
      zk[j] = NAN;
      if (i < nb) {
        if (e < gm.nW) {
          pos = e < gm.s1 ? e : gm.w0 + (e - gm.s1);
        } else {
          pos = __ldcg(irow + (e - gm.nW));
          if (zrow) zk[j] = __ldcg(zrow + (e - gm.nW));
        }
      }
      pp[j] = (pos >= 0 && pos < gm.N) ? static_cast<int>(pos) : -1;   // always, for a complete idx
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = tid + j * kSaThreads;
      const float z = pp[j] < 0 ? -INFINITY : (zk[j] == zk[j] ? zk[j] : __ldcg(srow + pp[j]));
      if (i < nb) {
        spos[i] = pp[j] >= 0 ? v_index(p, pg, b, h / p.G, pp[j]) : -1;
        sz[i] = z;
      }
    }
    __syncthreads();
    for (int g = warp * kRows; g < nb; g += kRows * kSaWarps) {
      const bool mine = lane < kRows && g + lane < nb;
      attend_rows<D>(Vb, mine ? spos[g + lane] : -1, mine ? sz[g + lane] : -INFINITY, m, zs, acc);
    }
    __syncthreads();   // the staging area is reused by the next block
  }
  combine_and_merge<D>(p, sm, cl, rank, ncl, row, m, zs, acc);
}

// Waits (rank 0's first thread, polling with a time limit) until every score CTA is done with
// this row's KV head, then tells every CTA of the cluster whether it may go on.  The row group's
// last cluster to get through sets the counter back to zero for the next step (the next score
// launch adds to it only after this kernel has finished).  Returns false on a timeout (error
// bit kErrReadyWait); every CTA of the cluster returns the same.
template <int D>
__device__ bool wait_ready(const SaParams &p, SaSmem<D> &sm, cg::cluster_group &cl, int rank, int ncl,
                           int row) {
  constexpr unsigned long long kLimitNs = 1000000000ull;   // one second
  if (rank == 0 && threadIdx.x == 0) {
    uint32_t *ctr = p.ready + static_cast<long long>(row / p.G) * p.ready_stride;
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    uint32_t ok = 1u;
    for (;;) {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
      if (v >= p.ready_target) break;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > kLimitNs) {
        ok = 0u;
        atomicOr(p.err, kErrReadyWait);
        break;
      }
      __nanosleep(256);
    }
    // the G clusters of this KV head pass here once each; the last one resets the counters
    const uint32_t prev = atomicAdd(ctr + 1, 1u);
    if (prev == static_cast<uint32_t>(p.G - 1)) {
      ctr[0] = 0u;
      ctr[1] = 0u;
    }
    for (int c = 0; c < ncl; ++c) cl.map_shared_rank(&sm, c)->x_ok = ok;
  }
  cl.sync();   // the verdict is in every CTA (and rank 0's acquire orders the cluster's reads)
  return sm.x_ok != 0u;
}

// kFull = false: the plain decode step (the score kernel's histogram, the cache's own score rows
// and positions); the threshold budget, the self-built histogram and candidate lists take the
// kFull = true instantiation, so the plain one carries none of their code.
template <int D, class Pg, bool kFull>
__device__ __forceinline__ void select_attend_body(const SaParams &p, const Pg &pg) {
  __shared__ SaSmem<D> sm;
  cg::cluster_group cl = cg::this_cluster();
  const int ncl = static_cast<int>(cl.num_blocks());
  const int rank = static_cast<int>(cl.block_rank());
  const int row = blockIdx.y;
  pdl_trigger();
  if (p.ready != nullptr) {
    // the scan is still running: start once this row's KV head is scored
    if (!wait_ready(p, sm, cl, rank, ncl, row)) return;
  } else {
    pdl_wait();   // the scores, histograms and (attention only) idx come from earlier kernels
  }
  // each phase computes the row geometry afresh (nothing stays live across the selection)
  if (p.mode & kSaSelect)
    select_phase<D, kFull>(p, row_geo<kFull>(p, pg, row, ncl), sm, cl, rank, ncl, row);
  if (p.mode & kSaAttend) {
    if (p.mode & kSaSelect) cl.sync();   // Omega complete in idx (release/acquire at cluster scope)
    attend_phase<D, kFull>(p, attend_geo<kFull>(p, pg, row, ncl), pg, sm, cl, rank, ncl, row);
  } else {
    cl.sync();   // no CTA leaves while the cluster may still use its shared memory
  }
}

// Two register bounds over the same body.  A launch whose clusters all run at once (one wave)
// is latency-bound: it takes 96 registers a thread and spills nothing, and a CTA of it still
// fits on an SM sub-partition beside a score CTA (the score kernel's bound states the sum).
// A launch of more clusters than that is throughput-bound: it keeps three CTAs an SM (at most
// 80 registers a thread, a few spilled words).
template <int D, class Pg, bool kFull>
__global__ void __maxnreg__(96) select_attend_kernel(const SaParams p, const Pg pg) {
  select_attend_body<D, Pg, kFull>(p, pg);
}

template <int D, class Pg, bool kFull>
__global__ void __launch_bounds__(kSaThreads, 3) select_attend_wide_kernel(const SaParams p,
                                                                           const Pg pg) {
  select_attend_body<D, Pg, kFull>(p, pg);
}

template <int D, class Pg, bool kFull, bool kWide>
struct SaKernel {
  static constexpr auto fn = select_attend_kernel<D, Pg, kFull>;
};
template <int D, class Pg, bool kFull>
struct SaKernel<D, Pg, kFull, true> {
  static constexpr auto fn = select_attend_wide_kernel<D, Pg, kFull>;
};

// ------------------------------------------------------------------ host

// Clusters of `ncl` CTAs of this kernel that the device runs at once (0 if it cannot run
// them), queried once per device and size.
template <int D>
static int active_clusters_t(int ncl) {
  static int cache[64][5];
  static bool done[64][5] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ncl <= 8 ? 1 : 0;
  int li = 0;
  while ((1 << li) < ncl) ++li;
  if (!done[dev][li]) {
    if (ncl > 8)
      (void)cudaFuncSetAttribute(select_attend_kernel<D, NoPaging, false>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ncl), 1);
    cfg.blockDim = dim3(kSaThreads);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(ncl);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, select_attend_kernel<D, NoPaging, false>, &cfg) !=
        cudaSuccess)
      n = 0;
    (void)cudaGetLastError();   // a refused query leaves no error behind
    cache[dev][li] = n;
    done[dev][li] = true;
  }
  return cache[dev][li];
}

// The cluster size of a query head (a power of two <= kMaxCluster): chunks of at most 64K
// candidates (a head whose threshold bin is crowded then spreads over several CTAs), grown while
// the clusters of all R heads still run in one wave and chunks keep at least 4096 candidates;
// a size whose last wave would be nearly empty is halved.
int select_cluster_size(long long nC, int R, int d) {
  auto active = [d](int n) { return d == 128 ? active_clusters_t<128>(n) : active_clusters_t<64>(n); };
  int n = 1;
  while (n < kMaxCluster && 65536LL * n < nC && active(2 * n) > 0) n *= 2;
  while (n < kMaxCluster && nC >= 8192LL * n && active(2 * n) >= R) n *= 2;
  const int a = active(n);
  if (n > 1 && a > 0 && R > a && (R % a) * 4 < a && active(n / 2) > 0) n /= 2;
  return n;
}

template <int D, class Pg, bool kFull, bool kWide>
static cudaError_t launch_sa_k(const SaParams &p, const Pg &pg, int R, int ncl, cudaStream_t s) {
  static bool attr_done[64] = {};
  static bool carve_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
    if (ncl > 8 && !attr_done[dev]) {
      const cudaError_t e = cudaFuncSetAttribute(SaKernel<D, Pg, kFull, kWide>::fn,
                                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      attr_done[dev] = true;
    }
    if (!carve_done[dev]) {   // the same carveout as the scan, so both fit on one SM
      const cudaError_t e = cudaFuncSetAttribute(SaKernel<D, Pg, kFull, kWide>::fn,
                                                 cudaFuncAttributePreferredSharedMemoryCarveout,
                                                 cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
      carve_done[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ncl), static_cast<unsigned>(R),
                     static_cast<unsigned>(p.nsplit < 1 ? 1 : p.nsplit));
  cfg.blockDim = dim3(kSaThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ncl);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, SaKernel<D, Pg, kFull, kWide>::fn, p, pg);
}

template <int D, class Pg>
static cudaError_t launch_sa_t(const SaParams &p, const Pg &pg, int R, int ncl, cudaStream_t s) {
  const bool full = (p.mode & (kSaEps | kSaBuildHist)) != 0 || p.row_n != nullptr ||
                    p.pos_map != nullptr || p.S_att != nullptr;
  // more clusters than the 96-register kernel runs at once: the three-CTA bound
  const long long clusters = static_cast<long long>(R) * (p.nsplit < 1 ? 1 : p.nsplit);
  const bool wide = clusters > active_clusters_t<D>(ncl);
  if (full)
    return wide ? launch_sa_k<D, Pg, true, true>(p, pg, R, ncl, s)
                : launch_sa_k<D, Pg, true, false>(p, pg, R, ncl, s);
  return wide ? launch_sa_k<D, Pg, false, true>(p, pg, R, ncl, s)
              : launch_sa_k<D, Pg, false, false>(p, pg, R, ncl, s);
}

size_t select_smem_bytes(int d) { return d == 128 ? sizeof(SaSmem<128>) : sizeof(SaSmem<64>); }

int attn_split(long long nU, int R, int ncl, int d) {
  if (nU <= 1024LL * ncl) return 1;
  const int a = d == 128 ? active_clusters_t<128>(ncl) : active_clusters_t<64>(ncl);
  int n = 1;
  while (2 * n <= kMaxAttnSplit && static_cast<long long>(R) * 2 * n <= a && nU > 512LL * ncl * n) n *= 2;
  return n;
}

static bool valid_launch(const SaParams &p, int ncl) {
  if (ncl < 1 || ncl > kMaxCluster || (ncl & (ncl - 1)) != 0) return false;
  return p.nsplit >= 1 && p.nsplit <= kMaxAttnSplit && !(p.nsplit > 1 && (p.mode & kSaSelect));
}

cudaError_t launch_select_attend(const SaParams &p, int d, int R, int ncl, cudaStream_t s) {
  if (!valid_launch(p, ncl)) return cudaErrorInvalidValue;
  const NoPaging pg{};
  return d == 128 ? launch_sa_t<128>(p, pg, R, ncl, s) : launch_sa_t<64>(p, pg, R, ncl, s);
}

cudaError_t launch_select_attend_paged(const SaParams &p, const PagedInfo &pg, int d, int R, int ncl,
                                       cudaStream_t s) {
  if (!valid_launch(p, ncl)) return cudaErrorInvalidValue;
  return d == 128 ? launch_sa_t<128>(p, pg, R, ncl, s) : launch_sa_t<64>(p, pg, R, ncl, s);
}

}  // namespace ra
