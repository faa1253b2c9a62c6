// C ABI of libra: argument validation, workspace layout and kernel sequencing.
// Every check runs on the host before anything is enqueued; the library allocates nothing.
#include <cuda_runtime.h>
#include <stdint.h>
#include <math.h>
#include <stdio.h>

#include <algorithm>

#include "../../include/ra.h"
#include "common.cuh"
#include "kernels.h"

namespace ra {

static thread_local char g_last_error[256] = "";

void set_last_error(const char *msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

static ra_status cuda_fail(cudaError_t e, const char *where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e),
           static_cast<int>(e));
  return RA_ERR_CUDA;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

cudaError_t ensure_smem_limit(const void *kernel, int bytes, bool (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  // the largest shared-memory carveout, so that an SM running this kernel's CTA keeps room for
  // a CTA of a kernel launched behind it (the selection beside the scan)
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

static constexpr size_t kAlign = 256;

size_t counter_block_bytes(size_t rows) {
  const size_t h = (rows * kHistBins * 4 + kAlign - 1) / kAlign * kAlign;
  const size_t m = (rows * kMetaWords * 4 + kAlign - 1) / kAlign * kAlign;
  return h + m;
}
static size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
static long long round4(long long x) { return (x + 3) / 4 * 4; }
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Derived sizes of one decode step (positions follow the slide "The GPU keeps 640 fixed
// positions": W = [0, s1) u [w0, N), candidates C = [s1, w0)).
struct Step {
  int B, Hq, Hkv, G, d, k, n_sink, n_window, R, ncl;
  long long N, cap, s1, w0, nW, nC, k_eff, ldS, ldL, cbase, cper;
  size_t off_S, off_hist, off_meta, off_list, off_selz, off_part, total;
};

static ra_status plan_shape(int B, int Hq, int Hkv, long long N, int d, int k, int n_sink,
                            int n_window, Step &st) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 0 || k < 0 || n_sink < 0 || n_window < 0) return RA_ERR_ARG;
  if (d != 64 && d != 128) return RA_ERR_SHAPE;
  if (Hq % Hkv != 0 || Hq / Hkv > kMaxGroup) return RA_ERR_SHAPE;
  if (N >= (1LL << 31) - 1) return RA_ERR_SHAPE;
  if (static_cast<long long>(B) * Hq > 65535) return RA_ERR_SHAPE;
  st.B = B; st.Hq = Hq; st.Hkv = Hkv; st.G = Hq / Hkv; st.d = d; st.k = k;
  st.n_sink = n_sink; st.n_window = n_window; st.N = N;
  st.R = B * Hq;
  st.s1 = std::min<long long>(n_sink, N);
  st.w0 = std::max<long long>(st.s1, N - n_window);
  st.nW = st.s1 + (N - st.w0);
  st.nC = st.w0 - st.s1;
  st.k_eff = std::min<long long>(k, st.nC);
  st.ldS = round4(std::max<long long>(N, 1));
  st.ldL = round4(std::max<long long>(st.nC, 1));
  st.ncl = 1;
  st.cbase = st.s1 & ~3LL;
  st.cper = round4(std::max<long long>(st.w0 - st.cbase, 1));
  size_t off = 0;
  st.off_hist = off;  off = align_up(off + static_cast<size_t>(st.R) * kHistBins * 4);
  st.off_meta = off;  off = align_up(off + static_cast<size_t>(st.R) * kMetaWords * 4);
  st.off_S = off;     off = align_up(off + static_cast<size_t>(st.R) * st.ldS * 4);
  // the threshold-bin lists (and the scores of the keys above the bin), whenever a selection
  // may stream over C: with a budget under |C|, and under a threshold budget, which can keep
  // fewer keys than a budget of |C| or more
  st.off_list = off;
  if (st.k_eff > 0) off = align_up(off + static_cast<size_t>(st.R) * st.ldL * 8);
  // the score of each selected entry, beside idx
  st.off_selz = off;
  if (st.k > 0) off = align_up(off + static_cast<size_t>(st.R) * st.k * 4);
  st.off_part = off;  off = align_up(off + static_cast<size_t>(st.R) * kMaxAttnSplit * (d + 4) * 4);
  st.total = off;
  return RA_OK;
}

// The selection's cluster split of C (host only, so the workspace size stays a pure function of
// the shape): chunks start at multiples of 4 so the CTAs read the score row in float4 units.
static void plan_clusters(Step &st) {
  st.ncl = select_cluster_size(st.nC, st.R, st.d);
  const long long span = std::max<long long>(st.w0 - st.cbase, 1);
  st.cper = round4((span + st.ncl - 1) / st.ncl);
}

static ra_status check_kv(const ra_kv *kv) {
  if (!kv || !kv->K || !kv->V) return RA_ERR_ARG;
  if (!aligned16(kv->K) || !aligned16(kv->V)) return RA_ERR_ARG;
  if (kv->B < 1 || kv->Hkv < 1 || kv->cap < 0 || kv->N < 0) return RA_ERR_ARG;
  if (kv->d != 64 && kv->d != 128) return RA_ERR_SHAPE;
  if (kv->N > kv->cap) return RA_ERR_SHAPE;
  return RA_OK;
}

// Validation common to the decode step and its phases.
static ra_status plan_step(const ra_kv *kv, int Hq, int k, int n_sink, int n_window, void *ws,
                           size_t ws_bytes, Step &st) {
  ra_status s = check_kv(kv);
  if (s != RA_OK) return s;
  s = plan_shape(kv->B, Hq, kv->Hkv, kv->N, kv->d, k, n_sink, n_window, st);
  if (s != RA_OK) return s;
  st.cap = kv->cap;
  if (kv->N == 0 || st.nW + st.k_eff == 0) return RA_ERR_EMPTY;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return RA_ERR_WORKSPACE;
  if (ws_bytes < st.total) return RA_ERR_WORKSPACE;
  plan_clusters(st);
  return RA_OK;
}

static uint8_t *at(void *ws, size_t off) { return static_cast<uint8_t *>(ws) + off; }

// Per-KV-head completion counters of an overlapped step: the meta words (slots 0 and 1) of the
// head group's first query head.
static uint32_t *ready_counters(void *ws, const Step &st) {
  return reinterpret_cast<uint32_t *>(at(ws, st.off_meta));
}
static long long ready_stride(const Step &st) { return static_cast<long long>(st.G) * kMetaWords; }

// The scan.  With `overlap` set, the score CTAs publish each KV head as they finish it and
// *overlap receives the count a selection waiting on them needs (the launch's CTA count).
static ra_status run_score(const ra_kv *kv, const void *q, const Step &st, void *ws,
                           cudaStream_t stream, bool hist = true, const void *k_new = nullptr,
                           const void *v_new = nullptr, uint32_t *overlap = nullptr) {
  ScoreParams p{};
  p.K = static_cast<const __nv_bfloat16 *>(kv->K);
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.S = reinterpret_cast<float *>(at(ws, st.off_S));
  p.hist = reinterpret_cast<uint32_t *>(at(ws, st.off_hist));
  p.N = st.N; p.cap = st.cap; p.ldS = st.ldS;
  p.cand_lo = st.s1; p.cand_hi = st.w0;
  p.tiles_per_head = (st.N + kScoreTile - 1) / kScoreTile;
  p.total_tiles = p.tiles_per_head * st.B * st.Hkv;
  p.B = st.B; p.Hkv = st.Hkv; p.G = st.G; p.Hq = st.Hq;
  p.scale = 1.0f / sqrtf(static_cast<float>(st.d));
  p.do_hist = hist && st.k_eff > 0 && st.k_eff < st.nC;
  p.err = reinterpret_cast<uint32_t *>(at(ws, st.off_meta)) + kError;
  if (k_new != nullptr) {   // the step's token is appended inside the scan (position N - 1)
    p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    p.K_cache = static_cast<__nv_bfloat16 *>(kv->K);
    p.V_cache = static_cast<__nv_bfloat16 *>(kv->V);
  }
  if (overlap != nullptr) {
    p.ready = ready_counters(ws, st);
    p.ready_stride = ready_stride(st);
  }
  int grid = 0;
  const cudaError_t e = launch_score(p, st.d, stream, &grid);
  if (overlap != nullptr) *overlap = static_cast<uint32_t>(grid);
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "score");
}

// Selection (kSaSelect), attention (kSaAttend) or both.  Both run in one launch unless the
// attention is large enough to want more clusters per head than the selection uses (then it is
// a second launch with nsplit clusters per head).
// ready_target > 0: the preceding scan publishes its KV heads (run_score with `overlap`), and
// the selection launch starts on each head as soon as its counter reaches ready_target.
static ra_status run_select_attend(const ra_kv *kv, const Step &st, int mode, int32_t *idx,
                                   float *out, void *ws, cudaStream_t stream,
                                   float log_eps = 0.f, uint32_t ready_target = 0) {
  if (mode == kSaSelect && st.k == 0) return RA_OK;
  SaParams p{};
  p.S = reinterpret_cast<const float *>(at(ws, st.off_S));
  p.hist = reinterpret_cast<uint32_t *>(at(ws, st.off_hist));
  p.list = reinterpret_cast<unsigned long long *>(at(ws, st.off_list));
  p.V = static_cast<const __nv_bfloat16 *>(kv->V);
  p.idx = idx;
  p.out = out;
  p.part = reinterpret_cast<float *>(at(ws, st.off_part));
  p.meta = reinterpret_cast<uint32_t *>(at(ws, st.off_meta));
  p.err = reinterpret_cast<uint32_t *>(at(ws, st.off_meta)) + kError;
  p.ldS = st.ldS; p.ldL = st.ldL; p.cap = st.cap; p.N = st.N;
  p.s1 = st.s1; p.w0 = st.w0; p.nW = st.nW; p.nC = st.nC; p.k_eff = st.k_eff;
  p.cbase = st.cbase; p.cper = st.cper;
  p.k = st.k; p.Hq = st.Hq; p.G = st.G; p.Hkv = st.Hkv;
  p.log_eps = log_eps;
  // a selection in this call keeps the selected scores beside idx for the attention; an
  // attention over a caller's idx (ra_sparse_attn) reads the score rows
  if ((mode & kSaSelect) && st.k > 0) p.sel_z = reinterpret_cast<float *>(at(ws, st.off_selz));
  const int split = (mode & kSaAttend) ? attn_split(st.nW + st.k_eff, st.R, st.ncl, st.d) : 1;
  if (mode & kSaSelect) {
    // the attention joins the launch when it can
    p.mode = split == 1 ? mode : (mode & ~kSaAttend);
    p.nsplit = 1;
    if (ready_target > 0) {
      p.ready = ready_counters(ws, st);
      p.ready_stride = ready_stride(st);
      p.ready_target = ready_target;
    }
    const cudaError_t e = launch_select_attend(p, st.d, st.R, st.ncl, stream);
    if (e != cudaSuccess) return cuda_fail(e, "select_attend");
    if (p.mode == mode) return RA_OK;
  }
  p.ready = nullptr;
  p.mode = kSaAttend;
  p.log_eps = 0.f;
  p.nsplit = split;
  const cudaError_t e = launch_select_attend(p, st.d, st.R, st.ncl, stream);
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "attend");
}

// Dense flash-decode split plan: as many splits per KV head as keep the grid close to a
// whole number of waves of one CTA per SM, at most kDenseMaxSplit.
static constexpr int kDenseMaxSplit = 256;

static int dense_nsplit_cap(long long N) {
  const long long tiles = std::max<long long>(1, (N + kDenseTile - 1) / kDenseTile);
  return static_cast<int>(std::min<long long>(tiles, kDenseMaxSplit));
}

// Counter block: per-row histograms then per-row counters, at the front of every workspace.
// Kernels leave it zero when they finish, so a workspace zero-filled once stays usable by
// later calls with the same B * Hq (whatever N), sparse and dense alike.
static size_t counter_bytes(int R, size_t *off_meta) {
  const size_t m = align_up(static_cast<size_t>(R) * kHistBins * 4);
  if (off_meta) *off_meta = m;
  return align_up(m + static_cast<size_t>(R) * kMetaWords * 4);
}

static size_t dense_bytes(int R, int nsplit_cap, int d, size_t *off_meta, size_t *off_part) {
  const size_t c = counter_bytes(R, off_meta);
  if (off_part) *off_part = c;
  return align_up(c + static_cast<size_t>(R) * nsplit_cap * (d + 4) * 4);
}

}  // namespace ra

using namespace ra;

extern "C" {

const char *ra_status_str(ra_status s) {
  switch (s) {
    case RA_OK: return "RA_OK";
    case RA_ERR_ARG: return "RA_ERR_ARG";
    case RA_ERR_SHAPE: return "RA_ERR_SHAPE";
    case RA_ERR_CAPACITY: return "RA_ERR_CAPACITY";
    case RA_ERR_WORKSPACE: return "RA_ERR_WORKSPACE";
    case RA_ERR_CUDA: return "RA_ERR_CUDA";
    case RA_ERR_EMPTY: return "RA_ERR_EMPTY";
  }
  return "RA_ERR_UNKNOWN";
}

const char *ra_version(void) { return "libra 0.1 (sm_100a)"; }

const char *ra_last_error(void) { return g_last_error; }

ra_status ra_append_kv(ra_kv *kv, const void *k_new, const void *v_new, int32_t T,
                       ra_stream_t stream) {
  ra_status s = check_kv(kv);
  if (s != RA_OK) return s;
  if (T < 0) return RA_ERR_ARG;
  if (T == 0) return RA_OK;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return RA_ERR_ARG;
  if (kv->N + T > kv->cap) return RA_ERR_CAPACITY;
  AppendParams p{};
  p.K = static_cast<__nv_bfloat16 *>(kv->K);
  p.V = static_cast<__nv_bfloat16 *>(kv->V);
  p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
  p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
  p.cap = kv->cap; p.N = kv->N; p.B = kv->B; p.Hkv = kv->Hkv; p.d = kv->d; p.T = T;
  cudaError_t e = launch_append(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append");
  kv->N += T;
  return RA_OK;
}

size_t ra_decode_workspace_bytes(int32_t B, int32_t Hq, int64_t N, int32_t d, int32_t k,
                                 int32_t n_sink, int32_t n_window) {
  Step st{};
  // the layout does not depend on the KV head count: plan it with one query head per KV head
  if (plan_shape(B, Hq, Hq, N, d, k, n_sink, n_window, st) != RA_OK) return 0;
  return st.total;
}

ra_status ra_score_gqa(const ra_kv *kv, const void *q, int32_t Hq, int32_t k, int32_t n_sink,
                       int32_t n_window, void *ws, size_t ws_bytes, ra_stream_t stream) {
  Step st{};
  ra_status s = plan_step(kv, Hq, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if (!q || !aligned16(q)) return RA_ERR_ARG;
  return run_score(kv, q, st, ws, reinterpret_cast<cudaStream_t>(stream));
}

// Validation of the fused append + decode entry points: kv grows by one token, which must fit.
static ra_status plan_append_step(ra_kv *kv, const void *k_new, const void *v_new, int32_t Hq,
                                  int32_t k, int32_t n_sink, int32_t n_window, void *ws,
                                  size_t ws_bytes, ra_kv &grown, Step &st) {
  ra_status s = check_kv(kv);
  if (s != RA_OK) return s;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return RA_ERR_ARG;
  if (kv->N + 1 > kv->cap) return RA_ERR_CAPACITY;
  grown = *kv;
  grown.N = kv->N + 1;
  return plan_step(&grown, Hq, k, n_sink, n_window, ws, ws_bytes, st);
}

ra_status ra_score_gqa_append(ra_kv *kv, const void *q, const void *k_new, const void *v_new,
                              int32_t Hq, int32_t k, int32_t n_sink, int32_t n_window, void *ws,
                              size_t ws_bytes, ra_stream_t stream) {
  ra_kv grown{};
  Step st{};
  ra_status s = plan_append_step(kv, k_new, v_new, Hq, k, n_sink, n_window, ws, ws_bytes, grown, st);
  if (s != RA_OK) return s;
  if (!q || !aligned16(q)) return RA_ERR_ARG;
  s = run_score(&grown, q, st, ws, reinterpret_cast<cudaStream_t>(stream), true, k_new, v_new);
  if (s == RA_OK) kv->N = grown.N;
  return s;
}

ra_status ra_decode_step_append(ra_kv *kv, const void *q, const void *k_new, const void *v_new,
                                int32_t Hq, int32_t k, int32_t n_sink, int32_t n_window,
                                float *out, int32_t *idx, void *ws, size_t ws_bytes,
                                ra_stream_t stream) {
  ra_kv grown{};
  Step st{};
  ra_status s = plan_append_step(kv, k_new, v_new, Hq, k, n_sink, n_window, ws, ws_bytes, grown, st);
  if (s != RA_OK) return s;
  if (!q || !aligned16(q) || !out || !aligned16(out)) return RA_ERR_ARG;
  if (k > 0 && (!idx || !aligned16(idx))) return RA_ERR_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint32_t target = 0;
  s = run_score(&grown, q, st, ws, cs, true, k_new, v_new, &target);
  if (s != RA_OK) return s;
  kv->N = grown.N;   // the token is in the cache once the scan has run
  return run_select_attend(&grown, st, kSaSelect | kSaAttend, idx, out, ws, cs, 0.f, target);
}

ra_status ra_decode_step_append_host(ra_kv *kv, const void *q_host, const void *k_new_host,
                                     const void *v_new_host, int32_t Hq, int32_t k,
                                     int32_t n_sink, int32_t n_window, float *out_host,
                                     int32_t *idx_host, const ra_step_io *dev, void *ws,
                                     size_t ws_bytes, ra_stream_t stream) {
  if (!dev || !q_host || !k_new_host || !v_new_host || !out_host || (k > 0 && !idx_host))
    return RA_ERR_ARG;
  // every check of the step first (nothing enqueued, kv unchanged on an error)
  ra_kv grown{};
  Step st{};
  ra_status s = plan_append_step(kv, dev->k_new, dev->v_new, Hq, k, n_sink, n_window, ws, ws_bytes,
                                 grown, st);
  if (s != RA_OK) return s;
  if (!dev->q || !aligned16(dev->q) || !dev->out || !aligned16(dev->out)) return RA_ERR_ARG;
  if (k > 0 && (!dev->idx || !aligned16(dev->idx))) return RA_ERR_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const size_t qb = static_cast<size_t>(kv->B) * Hq * kv->d * 2;
  const size_t rowb = static_cast<size_t>(kv->B) * kv->Hkv * kv->d * 2;
  const size_t ob = static_cast<size_t>(kv->B) * Hq * kv->d * 4;
  const size_t ib = static_cast<size_t>(kv->B) * Hq * (k > 0 ? k : 0) * 4;
  cudaError_t e = cudaMemcpyAsync(dev->q, q_host, qb, cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dev->k_new, k_new_host, rowb, cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dev->v_new, v_new_host, rowb, cudaMemcpyHostToDevice, cs);
  if (e != cudaSuccess) return cuda_fail(e, "decode_step_append_host: copy in");
  s = ra_decode_step_append(kv, dev->q, dev->k_new, dev->v_new, Hq, k, n_sink, n_window, dev->out,
                            dev->idx, ws, ws_bytes, stream);
  if (s != RA_OK) return s;
  e = cudaMemcpyAsync(out_host, dev->out, ob, cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess && ib > 0) e = cudaMemcpyAsync(idx_host, dev->idx, ib, cudaMemcpyDeviceToHost, cs);
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "decode_step_append_host: copy out");
}

int32_t ra_decode_step_launches(int32_t B, int32_t Hq, int32_t Hkv, int64_t N, int32_t d,
                                int32_t k, int32_t n_sink, int32_t n_window) {
  Step st{};
  if (plan_shape(B, Hq, Hkv, N, d, k, n_sink, n_window, st) != RA_OK) return -1;
  if (N == 0 || st.nW + st.k_eff == 0) return -1;
  plan_clusters(st);
  // the scan, then selection + attention in one launch unless the attention is split
  return attn_split(st.nW + st.k_eff, st.R, st.ncl, st.d) == 1 ? 2 : 3;
}

ra_status ra_topk_select(const ra_kv *kv, int32_t Hq, int32_t k, int32_t n_sink,
                         int32_t n_window, int32_t *idx, void *ws, size_t ws_bytes,
                         ra_stream_t stream) {
  Step st{};
  ra_status s = plan_step(kv, Hq, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if (k > 0 && (!idx || !aligned16(idx))) return RA_ERR_ARG;
  return run_select_attend(kv, st, kSaSelect, idx, nullptr, ws, reinterpret_cast<cudaStream_t>(stream));
}

ra_status ra_sparse_attn(const ra_kv *kv, int32_t Hq, int32_t k, int32_t n_sink,
                         int32_t n_window, const int32_t *idx, float *out, void *ws,
                         size_t ws_bytes, ra_stream_t stream) {
  Step st{};
  ra_status s = plan_step(kv, Hq, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if ((k > 0 && (!idx || !aligned16(idx))) || !out || !aligned16(out)) return RA_ERR_ARG;
  return run_select_attend(kv, st, kSaAttend, const_cast<int32_t *>(idx), out, ws,
                           reinterpret_cast<cudaStream_t>(stream));
}

ra_status ra_select_attend(const ra_kv *kv, int32_t Hq, int32_t k, int32_t n_sink,
                           int32_t n_window, int32_t *idx, float *out, void *ws, size_t ws_bytes,
                           ra_stream_t stream) {
  Step st{};
  ra_status s = plan_step(kv, Hq, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if ((k > 0 && (!idx || !aligned16(idx))) || !out || !aligned16(out)) return RA_ERR_ARG;
  return run_select_attend(kv, st, kSaSelect | kSaAttend, idx, out, ws,
                           reinterpret_cast<cudaStream_t>(stream));
}

ra_status ra_decode_step(const ra_kv *kv, const void *q, int32_t Hq, int32_t k, int32_t n_sink,
                         int32_t n_window, float *out, int32_t *idx, void *ws, size_t ws_bytes,
                         ra_stream_t stream) {
  Step st{};
  ra_status s = plan_step(kv, Hq, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if (!q || !aligned16(q) || !out || !aligned16(out)) return RA_ERR_ARG;
  if (k > 0 && (!idx || !aligned16(idx))) return RA_ERR_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint32_t target = 0;
  s = run_score(kv, q, st, ws, cs, true, nullptr, nullptr, &target);
  if (s != RA_OK) return s;
  return run_select_attend(kv, st, kSaSelect | kSaAttend, idx, out, ws, cs, 0.f, target);
}

// ---- paged caches

static ra_status check_paged(const ra_paged_kv *kv, long long *max_n) {
  if (!kv || !kv->K || !kv->V || !kv->block_table || !kv->seq_len) return RA_ERR_ARG;
  if (!aligned16(kv->K) || !aligned16(kv->V)) return RA_ERR_ARG;
  if (kv->B < 1 || kv->Hkv < 1 || kv->max_pages < 1 || kv->num_pages < 1) return RA_ERR_ARG;
  if (kv->B > kMaxPagedBatch) return RA_ERR_SHAPE;
  if (kv->d != 64 && kv->d != 128) return RA_ERR_SHAPE;
  long long m = 0;
  for (int b = 0; b < kv->B; ++b) {
    if (kv->seq_len[b] < 0 || static_cast<long long>(kv->seq_len[b]) > 1LL * kv->max_pages * kPageSize)
      return RA_ERR_SHAPE;
    m = std::max<long long>(m, kv->seq_len[b]);
  }
  *max_n = m;
  return RA_OK;
}

static void fill_paged_info(const ra_paged_kv *kv, int k, int n_sink, int n_window, PagedInfo &pg) {
  pg.block_table = kv->block_table;
  pg.max_pages = kv->max_pages;
  pg.n_sink = n_sink;
  pg.n_window = n_window;
  pg.k = k;
  int32_t off = 0;
  for (int b = 0; b < kv->B; ++b) {
    pg.seq_len[b] = kv->seq_len[b];
    pg.tile_off[b] = off;
    off += kv->Hkv * ((kv->seq_len[b] + kScoreTile - 1) / kScoreTile);
  }
  pg.tile_off[kv->B] = off;
}

// ---- prefill: exact top-k of a batch of queries (rows (b, h, m) of Q [B, Hq, M, d])

// The prefill plan is the decode plan with one row per query: B * M "sequences" of Hq heads.
static ra_status plan_prefill(const ra_kv *kv, int Hq, int M, int k, int n_sink, int n_window,
                              void *ws, size_t ws_bytes, Step &st) {
  ra_status s = check_kv(kv);
  if (s != RA_OK) return s;
  if (M < 1) return RA_ERR_ARG;
  if (static_cast<long long>(kv->B) * M > 65535) return RA_ERR_SHAPE;
  s = plan_shape(kv->B * M, Hq, kv->Hkv, kv->N, kv->d, k, n_sink, n_window, st);
  if (s != RA_OK) return s;
  st.cap = kv->cap;
  if (kv->N == 0) return RA_ERR_EMPTY;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return RA_ERR_WORKSPACE;
  if (ws_bytes < st.total) return RA_ERR_WORKSPACE;
  plan_clusters(st);
  return RA_OK;
}

static ra_status run_prefill_score(const ra_kv *kv, const void *q, int Hq, int M, const Step &st,
                                   void *ws, cudaStream_t stream) {
  PfParams p{};
  p.Q = static_cast<const __nv_bfloat16 *>(q);
  p.K = static_cast<const __nv_bfloat16 *>(kv->K);
  p.S = reinterpret_cast<float *>(at(ws, st.off_S));
  p.err = reinterpret_cast<uint32_t *>(at(ws, st.off_meta)) + kError;
  p.N = st.N; p.cap = st.cap; p.ldS = st.ldS;
  p.B = kv->B; p.Hq = Hq; p.Hkv = kv->Hkv; p.G = Hq / kv->Hkv; p.M = M;
  p.scale = 1.0f / sqrtf(static_cast<float>(kv->d));
  const cudaError_t e = launch_prefill_score(p, kv->d, stream);
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "prefill_score");
}

static ra_status run_prefill_select(const Step &st, int32_t *idx, void *ws, cudaStream_t stream) {
  if (st.k == 0) return RA_OK;
  SaParams p{};
  p.S = reinterpret_cast<const float *>(at(ws, st.off_S));
  p.hist = reinterpret_cast<uint32_t *>(at(ws, st.off_hist));
  p.list = reinterpret_cast<unsigned long long *>(at(ws, st.off_list));
  p.idx = idx;
  p.part = reinterpret_cast<float *>(at(ws, st.off_part));
  p.meta = reinterpret_cast<uint32_t *>(at(ws, st.off_meta));
  p.err = reinterpret_cast<uint32_t *>(at(ws, st.off_meta)) + kError;
  p.ldS = st.ldS; p.ldL = st.ldL; p.cap = st.cap; p.N = st.N;
  p.s1 = st.s1; p.w0 = st.w0; p.nW = st.nW; p.nC = st.nC; p.k_eff = st.k_eff;
  p.cbase = st.cbase; p.cper = st.cper;
  p.k = st.k; p.Hq = st.Hq; p.G = st.G; p.Hkv = st.Hkv;
  p.mode = kSaSelect | kSaBuildHist;
  p.nsplit = 1;
  const cudaError_t e = launch_select_attend(p, st.d, st.R, st.ncl, stream);
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "prefill_select");
}

ra_status ra_decode_step_eps(const ra_kv *kv, const void *q, int32_t Hq, int32_t k, float eps,
                             int32_t n_sink, int32_t n_window, float *out, int32_t *idx,
                             void *ws, size_t ws_bytes, ra_stream_t stream) {
  if (!(eps > 0.0f && eps < 1.0f)) return RA_ERR_ARG;
  Step st{};
  ra_status s = plan_step(kv, Hq, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if (st.nW == 0) return RA_ERR_EMPTY;   // the threshold may keep no key: W must be non-empty
  if (!q || !aligned16(q) || !out || !aligned16(out)) return RA_ERR_ARG;
  if (k > 0 && (!idx || !aligned16(idx))) return RA_ERR_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  s = run_score(kv, q, st, ws, cs, /*hist=*/false);   // the selection counts against the threshold
  if (s != RA_OK) return s;
  return run_select_attend(kv, st, kSaSelect | kSaAttend | kSaEps, idx, out, ws, cs, logf(eps));
}

size_t ra_dense_workspace_bytes(int32_t B, int32_t Hq, int64_t N, int32_t d) {
  if (B < 1 || Hq < 1 || N < 0 || (d != 64 && d != 128)) return 0;
  if (N >= (1LL << 31) - 1) return 0;
  return dense_bytes(B * Hq, dense_nsplit_cap(N), d, nullptr, nullptr);
}

ra_status ra_dense_decode(const ra_kv *kv, const void *q, int32_t Hq, float *out, void *ws,
                          size_t ws_bytes, ra_stream_t stream) {
  ra_status s = check_kv(kv);
  if (s != RA_OK) return s;
  if (Hq < 1 || Hq % kv->Hkv != 0 || Hq / kv->Hkv > kMaxGroup) return RA_ERR_SHAPE;
  if (kv->N >= (1LL << 31) - 1 || static_cast<long long>(kv->B) * Hq > 65535) return RA_ERR_SHAPE;
  if (kv->N == 0) return RA_ERR_EMPTY;
  if (!q || !aligned16(q) || !out || !aligned16(out)) return RA_ERR_ARG;
  const int R = kv->B * Hq;
  const int cap_split = dense_nsplit_cap(kv->N);
  size_t off_meta = 0, off_part = 0;
  const size_t need = dense_bytes(R, cap_split, kv->d, &off_meta, &off_part);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0 || ws_bytes < need)
    return RA_ERR_WORKSPACE;

  // splits: the smallest whole number of waves (one CTA per SM) that is >= 95% full
  const long long tiles = (kv->N + kDenseTile - 1) / kDenseTile;
  const int BH = kv->B * kv->Hkv;
  const int sms = num_sms();
  int best = 1;
  double best_eff = -1.0;
  for (int w = 1; w <= 8; ++w) {
    int ns = std::max(1, (sms * w) / BH);
    ns = static_cast<int>(std::min<long long>(ns, std::min<long long>(tiles, cap_split)));
    const long long ctas = static_cast<long long>(BH) * ns;
    const long long waves = (ctas + sms - 1) / sms;
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * sms);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = ns;
    }
    if (eff >= 0.95) break;
  }
  const long long kps = (tiles + best - 1) / best * kDenseTile;
  const int nsplit = static_cast<int>((kv->N + kps - 1) / kps);

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  DenseParams p{};
  p.K = static_cast<const __nv_bfloat16 *>(kv->K);
  p.V = static_cast<const __nv_bfloat16 *>(kv->V);
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.part = reinterpret_cast<float *>(at(ws, off_part));
  p.out = out;
  p.meta = reinterpret_cast<uint32_t *>(at(ws, off_meta));
  p.N = kv->N; p.cap = kv->cap; p.keys_per_split = kps;
  p.B = kv->B; p.Hkv = kv->Hkv; p.G = Hq / kv->Hkv; p.Hq = Hq; p.nsplit = nsplit;
  p.scale = 1.0f / sqrtf(static_cast<float>(kv->d));
  p.err = reinterpret_cast<uint32_t *>(at(ws, off_meta)) + kError;
  const cudaError_t e = launch_dense(p, kv->d, cs);
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "dense_decode");
}

size_t ra_prefill_workspace_bytes(int32_t B, int32_t Hq, int32_t M, int64_t N, int32_t d,
                                  int32_t k, int32_t n_sink, int32_t n_window) {
  if (B < 1 || M < 1 || static_cast<long long>(B) * M > 65535) return 0;
  Step st{};
  if (plan_shape(B * M, Hq, Hq, N, d, k, n_sink, n_window, st) != RA_OK) return 0;
  return st.total;
}

ra_status ra_prefill_score(const ra_kv *kv, const void *q, int32_t Hq, int32_t M, int32_t k,
                           int32_t n_sink, int32_t n_window, void *ws, size_t ws_bytes,
                           ra_stream_t stream) {
  Step st{};
  ra_status s = plan_prefill(kv, Hq, M, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if (!q || !aligned16(q)) return RA_ERR_ARG;
  return run_prefill_score(kv, q, Hq, M, st, ws, reinterpret_cast<cudaStream_t>(stream));
}

ra_status ra_prefill_select(const ra_kv *kv, int32_t Hq, int32_t M, int32_t k, int32_t n_sink,
                            int32_t n_window, int32_t *idx, void *ws, size_t ws_bytes,
                            ra_stream_t stream) {
  Step st{};
  ra_status s = plan_prefill(kv, Hq, M, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if (k > 0 && (!idx || !aligned16(idx))) return RA_ERR_ARG;
  return run_prefill_select(st, idx, ws, reinterpret_cast<cudaStream_t>(stream));
}

ra_status ra_prefill_topk(const ra_kv *kv, const void *q, int32_t Hq, int32_t M, int32_t k,
                          int32_t n_sink, int32_t n_window, int32_t *idx, void *ws,
                          size_t ws_bytes, ra_stream_t stream) {
  Step st{};
  ra_status s = plan_prefill(kv, Hq, M, k, n_sink, n_window, ws, ws_bytes, st);
  if (s != RA_OK) return s;
  if (!q || !aligned16(q)) return RA_ERR_ARG;
  if (k > 0 && (!idx || !aligned16(idx))) return RA_ERR_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  s = run_prefill_score(kv, q, Hq, M, st, ws, cs);
  if (s != RA_OK) return s;
  return run_prefill_select(st, idx, ws, cs);
}

ra_status ra_pyramid_budgets(int32_t L, int32_t k_mean, double ratio, int32_t *k_out) {
  if (L < 1 || k_mean < 0 || !(ratio > 0.0 && ratio <= 1.0) || !k_out) return RA_ERR_ARG;
  if (L == 1) {
    k_out[0] = k_mean;
    return RA_OK;
  }
  const double k_max = 2.0 * k_mean / (1.0 + ratio);
  long long total = 0;
  for (int32_t l = 0; l < L; ++l) {
    const double x = k_max * (1.0 - (1.0 - ratio) * l / (L - 1));
    k_out[l] = static_cast<int32_t>(floor(x));
    total += k_out[l];
  }
  // the rounding remainder goes one by one to the lowest layers: the total is L * k_mean
  const long long rem = static_cast<long long>(L) * k_mean - total;
  for (long long l = 0; l < rem && l < L; ++l) k_out[l] += 1;
  return RA_OK;
}

ra_status ra_paged_append_kv(ra_paged_kv *kv, const void *k_new, const void *v_new, int32_t T,
                             ra_stream_t stream) {
  long long max_n = 0;
  ra_status s = check_paged(kv, &max_n);
  if (s != RA_OK) return s;
  if (T < 0) return RA_ERR_ARG;
  if (T == 0) return RA_OK;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return RA_ERR_ARG;
  for (int b = 0; b < kv->B; ++b)
    if (static_cast<long long>(kv->seq_len[b]) + T > 1LL * kv->max_pages * kPageSize)
      return RA_ERR_CAPACITY;
  AppendParams p{};
  p.K = static_cast<__nv_bfloat16 *>(kv->K);
  p.V = static_cast<__nv_bfloat16 *>(kv->V);
  p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
  p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
  p.B = kv->B; p.Hkv = kv->Hkv; p.d = kv->d; p.T = T;
  PagedInfo pg{};
  fill_paged_info(kv, 0, 0, 0, pg);
  const cudaError_t e = launch_append_paged(p, pg, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "paged_append");
  for (int b = 0; b < kv->B; ++b) kv->seq_len[b] += T;
  return RA_OK;
}

size_t ra_paged_workspace_bytes(int32_t B, int32_t Hq, int64_t max_N, int32_t d, int32_t k,
                                int32_t n_sink, int32_t n_window) {
  if (B > kMaxPagedBatch) return 0;
  return ra_decode_workspace_bytes(B, Hq, max_N, d, k, n_sink, n_window);
}

ra_status ra_paged_decode_step(const ra_paged_kv *kv, const void *q, int32_t Hq, int32_t k,
                               int32_t n_sink, int32_t n_window, float *out, int32_t *idx,
                               void *ws, size_t ws_bytes, ra_stream_t stream) {
  long long max_n = 0;
  ra_status s = check_paged(kv, &max_n);
  if (s != RA_OK) return s;
  for (int b = 0; b < kv->B; ++b)
    if (kv->seq_len[b] < 1) return RA_ERR_EMPTY;
  // the plan of the longest sequence bounds every row's (scores, lists, cluster split)
  Step st{};
  s = plan_shape(kv->B, Hq, kv->Hkv, max_n, kv->d, k, n_sink, n_window, st);
  if (s != RA_OK) return s;
  for (int b = 0; b < kv->B; ++b) {   // every row's union must be non-empty
    const long long N = kv->seq_len[b];
    const long long s1 = std::min<long long>(n_sink, N), w0 = std::max<long long>(s1, N - n_window);
    if (s1 + (N - w0) + std::min<long long>(k, w0 - s1) == 0) return RA_ERR_EMPTY;
  }
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0 || ws_bytes < st.total)
    return RA_ERR_WORKSPACE;
  if (!q || !aligned16(q) || !out || !aligned16(out)) return RA_ERR_ARG;
  if (k > 0 && (!idx || !aligned16(idx))) return RA_ERR_ARG;
  plan_clusters(st);
  st.cap = 0;
  PagedInfo pg{};
  fill_paged_info(kv, k, n_sink, n_window, pg);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int grid = 0;
  {
    ScoreParams p{};
    p.K = static_cast<const __nv_bfloat16 *>(kv->K);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.S = reinterpret_cast<float *>(at(ws, st.off_S));
    p.hist = reinterpret_cast<uint32_t *>(at(ws, st.off_hist));
    p.N = st.N; p.cap = 0; p.ldS = st.ldS;
    p.total_tiles = pg.tile_off[kv->B];
    p.B = st.B; p.Hkv = st.Hkv; p.G = st.G; p.Hq = st.Hq;
    p.scale = 1.0f / sqrtf(static_cast<float>(st.d));
    p.do_hist = k > 0;   // each head decides from its own length
    p.err = reinterpret_cast<uint32_t *>(at(ws, st.off_meta)) + kError;
    p.ready = ready_counters(ws, st);   // the selection starts on each head as it is scored
    p.ready_stride = ready_stride(st);
    const cudaError_t e = launch_score_paged(p, pg, kv->num_pages, st.d, cs, &grid);
    if (e != cudaSuccess) return cuda_fail(e, "paged_score");
  }
  SaParams p{};
  p.S = reinterpret_cast<const float *>(at(ws, st.off_S));
  p.hist = reinterpret_cast<uint32_t *>(at(ws, st.off_hist));
  p.list = reinterpret_cast<unsigned long long *>(at(ws, st.off_list));
  p.V = static_cast<const __nv_bfloat16 *>(kv->V);
  p.idx = idx;
  p.out = out;
  p.part = reinterpret_cast<float *>(at(ws, st.off_part));
  p.meta = reinterpret_cast<uint32_t *>(at(ws, st.off_meta));
  p.err = reinterpret_cast<uint32_t *>(at(ws, st.off_meta)) + kError;
  p.ldS = st.ldS; p.ldL = st.ldL; p.cap = 0; p.N = st.N;
  p.k = st.k; p.Hq = st.Hq; p.G = st.G; p.Hkv = st.Hkv;
  if (k > 0) p.sel_z = reinterpret_cast<float *>(at(ws, st.off_selz));
  const int split = attn_split(st.nW + st.k_eff, st.R, st.ncl, st.d);
  p.mode = split == 1 ? (kSaSelect | kSaAttend) : kSaSelect;
  p.nsplit = 1;
  p.ready = ready_counters(ws, st);
  p.ready_stride = ready_stride(st);
  p.ready_target = static_cast<uint32_t>(grid);
  cudaError_t e = launch_select_attend_paged(p, pg, st.d, st.R, st.ncl, cs);
  if (e != cudaSuccess) return cuda_fail(e, "paged_select_attend");
  if (split > 1) {
    p.ready = nullptr;
    p.mode = kSaAttend;
    p.nsplit = split;
    e = launch_select_attend_paged(p, pg, st.d, st.R, st.ncl, cs);
    if (e != cudaSuccess) return cuda_fail(e, "paged_attend");
  }
  return RA_OK;
}

// ---- IVF index

// Build workspace: the key-centroid scores of one chunk of keys (at most kIvfScoreBytes, so the
// workspace stays bounded at any N), the assignment, and the sort's per-chunk slot table.
static constexpr size_t kIvfScoreBytes = size_t(256) << 20;

struct IvfBuildLayout {
  size_t off_A, off_assign, off_cc, off_err, total;
  long long ldA, M;   // score row stride, keys scored per chunk
  int nsort;          // sort chunks per head
};
static bool ivf_build_layout(int B, int Hkv, long long N, int d, int nlist, IvfBuildLayout &L) {
  if (B < 1 || Hkv < 1 || N < 1 || (d != 64 && d != 128) || nlist < 1 || nlist > 4096) return false;
  if (N >= (1LL << 31) - 1) return false;
  const size_t BH = static_cast<size_t>(B) * Hkv;
  L.ldA = round4(nlist);
  // keys per score chunk: a multiple of the 128-row score tile, at least one tile
  const long long per_row = static_cast<long long>(BH) * L.ldA * 4;
  long long M = static_cast<long long>(kIvfScoreBytes) / per_row / 128 * 128;
  if (M < 128) M = 128;
  L.M = std::min<long long>(M, N);
  L.nsort = static_cast<int>((N + kIvfSortChunk - 1) / kIvfSortChunk);
  size_t off = 0;
  L.off_A = off;      off = align_up(off + BH * L.M * L.ldA * 4);
  L.off_assign = off; off = align_up(off + BH * N * 4);
  L.off_cc = off;     off = align_up(off + BH * L.nsort * nlist * 4);
  L.off_err = off;    off = align_up(off + 4);
  L.total = off;
  return true;
}

size_t ra_ivf_build_workspace_bytes(int32_t B, int32_t Hkv, int64_t N, int32_t d, int32_t nlist) {
  IvfBuildLayout L{};
  return ivf_build_layout(B, Hkv, N, d, nlist, L) ? L.total : 0;
}

ra_status ra_ivf_build(const ra_kv *kv, ra_ivf *ix, int32_t iters, void *ws, size_t ws_bytes,
                       ra_stream_t stream) {
  ra_status s = check_kv(kv);
  if (s != RA_OK) return s;
  if (!ix || !ix->Ksorted || !ix->pos || !ix->offsets || !ix->centroids || iters < 0) return RA_ERR_ARG;
  if (!aligned16(ix->Ksorted) || !aligned16(ix->centroids)) return RA_ERR_ARG;
  if (ix->B != kv->B || ix->Hkv != kv->Hkv || ix->d != kv->d || ix->N < 1 || ix->N > kv->N)
    return RA_ERR_SHAPE;
  IvfBuildLayout L{};
  if (!ivf_build_layout(kv->B, kv->Hkv, ix->N, kv->d, ix->nlist, L)) return RA_ERR_SHAPE;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0 || ws_bytes < L.total)
    return RA_ERR_WORKSPACE;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  IvfParams p{};
  p.K = static_cast<const __nv_bfloat16 *>(kv->K);
  p.cent = static_cast<__nv_bfloat16 *>(ix->centroids);
  p.A = reinterpret_cast<const float *>(at(ws, L.off_A));
  p.assign = reinterpret_cast<int32_t *>(at(ws, L.off_assign));
  p.chunk_cnt = reinterpret_cast<uint32_t *>(at(ws, L.off_cc));
  p.offsets = ix->offsets;
  p.pos = ix->pos;
  p.Ksorted = static_cast<__nv_bfloat16 *>(ix->Ksorted);
  p.N = ix->N; p.cap = kv->cap; p.ldA = L.ldA;
  p.BH = kv->B * kv->Hkv; p.nlist = ix->nlist; p.d = kv->d; p.nsort = L.nsort;
  // the key-centroid scores of a chunk of keys: those keys as the query rows of the
  // tensor-core score kernel, the centroids as its keys
  PfParams f{};
  f.K = p.cent;
  f.S = reinterpret_cast<float *>(at(ws, L.off_A));
  f.err = reinterpret_cast<uint32_t *>(at(ws, L.off_err));
  f.N = ix->nlist; f.cap = ix->nlist; f.ldS = L.ldA; f.q_plane_rows = kv->cap;
  f.B = kv->B; f.Hq = kv->Hkv; f.Hkv = kv->Hkv; f.G = 1;
  f.scale = 1.0f;
  cudaError_t e = cudaMemsetAsync(at(ws, L.off_err), 0, 4, cs);
  if (e == cudaSuccess) e = launch_ivf_init(p, cs);
  for (int it = 0; it <= iters && e == cudaSuccess; ++it) {
    for (long long c0 = 0; c0 < ix->N && e == cudaSuccess; c0 += L.M) {
      const long long m = std::min<long long>(L.M, ix->N - c0);
      f.Q = static_cast<const __nv_bfloat16 *>(kv->K) + c0 * kv->d;
      f.M = static_cast<int>(m);
      e = launch_prefill_score(f, kv->d, cs);
      p.c0 = c0;
      p.M = m;
      if (e == cudaSuccess) e = launch_ivf_assign(p, cs);
    }
    if (e == cudaSuccess) e = launch_ivf_sort(p, it == iters, cs);
    if (e == cudaSuccess && it < iters) e = launch_ivf_update(p, cs);
  }
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "ivf_build");
}

struct IvfSearchLayout {
  Step st;                  // the selection's plan over candidate rows of up to N entries
  size_t off_Sfull, off_poscand, off_probe, off_candoff, off_ncand, total;
};
static bool ivf_search_layout(int B, int Hq, long long N, int d, int k, int nprobe,
                              IvfSearchLayout &L) {
  if (nprobe < 1 || nprobe > 64) return false;
  if (plan_shape(B, Hq, Hq, N, d, k, 0, 0, L.st) != RA_OK) return false;
  const size_t R = static_cast<size_t>(B) * Hq;
  size_t off = L.st.total;
  L.off_Sfull = off;   off = align_up(off + R * L.st.ldS * 4);
  L.off_poscand = off; off = align_up(off + R * L.st.ldS * 4);
  L.off_probe = off;   off = align_up(off + R * nprobe * 4);
  L.off_candoff = off; off = align_up(off + R * (nprobe + 1) * 4);
  L.off_ncand = off;   off = align_up(off + R * 4);
  L.total = off;
  return true;
}

size_t ra_ivf_search_workspace_bytes(int32_t B, int32_t Hq, int64_t N, int32_t d, int32_t k,
                                     int32_t nprobe) {
  IvfSearchLayout L{};
  return ivf_search_layout(B, Hq, N, d, k, nprobe, L) ? L.total : 0;
}

ra_status ra_ivf_decode_step(const ra_kv *kv, const ra_ivf *ix, const void *q, int32_t Hq,
                             int32_t k, int32_t nprobe, int32_t n_sink, int32_t n_window,
                             float *out, int32_t *idx, void *ws, size_t ws_bytes,
                             ra_stream_t stream) {
  ra_status s = check_kv(kv);
  if (s != RA_OK) return s;
  if (!ix || !ix->Ksorted || !ix->pos || !ix->offsets || !ix->centroids) return RA_ERR_ARG;
  if (!aligned16(ix->Ksorted) || !aligned16(ix->centroids)) return RA_ERR_ARG;
  if (ix->B != kv->B || ix->Hkv != kv->Hkv || ix->d != kv->d) return RA_ERR_SHAPE;
  if (nprobe < 1 || nprobe > 64 || nprobe > ix->nlist || ix->nlist > 4096) return RA_ERR_ARG;
  if (ix->N < 1 || ix->N > kv->N || kv->N - ix->N > n_window) return RA_ERR_ARG;
  Step dec{};   // the step's own geometry (W, C, the attention)
  s = plan_step(kv, Hq, k, n_sink, n_window, ws, ws_bytes, dec);
  if (s != RA_OK && s != RA_ERR_WORKSPACE) return s;
  IvfSearchLayout L{};
  if (!ivf_search_layout(kv->B, Hq, kv->N, kv->d, k, nprobe, L)) return RA_ERR_SHAPE;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0 || ws_bytes < L.total)
    return RA_ERR_WORKSPACE;
  if (!q || !aligned16(q) || !out || !aligned16(out)) return RA_ERR_ARG;
  if (k > 0 && (!idx || !aligned16(idx))) return RA_ERR_ARG;
  // one cluster size for the selection and the attention, sized for the expected candidates
  // (twice the probed clusters' mean share; rows with more take longer chunks) and grown until
  // a CTA attends over at most 256 entries of U
  const long long expect = std::min<long long>(
      ix->N, std::max<long long>(4096, 2 * ix->N * nprobe / ix->nlist));
  int ncl = select_cluster_size(expect, dec.R, dec.d);
  const long long nU = dec.nW + std::min<long long>(k, expect);
  while (ncl < 8 && nU > 256LL * ncl) ncl *= 2;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  IvfSearchParams v{};
  v.q = static_cast<const __nv_bfloat16 *>(q);
  v.K = static_cast<const __nv_bfloat16 *>(kv->K);
  v.Ksorted = static_cast<const __nv_bfloat16 *>(ix->Ksorted);
  v.cent = static_cast<const __nv_bfloat16 *>(ix->centroids);
  v.pos = ix->pos;
  v.offsets = ix->offsets;
  v.probe = reinterpret_cast<int32_t *>(at(ws, L.off_probe));
  v.cand_off = reinterpret_cast<int32_t *>(at(ws, L.off_candoff));
  v.n_cand = reinterpret_cast<int32_t *>(at(ws, L.off_ncand));
  v.S = reinterpret_cast<float *>(at(ws, L.off_Sfull));
  v.S_cand = reinterpret_cast<float *>(at(ws, L.st.off_S));
  v.pos_cand = reinterpret_cast<int32_t *>(at(ws, L.off_poscand));
  v.N = ix->N; v.cap = kv->cap; v.ldS = L.st.ldS; v.ldC = L.st.ldS;
  v.s1 = dec.s1; v.w0 = dec.w0; v.nW = dec.nW;
  v.R = dec.R; v.Hq = Hq; v.Hkv = kv->Hkv; v.G = Hq / kv->Hkv; v.d = kv->d;
  v.nlist = ix->nlist; v.nprobe = nprobe; v.k = k;
  v.scale = 1.0f / sqrtf(static_cast<float>(kv->d));
  cudaError_t e = launch_ivf_probe(v, cs);
  if (e == cudaSuccess) e = launch_ivf_cand(v, kv->d, cs);
  if (e != cudaSuccess) return cuda_fail(e, "ivf_search");
  // the exact top-k of each row's candidates (idx: their cache positions), then softmax
  // attention over W u Omega from the full-length score rows; one launch unless the attention
  // wants more clusters per head than the selection has
  SaParams p{};
  p.S = v.S_cand;
  p.S_att = v.S;
  p.pos_map = v.pos_cand;
  p.row_n = v.n_cand;
  p.hist = reinterpret_cast<uint32_t *>(at(ws, L.st.off_hist));
  p.list = reinterpret_cast<unsigned long long *>(at(ws, L.st.off_list));
  p.V = static_cast<const __nv_bfloat16 *>(kv->V);
  p.idx = idx;
  p.out = out;
  p.part = reinterpret_cast<float *>(at(ws, L.st.off_part));
  p.meta = reinterpret_cast<uint32_t *>(at(ws, L.st.off_meta));
  p.err = reinterpret_cast<uint32_t *>(at(ws, L.st.off_meta)) + kError;
  p.ldS = L.st.ldS; p.ldL = L.st.ldL; p.cap = kv->cap; p.N = dec.N;
  p.s1 = dec.s1; p.w0 = dec.w0; p.nW = dec.nW; p.nC = dec.nC; p.k_eff = dec.k_eff;
  p.cbase = dec.cbase; p.cper = dec.cper;
  p.k = k; p.Hq = Hq; p.G = dec.G; p.Hkv = dec.Hkv;
  if (k > 0) p.sel_z = reinterpret_cast<float *>(at(ws, L.st.off_selz));
  const int split = attn_split(nU, dec.R, ncl, dec.d);
  if (k > 0) {
    p.mode = kSaSelect | kSaBuildHist | (split == 1 ? kSaAttend : 0);
    p.nsplit = 1;
    e = launch_select_attend(p, kv->d, dec.R, ncl, cs);
    if (e != cudaSuccess) return cuda_fail(e, "ivf_select_attend");
    if (split == 1) return RA_OK;
  }
  p.mode = kSaAttend;
  p.nsplit = split;
  e = launch_select_attend(p, kv->d, dec.R, ncl, cs);
  return e == cudaSuccess ? RA_OK : cuda_fail(e, "ivf_attend");
}

}  // extern "C"
