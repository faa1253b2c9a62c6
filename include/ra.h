/*
 * ra.h -- C ABI of libra: exact top-k retrieval attention for one decode step on B200.
 *
 * The operation is the decode step of RetrievalAttention ("RetrievalAttention:
 * Accelerating Long-Context LLM Inference via Vector Retrieval", arXiv 2409.10516v3 slides):
 *
 *   z_i = q_t k_i^T / sqrt(d)                          slide "Sparse attention renormalizes
 *                                                       selected tokens", Eq. (1)
 *   W   = first n_sink tokens + last n_window tokens    slide "The GPU keeps 640 fixed
 *                                                       positions" (128 + 512 there)
 *   C   = [0, N) \ W;  Omega = the k largest z in C     same slide: W and Omega disjoint,
 *                                                       a fixed top-k budget, one index
 *                                                       per query head under GQA
 *   o   = softmax over U = W u Omega of z, times v      Eq. (2) renormalised over U, computed
 *                                                       as split partial states merged by
 *                                                       Eqs. (3)-(5) (slide "Two local softmax
 *                                                       outputs need global weights")
 *
 * Retrieval here is exact (a full scan of K in HBM), not the slides' CPU-side ANN index.
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller owns every buffer (device memory unless stated).  The library
 *     allocates nothing; the only state carried between calls is the zeroed counter block at
 *     the front of a workspace (see ra_decode_step).
 *   - Ordering: all work is enqueued on `stream` (a cudaStream_t, may be NULL for the legacy
 *     default stream); no call synchronises the host.  Results are valid once the stream
 *     reaches that point.
 *   - Errors: arguments are validated on the host before anything is enqueued; on any error
 *     status nothing has been enqueued, except RA_ERR_CUDA, which reports a failed launch.
 *     No C++ exception crosses this interface.
 *   - Layouts are dense row-major.  bf16 is IEEE bfloat16 (raw 16-bit patterns).
 *   - Device pointers must be 16-byte aligned.
 */
#ifndef RA_H
#define RA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t is `struct CUstream_st *`; declared here so the header needs no CUDA headers. */
struct CUstream_st;
typedef struct CUstream_st *ra_stream_t;

typedef enum {
  RA_OK = 0,
  RA_ERR_ARG = 1,        /* null or misaligned pointer, negative size or budget            */
  RA_ERR_SHAPE = 2,      /* unsupported shape: d not 64/128, Hq % Hkv != 0, G > 8, N > cap */
  RA_ERR_CAPACITY = 3,   /* append would exceed the cache capacity                         */
  RA_ERR_WORKSPACE = 4,  /* ws is NULL or ws_bytes is below the required size              */
  RA_ERR_CUDA = 5,       /* a CUDA call or kernel launch failed                            */
  RA_ERR_EMPTY = 6       /* empty selected union (N == 0, or W empty and k == 0)           */
} ra_status;

/*
 * A per-layer KV cache resident in device memory.
 *   K, V : bf16 [B, Hkv, cap, d], device, caller-owned.  Row (b, g, i) holds key/value i of
 *          KV head g of sequence b.
 *   B    : sequences (batch), >= 1.       Hkv : KV heads, >= 1.
 *   d    : head dimension, 64 or 128.     cap : rows allocated per (b, g), >= N.
 *   N    : tokens currently cached (host-side; ra_append_kv advances it).
 */
typedef struct {
  void *K;
  void *V;
  int32_t B, Hkv, d, cap;
  int64_t N;
} ra_kv;

/*
 * A per-layer KV cache in pages (the serving layout: sequences of different lengths share one
 * pool of fixed-size pages, a block table maps each sequence's token i to its page).
 *   K, V        : bf16 page pools [num_pages, Hkv, 128, d], device, caller-owned.  Token i of
 *                 sequence b, KV head g, is row i % 128 of page block_table[b * max_pages +
 *                 i / 128] (pool row (page * Hkv + g) * 128 + i % 128).
 *   block_table : int32 [B, max_pages], device, caller-owned; entries for the pages a
 *                 sequence uses must be valid page indices (< num_pages).
 *   seq_len     : int32 [B], HOST, caller-owned: tokens cached per sequence (>= 1 for a decode
 *                 step, <= max_pages * 128); ra_paged_append_kv advances it.
 *   B <= 256, d 64 or 128.
 */
typedef struct {
  void *K;
  void *V;
  const int32_t *block_table;
  int32_t *seq_len;
  int32_t B, Hkv, d, max_pages, num_pages;
} ra_paged_kv;

/* Human-readable name of a status (static string). */
const char *ra_status_str(ra_status s);

/* Library version string (static). */
const char *ra_version(void);

/* Detail of the last RA_ERR_CUDA on the calling thread, or of a refused first call of
 * ra_decode_step_static inside a stream capture (static thread-local string). */
const char *ra_last_error(void);

/*
 * Append T new tokens: K[b, g, N + t, :] = k_new[b, g, t, :] (same for V), then kv->N += T.
 * Eq. (1)'s sum runs over j <= t, so the current token is appended before the decode step.
 *   k_new, v_new : bf16 [B, Hkv, T, d], device.   T >= 0 (T == 0 is a no-op).
 * Errors: RA_ERR_ARG (null kv/pointers, T < 0), RA_ERR_CAPACITY (N + T > cap; kv unchanged).
 */
ra_status ra_append_kv(ra_kv *kv, const void *k_new, const void *v_new, int32_t T,
                       ra_stream_t stream);

/*
 * Workspace bytes that ra_decode_step (and its three phases) need for this shape.
 * Returns 0 for an invalid shape.  The size grows with B*Hq*N (the fp32 scores).
 */
size_t ra_decode_workspace_bytes(int32_t B, int32_t Hq, int64_t N, int32_t d, int32_t k,
                                 int32_t n_sink, int32_t n_window);

/*
 * One decode step of exact top-k retrieval attention (all four parts above).
 *   kv       : cache of this layer (N >= 1).
 *   q        : bf16 [B, Hq, d], device.  Query head h reads KV head h / (Hq / Hkv).
 *   Hq       : query heads; Hq % Hkv == 0 and G = Hq / Hkv <= 8.
 *   k        : retrieval budget per query head (>= 0); clamped to |C|, so k >= N is legal
 *              and makes the step full attention.
 *   n_sink   : leading tokens always attended (>= 0).
 *   n_window : trailing tokens always attended (>= 0).  The two ranges may overlap.
 *   out      : float32 [B, Hq, d], device: the attention output.
 *   idx      : int32 [B, Hq, k], device (may be NULL only when k == 0): Omega, the retrieved
 *              positions of each query head, in unspecified order (a set); entries past
 *              min(k, |C|) are -1.  Ties in score go to the lower position.
 *   ws       : device workspace of at least ra_decode_workspace_bytes(...) bytes, 256-byte
 *              aligned, zero-filled once before its first use (cudaMemsetAsync(ws, 0, n)).
 *              It starts with a counter block (per query head: a 2048-bin histogram and 8
 *              counters) whose place depends on B*Hq only; every completed call leaves that
 *              block zero again, so one workspace serves any later call with the same B*Hq
 *              (N may grow; the dense path's workspace follows the same rule).
 * Errors: RA_ERR_ARG, RA_ERR_SHAPE, RA_ERR_EMPTY (N == 0), RA_ERR_WORKSPACE, RA_ERR_CUDA.
 * Calls that share one workspace must not overlap on the device.
 */
ra_status ra_decode_step(const ra_kv *kv, const void *q, int32_t Hq, int32_t k, int32_t n_sink,
                         int32_t n_window, float *out, int32_t *idx, void *ws, size_t ws_bytes,
                         ra_stream_t stream);

/*
 * Append one token and run the decode step over the grown cache, with the append done inside
 * the scan instead of as a launch of its own: ra_append_kv(kv, k_new, v_new, 1) followed by
 * ra_decode_step, with the same results.  The CTA of the score kernel whose tile holds the new
 * position writes the token's K and V rows to the cache and scores the key from its staged
 * tile (Eq. (1) sums over j <= t: the current token is attended, here through the window).
 *   k_new, v_new : bf16 [B, Hkv, 1, d], device, 16-byte aligned.
 *   Other arguments as ra_decode_step; the workspace is sized for kv->N + 1 tokens.
 * On success kv->N has grown by one.  Errors: as ra_decode_step, checked before any launch
 * (kv unchanged); RA_ERR_CAPACITY when kv->N + 1 > cap.
 */
ra_status ra_decode_step_append(ra_kv *kv, const void *q, const void *k_new, const void *v_new,
                                int32_t Hq, int32_t k, int32_t n_sink, int32_t n_window,
                                float *out, int32_t *idx, void *ws, size_t ws_bytes,
                                ra_stream_t stream);
/*
 * ra_decode_step_append for a caller whose step inputs and outputs live in host memory: the
 * query and the token's K / V rows are copied from host memory into the caller's device
 * staging buffers, the step runs, and out and idx are copied back, all enqueued on `stream`
 * (one cudaMemcpyAsync per buffer); nothing waits on the host, so the caller synchronises
 * `stream` before reading out_host / idx_host.  Host buffers should be pinned (page-locked)
 * for the copies to be asynchronous.
 *   dev : device staging of the step's inputs and outputs (shapes and alignment as
 *         ra_decode_step_append's q, k_new, v_new, out, idx), caller-owned.
 *   q_host bf16 [B, Hq, d]; k_new_host, v_new_host bf16 [B, Hkv, 1, d]; out_host fp32
 *   [B, Hq, d]; idx_host int32 [B, Hq, k] (may be null when k = 0).
 * Errors: as ra_decode_step_append, checked before anything is enqueued; RA_ERR_ARG for a
 * null host pointer; RA_ERR_CUDA if a copy cannot be enqueued.
 */
typedef struct {
  void *q, *k_new, *v_new;
  float *out;
  int32_t *idx;
} ra_step_io;
ra_status ra_decode_step_append_host(ra_kv *kv, const void *q_host, const void *k_new_host,
                                     const void *v_new_host, int32_t Hq, int32_t k,
                                     int32_t n_sink, int32_t n_window, float *out_host,
                                     int32_t *idx_host, const ra_step_io *dev, void *ws,
                                     size_t ws_bytes, ra_stream_t stream);

/*
 * Kernel launches that ra_decode_step (or ra_decode_step_append) makes for this shape: 2 (the
 * scan, then the selection fused with the attention) or 3 (the attention split across several
 * clusters per head, as a launch of its own).  Host only; it queries the current device's
 * occupancy like the step itself.  -1 for a shape the step rejects.
 */
int32_t ra_decode_step_launches(int32_t B, int32_t Hq, int32_t Hkv, int64_t N, int32_t d,
                                int32_t k, int32_t n_sink, int32_t n_window);

/* The scan phase of ra_decode_step_append alone (then ra_select_attend over the grown kv). */
ra_status ra_score_gqa_append(ra_kv *kv, const void *q, const void *k_new, const void *v_new,
                              int32_t Hq, int32_t k, int32_t n_sink, int32_t n_window, void *ws,
                              size_t ws_bytes, ra_stream_t stream);

/*
 * ra_decode_step with the retrieval set cut at a softmax-weight threshold (Eq. (2), slide
 * "Sparse attention renormalizes selected tokens"): Omega = the candidates i of C whose full
 * softmax weight a_i = e^{z_i} / sum_{j < N} e^{z_j} exceeds eps, the k largest of them when
 * more than k pass (k is the budget cap).  U = W u Omega as in ra_decode_step.
 *   eps : 0 < eps < 1.   idx : entries past |Omega| are -1 (|Omega| <= min(k, |C|)).
 *   ws  : the ra_decode_workspace_bytes(...) workspace of the same k.
 * Errors: as ra_decode_step; RA_ERR_ARG for eps outside (0, 1); RA_ERR_EMPTY when W is empty
 * (the threshold may keep no key at all).
 */
ra_status ra_decode_step_eps(const ra_kv *kv, const void *q, int32_t Hq, int32_t k, float eps,
                             int32_t n_sink, int32_t n_window, float *out, int32_t *idx,
                             void *ws, size_t ws_bytes, ra_stream_t stream);

/*
 * Per-layer retrieval budgets in the PyramidKV style (slide "Extra experiments show where
 * budget matters": an adaptive layer budget): k_out[l], l < L, falls linearly from k_max at
 * layer 0 to ratio * k_max at layer L - 1 with mean k_mean (k_max = 2 k_mean / (1 + ratio)),
 * each rounded down and the remainder given one each to the lowest layers, so that the budgets
 * sum to exactly L * k_mean.  Host only (no device work).  Pass k_out[l] as layer l's k.
 *   ratio in (0, 1] (1: every layer gets k_mean).   k_out: int32 [L], host, caller-owned.
 * Errors: RA_ERR_ARG.
 */
ra_status ra_pyramid_budgets(int32_t L, int32_t k_mean, double ratio, int32_t *k_out);

/*
 * The decode step on a paged cache (ragged sequence lengths): per sequence b, exactly
 * ra_decode_step over its seq_len[b] tokens (its own W, C and min(k, |C|)).
 *   ra_paged_append_kv : token seq_len[b] + t of every sequence from k_new / v_new [B, Hkv, T, d]
 *                        (bf16, device), then seq_len[b] += T on the host.  The pages must
 *                        already be in the block table.  RA_ERR_CAPACITY past max_pages * 128.
 *   ra_paged_workspace_bytes : the workspace of the longest sequence (max_N = max seq_len).
 *   ra_paged_decode_step : q [B, Hq, d], out [B, Hq, d] fp32, idx [B, Hq, k] (-1 past each
 *                        sequence's min(k, |C|)), ws as in ra_decode_step (zero-filled once).
 * Errors: as ra_decode_step; RA_ERR_SHAPE for B > 256 or a length outside [1, max_pages * 128].
 */
ra_status ra_paged_append_kv(ra_paged_kv *kv, const void *k_new, const void *v_new, int32_t T,
                             ra_stream_t stream);
size_t ra_paged_workspace_bytes(int32_t B, int32_t Hq, int64_t max_N, int32_t d, int32_t k,
                                int32_t n_sink, int32_t n_window);
ra_status ra_paged_decode_step(const ra_paged_kv *kv, const void *q, int32_t Hq, int32_t k,
                               int32_t n_sink, int32_t n_window, float *out, int32_t *idx,
                               void *ws, size_t ws_bytes, ra_stream_t stream);

/*
 * The phases of ra_decode_step, exposed so a caller can time or interleave them.  All take the
 * arguments of ra_decode_step and the same workspace, and must run as one of the complete
 * sequences  ra_score_gqa, ra_select_attend  (which is ra_decode_step)  or
 * ra_score_gqa, ra_topk_select, ra_sparse_attn  (ra_topk_select re-zeroes what ra_score_gqa
 * counted).
 *   ra_score_gqa     : z for every (query head, position) into ws, plus the per-head score
 *                      histogram of the candidates (one pass over K per KV head).
 *   ra_topk_select   : Omega into idx from the scores in ws (radix select over the histogram,
 *                      bitonic finish).
 *   ra_sparse_attn   : out from the scores in ws, the V rows of U = W u Omega (Omega read from
 *                      idx), and the merge of the split partial states (Eqs. (3)-(5)).
 *   ra_select_attend : ra_topk_select then ra_sparse_attn in one launch.
 */
ra_status ra_score_gqa(const ra_kv *kv, const void *q, int32_t Hq, int32_t k, int32_t n_sink,
                       int32_t n_window, void *ws, size_t ws_bytes, ra_stream_t stream);
ra_status ra_topk_select(const ra_kv *kv, int32_t Hq, int32_t k, int32_t n_sink,
                         int32_t n_window, int32_t *idx, void *ws, size_t ws_bytes,
                         ra_stream_t stream);
ra_status ra_sparse_attn(const ra_kv *kv, int32_t Hq, int32_t k, int32_t n_sink,
                         int32_t n_window, const int32_t *idx, float *out, void *ws,
                         size_t ws_bytes, ra_stream_t stream);
ra_status ra_select_attend(const ra_kv *kv, int32_t Hq, int32_t k, int32_t n_sink,
                           int32_t n_window, int32_t *idx, float *out, void *ws, size_t ws_bytes,
                           ra_stream_t stream);

/*
 * ra_decode_step without a caller workspace, for callers that cannot allocate device memory
 * (for example a plugin that its host engine hands only input and output pointers, or a serving
 * loop that bans cudaMalloc after start-up because it can synchronise the device).  The paper
 * has no counterpart: this is a packaging variant of ra_decode_step.
 *   Arguments, outputs and errors are those of ra_decode_step, without ws / ws_bytes.
 *   Scratch: a 64 MiB array inside libra (a file-scope __device__ array), held on every GPU
 *     that loads the library until the process exits.  A shape whose
 *     ra_decode_workspace_bytes(...) exceeds 64 MiB is rejected with RA_ERR_WORKSPACE before
 *     anything is enqueued (the 128K Llama-3-8B layer, 32 query heads, needs about 48 MiB).
 *   The first call on each device looks up the array's device address (cudaGetSymbolAddress
 *     with that device current); make that first call before any stream capture.  A first
 *     call on a capturing stream is refused with RA_ERR_ARG (ra_last_error() says why) and
 *     enqueues nothing.  Host threads may make first calls concurrently.
 *   Each call clears the scratch's counter block with cudaMemsetAsync on `stream`; nothing is
 *     allocated.  All calls on a device share the one array and it keeps the last call's
 *     contents, so calls that overlap on the GPU (other streams, other host threads) race.
 */
ra_status ra_decode_step_static(const ra_kv *kv, const void *q, int32_t Hq, int32_t k,
                                int32_t n_sink, int32_t n_window, float *out, int32_t *idx,
                                ra_stream_t stream);

/*
 * Exact top-k of a batch of prefill queries: for every query row (b, h, m) of q, Omega = the
 * min(k, |C|) largest z_i = q[b,h,m] . K[b,h/G,i] / sqrt(d) over the candidates C = [0,N) \ W,
 * ties to the lower position (the decode step's selection, one query at a time; no causal mask).
 * These are the nearest-key lists the slides build the query-aware index from (slide
 * "Prefill queries teach the key graph what matters": prefill queries and their top-k keys,
 * found on the GPU).  With G * M query
 * rows per KV head the scores are a dense contraction, computed on the tcgen05 tensor cores
 * (bf16 x bf16 -> fp32 in tensor memory).
 *   q   : bf16 [B, Hq, M, d], device.   M >= 1, B * M <= 65535.
 *   idx : int32 [B, Hq, M, k], device (may be NULL only when k == 0); entries past
 *         min(k, |C|) are -1; order within a row unspecified.
 *   ws  : at least ra_prefill_workspace_bytes(...) bytes, 256-byte aligned (no zero-fill
 *         needed).  It holds the fp32 scores of every query row (B * Hq * M * N * 4 bytes).
 * The two phases ra_prefill_score (scores into ws) and ra_prefill_select (idx from ws), run in
 * that order with the same arguments, are ra_prefill_topk.
 * Errors: RA_ERR_ARG, RA_ERR_SHAPE, RA_ERR_EMPTY (N == 0), RA_ERR_WORKSPACE, RA_ERR_CUDA.
 */
size_t ra_prefill_workspace_bytes(int32_t B, int32_t Hq, int32_t M, int64_t N, int32_t d,
                                  int32_t k, int32_t n_sink, int32_t n_window);
ra_status ra_prefill_topk(const ra_kv *kv, const void *q, int32_t Hq, int32_t M, int32_t k,
                          int32_t n_sink, int32_t n_window, int32_t *idx, void *ws,
                          size_t ws_bytes, ra_stream_t stream);
ra_status ra_prefill_score(const ra_kv *kv, const void *q, int32_t Hq, int32_t M, int32_t k,
                           int32_t n_sink, int32_t n_window, void *ws, size_t ws_bytes,
                           ra_stream_t stream);
ra_status ra_prefill_select(const ra_kv *kv, int32_t Hq, int32_t M, int32_t k, int32_t n_sink,
                            int32_t n_window, int32_t *idx, void *ws, size_t ws_bytes,
                            ra_stream_t stream);

/*
 * Device-side approximate retrieval: an inverted-file (IVF) index of one layer's keys (the
 * pages' IVF baseline over the keys, probed with the decode query; slide "Available GPU memory
 * changes the comparison"), built and searched on the GPU.  Not exact: a key of a cluster that
 * is not probed is never retrieved.
 *   Ksorted   : bf16 [B, Hkv, N, d], the keys ordered by cluster.
 *   pos       : int32 [B, Hkv, N], the cache position of each sorted key.
 *   offsets   : int32 [B, Hkv, nlist + 1], cluster c's keys are sorted entries
 *               [offsets[c], offsets[c + 1]).
 *   centroids : bf16 [B, Hkv, nlist, d], unit-norm (spherical k-means: keys are assigned to the
 *               centroid of largest inner product, ties to the lower index).
 *   All device, caller-owned.  N is the number of keys indexed; 1 <= nlist <= 4096.
 */
typedef struct {
  void *Ksorted;
  int32_t *pos;
  int32_t *offsets;
  void *centroids;
  int32_t B, Hkv, d, nlist;
  int64_t N;
} ra_ivf;

/*
 * Build the index of kv's first ix->N keys (ix->N <= kv->N; B, Hkv, d as kv's): `iters` Lloyd
 * iterations of spherical k-means from centroids at the unit keys of positions
 * floor(c * N / nlist) (the key-centroid scores on the tcgen05 tensor cores, an empty cluster
 * keeping its centroid, each centroid the unit direction of its keys' sum rounded to bf16),
 * then the final assignment and the sort by cluster, keys of a cluster in increasing position.
 * Deterministic: the same cache gives the same index bit for bit (integer counts, a stable
 * sort, sums in position order).  The key-centroid scores are computed over chunks of keys, so
 * the workspace is about 256 MB plus 4 * B * Hkv * (N + nlist * ceil(N / 1024)) bytes at any N
 * (the 256 MB score block grows to one 128-key tile, B * Hkv * nlist * 512 bytes, if that is larger).
 *   ws : at least ra_ivf_build_workspace_bytes(...) bytes, 256-byte aligned (no zeroing needed).
 * Errors: RA_ERR_ARG, RA_ERR_SHAPE, RA_ERR_WORKSPACE, RA_ERR_CUDA.
 */
size_t ra_ivf_build_workspace_bytes(int32_t B, int32_t Hkv, int64_t N, int32_t d, int32_t nlist);
ra_status ra_ivf_build(const ra_kv *kv, ra_ivf *ix, int32_t iters, void *ws, size_t ws_bytes,
                       ra_stream_t stream);

/*
 * A decode step that retrieves through the index: per query head, the nprobe clusters whose
 * centroids score highest (ties to the lower cluster), the exact top-k of their keys outside W,
 * and softmax attention over W u Omega as ra_decode_step.  Keys of equal score are taken in
 * candidate order (probe order, then the order inside a cluster), not by position.  Keys
 * appended after the build are only attended through the window: kv->N - ix->N <= n_window is
 * required.  Three launches: the centroid probe, the candidate scores, and the selection fused
 * with the attention (a fourth when the attention is split across several clusters per head).
 *   nprobe : 1 <= nprobe <= min(nlist, 64).
 *   idx    : int32 [B, Hq, k], cache positions; -1 in slots that retrieve nothing (when the
 *            probed clusters hold fewer than k keys outside W).
 *   ws     : at least ra_ivf_search_workspace_bytes(...) bytes, 256-byte aligned, zero-filled
 *            once (it holds a decode workspace's counter block).
 * Errors: as ra_decode_step; RA_ERR_ARG for nprobe or an index that does not cover the cache.
 */
size_t ra_ivf_search_workspace_bytes(int32_t B, int32_t Hq, int64_t N, int32_t d, int32_t k,
                                     int32_t nprobe);
ra_status ra_ivf_decode_step(const ra_kv *kv, const ra_ivf *ix, const void *q, int32_t Hq,
                             int32_t k, int32_t nprobe, int32_t n_sink, int32_t n_window,
                             float *out, int32_t *idx, void *ws, size_t ws_bytes,
                             ra_stream_t stream);

/* Workspace bytes for ra_dense_decode (split partial states).  0 for an invalid shape. */
size_t ra_dense_workspace_bytes(int32_t B, int32_t Hq, int64_t N, int32_t d);

/*
 * Full attention over all N cached tokens (Eq. (1)): the dense flash-decode comparison path.
 *   q : bf16 [B, Hq, d], device.   out : float32 [B, Hq, d], device.
 *   ws: at least ra_dense_workspace_bytes(...) bytes, 256-byte aligned, zero-filled once
 *       before first use (same counter-block rule as ra_decode_step).
 * Errors: as ra_decode_step.
 */
ra_status ra_dense_decode(const ra_kv *kv, const void *q, int32_t Hq, float *out, void *ws,
                          size_t ws_bytes, ra_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RA_H */
