// Kernel parameter blocks and host-side launchers of libra (internal, not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace ra {

// Launches `kernel` on `s` with programmatic stream serialisation allowed, so it may be
// scheduled while its predecessor in the stream is still finishing (it synchronises with
// griddepcontrol.wait before reading the predecessor's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Scores of every (query head, position) of one layer, plus the first radix digit's
// histogram of the candidates (z in S is already scaled by 1/sqrt(d)).
struct ScoreParams {
  const __nv_bfloat16 *K;   // [B, Hkv, cap, d]
  const __nv_bfloat16 *q;   // [B, Hq, d]
  float *S;                 // [B*Hq, ldS]
  uint32_t *hist;           // [B*Hq, kHistBins] (zeroed before the launch)
  long long N, cap, ldS;
  long long cand_lo, cand_hi;   // candidates are positions in [cand_lo, cand_hi)
  long long tiles_per_head;
  long long total_tiles;
  int B, Hkv, G, Hq;
  float scale;
  int do_hist;
  uint32_t *err;            // error word (bit kErrScoreWait: a load never landed)
  // Appending the step's token inside the scan (dense caches; all null otherwise): position
  // N - 1 of every head is the new token, whose K / V rows ([B * Hkv, d]) the CTA scanning
  // that tile writes to the cache and patches into its staged tile before scoring it.
  const __nv_bfloat16 *k_new, *v_new;
  __nv_bfloat16 *K_cache, *V_cache;
  // Completion counters (null: none): when a CTA is done with every tile of the head bg that it
  // scores, it adds 1 to ready[bg * ready_stride] (after its score and histogram writes of that
  // head are visible device-wide), so a kernel running concurrently can start on that head.
  uint32_t *ready;
  long long ready_stride;
};

// Paged KV caches: K and V in pages of kPageSize tokens, [num_pages, Hkv, kPageSize, d]; sequence
// b's token i lives in page block_table[b * max_pages + i / kPageSize].  The lengths travel in
// the kernels' parameter blocks (at most kMaxPagedBatch sequences per call).
constexpr int kPageSize = 128;
constexpr int kMaxPagedBatch = 256;
struct PagedInfo {
  const int32_t *block_table;               // [B, max_pages], device
  int max_pages, n_sink, n_window, k;
  int32_t seq_len[kMaxPagedBatch];          // tokens of sequence b
  int32_t tile_off[kMaxPagedBatch + 1];     // score tiles before sequence b (all its KV heads)
};
struct NoPaging {};   // the dense [B, Hkv, cap, d] layout

// Top-k selection and sparse attention of one decode step, one thread-block cluster per query
// head (row = b * Hq + h).  mode: kSaSelect writes idx from the scores; kSaAttend computes out
// from the scores, idx and V; both in one launch for the decode step.
constexpr int kSaSelect = 1;
constexpr int kSaAttend = 2;
constexpr int kSaBuildHist = 4;        // with kSaSelect: build the digit-1 histogram from S first
constexpr int kSaEps = 8;              // with kSaSelect: keep only keys whose softmax weight > eps
constexpr int kMaxCluster = 16;        // CTAs per query head at most
constexpr int kMaxAttnSplit = 4;       // clusters per query head in the attention-only launch
constexpr uint32_t kErrSelect = 4u;    // error bit: the selection's counts were inconsistent

struct SaParams {
  const float *S;           // [B*Hq, ldS] scores
  uint32_t *hist;           // [B*Hq, kHistBins] digit-1 histogram (left zero by the select)
  unsigned long long *list; // [B*Hq, ldL] composites (order key << 32 | ~position) of threshold-bin keys
  const __nv_bfloat16 *V;   // [B, Hkv, cap, d]
  int32_t *idx;             // [B*Hq, k]: written (select) or read (attention only)
  float *out;               // [B*Hq, d]
  float *part;              // [B*Hq, kMaxAttnSplit, d + 4] partial states of the clusters
  uint32_t *meta;           // [B*Hq, kMetaWords] counters (kDone left zero)
  uint32_t *err;            // error word
  long long ldS, ldL, cap, N;
  long long s1, w0, nW, nC, k_eff;   // W = [0, s1) u [w0, N), C = [s1, w0)
  long long cbase, cper;    // CTA r of a cluster owns candidates [cbase + r cper, + cper)
  int k, Hq, G, Hkv, mode;
  int nsplit;               // clusters per query head (grid z); > 1 only for attention alone
  float log_eps;            // kSaEps: ln(eps)
  const int32_t *row_n;     // if set: row r's candidates are [0, row_n[r]) of its score row,
                            // with no static set (the IVF candidate lists)
  const int32_t *pos_map;   // with row_n: [B*Hq, ldS] cache position of each candidate (-1: a
                            // static-set key); idx reports these positions
  const float *S_att;       // with row_n: [B*Hq, ldS] full-length score rows for the attention
  float *sel_z;             // if set: [B*Hq, k] the score of each selected entry, beside idx (the
                            // selection writes it; the attention reads it instead of the rows)
  // Overlap with the score kernel (null: none; the kernel waits for its predecessor instead):
  // the cluster of row r starts once ready[(r / G) * ready_stride] reaches ready_target (every
  // score CTA is done with that KV head), and the row group's last cluster sets it back to 0.
  uint32_t *ready;
  long long ready_stride;
  uint32_t ready_target;
};
constexpr uint32_t kErrReadyWait = 16u;   // error bit: a head's scores never became ready

// Scores of prefill queries (rows (b, h, m) of Q [B, Hq, M, d]) against the keys of their KV
// head, on the tensor cores.
struct PfParams {
  const __nv_bfloat16 *Q;   // [B, Hq, M, d]
  const __nv_bfloat16 *K;   // [B, Hkv, cap, d]
  float *S;                 // [B*Hq*M, ldS]
  uint32_t *err;            // error word (bit kErrPrefillWait: a copy or the MMAs never landed)
  long long N, cap, ldS;
  long long q_plane_rows;   // rows between KV heads' query blocks in Q (0: G * M, contiguous)
  int B, Hq, Hkv, G, M;
  float scale;
};
constexpr uint32_t kErrPrefillWait = 8u;

// IVF index build over one layer's keys (per KV head, bg = b * Hkv + g).  Every step is
// deterministic: integer counts, a stable counting sort and fixed-order sums.
constexpr int kIvfSortChunk = 1024;   // keys one warp places in the stable scatter
struct IvfParams {
  const __nv_bfloat16 *K;   // cache keys [BH, cap, d]
  __nv_bfloat16 *cent;      // [BH, nlist, d] unit-norm centroids
  const float *A;           // [BH * M, ldA] key-centroid scores of the key chunk [c0, c0 + M)
  int32_t *assign;          // [BH * N] cluster of each key
  uint32_t *chunk_cnt;      // [BH, nsort, nlist]: per sort chunk, counts, then first slots
  int32_t *offsets;         // [BH, nlist + 1]
  int32_t *pos;             // [BH, N] cache position of each sorted key
  __nv_bfloat16 *Ksorted;   // [BH, N, d] (written by the final sort)
  long long N, cap, ldA, c0, M;
  int BH, nlist, d, nsort;
};

// IVF search of one decode step (rows = b * Hq + h).
struct IvfSearchParams {
  const __nv_bfloat16 *q, *K, *Ksorted, *cent;
  const int32_t *pos, *offsets;
  int32_t *probe, *cand_off, *n_cand;   // [R, nprobe], [R, nprobe + 1], [R]
  float *S;                 // [R, ldS] full-length score rows (written at candidate and W positions)
  float *S_cand;            // [R, ldC] candidate scores (-inf: a W key)
  int32_t *pos_cand;        // [R, ldC] cache position of each candidate (-1: a W key)
  long long N, cap, ldS, ldC, s1, w0, nW;
  int R, Hq, Hkv, G, d, nlist, nprobe, k;
  float scale;
};

struct DenseParams {
  const __nv_bfloat16 *K, *V, *q;
  float *part;              // [B*Hq, nsplit, d + 4] partial states (m, Z, pad, pad, N[d])
  float *out;               // [B*Hq, d]
  uint32_t *meta;           // [B*Hq, kMetaWords] counters (left zero by the merging CTA)
  long long N, cap, keys_per_split;
  int B, Hkv, G, Hq, nsplit;
  float scale;
  uint32_t *err;            // error word (bit kErrDenseWait: a load never landed)
};

struct AppendParams {
  __nv_bfloat16 *K, *V;
  const __nv_bfloat16 *k_new, *v_new;
  long long cap, N;
  int B, Hkv, d, T;
};

// tuning constants the host layout needs
constexpr int kScoreTile = 128;
constexpr int kDenseTile = 128;

int num_sms();

// Sets the calling thread's ra_last_error() text.
void set_last_error(const char *msg);

// Bytes of the counter block at the front of every workspace for `rows` query heads (the
// digit-1 histograms, then the per-row counters), 256-byte aligned sections.
size_t counter_block_bytes(size_t rows);

// Raises a kernel's dynamic shared-memory limit once per device (so that later launches,
// including launches inside a stream capture, make no attribute call).
cudaError_t ensure_smem_limit(const void *kernel, int bytes, bool (&done)[64]);

// CTAs of a score launch over `total_tiles` tiles.
int score_grid(long long total_tiles);
// Bytes of static shared memory of one selection CTA (a score CTA leaves room for one).
size_t select_smem_bytes(int d);
// grid (optional): the launch's CTA count, the value a selection overlapping it waits for.
cudaError_t launch_score(const ScoreParams &p, int d, cudaStream_t s, int *grid = nullptr);
cudaError_t launch_score_paged(const ScoreParams &p, const PagedInfo &pg, long long num_pages, int d,
                               cudaStream_t s, int *grid = nullptr);
// Cluster size for one query head: a power of two <= kMaxCluster (16 only where the device
// schedules 16-CTA clusters of this kernel), chunks of at most 64K scores, grown to fill the GPU.
int select_cluster_size(long long nC, int R, int d);
// Clusters per query head for the attention over nU entries on its own: 1 while a CTA of one
// cluster takes at most 1024 entries, else up to kMaxAttnSplit while all clusters run in one wave.
int attn_split(long long nU, int R, int ncl, int d);
cudaError_t launch_select_attend(const SaParams &p, int d, int R, int ncl, cudaStream_t s);
cudaError_t launch_select_attend_paged(const SaParams &p, const PagedInfo &pg, int d, int R, int ncl,
                                       cudaStream_t s);
cudaError_t launch_dense(const DenseParams &p, int d, cudaStream_t s);
cudaError_t launch_prefill_score(const PfParams &p, int d, cudaStream_t s);
cudaError_t launch_ivf_init(const IvfParams &p, cudaStream_t s);
cudaError_t launch_ivf_assign(const IvfParams &p, cudaStream_t s);   // keys [c0, c0 + M)
cudaError_t launch_ivf_sort(const IvfParams &p, bool copy_rows, cudaStream_t s);
cudaError_t launch_ivf_update(const IvfParams &p, cudaStream_t s);
cudaError_t launch_ivf_probe(const IvfSearchParams &p, cudaStream_t s);
cudaError_t launch_ivf_cand(const IvfSearchParams &p, int d, cudaStream_t s);
cudaError_t launch_append(const AppendParams &p, cudaStream_t s);
cudaError_t launch_append_paged(const AppendParams &p, const PagedInfo &pg, cudaStream_t s);

}  // namespace ra
