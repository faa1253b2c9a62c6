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
};

struct TopkParams {
  const float *S;
  uint32_t *hist;           // [B*Hq, kHistBins] digit-1 histogram (left zero by the select)
  uint32_t *hist2;          // [B*Hq, kHistBins] digit-2 histogram of the listed keys (same)
  uint32_t *meta;           // [B*Hq, kMetaWords] counters (left zero by the select)
  uint2 *cand;              // [B*Hq, ldC] (position, order key) of the keys in bin b1
  uint2 *bucket;            // [B*Hq, kTopkBucket] the keys in (b1, b2)
  int32_t *idx;             // [B*Hq, k]
  long long ldS, ldC, N;
  long long cand_lo, cand_hi, nC, k_eff;
  int k, R;
};

struct AttnParams {
  const float *S;
  const __nv_bfloat16 *V;
  const int32_t *idx;
  float *part;              // [B*Hq, nsplit, d + 4] partial states (m, Z, pad, pad, N[d])
  float *out;               // [B*Hq, d]
  uint32_t *meta;
  long long ldS, cap, N;
  long long s1, w0, nW, k_eff;
  int k, Hq, G, Hkv, nsplit, R, B;
  int nWsplit;              // static-set CTAs per KV head, wrange rows of W each
  int nOsplit;              // retrieved-set CTAs per query head, orange rows of Omega each
  long long wrange, orange; // multiples of kAttnRange
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
constexpr int kAttnRange = 64;      // entries of U a sparse-attention CTA takes at a time
constexpr int kAttnWave = 768;      // about one wave of sparse-attention CTAs on 148 SMs
constexpr int kTopkChunk = 8192;    // positions per top-k CTA
constexpr int kTopkBucket = 4096;   // (b1, b2) bucket entries kept per query head
constexpr int kDenseTile = 128;

int num_sms();

// Bytes of the counter block at the front of every workspace for `rows` query heads
// (digit-1 and digit-2 histograms, then the per-row counters), 256-byte aligned sections.
size_t counter_block_bytes(size_t rows);

// Raises a kernel's dynamic shared-memory limit once per device (so that later launches,
// including launches inside a stream capture, make no attribute call).
cudaError_t ensure_smem_limit(const void *kernel, int bytes, bool (&done)[64]);

cudaError_t launch_score(const ScoreParams &p, int d, cudaStream_t s);
cudaError_t launch_topk(const TopkParams &p, cudaStream_t s);
cudaError_t launch_sparse_attn(const AttnParams &p, int d, cudaStream_t s);
cudaError_t launch_dense(const DenseParams &p, int d, cudaStream_t s);
cudaError_t launch_append(const AppendParams &p, cudaStream_t s);

}  // namespace ra
