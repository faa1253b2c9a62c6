// Kernel parameter blocks and host-side launchers of libra (internal, not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ra {

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
};

struct TopkParams {
  const float *S;
  const uint32_t *hist;
  uint32_t *meta;           // [B*Hq, kMetaWords] (zeroed before the score launch)
  uint32_t *cand;           // [B*Hq, ldC]
  int32_t *idx;             // [B*Hq, k]
  long long ldS, ldC, N;
  long long cand_lo, cand_hi, nC, k_eff;
  long long chunk;          // positions per collect CTA
  int k, R;
};

struct AttnParams {
  const float *S;
  const __nv_bfloat16 *V;
  const int32_t *idx;
  float *part;              // [B*Hq, nsplit, d + 2]
  float *out;               // [B*Hq, d]
  uint32_t *meta;
  long long ldS, cap, N;
  long long s1, w0, nW, k_eff;
  int k, Hq, G, Hkv, nsplit, R;
};

struct DenseParams {
  const __nv_bfloat16 *K, *V, *q;
  float *part;              // [B*Hq, nsplit, d + 2]
  float *out;               // [B*Hq, d]
  uint32_t *meta;           // [B*Hq, kMetaWords] (zeroed before the launch)
  long long N, cap, keys_per_split;
  int B, Hkv, G, Hq, nsplit;
  float scale;
};

struct AppendParams {
  __nv_bfloat16 *K, *V;
  const __nv_bfloat16 *k_new, *v_new;
  long long cap, N;
  int B, Hkv, d, T;
};

// tuning constants the host layout needs
constexpr int kScoreTile = 128;
constexpr int kAttnChunk = 64;      // U entries per sparse-attention CTA
constexpr int kCollectChunk = 4096; // positions per collect CTA
constexpr int kDenseTile = 128;

int num_sms();

// Raises a kernel's dynamic shared-memory limit once per device (so that later launches,
// including launches inside a stream capture, make no attribute call).
cudaError_t ensure_smem_limit(const void *kernel, int bytes, bool (&done)[64]);

cudaError_t launch_score(const ScoreParams &p, int d, cudaStream_t s);
cudaError_t launch_topk(const TopkParams &p, cudaStream_t s);
cudaError_t launch_sparse_attn(const AttnParams &p, int d, cudaStream_t s);
cudaError_t launch_dense(const DenseParams &p, int d, cudaStream_t s);
cudaError_t launch_append(const AppendParams &p, cudaStream_t s);

}  // namespace ra
