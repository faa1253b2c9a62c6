// Scores of a batch of prefill queries against every cached key, on the tcgen05 tensor cores:
// S[(b, h, m), i] = q[b, h, m] . K[b, h / G, i] / sqrt(d) (RetrievalAttention slides, Eq. (1);
// the index is built from the prefill queries' nearest keys, slide "Query-aware index
// construction").  With G * M query rows per KV head this is a dense contraction
// [G*M, d] x [d, N], unlike the single-query decode scan.
//
// One CTA per output tile of 128 query rows x 256 keys of one KV head:
//   * one thread loads the query tile and the key tile with TMA bulk tensor copies (128-byte
//     swizzled boxes of 64 channels) onto one mbarrier;
//   * the same thread issues d / 16 tcgen05.mma (M 128, N 256, K 16, bf16 x bf16 -> fp32) into
//     256 columns of tensor memory and commits them to a second mbarrier;
//   * the four warps read their 32 tensor-memory lanes (one query row per thread) with
//     tcgen05.ld, 32 columns at a time, scale, and write them into a 128-byte-swizzled
//     [128 rows][32 columns] fp32 box in shared memory (the key tile's buffer, free once the
//     products are done); one thread stores each box with a TMA tensor store (full lines; rows
//     past the KV head's G * M and keys past N are clipped by the tensor map), two boxes in
//     flight.
// Every wait is bounded (an error bit and an orderly exit instead of a hang); the tensor memory
// is freed on every path.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace ra {

constexpr int kPfM = 128;          // query rows per tile (UMMA M)
constexpr int kPfN = 256;          // keys per tile (UMMA N)
constexpr int kPfThreads = 128;    // four warps: one tensor-memory lane quarter each

template <int D>
struct PfCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kABox = kPfM * 128;              // bytes of one 64-channel box
  static constexpr int kBBox = kPfN * 128;
  static constexpr int kABytes = kBoxes * kABox;
  static constexpr int kBBytes = kBoxes * kBBox;
  static constexpr size_t smem_bytes() { return 1024 + kABytes + kBBytes + 64; }
};

constexpr int kPfCols = 32;                   // columns per stored box
constexpr int kPfBox = kPfM * kPfCols * 4;    // 16 KB

template <int D>
__global__ void __launch_bounds__(kPfThreads, 2)
    prefill_score_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmS, const PfParams p) {
  using C = PfCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sA = (raw + 1023u) & ~1023u;   // swizzled boxes need 1024-byte alignment
  const uint32_t sB = sA + C::kABytes;
  const uint32_t bar_load = sB + C::kBBytes;
  const uint32_t bar_mma = bar_load + 8;
  const uint32_t slot = bar_mma + 8;
  const uint32_t *slot_ptr = reinterpret_cast<const uint32_t *>(smem_raw + (slot - raw));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long key0 = static_cast<long long>(blockIdx.x) * kPfN;
  const int qb = blockIdx.y;                               // 128-row block of the head's rows
  const int bg = blockIdx.z;                               // b * Hkv + g

  pdl_trigger();
  if (warp == 0) tmem_alloc(slot, kPfN);
  if (tid == 32) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *slot_ptr;
  pdl_wait();   // the keys (appended rows) and queries come from earlier work on the stream

  if (tid == 0) {
    const uint64_t pol = policy_evict_first();
    mbar_arrive_expect_tx(bar_load, C::kABytes + C::kBBytes);
#pragma unroll
    for (int bx = 0; bx < C::kBoxes; ++bx) {
      tma_load_3d(sA + bx * C::kABox, &tmQ, bx * 64, qb * kPfM, bg, bar_load, pol);
      tma_load_3d(sB + bx * C::kBBox, &tmK, bx * 64, static_cast<int>(key0), bg, bar_load, pol);
    }
    if (mbar_wait(bar_load, 0)) {
      tc_fence_after_sync();
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kPfM, kPfN);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk & 3) * 32;   // 16 bf16 = 32 bytes per K step within a row
        const uint64_t da = umma_desc_k_sw128(sA + (kk >> 2) * C::kABox + koff);
        const uint64_t db = umma_desc_k_sw128(sB + (kk >> 2) * C::kBBox + koff);
        umma_bf16(tmem, da, db, idesc, kk > 0);
      }
      umma_commit(bar_mma);
    } else {
      atomicOr(p.err, kErrPrefillWait);
    }
  }
  const bool done = mbar_wait(bar_mma, 0);
  tc_fence_after_sync();
  if (!__syncthreads_and(done)) {
    // the MMAs (or the loads) never completed: leave without reading tensor memory; the
    // copies still in flight are waited for (bounded) so that nothing lands after exit
    if (tid == 0) {
      atomicOr(p.err, kErrPrefillWait);
      mbar_wait(bar_load, 0);
    }
  } else {
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int r = warp * 32 + lane;   // this thread's row in the tile and in the stored box
#pragma unroll 1
    for (int ch = 0; ch < kPfN / kPfCols; ++ch) {
      const uint32_t buf = sB + (ch & 1) * kPfBox;
      if (ch >= 2 && tid == 0) bulk_wait_group_read<1>();   // box ch - 2 has left this buffer
      __syncthreads();
      uint32_t v0[16], v1[16];
      tmem_ld16(tmem + lane_base + static_cast<uint32_t>(ch * kPfCols), v0);
      tmem_ld16(tmem + lane_base + static_cast<uint32_t>(ch * kPfCols + 16), v1);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 8; ++c) {   // 16-byte chunk c of the row, at swizzled chunk c ^ (r % 8)
        const uint32_t *w = c < 4 ? v0 + 4 * c : v1 + 4 * (c - 4);
        const float4 f = make_float4(canon_zero(__uint_as_float(w[0]) * p.scale),
                                     canon_zero(__uint_as_float(w[1]) * p.scale),
                                     canon_zero(__uint_as_float(w[2]) * p.scale),
                                     canon_zero(__uint_as_float(w[3]) * p.scale));
        const uint32_t dst = buf + r * 128 + ((c ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"r"(dst), "f"(f.x), "f"(f.y),
                     "f"(f.z), "f"(f.w)
                     : "memory");
      }
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        tma_store_3d(&tmS, buf, static_cast<int>(key0) + ch * kPfCols, qb * kPfM, bg);
        bulk_commit_group();
      }
    }
    if (tid == 0) bulk_wait_group<0>();   // every store has finished before the CTA leaves
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kPfN);
}

// Host: 3-D fp32 tensor map over the scores viewed as [B * Hkv heads][G * M rows][N keys] (rows
// ldS floats apart) with a box of [1][128][32] and the 128-byte swizzle.
static bool encode_scores_tmap(CUtensorMap *out, float *S, long long heads, long long head_rows,
                               long long N, long long ldS) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(head_rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ldS) * 4,
                                 static_cast<cuuint64_t>(ldS) * 4 * head_rows};
  const cuuint32_t box[3] = {kPfCols, kPfM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, S, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_prefill_t(const PfParams &p, cudaStream_t s) {
  using C = PfCfg<D>;
  static bool done[64] = {};
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(prefill_score_kernel<D>),
                                    static_cast<int>(C::smem_bytes()), done);
  if (e != cudaSuccess) return e;
  // queries as [B * Hkv planes][G * M rows][d] (planes q_plane_rows rows apart): the G * M rows
  // of a KV head's query heads are contiguous in [B, Hq, M, d]; rows past G * M read as zeros
  const long long head_rows_q = static_cast<long long>(p.G) * p.M;
  CUtensorMap tq, tk;
  if (!encode_rows_tmap(&tq, p.Q, D, static_cast<uint64_t>(head_rows_q),
                        static_cast<uint64_t>(p.B) * p.Hkv, kPfM,
                        static_cast<uint64_t>(p.q_plane_rows > 0 ? p.q_plane_rows : head_rows_q)))
    return cudaErrorInvalidValue;
  if (!encode_rows_tmap(&tk, p.K, D, static_cast<uint64_t>(p.N),
                        static_cast<uint64_t>(p.B) * p.Hkv, kPfN, static_cast<uint64_t>(p.cap)))
    return cudaErrorInvalidValue;
  const long long head_rows = static_cast<long long>(p.G) * p.M;
  CUtensorMap ts;
  if (!encode_scores_tmap(&ts, p.S, static_cast<long long>(p.B) * p.Hkv, head_rows, p.N, p.ldS))
    return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>((p.N + kPfN - 1) / kPfN),
                  static_cast<unsigned>((head_rows + kPfM - 1) / kPfM),
                  static_cast<unsigned>(p.B * p.Hkv));
  return launch_pdl(prefill_score_kernel<D>, grid, dim3(kPfThreads), C::smem_bytes(), s, tq, tk,
                    ts, p);
}

cudaError_t launch_prefill_score(const PfParams &p, int d, cudaStream_t s) {
  return d == 128 ? launch_prefill_t<128>(p, s) : launch_prefill_t<64>(p, s);
}

}  // namespace ra
