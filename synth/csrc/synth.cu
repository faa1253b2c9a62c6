// Device fill of the seeded synthetic workloads: the same bits as synth/gen.py.
// Input generation only; none of the attention method's arithmetic lives here.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ra_synth.h"

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kMix1 = 0xBF58476D1CE4E5B9ull;
constexpr uint64_t kMix2 = 0x94D049BB133111EBull;
constexpr double kIhScale = 0x1.bb67ae8584caap-16;   // sqrt(3) / 65536
constexpr double kOffStd = 0x1.6a09e667f3bcdp+0;     // sqrt(2)
constexpr int kKindQ = 1, kKindK = 2, kKindKoff = 3, kKindV = 4;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * kMix1;
  z = (z ^ (z >> 27)) * kMix2;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, int kind, int layer, int b, int head) {
  const uint64_t tag = (static_cast<uint64_t>(kind & 0xFF) << 56) |
                       (static_cast<uint64_t>(layer & 0xFFF) << 44) |
                       (static_cast<uint64_t>(b & 0xFFFF) << 28) |
                       (static_cast<uint64_t>(head & 0xFFFF) << 12);
  return mix64(seed * kGamma + tag);
}

__device__ inline double normal_at(uint64_t key, uint64_t i) {
  const uint64_t u = mix64(key + (i + 1) * kGamma);
  const int64_t s = static_cast<int64_t>((u & 0xFFFF) + ((u >> 16) & 0xFFFF) +
                                         ((u >> 32) & 0xFFFF) + ((u >> 48) & 0xFFFF));
  return __dmul_rn(static_cast<double>(s - 131070), kIhScale);
}

__device__ inline uint16_t to_bf16_bits(double x) {
  const uint32_t bits = __float_as_uint(__double2float_rn(x));
  return static_cast<uint16_t>((bits + 0x7FFFu + ((bits >> 16) & 1u)) >> 16);
}

// Block (x, bg): a thread owns 8 consecutive channels (c8) of every row r = row0 + phase
// (mod rows in flight); the stream keys and the channel offsets are computed once per thread.
__global__ void __launch_bounds__(256) fill_kv_kernel(uint16_t *K, uint16_t *V, int Hkv,
                                                      long long cap, int d, long long row0,
                                                      long long nrows, uint64_t seed, int layer,
                                                      int with_offset) {
  const int per_row = d / 8;                     // threads per row
  const int phases = 256 / per_row;              // rows in flight per block
  const int bg = blockIdx.y;
  const int b = bg / Hkv, g = bg % Hkv;
  const int c8 = threadIdx.x % per_row;
  const int phase = threadIdx.x / per_row;
  const uint64_t kk = stream_key(seed, kKindK, layer, b, g);
  const uint64_t kv = stream_key(seed, kKindV, layer, b, g);
  double off[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    off[j] = with_offset ? __dmul_rn(kOffStd, normal_at(stream_key(seed, kKindKoff, layer, b, g),
                                                        static_cast<uint64_t>(c8 * 8 + j)))
                         : 0.0;
  const long long step = static_cast<long long>(gridDim.x) * phases;
  for (long long r = static_cast<long long>(blockIdx.x) * phases + phase; r < nrows; r += step) {
    const long long i = row0 + r;
    uint16_t outk[8], outv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint64_t e = static_cast<uint64_t>(i) * d + c8 * 8 + j;
      double xk = normal_at(kk, e);
      if (with_offset) xk = __dadd_rn(xk, off[j]);
      outk[j] = to_bf16_bits(xk);
      outv[j] = to_bf16_bits(normal_at(kv, e));
    }
    const long long o = (static_cast<long long>(bg) * cap + i) * d + c8 * 8;
    uint4 pk, pv;
    pk.x = outk[0] | (static_cast<uint32_t>(outk[1]) << 16);
    pk.y = outk[2] | (static_cast<uint32_t>(outk[3]) << 16);
    pk.z = outk[4] | (static_cast<uint32_t>(outk[5]) << 16);
    pk.w = outk[6] | (static_cast<uint32_t>(outk[7]) << 16);
    pv.x = outv[0] | (static_cast<uint32_t>(outv[1]) << 16);
    pv.y = outv[2] | (static_cast<uint32_t>(outv[3]) << 16);
    pv.z = outv[4] | (static_cast<uint32_t>(outv[5]) << 16);
    pv.w = outv[6] | (static_cast<uint32_t>(outv[7]) << 16);
    *reinterpret_cast<uint4 *>(K + o) = pk;
    *reinterpret_cast<uint4 *>(V + o) = pv;
  }
}

__global__ void fill_q_kernel(uint16_t *q, int B, int Hq, int d, uint64_t seed) {
  const long long total = static_cast<long long>(B) * Hq * d;
  for (long long w = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; w < total;
       w += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(w % d);
    const long long bh = w / d;
    const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
    q[w] = to_bf16_bits(normal_at(stream_key(seed, kKindQ, 0, b, h), c));
  }
}

}  // namespace

extern "C" {

int synth_fill_kv(void *K, void *V, int32_t B, int32_t Hkv, int32_t cap, int32_t d, int64_t row0,
                  int64_t nrows, uint64_t seed, int32_t layer, int32_t with_offset,
                  struct CUstream_st *stream) {
  if (!K || !V || B < 1 || Hkv < 1 || (d != 64 && d != 128) || row0 < 0 || nrows < 0 ||
      row0 + nrows > cap)
    return -1;
  if (nrows == 0) return 0;
  if (static_cast<long long>(B) * Hkv > 65535) return -1;
  const int phases = 256 / (d / 8);
  long long bx = (nrows + phases - 1) / phases;
  const long long want = (148LL * 16 + static_cast<long long>(B) * Hkv - 1) / (static_cast<long long>(B) * Hkv);
  if (bx > want) bx = want;
  const dim3 grid(static_cast<unsigned>(bx < 1 ? 1 : bx), static_cast<unsigned>(B * Hkv));
  fill_kv_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint16_t *>(K), static_cast<uint16_t *>(V), Hkv, cap, d, row0, nrows, seed,
      layer, with_offset);
  return static_cast<int>(cudaGetLastError());
}

int synth_fill_q(void *q, int32_t B, int32_t Hq, int32_t d, uint64_t seed,
                 struct CUstream_st *stream) {
  if (!q || B < 1 || Hq < 1 || d < 1) return -1;
  const long long total = static_cast<long long>(B) * Hq * d;
  const long long blocks = (total + 255) / 256;
  fill_q_kernel<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint16_t *>(q), B, Hq, d, seed);
  return static_cast<int>(cudaGetLastError());
}

void synth_constants(double out[2]) {
  out[0] = kIhScale;
  out[1] = kOffStd;
}

}  // extern "C"
