// Shared device helpers for libra (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ra {

constexpr int kHistBits = 11;                 // radix digits of 11 bits (digit 1: digit1_bin)
constexpr int kHistBins = 1 << kHistBits;     // 2048 bins per query head
constexpr int kMaxGroup = 8;                  // query heads per KV head (one n8 MMA tile)
constexpr int kMetaWords = 8;                 // per-row counters in the workspace

// per-row counters (uint32) in the workspace's meta block: the error word (row 0) and the
// dense merge's CTA counter (left zero by the merging CTA)
enum MetaSlot { kError = 6, kDone = 7 };

// ------------------------------------------------------------------ programmatic dependent launch

// Kernels of a decode step are launched with programmatic stream serialisation: each lets the
// next kernel of the stream be scheduled as soon as all of its own CTAs are running, and
// waits for its predecessor (completion and memory visibility) before touching its outputs.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// ------------------------------------------------------------------ order-preserving keys

// Maps a float to a uint32 whose unsigned order equals the float order (-0 sorts below +0;
// scores are canonicalised so that zero is always +0).
__device__ __forceinline__ uint32_t order_key(float z) {
  uint32_t u = __float_as_uint(z);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float canon_zero(float z) { return z == 0.0f ? 0.0f : z; }

// The float whose order key is `key` (the inverse bijection of order_key on bit patterns): for
// finite scores z >= key_float(K) exactly when order_key(z) >= K.
__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// ------------------------------------------------------------------ digit 1 of the top-k select
//
// The first digit of the selection's radix select is a bin of the score that is fine where top-k
// thresholds lie.  Let a = bits [17, 31) of |z| (its exponent and top 6 mantissa bits) and
// m = clamp(a - kD1A0, 0, 1023): m = 1 .. 1022 cover |z| in [2^-8, 2^8) at 64 steps an octave,
// m = 0 holds |z| < 2^-8 and m = 1023 holds |z| >= 2^8 (less the top two steps).  The bin is
// 1024 + m for z >= +0 and 1023 - m for z < 0, so bins rise with z; a bin with 1 <= m <= 1022
// is one value of the order key's top 15 bits (sign and a), the four others (0, 1023, 1024,
// 2047) share no key prefix.  (A plain top-11-bit digit has 4 bins an octave: at 1 % of 128K
// keys its threshold bin holds thousands of a head's keys.)
constexpr uint32_t kD1A0 = (127u - 8u) * 64u - 1u;   // a of 2^-8, less one
constexpr uint32_t kD1PrefixBits = 15;

// From the score itself (canonical zero): two float clamps, a shift, a subtraction, a sign flip.
__device__ __forceinline__ uint32_t digit1_bin_z(float z) {
  const float c = fminf(fmaxf(fabsf(z), __uint_as_float(kD1A0 << 17)),
                        __uint_as_float((kD1A0 + 1023u) << 17));
  const int m = static_cast<int>(__float_as_uint(c) >> 17) - static_cast<int>(kD1A0);
  const int s = static_cast<int>(__float_as_uint(z)) >> 31;   // 0, or -1 for z < 0
  return static_cast<uint32_t>(1024 + (m ^ s));
}
// The same bin from an order key (the inverse of order_key, then the rule above).
__host__ __device__ __forceinline__ uint32_t digit1_bin(uint32_t key) {
  const uint32_t u = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;   // the float's bits
  const uint32_t a = (u >> 17) & 0x3FFFu;
  const uint32_t m = a <= kD1A0 ? 0u : (a - kD1A0 > 1023u ? 1023u : a - kD1A0);
  return (u & 0x80000000u) ? 1023u - m : 1024u + m;
}
// The smallest key of bin b (b = 2048: 2^32, past every key).
__host__ __device__ __forceinline__ unsigned long long digit1_floor(uint32_t b) {
  if (b >= 2048u) return 1ull << 32;
  if (b >= 1024u) {   // z >= +0: the smallest |z| of its m
    const uint32_t m = b - 1024u;
    return m == 0u ? 0x80000000ull : (0x80000000ull | (static_cast<unsigned long long>(kD1A0 + m) << 17));
  }
  const uint32_t m = 1023u - b;   // z < 0: the largest |z| of its m
  return m == 1023u ? 0ull : static_cast<unsigned long long>(0x3FFFu - (kD1A0 + m)) << 17;
}
// Key bits every key of bin b shares from the top: 15, or 0 for the four catch-all bins.
__host__ __device__ __forceinline__ int digit1_prefix_bits(uint32_t b) {
  return (b == 0u || b == 1023u || b == 1024u || b >= 2047u) ? 0 : static_cast<int>(kD1PrefixBits);
}

// ------------------------------------------------------------------ shared-memory addresses

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}


// ------------------------------------------------------------------ tensor-core fragments

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                            uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ bf16 pairs

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------------ warp reductions

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

}  // namespace ra
