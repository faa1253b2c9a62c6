// Tensor-memory-accelerator (TMA) loads and mbarrier helpers for sm_100a, plus the host-side
// tensor-map encoder (fetched from the driver at run time, so libra does not link libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ra {

// Bounded-wait budget: mbarrier.try_wait polls (each may suspend for a while) before a wait
// is declared lost.  Far above any legitimate wait; it only turns a hang into an error flag.
constexpr uint32_t kWaitPolls = 1u << 24;

// Error bits in the workspace's error word.
constexpr uint32_t kErrScoreWait = 1u;
constexpr uint32_t kErrDenseWait = 2u;

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Plain arrival (no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

// Returns true once the barrier's phase with the given parity has completed, false if the
// poll budget ran out first.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitPolls; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// As mbar_wait, but also gives up (false) once *abort is non-zero: a CTA whose pipeline broke
// stops all its waits at once instead of each running out its own budget.
__device__ __forceinline__ bool mbar_wait_or_abort(uint32_t bar, uint32_t parity,
                                                   const volatile int *abort) {
  for (uint32_t i = 0; i < kWaitPolls; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    if ((i & 15u) == 15u && *abort) return false;
  }
  return false;
}

// 1-D bulk copy global -> shared (this CTA), completion counted in bytes on the mbarrier; both
// addresses 16-byte aligned and `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Barrier 1 over the first `threads` threads of the CTA (barrier 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(int threads) {
  asm volatile("bar.sync 1, %0;\n" ::"r"(threads) : "memory");
}

// Adds 1 to a device-wide counter with release semantics: writes this thread has made or
// observed (a preceding barrier) are visible to any thread that acquires the new value.
__device__ __forceinline__ void red_release_add1(uint32_t *ctr) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;\n" ::"l"(ctr) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *m) {
  asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled bulk tensor load global -> shared (this CTA only), completion counted in bytes on
// the mbarrier.  x is the innermost coordinate (in elements; x * 2 bytes is a multiple of 16).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *m, int x, int y, int z,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy)
      : "memory");
}

// 16-byte shared-memory store at a shared-space address.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later async-proxy (TMA)
// accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// L2 policy for data read once per step (the K stream): evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}

// Host: encode a 3-D bf16 tensor map over [planes][rows][cols] (cols innermost; planes are
// plane_rows rows apart, plane_rows >= rows) with a box of [1][box_rows][64] and 128-byte
// swizzle.  Rows at or past `rows` read as zeros.  Returns false if the driver refused it.
bool encode_rows_tmap(CUtensorMap *out, const void *base, uint64_t cols, uint64_t rows,
                      uint64_t planes, uint32_t box_rows, uint64_t plane_rows);

}  // namespace ra
