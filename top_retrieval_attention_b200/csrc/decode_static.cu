// ra_decode_step_static: the decode step for callers that cannot allocate device memory.
//
// Some callers never get to call cudaMalloc: a plugin that an inference engine invokes with
// nothing but input and output pointers (the engine owns all device memory), or a serving loop
// that forbids allocation after start-up because cudaMalloc can synchronise the device and
// stall every stream.  This entry point runs the same kernels as ra_decode_step, with the
// workspace taken from a scratch array that lives in the library itself.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes (64 MiB).  Every GPU on
// which the library is loaded holds it until the process exits.  All calls on a device share
// it and it keeps the last call's contents, so calls whose work overlaps on the GPU (two
// streams, two host threads) race and must be serialised by the caller.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/ra.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;

__device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

// Device address of g_scratch per device.  In host code `g_scratch` names a host-side stand-in,
// not device memory, so the address is looked up once per device with that device current.
// Host threads may make their first calls at the same time: the cache is atomic (two threads
// may both look the address up; both store the same value).
std::atomic<void *> g_scratch_addr[64] = {};

}  // namespace

extern "C" ra_status ra_decode_step_static(const ra_kv *kv, const void *q, int32_t Hq, int32_t k,
                                           int32_t n_sink, int32_t n_window, float *out,
                                           int32_t *idx, ra_stream_t stream) {
  if (!kv) return RA_ERR_ARG;
  // Argument and shape errors first, reported exactly as ra_decode_step reports them: with no
  // workspace it validates everything else and stops at RA_ERR_WORKSPACE, enqueuing nothing.
  const ra_status pre = ra_decode_step(kv, q, Hq, k, n_sink, n_window, out, idx, nullptr, 0, stream);
  if (pre != RA_ERR_WORKSPACE) return pre;
  const auto misaligned = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (!q || misaligned(q) || !out || misaligned(out)) return RA_ERR_ARG;
  if (k > 0 && (!idx || misaligned(idx))) return RA_ERR_ARG;
  const size_t need = ra_decode_workspace_bytes(kv->B, Hq, kv->N, kv->d, k, n_sink, n_window);
  if (need == 0 || need > kStaticScratchBytes) return RA_ERR_WORKSPACE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RA_ERR_CUDA;
  void *ws = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (ws == nullptr) {
    // the look-up is a runtime call that a stream capture may not allow: refuse it there
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(reinterpret_cast<cudaStream_t>(stream), &cap) != cudaSuccess)
      return RA_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) {
      ra::set_last_error("ra_decode_step_static: the first call on a device must come before "
                         "any stream capture (it looks up the scratch's device address)");
      return RA_ERR_ARG;
    }
    if (cudaGetSymbolAddress(&ws, g_scratch) != cudaSuccess || ws == nullptr) return RA_ERR_CUDA;
    g_scratch_addr[dev].store(ws, std::memory_order_release);
  }

  // The counter block at the front of the workspace (per query head: histogram and
  // counters) must start at zero; clear it on every call rather than trusting the last one.
  const size_t rows = static_cast<size_t>(kv->B) * static_cast<size_t>(Hq);
  const size_t counters = ra::counter_block_bytes(rows);
  if (cudaMemsetAsync(ws, 0, counters, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RA_ERR_CUDA;
  return ra_decode_step(kv, q, Hq, k, n_sink, n_window, out, idx, ws, kStaticScratchBytes, stream);
}
