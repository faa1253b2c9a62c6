// Append T new tokens to a layer's KV cache: K[b, g, N + t, :] = k_new[b, g, t, :], same for
// V.  The decode step attends over j <= t including the current token (RetrievalAttention
// slides, Eq. (1)), so a step appends before it scores.
#include "common.cuh"
#include "kernels.h"

namespace ra {

__global__ void __launch_bounds__(256) append_kv_kernel(const AppendParams p) {
  pdl_trigger();
  pdl_wait();   // the previous step may still read the rows this append overwrites
  // one 16-byte unit per thread: units per row = d / 8
  const int upr = p.d / 8;
  const long long units = static_cast<long long>(p.B) * p.Hkv * p.T * upr;
  for (long long u = blockIdx.x * 256LL + threadIdx.x; u < 2 * units;
       u += static_cast<long long>(gridDim.x) * 256) {
    const bool is_v = u >= units;
    const long long w = is_v ? u - units : u;
    const int c = static_cast<int>(w % upr);
    const long long rt = w / upr;               // (b*Hkv + g) * T + t
    const long long t = rt % p.T;
    const long long bg = rt / p.T;
    const uint4 *src = reinterpret_cast<const uint4 *>(is_v ? p.v_new : p.k_new) + w;
    __nv_bfloat16 *dst_base = is_v ? p.V : p.K;
    uint4 *dst = reinterpret_cast<uint4 *>(dst_base + (bg * p.cap + p.N + t) * p.d) + c;
    *dst = __ldg(src);
  }
}

cudaError_t launch_append(const AppendParams &p, cudaStream_t s) {
  const long long units = 2LL * p.B * p.Hkv * p.T * (p.d / 8);
  long long blocks = (units + 255) / 256;
  if (blocks > 4LL * num_sms()) blocks = 4LL * num_sms();
  if (blocks < 1) blocks = 1;
  return launch_pdl(append_kv_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, p);
}

}  // namespace ra

namespace ra {

// Paged caches: token N_b + t of sequence b goes to row (N_b + t) % kPageSize of page
// block_table[b][(N_b + t) / kPageSize], KV head g: pool row (page * Hkv + g) * kPageSize + ...
__global__ void __launch_bounds__(256) append_kv_paged_kernel(const AppendParams p,
                                                              const PagedInfo pg) {
  pdl_trigger();
  pdl_wait();   // the previous step may still read the rows this append overwrites
  const int upr = p.d / 8;   // 16-byte units per row
  const long long units = static_cast<long long>(p.B) * p.Hkv * p.T * upr;
  for (long long u = blockIdx.x * 256LL + threadIdx.x; u < 2 * units;
       u += static_cast<long long>(gridDim.x) * 256) {
    const bool is_v = u >= units;
    const long long w = is_v ? u - units : u;
    const int c = static_cast<int>(w % upr);
    const long long rt = w / upr;               // (b * Hkv + g) * T + t
    const long long t = rt % p.T;
    const long long bg = rt / p.T;
    const long long b = bg / p.Hkv, g = bg - b * p.Hkv;
    const long long pos = pg.seq_len[b] + t;
    const long long page = __ldg(pg.block_table + b * pg.max_pages + pos / kPageSize);
    const long long row = (page * p.Hkv + g) * kPageSize + pos % kPageSize;
    const uint4 *src = reinterpret_cast<const uint4 *>(is_v ? p.v_new : p.k_new) + w;
    __nv_bfloat16 *dst_base = is_v ? p.V : p.K;
    reinterpret_cast<uint4 *>(dst_base + row * p.d)[c] = __ldg(src);
  }
}

cudaError_t launch_append_paged(const AppendParams &p, const PagedInfo &pg, cudaStream_t s) {
  const long long units = 2LL * p.B * p.Hkv * p.T * (p.d / 8);
  long long blocks = (units + 255) / 256;
  if (blocks > 4LL * num_sms()) blocks = 4LL * num_sms();
  if (blocks < 1) blocks = 1;
  return launch_pdl(append_kv_paged_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, p,
                    pg);
}

}  // namespace ra
