/*
 * ra_synth.h -- device fill of the seeded synthetic decode workloads (input generation only;
 * contains none of the attention method's arithmetic).
 *
 * Produces, in device memory, exactly the bf16 bit patterns that the host generator
 * (synth/gen.py) produces for the same (seed, layer, b, head, position, channel): SplitMix64
 * outputs (Steele, Lea and Flood, OOPSLA 2014) turned into Irwin-Hall(4) normal deviates with
 * integer and correctly rounded IEEE double operations only, then rounded double -> float ->
 * bf16 (round to nearest even at each step).
 *
 * All calls are asynchronous on `stream` and return 0 on success, a CUDA error code otherwise,
 * or -1 for invalid arguments (nothing enqueued).
 */
#ifndef RA_SYNTH_H
#define RA_SYNTH_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;

/* Rows [row0, row0 + nrows) of K and V ([B, Hkv, cap, d] bf16, device) of one layer:
 * K = bf16(x + off[c]) (off = sqrt(2) * N(0,1) per (layer, b, g, c); omitted when
 * with_offset == 0), V = bf16(x').  Needles are planted separately by the caller. */
int synth_fill_kv(void *K, void *V, int32_t B, int32_t Hkv, int32_t cap, int32_t d,
                  int64_t row0, int64_t nrows, uint64_t seed, int32_t layer, int32_t with_offset,
                  struct CUstream_st *stream);

/* q [B, Hq, d] bf16, device. */
int synth_fill_q(void *q, int32_t B, int32_t Hq, int32_t d, uint64_t seed,
                 struct CUstream_st *stream);

/* The two double constants of the generator (sqrt(3)/65536 and sqrt(2)), for host checks. */
void synth_constants(double out[2]);

#ifdef __cplusplus
}
#endif

#endif /* RA_SYNTH_H */
