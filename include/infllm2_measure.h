/*
 * libinfllm2 measurement export — not part of the attention path.
 *
 * libinfllm2.so also exports one measurement routine used by the benchmark
 * to obtain a roofline denominator that no vendor figure provides: the
 * L2 -> SM gather bandwidth with the block-sparse attention's access
 * pattern.  It computes nothing of the method (the pages have no
 * counterpart) and no call of the attention path uses it.  Types and error
 * codes come from infllm2.h.
 */
#ifndef INFLLM2_MEASURE_H_
#define INFLLM2_MEASURE_H_

#include "infllm2.h"

#ifdef __cplusplus
extern "C" {
#endif

/* L2 -> SM gather bandwidth with the block-sparse attention's
 * access pattern: the roofline denominator of the gather-bound attention
 * kernel.  K, V: [rows, h_kv, 128] bf16 device tensors (any contents).
 * One CTA per SM; `producers` (1, 2, 3 or 6) warps each gather `tiles`
 * tiles of two random 64-key blocks (32 KB) of kv group 0 from the first
 * nblk blocks, with 192 KB in flight per SM, and discard them.  The caller
 * times the call (bytes = num_SMs * producers * tiles * 32768).  Returns
 * INFLLM2_ERR_INVALID_ARG for null or misaligned tensors, nblk * 64 > rows
 * or tiles < 1. */
int infllm2_probe_l2_gather(const void* K, const void* V, int64_t rows, int32_t h_kv, int32_t nblk,
                            int32_t tiles, int32_t producers, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* INFLLM2_MEASURE_H_ */
