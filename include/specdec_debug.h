/*
 * specdec debug entry points: expose the random stream so that tests can pin
 * it.  Not needed to run the method.
 */
#ifndef SPECDEC_DEBUG_H
#define SPECDEC_DEBUG_H

#include "specdec.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Philox4x32-10 block function as the kernels use it (Salmon et al., SC'11):
 * out[i, 0..3] = Philox(ctr[i, 0..3], key[i, 0..1]).  Device arrays, n rows. */
spec_status spec_debug_philox(const uint32_t *ctr, const uint32_t *key, uint32_t *out, int32_t n,
                              spec_stream_t stream);

/* The same block function computed by the CUDA toolkit's curand Philox4_32_10
 * generator (seed = key, subsequence = counter words 2..3, offset = 4 x counter
 * words 0..1), an independent implementation of the published algorithm. */
spec_status spec_debug_curand_philox(const uint32_t *ctr, const uint32_t *key, uint32_t *out,
                                     int32_t n, spec_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
