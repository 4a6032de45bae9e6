/*
 * gauss_testing.h -- test hooks of libgauss_b200.so (not part of the
 * computation's API; used by the test-suite to check building blocks of the
 * kernels in isolation).
 */
#ifndef GAUSS_B200_TESTING_H
#define GAUSS_B200_TESTING_H

#include "gauss.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * out[i] = 2^x[i] evaluated on the device by the FMA-pipe exponential the
 * kernels use for part of their kernel values (exact base-2 argument reduction,
 * then a minimax polynomial of degree 3 or 5 for 2^f on [-1/2, 1/2], fitted by
 * the Remez exchange in csrc/gen_exp2_poly.py).  Inputs are clamped to >= -125.
 * x and out are device arrays of n floats (16-byte aligned); degree is 3 or 5.
 * Returns GS_ERR_INVALID_ARG for a bad degree or pointer, GS_OK otherwise.
 */
gs_status gs_test_exp2_poly(const float *x, float *out, int64_t n, int degree, gs_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GAUSS_B200_TESTING_H */
