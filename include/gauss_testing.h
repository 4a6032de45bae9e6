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

/*
 * The limit of the tensor-core kernels' bounded mbarrier waits (default
 * 2e9 ns) and a stall mode that makes those waits run out on purpose, so that
 * the abort path can be tested without a fault:
 *   stall 0  normal operation;
 *   stall 1  the MMA-issuing thread issues nothing: the TMA producer fills its
 *            stages and the exp warps wait for similarity tiles that never come;
 *   stall 2  the exp warps skip their loops: the issuer's first MMAs run, then
 *            it waits for exponentials that never come.
 * A kernel whose wait runs out raises the device error word (read and cleared
 * by gs_last_device_error, which then returns GS_ERR_TIMEOUT); its other warps
 * leave their loops; the producer waits (bounded) for the loads it issued and
 * the issuer for the MMAs it issued before TMEM is freed and the CTA exits.
 * Outputs of a call made in a stall mode are unspecified.  limit_ns must lie in
 * [1e3, 1e10] and stall in {0, 1, 2}, else GS_ERR_INVALID_ARG.  The setting is
 * per process and per device (the current one), synchronous, and applies to
 * launches made after it returns; restore (2000000000, 0) when done.
 */
gs_status gs_test_set_waits(uint64_t limit_ns, int stall);

/*
 * Synchronises `stream`, then reads and clears the raw device error word of the
 * tensor-core kernels into *word: bit 0 (1) a bounded wait ran out; bit 1 (2)
 * an fp32 kernel was launched with tensor-map boxes made for another
 * instantiation (it returned at once); bit 2 (4) a wait for work already issued
 * (the drain after an abort) ran out.  GS_ERR_INVALID_ARG for a NULL word,
 * GS_ERR_CUDA if the synchronisation or the read fails.
 */
gs_status gs_test_read_error_word(int *word, gs_stream_t stream);

/*
 * Measurement probe: the MUFU ex2 rate of an SM.  Launches `blocks` CTAs of
 * 1024 threads, one per SM (each holds 120 KB of shared memory); every thread
 * runs 8 independent chains v <- 2^(-v/2) for `iters` steps (8 * iters ex2 a
 * thread), and cycles[b] receives the SM cycles of CTA b's loop, so that
 * 1024 * 8 * iters / cycles[b] is the SM's ex2 results per clock.  cycles: device
 * array of `blocks` int64; sink: device array of blocks * 1024 floats (keeps the
 * results live).  blocks in [1, 4096], iters in [1, 2^20], else
 * GS_ERR_INVALID_ARG (checked before anything is launched).  Asynchronous on
 * `stream`.
 */
gs_status gs_test_ex2_probe(long long *cycles, float *sink, int blocks, int iters, gs_stream_t stream);

/*
 * Measurement probe: the cost of back-to-back tcgen05.mma instructions issued by
 * one thread.  Launches `blocks` CTAs of 128 threads, one per SM; in each, one
 * thread issues n_mma MMAs of M = 128, N = n_cols, K = 16 (kind::f16, zero
 * operands in shared memory, one TMEM accumulator), commits them and waits
 * (bounded: 2 s) for their completion; cycles[b] = the SM cycles from the first
 * issue to the completion (-1, and *status |= 1, if the wait ran out).  cycles:
 * device array of `blocks` int64; status: device int, zeroed by the caller.
 * blocks in [1, 4096], n_mma in [1, 65536], n_cols in {32, 64, 128, 256}, else
 * GS_ERR_INVALID_ARG (checked before anything is launched).  Asynchronous.
 */
gs_status gs_test_mma_probe(long long *cycles, int *status, int blocks, int n_mma, int n_cols,
                            gs_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GAUSS_B200_TESTING_H */
