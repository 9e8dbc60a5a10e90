/*
 * attn_diag.h -- diagnostic entry points of libattn_b200.so, kept apart from the compute ABI in
 * attn.h. They exercise parts of the kernels in isolation (the bounded waits and the FMA-pipe
 * exponential) so that tests can check them on the GPU; no compute path needs them.
 * Conventions (device pointers, streams, status codes) are those of attn.h.
 */
#ifndef ATTN_B200_DIAG_H
#define ATTN_B200_DIAG_H

#include "attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * attn_selftest_wait_timeout -- launches one CTA that waits on a shared-memory barrier nothing
 * ever arrives on, with a wall-clock limit of `limit_us` microseconds (1..1000000). The wait
 * runs out, the kernel records ATTN_ERR_TIMEOUT in the device error word and returns; the CUDA
 * context stays usable. Pair with attn_check_device() to observe the status. Enqueued on
 * `stream`; returns ATTN_ERR_INVALID_ARG for a limit outside the range.
 */
attn_status attn_selftest_wait_timeout(unsigned int limit_us, void *stream);

/*
 * attn_selftest_exp2 -- y[i] = 2^x[i] for n device floats, computed with the FMA-pipe polynomial
 * the prefill softmax uses for part of its exponentials (round-to-nearest range reduction,
 * degree-3 minimax polynomial; relative error below 1e-4 for x in [-125, 64]; for x below -126,
 * -inf included, the result is exactly 0; between -126 and -125 it is tiny but not accurate).
 * x and y are device pointers; enqueued on `stream`.
 */
attn_status attn_selftest_exp2(const float *x, float *y, int n, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_DIAG_H */
