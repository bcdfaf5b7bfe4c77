/*
 * flce_diag.h -- diagnostic entry points of libflce.so.
 *
 * These are not part of the method.  They exist so that the test suite can
 * check building blocks of the library in isolation: the tensor-core GEMM
 * core with each operand layout, and the bounded-wait failure path.  Same
 * conventions as flce.h (device pointers, caller-owned memory, work enqueued
 * on `stream`).
 */
#ifndef FLCE_DIAG_H_
#define FLCE_DIAG_H_

#include "flce.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * out[M x N] (float32, row-major) = scale * A * B^T, computed by the same
 * persistent tcgen05 kernel the loss uses, with a plain store epilogue.
 *
 *   A: a_mn == 0 -> [M x K] row-major (K contiguous)
 *      a_mn != 0 -> [K x M] row-major (M contiguous)
 *   B: b_mn == 0 -> [N x K] row-major;  b_mn != 0 -> [K x N] row-major
 *
 * M, N, K >= 1; the contiguous extent of each operand must be a multiple
 * of 8 elements.  `ws` is any device buffer of >= 256 bytes used for the
 * error word.
 */
FLCE_API flce_status flce_diag_gemm(const void* A, const void* B, float* out,
                           int64_t M, int64_t N, int64_t K, int dtype, int a_mn, int b_mn,
                           float scale, void* ws, size_t ws_bytes, flce_stream stream);

/*
 * Launches one block that waits on a pipeline barrier nothing ever completes,
 * with a limit of `limit_ns` nanoseconds.  The wait must give up, record
 * FLCE_ERR_TIMEOUT in the error word of `ws` and return; the call then
 * reports it through flce_device_status().  No fault, trap or hang is
 * involved.
 */
FLCE_API flce_status flce_diag_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, flce_stream stream);

/*
 * Computes y_poly[i] = ex2_poly(x[i]) (the exponential the epilogues evaluate
 * on the FMA pipe for small hidden sizes) and y_sfu[i] = ex2.approx(x[i])
 * (the special-function unit's), for accuracy tests.  Device pointers, n >= 0.
 */
FLCE_API flce_status flce_diag_exp2(const float* x, float* y_poly, float* y_sfu, int64_t n,
                                    flce_stream stream);

/*
 * Per-launch timing of the library's own kernels.  Between begin and end,
 * every kernel the library enqueues is bracketed by two CUDA events on the
 * caller's stream (this adds no synchronisation), except the backward's chain
 * of GEMM launches, which overlap one another (programmatic dependent launch)
 * and are timed as one span from before the first to after the last.  end()
 * waits for those events and returns, per kind k in [0, nkinds), the summed
 * duration in ms and the number of launches:
 *   0 = forward GEMM, 1 = backward GEMM chain, 2 = plain GEMM (diagnostic),
 *   3 = every other kernel (compaction, gather, merge, loss, sort, db, scatter).
 */
FLCE_API flce_status flce_diag_profile_begin(void);
FLCE_API flce_status flce_diag_profile_end(double* ms, int64_t* launches, int nkinds);

#ifdef __cplusplus
}
#endif

#endif /* FLCE_DIAG_H_ */
