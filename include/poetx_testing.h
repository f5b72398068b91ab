/*
 * poetx_testing.h — test hook of libpoetx: direct access to the batched GEMM core that every
 * contraction of the POET-X layer runs on (the block-diagonal products, the W0' products, the
 * per-block gradients, the Cayley–Neumann powers and the merge; replication review of POET-X,
 * "Summary": batch-parallel block-diagonal matmul).  Used by the tests to check each operand
 * layout and tile width against a plain fp32 matmul.  Not needed by users of the layer.
 *
 *   D[z][m][n] (+ split s) = alpha * sum_{k in split s} A[z][m][k] * B[z][n][k] + beta * C[z][m][n]
 *                            (+ 1 where m == n if diag)
 *   A (a_mn == 0): A[z][m][k] = a[(z*a_zrow + m) * a_ld + z*a_zcol + k]
 *     (a_mn == 1): A[z][m][k] = a[(z*a_zrow + k) * a_ld + z*a_zcol + m]      (B likewise with n)
 *   D[z][m][n] at d[(z*d_zrow + m) * d_ld + z*d_zcol + n + s*d_split_stride]; C like D (no split).
 * dtype selects the operand type (POETX_BF16: tcgen05 tensor cores; POETX_F32: fp32 CUDA cores);
 * d_dtype the output type; C is float32 or NULL.  All pointers are device pointers; the call
 * is asynchronous on `stream`.  a_rows/a_cols (b_rows/b_cols) are the extents of the whole
 * operand arrays; the call is rejected (POETX_ERR_INVALID_ARG) if any addressed element lies
 * outside them.
 */
#ifndef POETX_TESTING_H_
#define POETX_TESTING_H_

#include "poetx.h"

#ifdef __cplusplus
extern "C" {
#endif

poetx_status poetx_test_gemm(int dtype, int M, int N, int K, int batch, int splits,
                             const void* a, long long a_rows, long long a_cols, long long a_ld,
                             long long a_zrow, long long a_zcol, int a_mn,
                             const void* b, long long b_rows, long long b_cols, long long b_ld,
                             long long b_zrow, long long b_zcol, int b_mn,
                             void* d, int d_dtype, long long d_ld, long long d_zrow, long long d_zcol,
                             long long d_split_stride, float alpha, float beta, const float* c,
                             long long c_ld, long long c_zrow, long long c_zcol, int diag,
                             poetx_stream stream);

/* Failure-detection probe (the bounded device-side waits of every kernel; no GPU fault is
 * involved).  Launches one CTA that waits on a shared-memory mbarrier nothing arrives on, with the
 * wait bounded by limit_ns nanoseconds of the device's global timer (1 us .. 100 ms).  The wait
 * runs out, the kernel records a device timeout (poetx_device_status() then returns
 * POETX_ERR_DEVICE_TIMEOUT with detail (7 << 8) | 1) and writes 2 to *returned (a device int;
 * 1 would mean that the wait completed).  Errors: INVALID_ARG (NULL, limit out of range),
 * ALIGNMENT, CUDA. */
poetx_status poetx_test_wait_timeout(long long limit_ns, int* returned, poetx_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* POETX_TESTING_H_ */
