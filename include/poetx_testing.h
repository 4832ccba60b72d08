/*
 * poetx_testing.h — kernel-level test hook of libpoetx (not needed by users of the layer).
 *
 * poetx_testing_gemm_bf16 runs the library's bf16 tensor-core contraction (tcgen05.mma with TMEM
 * accumulators, operands staged by TMA) on one plain product, so unit tests can compare the
 * kernel against a reference matmul for each operand layout:
 *     C[i, j] = sum_k A(i, k) B(k, j),  0 <= i < M, 0 <= j < N, 0 <= k < K
 *   A: bf16 device tensor [a_rows][a_cols] row-major.  a_mn = 0: A(i, k) = A[i][k] (K-major,
 *      a_rows >= M rows, a_cols = K);  a_mn = 1: A(i, k) = A[k][i] (M-major, a_rows = K).
 *   B: bf16 device tensor [b_rows][b_cols].  b_mn = 0: B(k, j) = B[j][k] (K-major, b_cols = K);
 *      b_mn = 1: B(k, j) = B[k][j] (N-major, b_rows = K).
 *   C: [M][ldc] row-major, fp32 (c_f32 = 1) or bf16 (c_f32 = 0, round-to-nearest-even).
 *   splits > 1 splits K into that many ranges of whole 64-wide K blocks and writes fp32
 *   partial products to C + s * M * ldc (c_f32 must be 1); the caller adds them. A count that
 *   would leave a range empty (e.g. 5 ranges over 16 blocks) is rejected with INVALID_ARG.
 *   variant 0 runs the single-CTA kernel (128 x BN tiles); variant 1 runs the CTA-pair kernel
 *   (tcgen05.mma.cta_group::2 on a 2-CTA cluster, 256 x 256 tiles; N % 256 == 0, M >= 256);
 *   variants 2 and 3 run the dense CTA-pair kernel on 256 x 512 tiles (A K-major, bf16 C,
 *   splits = 1, N % 512 == 0, M >= 256), with (2) or without (3) the two MMAs of a K step
 *   sharing A through the tensor core's collector buffer.
 *   epi_wait_ns > 0 limits the epilogue warps' wait for a finished accumulator to that many
 *   nanoseconds (0: the kernels' default of 4 s). It exists to exercise the bounded-wait error
 *   path: with a limit shorter than the main loop the wait runs out, the epilogue writes a
 *   nonzero code into the device error word (poetx_device_status then returns
 *   POETX_ERR_TIMEOUT and clears it), skips its stores and leaves; the producer and MMA roles
 *   finish or drain their copies and MMAs, TMEM is freed and the kernel returns. C is then
 *   unspecified. Use a product of at most two tiles per CTA (cluster) for a clean drain:
 *   the MMA role then never waits for an accumulator the epilogue would have handed back.
 * Returns POETX_ERR_UNSUPPORTED when the chosen kernel's tiling does not cover the shape
 * (N % 64 != 0, K-major extents < 64, misaligned pointers or strides); it never falls back.
 * Asynchronous on `stream`.
 */
#ifndef POETX_TESTING_H
#define POETX_TESTING_H
#include "poetx.h"
#ifdef __cplusplus
extern "C" {
#endif

poetx_status poetx_testing_gemm_bf16(const void* A, int64_t a_rows, int64_t a_cols, int32_t a_mn,
                                     const void* B, int64_t b_rows, int64_t b_cols, int32_t b_mn,
                                     int64_t M, int64_t N, int64_t K, void* C, int32_t c_f32,
                                     int64_t ldc, int32_t splits, int32_t variant,
                                     uint64_t epi_wait_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif
