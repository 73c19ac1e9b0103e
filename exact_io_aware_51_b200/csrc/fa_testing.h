/*
 * Test-only entry points.  None of them is part of the library's public
 * interface (include/fa.h); the tests use them to check pieces of the kernels
 * on their own.
 *
 * In libfa.so (the product library):
 *   fa_debug_inject: 1 makes the next forward launches' first key-tile
 *     barrier expect 16 bytes that never arrive, so its waits expire and the
 *     launch reports FA_ERR_DEVICE_TIMEOUT; 2 (honoured only by the checking
 *     build libfa_debug.so) moves the forward's first key-tile row past N, so
 *     the loader's bounds check refuses the load and the launch reports
 *     FA_ERR_DEVICE_CHECK; 0 turns it off (process-wide).
 *
 * In libfa_probe.so (a separate test library built from fa_probe.cu):
 *   fa_debug_umma: one 128 x N x K tcgen05 MMA tile, D = A B^T, with A [128][K]
 *     and B [N][K] bf16 row-major device arrays and D [128][N] fp32.
 *     a_mn_major / b_mn_major choose how the operand is laid out in shared
 *     memory (0: the reduction dimension contiguous, 1: the M or N dimension
 *     contiguous); a_tmem reads A from tensor memory instead.  N and K must be
 *     64 or 128.  Asynchronous on `stream`.
 *   fa_debug_umma_f8: the same probe for the 8-bit MMA (kind::f8f6f4, e4m3
 *     operands, fp32 accumulation) with K = 128: A [128][128] and B [N][128]
 *     e4m3 bytes, D [128][N] fp32.  b_mn_major stores B with N contiguous;
 *     a_tmem reads A from tensor memory (four elements per column).  N must be
 *     64 or 128.
 * Return values are the fa_status codes of include/fa.h.
 */
#ifndef FA_TESTING_H
#define FA_TESTING_H

#ifdef __cplusplus
extern "C" {
#endif

void fa_debug_inject(int mode);

int fa_debug_umma(const void* A, const void* B, float* D, int N, int K, int a_mn_major, int b_mn_major,
                  int a_tmem, void* stream);
int fa_debug_umma_f8(const void* A, const void* B, float* D, int N, int b_mn_major, int a_tmem, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_TESTING_H */
