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
 *   fa_debug_umma_2cta: one M = 256 tile over a cluster of two CTAs with every
 *     tcgen05 instruction in its cta_group::2 form, D = A B^T with A [256][K],
 *     B [N][K] bf16 and D [256][N] fp32.  CTA r holds A's rows [128 r, 128 r +
 *     128) (K-major in shared memory, or in its tensor memory with a_tmem) and
 *     B's rows [r N / 2, (r + 1) N / 2) (K-major, or N-contiguous with
 *     b_mn_major).  N = 128, K = 64 or 128.  *status (device int) is set to 1
 *     if the MMAs did not complete within 2 s.
 *   fa_debug_mma_rate: tensor-pipe rate.  `grid` CTAs (mode 2: grid / 2 CTA
 *     pairs), one per SM, each issue reps x 8 back-to-back 128 x n x 16 bf16
 *     MMAs into one TMEM accumulator (mode 0: both operands in shared memory;
 *     1: A in tensor memory; 2: M = 256 over a CTA pair with cta_group::2,
 *     n = 128 or 256) and write the SM clocks until completion to
 *     cycles[grid].  With kind > 0 four more warps per CTA load the SM with
 *     one kind of traffic (1 tcgen05.ld, 2 tcgen05.st, 3 st.shared,
 *     4 ld.shared, 5 bulk copy shared -> global, 6 bulk fp32 reduce-add,
 *     7 red.global.add.v4.f32, 8 ld.global hitting L1, 9 a quad transpose
 *     then red.global.add.v4.f32) and add their operation count to
 *     ops[grid] (4 KB per operation, 16 KB for kind 9).  Kinds 10-13 run
 *     FFMA-bound warps instead: 10 one on every SMSP, 11 one on the issuer's
 *     SMSP only, 12 three on the other SMSPs, 13 as 10 with the MMAs split
 *     over two issuing threads on two SMSPs (modes 0 and 1, n <= 128), 14 as
 *     11 with the MMAs issued by a converged warp, one lane elected by
 *     elect.sync (modes 0 and 1).  scratch: device
 *     floats, grid x 4 x 16384 of them.  cycles and ops: device arrays of
 *     64-bit counters (ops zeroed by the caller).  *status set to 1 if the
 *     MMAs did not complete within 2 s.
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
int fa_debug_umma_2cta(const void* A, const void* B, float* D, int N, int K, int b_mn_major, int a_tmem, int* status,
                       void* stream);
int fa_debug_mma_rate(int mode, int n, int kind, int grid, int reps, unsigned long long* cycles,
                      unsigned long long* ops, float* scratch, int* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_TESTING_H */
