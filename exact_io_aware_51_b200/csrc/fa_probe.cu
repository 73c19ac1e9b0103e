// Test-only probe of one tcgen05 MMA tile: D[128][N] = A[128][K] * B[N][K]^T.
//
// It checks, on its own, each operand layout the attention kernels hand to the
// tensor cores: 128-byte swizzled K-major and MN-major shared-memory operands,
// and A read from tensor memory.  The threads place A and B in shared memory
// with the same swizzle the TMA produces, one thread issues the MMAs, and the
// fp32 result is read back through tcgen05.ld.
//
// It is built into its own test library (libfa_probe.so), outside the product
// library, and declared in fa_testing.h, not in the public header.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_testing.h"
#include "sm100.cuh"

namespace fa {
namespace {

__global__ void __launch_bounds__(128, 1)
    umma_probe_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B, float* __restrict__ D,
                      int N, int K, int a_mn, int b_mn, int a_tmem) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                 // up to 128 x 128 bf16 = 32 KB
  uint8_t* sB = smem + 32768;         // up to 128 x 128 bf16 = 32 KB
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;

  // ---- A into shared memory ----
  for (int e = tid; e < 128 * K; e += 128) {
    const int m = e / K, k = e % K;
    uint32_t off;
    if (a_mn == 0)
      off = (k / 64) * (128 * 128) + sw128_offset(m, (k % 64) / 8) + (k % 8) * 2;
    else
      off = (m / 64) * (K * 128) + sw128_offset(k, (m % 64) / 8) + (m % 8) * 2;
    *reinterpret_cast<__nv_bfloat16*>(sA + off) = A[e];
  }
  // ---- B into shared memory ----
  for (int e = tid; e < N * K; e += 128) {
    const int n = e / K, k = e % K;
    uint32_t off;
    if (b_mn == 0)
      off = (k / 64) * (N * 128) + sw128_offset(n, (k % 64) / 8) + (k % 8) * 2;
    else
      off = (n / 64) * (K * 128) + sw128_offset(k, (n % 64) / 8) + (n % 8) * 2;
    *reinterpret_cast<__nv_bfloat16*>(sB + off) = B[e];
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tbase, 512);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;

  if (a_tmem) {
    // row m = tid into lane m, two bf16 per column starting at column 256
    for (int c0 = 0; c0 < K / 2; c0 += 16) {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int k = 2 * (c0 + i);
        const __nv_bfloat162 v = __halves2bfloat162(A[tid * K + k], A[tid * K + k + 1]);
        r[i] = *reinterpret_cast<const uint32_t*>(&v);
      }
      tmem_st16(tmem + lane_bits + 256 + c0, r);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (tid == 0) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    const uint32_t idesc = idesc_bf16(128, N, a_tmem ? 0 : a_mn, b_mn);
    for (int kk = 0; kk < K / 16; ++kk) {
      const uint64_t bd = (b_mn == 0) ? sw128_desc(b0 + (kk / 4) * (N * 128) + (kk % 4) * 32, 16, 1024)
                                      : sw128_desc(b0 + kk * 2048, K * 128, 1024);
      if (a_tmem) {
        umma_ts(tmem, tmem + 256 + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
      } else {
        const uint64_t ad = (a_mn == 0) ? sw128_desc(a0 + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024)
                                        : sw128_desc(a0 + kk * 2048, K * 128, 1024);
        umma_ss(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
    }
    umma_commit(&bar);
  }
  // bounded wait for the MMAs (no other role can stall this one)
  const uint64_t t0 = globaltimer_ns();
  bool done = false;
  while (!(done = mbar_try_wait(&bar, 0)) && globaltimer_ns() - t0 < 2000000000ull) {
  }
  done = __all_sync(0xffffffffu, done);
  tc_fence_after();
  if (done) {
    for (int c0 = 0; c0 < N; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_bits + c0, r);
      tmem_wait_ld();
      reg_fence32(r);
#pragma unroll
      for (int i = 0; i < 32; ++i) D[tid * N + c0 + i] = __uint_as_float(r[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The same probe for the 8-bit (e4m3) MMA with K = 128: A [128][128] K-major in
// shared memory or in TMEM (four elements per column), B [N][128] K-major or
// stored MN-major ([128 k][N], N contiguous).  One 128-byte swizzled row holds
// all 128 elements of a K-major row.
__global__ void __launch_bounds__(128, 1)
    umma_probe_f8_kernel(const uint8_t* __restrict__ A, const uint8_t* __restrict__ B, float* __restrict__ D, int N,
                         int b_mn, int a_tmem) {
  constexpr int K = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;          // 128 x 128 bytes
  uint8_t* sB = smem + 16384;  // N x 128 bytes (N <= 128)
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;

  for (int e = tid; e < 128 * K; e += 128) {
    const int m = e / K, k = e % K;
    sA[sw128_offset(m, k / 16) + (k % 16)] = A[e];
  }
  for (int e = tid; e < N * K; e += 128) {
    const int n = e / K, k = e % K;
    const uint32_t off = (b_mn == 0) ? sw128_offset(n, k / 16) + (k % 16) : sw128_offset(k, n / 16) + (n % 16);
    sB[off] = B[e];
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tbase, 512);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;

  if (a_tmem) {
    // row m = tid into lane m; column 256 + c holds k = 4c .. 4c + 3 (k = 4c in the low byte)
    for (int c0 = 0; c0 < K / 4; c0 += 16) {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint8_t* a4 = A + tid * K + 4 * (c0 + i);
        r[i] = static_cast<uint32_t>(a4[0]) | (static_cast<uint32_t>(a4[1]) << 8) |
               (static_cast<uint32_t>(a4[2]) << 16) | (static_cast<uint32_t>(a4[3]) << 24);
      }
      tmem_st16(tmem + lane_bits + 256 + c0, r);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (tid == 0) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    const uint32_t idesc = idesc_e4m3(128, N, 0, b_mn);
    for (int kk = 0; kk < K / 32; ++kk) {
      const uint64_t bd = (b_mn == 0) ? sw128_desc(b0 + kk * 32, 16, 1024) : sw128_desc(b0 + kk * 4096, 16384, 1024);
      if (a_tmem)
        umma_ts_f8(tmem, tmem + 256 + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
      else
        umma_ss_f8(tmem, sw128_desc(a0 + kk * 32, 16, 1024), bd, idesc, kk > 0 ? 1u : 0u);
    }
    umma_commit(&bar);
  }
  const uint64_t t0 = globaltimer_ns();
  bool done = false;
  while (!(done = mbar_try_wait(&bar, 0)) && globaltimer_ns() - t0 < 2000000000ull) {
  }
  done = __all_sync(0xffffffffu, done);
  tc_fence_after();
  if (done) {
    for (int c0 = 0; c0 < N; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_bits + c0, r);
      tmem_wait_ld();
      reg_fence32(r);
#pragma unroll
      for (int i = 0; i < 32; ++i) D[tid * N + c0 + i] = __uint_as_float(r[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Two-CTA probe: one M = 256 tile over a cluster of two CTAs,
// D[256][N] = A[256][K] * B[N][K]^T, with every tcgen05 instruction in its
// cta_group::2 form.  CTA r holds rows [128 r, 128 r + 128) of A (in shared
// memory, K-major, or in its tensor memory) and rows [r N/2, (r + 1) N/2) of B
// (K-major, or MN-major with the N rows contiguous); CTA 0 issues the MMAs, the
// commit arrives on the barrier of both CTAs, and each CTA reads its 128 rows
// of D out of its own tensor memory.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
    umma2_probe_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B,
                       float* __restrict__ D, int N, int K, int b_mn, int a_tmem, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;          // 128 x K bf16, up to 32 KB
  uint8_t* sB = smem + 32768;  // N/2 x K bf16, up to 16 KB
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int rank = static_cast<int>(cluster_rank());
  const int nh = N / 2;
  const __nv_bfloat16* Ar = A + static_cast<size_t>(rank) * 128 * K;
  const __nv_bfloat16* Br = B + static_cast<size_t>(rank) * nh * K;

  if (!a_tmem) {
    for (int e = tid; e < 128 * K; e += 128) {
      const int m = e / K, k = e % K;
      *reinterpret_cast<__nv_bfloat16*>(sA + (k / 64) * (128 * 128) + sw128_offset(m, (k % 64) / 8) + (k % 8) * 2) =
          Ar[e];
    }
  }
  for (int e = tid; e < nh * K; e += 128) {
    const int n = e / K, k = e % K;
    uint32_t off;
    if (b_mn == 0)
      off = (k / 64) * (nh * 128) + sw128_offset(n, (k % 64) / 8) + (k % 8) * 2;
    else  // nh = 64: one 64-element chunk per reduction row
      off = sw128_offset(k, n / 8) + (n % 8) * 2;
    *reinterpret_cast<__nv_bfloat16*>(sB + off) = Br[e];
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&tbase))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
  if (a_tmem) {
    // row 128 rank + tid into lane tid, two bf16 per column from column 256
    for (int c0 = 0; c0 < K / 2; c0 += 16) {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int k = 2 * (c0 + i);
        const __nv_bfloat162 v = __halves2bfloat162(Ar[tid * K + k], Ar[tid * K + k + 1]);
        r[i] = *reinterpret_cast<const uint32_t*>(&v);
      }
      tmem_st16(tmem + lane_bits + 256 + c0, r);
    }
    tmem_wait_st();
  }
  // both CTAs' operands, barriers and tensor memory are in place
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();

  if (rank == 0 && tid == 0) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    const uint32_t idesc = idesc_bf16(256, N, 0, b_mn);
    for (int kk = 0; kk < K / 16; ++kk) {
      const uint64_t bd = (b_mn == 0) ? sw128_desc(b0 + (kk / 4) * (nh * 128) + (kk % 4) * 32, 16, 1024)
                                      : sw128_desc(b0 + kk * 2048, 16, 1024);
      const uint32_t acc = kk > 0 ? 1u : 0u;
      if (a_tmem) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem),
            "r"(tmem + 256 + kk * 8), "l"(bd), "r"(idesc), "r"(acc)
            : "memory");
      } else {
        const uint64_t ad = sw128_desc(a0 + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
            "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
            : "memory");
      }
    }
    const uint16_t mask = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(&bar)),
        "h"(mask)
        : "memory");
  }
  // bounded wait for the MMAs
  const uint64_t t0 = globaltimer_ns();
  bool done = false;
  while (!(done = mbar_try_wait(&bar, 0)) && globaltimer_ns() - t0 < 2000000000ull) {
  }
  done = __all_sync(0xffffffffu, done);
  if (!done && (tid & 31) == 0) atomicExch(status, 1);
  tc_fence_after();
  if (done) {
    for (int c0 = 0; c0 < N; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_bits + c0, r);
      tmem_wait_ld();
      reg_fence32(r);
#pragma unroll
      for (int i = 0; i < 32; ++i) D[(static_cast<size_t>(rank) * 128 + tid) * N + c0 + i] = __uint_as_float(r[i]);
    }
  }
  // neither CTA frees its tensor memory while the pair's MMAs may still use it
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

cudaError_t launch_umma_probe_f8(const void* A, const void* B, float* D, int N, int b_mn, int a_tmem,
                                 cudaStream_t s) {
  constexpr int smem = 32768 + 1024;
  cudaError_t e = cudaFuncSetAttribute(umma_probe_f8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  umma_probe_f8_kernel<<<1, 128, smem, s>>>(static_cast<const uint8_t*>(A), static_cast<const uint8_t*>(B), D, N,
                                            b_mn, a_tmem);
  return cudaGetLastError();
}

cudaError_t launch_umma_probe(const void* A, const void* B, float* D, int N, int K, int a_mn, int b_mn, int a_tmem,
                              cudaStream_t s) {
  constexpr int smem = 65536 + 1024;
  cudaError_t e = cudaFuncSetAttribute(umma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  umma_probe_kernel<<<1, 128, smem, s>>>(static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B),
                                         D, N, K, a_mn, b_mn, a_tmem);
  return cudaGetLastError();
}

cudaError_t launch_umma2_probe(const void* A, const void* B, float* D, int N, int K, int b_mn, int a_tmem, int* status,
                               cudaStream_t s) {
  constexpr int smem = 49152 + 1024;
  cudaError_t e = cudaFuncSetAttribute(umma2_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  umma2_probe_kernel<<<2, 128, smem, s>>>(static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B),
                                          D, N, K, b_mn, a_tmem, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Tensor-pipe rate probe.  One CTA (or CTA pair, MODE 2) per SM: warp 0 issues
// reps x 8 back-to-back 128 x N x 16 bf16 MMAs (256 x N x 16 for the pair)
// into one TMEM accumulator and records the SM clocks until they complete.
// Warps 4-7 can meanwhile load the SM with one kind of traffic and count
// their 4 KB operations (the drain pattern, kind 9, counts 16 KB):
//   1 tcgen05.ld, 2 tcgen05.st (TMEM columns 256-383), 3 st.shared,
//   4 ld.shared, 5 bulk copy shared -> global, 6 bulk fp32 reduce-add
//   shared -> global, 7 red.global.add.v4.f32 from registers, 8 ld.global
//   (L1 hits), 9 a 4 x 4 transpose in lane quads then red.global.add.v4.f32,
//   10 FFMA-bound code on warps 4-7 (one per SMSP), 11 the same on warp 4
//   only (the issuer's SMSP), 12 on warps 5-7 only (the other SMSPs), 13 as
//   10 with the MMAs split over two issuers (warps 0 and 1, SMSPs 0 and 1,
//   each into its own accumulator), 14 as 11 with the MMAs issued by all of
//   warp 0, converged, one lane elected by elect.sync (modes 0 and 1).
// Operand values are arbitrary: only the timing is read.
// ---------------------------------------------------------------------------
constexpr int kRateSmem = 200 * 1024;  // more than half the SM's shared memory: one CTA per SM

template <int MODE>  // 0: A and B in shared memory, 1: A in TMEM, 2: CTA pair, both in shared memory
__global__ void __launch_bounds__(256, 1)
    mma_rate_kernel(int N, int reps, int kind, unsigned long long* __restrict__ cycles,
                    unsigned long long* __restrict__ ops, float* __restrict__ scratch, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = smem_u32(smem);              // [128][128] bf16, two 16 KB K-chunks
  const uint32_t sB = smem_u32(smem + 32768);      // up to [256][128] bf16, two K-chunks
  const uint32_t sX = smem_u32(smem + 98304);      // 64 KB the traffic warps read and write
  __shared__ uint64_t bar, bar2;
  __shared__ uint32_t tbase;
  __shared__ volatile int stop;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 98304 / 4; i += 256)
    reinterpret_cast<uint32_t*>(smem)[i] = 0x3c003c00u ^ ((static_cast<uint32_t>(i) * 2654435761u) & 0x00ff00ffu);
  if (tid == 0) {
    stop = 0;
    mbar_init(&bar, 1);
    mbar_init(&bar2, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    if (MODE == 2) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&tbase))
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      tmem_alloc(&tbase, 512);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  if (MODE == 1 && warp < 4) {  // A: 128 x 128 bf16 in TMEM columns 384..447
    uint32_t r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = 0x3c003c00u ^ static_cast<uint32_t>(tid * 31 + i);
    for (int c0 = 0; c0 < 64; c0 += 16) tmem_st16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 384 + c0, r);
    tmem_wait_st();
  }
  tc_fence_before();
  if (MODE == 2) cluster_sync_all(); else __syncthreads();
  tc_fence_after();

  const bool two = kind == 13;  // a second issuer: lane 0 of warp 1, its own accumulator at column 128
  const bool conv = kind == 14;  // all of warp 0 issues, converged, through elect.sync
  const bool issuer = (tid == 0 && (MODE != 2 || cluster_rank() == 0)) || (two && tid == 32);
  const unsigned long long c0 = clock64();
  if (MODE != 2 && conv && warp == 0) {
    const uint32_t idesc = (MODE == 1) ? idesc_bf16(128, N, 0, 1) : idesc_bf16(128, N, 0, 0);
    for (int r = 0; r < reps; ++r) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = (r > 0 || kk > 0) ? 1u : 0u;
        if (MODE == 1)
          umma_ts_w(tmem, tmem + 384 + kk * 8, sw128_desc(sB + kk * 2048, 16384, 1024), idesc, acc);
        else
          umma_ss_w(tmem, sw128_desc(sA + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                    sw128_desc(sB + (kk >> 2) * (N * 128) + (kk & 3) * 32, 16, 1024), idesc, acc);
      }
    }
    umma_commit_w(&bar);
    __syncwarp();
  } else if (issuer && !conv) {
    const int nb = (MODE == 2) ? N / 2 : N;  // B rows in this CTA
    const uint32_t idesc = (MODE == 1) ? idesc_bf16(128, N, 0, 1) : idesc_bf16(MODE == 2 ? 256 : 128, N, 0, 0);
    if (!two) {
      // the plain stream: nothing between the MMAs but their constant offsets
      for (int r = 0; r < reps; ++r) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (r > 0 || kk > 0) ? 1u : 0u;
          const uint64_t ad = sw128_desc(sA + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(sB + (kk >> 2) * (nb * 128) + (kk & 3) * 32, 16, 1024);
          if (MODE == 0) {
            umma_ss(tmem, ad, bd, idesc, acc);
          } else if (MODE == 1) {
            // B MN-major: 16 K-rows of 128 bytes per step, N groups of 64 at 16 KB
            umma_ts(tmem, tmem + 384 + kk * 8, sw128_desc(sB + kk * 2048, 16384, 1024), idesc, acc);
          } else {
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
                : "memory");
          }
        }
      }
    } else {
      // two issuers (modes 0 and 1): half the groups each, each into its own accumulator
      const uint32_t d = tmem + ((tid == 32) ? 128u : 0u);
      const int my_reps = (tid == 32) ? reps - reps / 2 : reps / 2;
      for (int r = 0; r < my_reps; ++r) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (r > 0 || kk > 0) ? 1u : 0u;
          if (MODE == 1)
            umma_ts(d, tmem + 384 + kk * 8, sw128_desc(sB + kk * 2048, 16384, 1024), idesc, acc);
          else
            umma_ss(d, sw128_desc(sA + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                    sw128_desc(sB + (kk >> 2) * (nb * 128) + (kk & 3) * 32, 16, 1024), idesc, acc);
        }
      }
    }
    if (MODE == 2) {
      const uint16_t mask = 0x3;
      asm volatile(
          "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
              smem_u32(&bar)),
          "h"(mask)
          : "memory");
    } else {
      umma_commit(tid == 32 ? &bar2 : &bar);
    }
  }
  if (kind >= 10) {
    // FFMA-bound warps: eight independent chains, so every cycle has an instruction ready
    const bool busy = (kind == 11 || kind == 14) ? warp == 4 : (kind == 12) ? (warp >= 5 && warp <= 7) : (warp >= 4 && warp <= 7);
    if (busy) {
      float f[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = static_cast<float>(lane + i);
      unsigned long long n = 0;
      for (int it = 0; it < 1000000 && !stop; ++it, ++n) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = fmaf(f[i], 0.999f, 0.5f);
        }
      }
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) sum += f[i];
      if (lane == 0) atomicAdd(ops + blockIdx.x, n + (sum == 12345.f ? 1u : 0u));
    }
  } else if (warp >= 4 && kind > 0) {
    const int w4 = warp - 4;
    const uint32_t lane_bits = static_cast<uint32_t>(w4 * 32) << 16;
    float* mine = scratch + (static_cast<size_t>(blockIdx.x) * 4 + w4) * 16384;  // this warp's 64 KB
    unsigned long long n = 0;
    uint32_t acc = 0;
    for (int it = 0; it < 200000 && !stop; ++it, ++n) {
      if (kind == 1) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_bits + 256 + (it & 3) * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) acc += r[i];
      } else if (kind == 2) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = static_cast<uint32_t>(it + i);
        tmem_st32(tmem + lane_bits + 256 + (it & 3) * 32, r);
        tmem_wait_st();
      } else if (kind == 3 || kind == 4) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t addr = sX + (((w4 * 8 + u) * 512 + lane * 16 + (it & 3) * 16384) & 65535);
          if (kind == 3) {
            st_shared_v4(addr, it, u, acc, 1u);
          } else {
            uint32_t x, y, z, q;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(x), "=r"(y), "=r"(z), "=r"(q) : "r"(addr));
            acc += x ^ y ^ z ^ q;
          }
        }
      } else if (kind == 5 || kind == 6) {
        if (lane == 0) {
          float* dst = mine + (it & 15) * 1024;
          const uint32_t src = sX + w4 * 16384 + (it & 3) * 4096;
          if (kind == 5)
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], 4096;" ::"l"(dst), "r"(src)
                         : "memory");
          else
            asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], 4096;" ::"l"(dst),
                         "r"(src)
                         : "memory");
          bulk_commit();
          asm volatile("cp.async.bulk.wait_group.read 4;" ::: "memory");
        }
        __syncwarp();
      } else if (kind == 7) {
        // rows of 128 floats: lanes with the same (lane & 3) cover 128 contiguous bytes of one row
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float* pp = mine + (((it & 3) * 8 + u) * 4 + (lane & 3)) * 128 + (lane >> 2) * 4;
          asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(pp), "f"(1.f), "f"(2.f),
                       "f"(3.f), "f"(4.f)
                       : "memory");
        }
      } else if (kind == 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float x, y, z, q;
          asm volatile("ld.global.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(x), "=f"(y), "=f"(z), "=f"(q)
                       : "l"(mine + u * 128 + lane * 4));
          acc += __float_as_uint(x) ^ __float_as_uint(q);
        }
      } else {
        // 128 columns per lane; per 4 columns two butterfly stages (xor 2, xor 1) leave
        // lane 4 k + j holding column j of its quad's 4 x 4 block, added as one vector
        const int j = lane & 3;
        const bool hi = (j & 2) != 0, odd = (j & 1) != 0;
#pragma unroll 4
        for (int c = 0; c < 128; c += 4) {
          const float x0 = static_cast<float>(c + it), x1 = x0 + 1.f, x2 = x0 + 2.f, x3 = x0 + 3.f;
          const float r0 = __shfl_xor_sync(0xffffffffu, hi ? x0 : x2, 2);
          const float r1 = __shfl_xor_sync(0xffffffffu, hi ? x1 : x3, 2);
          const float w0 = hi ? r0 : x0, w1 = hi ? r1 : x1, w2 = hi ? x2 : r0, w3 = hi ? x3 : r1;
          const float q0 = __shfl_xor_sync(0xffffffffu, odd ? w0 : w1, 1);
          const float q1 = __shfl_xor_sync(0xffffffffu, odd ? w2 : w3, 1);
          float* pp = mine + (c + j) * 128 + 4 * (lane >> 2);
          asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(pp),
                       "f"(odd ? q0 : w0), "f"(odd ? w1 : q0), "f"(odd ? q1 : w2), "f"(odd ? w3 : q1)
                       : "memory");
        }
      }
    }
    if ((kind == 5 || kind == 6) && lane == 0) bulk_wait_all();
    if (lane == 0) atomicAdd(ops + blockIdx.x, n + (acc == 0xdeadbeefu ? 1u : 0u));
  }
  if (tid == 0) {
    const uint64_t t0 = globaltimer_ns();
    bool done = false;
    while (!(done = mbar_try_wait(&bar, 0)) && globaltimer_ns() - t0 < 2000000000ull) {
    }
    if (done && two) {
      while (!(done = mbar_try_wait(&bar2, 0)) && globaltimer_ns() - t0 < 2000000000ull) {
      }
    }
    if (!done) atomicExch(status, 1);
    cycles[blockIdx.x] = clock64() - c0;
    stop = 1;
  }
  __syncwarp();
  tc_fence_before();
  if (MODE == 2) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    if (MODE == 2)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    else
      tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_mma_rate(int mode, int N, int kind, int grid, int reps, unsigned long long* cycles,
                            unsigned long long* ops, float* scratch, int* status, cudaStream_t s) {
  auto go = [&](auto kernel) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRateSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = kRateSmem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (mode == 2) ? 2 : 1;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, N, reps, kind, cycles, ops, scratch, status);
  };
  if (mode == 0) return go(mma_rate_kernel<0>);
  if (mode == 1) return go(mma_rate_kernel<1>);
  return go(mma_rate_kernel<2>);
}

// The current device must be an sm_100 part (tcgen05).
int probe_device_ok() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FA_ERR_LAUNCH;
  return (major == 10 && minor == 0) ? FA_OK : FA_ERR_ARCH;
}

}  // namespace
}  // namespace fa

extern "C" {

int fa_debug_umma(const void* A, const void* B, float* D, int N, int K, int a_mn_major, int b_mn_major, int a_tmem,
                  void* stream) {
  if (!A || !B || !D) return FA_ERR_INVALID_ARG;
  if ((N != 64 && N != 128) || (K != 64 && K != 128)) return FA_ERR_UNSUPPORTED;
  const int rc = fa::probe_device_ok();
  if (rc != FA_OK) return rc;
  const cudaError_t e = fa::launch_umma_probe(A, B, D, N, K, a_mn_major ? 1 : 0, b_mn_major ? 1 : 0, a_tmem ? 1 : 0,
                                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

int fa_debug_umma_f8(const void* A, const void* B, float* D, int N, int b_mn_major, int a_tmem, void* stream) {
  if (!A || !B || !D) return FA_ERR_INVALID_ARG;
  if (N != 64 && N != 128) return FA_ERR_UNSUPPORTED;
  const int rc = fa::probe_device_ok();
  if (rc != FA_OK) return rc;
  const cudaError_t e =
      fa::launch_umma_probe_f8(A, B, D, N, b_mn_major ? 1 : 0, a_tmem ? 1 : 0, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

int fa_debug_umma_2cta(const void* A, const void* B, float* D, int N, int K, int b_mn_major, int a_tmem, int* status,
                       void* stream) {
  if (!A || !B || !D || !status) return FA_ERR_INVALID_ARG;
  if (N != 128 || (K != 64 && K != 128)) return FA_ERR_UNSUPPORTED;
  const int rc = fa::probe_device_ok();
  if (rc != FA_OK) return rc;
  const cudaError_t e = fa::launch_umma2_probe(A, B, D, N, K, b_mn_major ? 1 : 0, a_tmem ? 1 : 0, status,
                                               static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

int fa_debug_mma_rate(int mode, int n, int kind, int grid, int reps, unsigned long long* cycles,
                      unsigned long long* ops, float* scratch, int* status, void* stream) {
  if (!cycles || !ops || !scratch || !status) return FA_ERR_INVALID_ARG;
  if (mode < 0 || mode > 2 || kind < 0 || kind > 14 || grid < 1 || grid > 4096 || reps < 1 || reps > 100000)
    return FA_ERR_INVALID_ARG;
  if (kind == 13 && (mode == 2 || n > 128)) return FA_ERR_UNSUPPORTED;  // the second accumulator sits at column 128
  if (kind == 14 && mode == 2) return FA_ERR_UNSUPPORTED;
  if (mode == 2 ? (n != 128 && n != 256) || grid % 2 != 0 : (n != 64 && n != 128 && n != 256))
    return FA_ERR_UNSUPPORTED;
  const int rc = fa::probe_device_ok();
  if (rc != FA_OK) return rc;
  const cudaError_t e = fa::launch_mma_rate(mode, n, kind, grid, reps, cycles, ops, scratch, status,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

}  // extern "C"
