// Elementwise kernels for attention over a sequence split into chunks (ring
// attention: "Flash Attention" (Ultralytics glossary), "Flash Attention и
// смежные понятия" -- each device computes blockwise attention for its part of
// a long sequence while key/value blocks travel around a ring of devices).
//
// A query chunk's output is assembled from one partial result per key chunk.
// Each partial (O_c, LSE_c) is exact attention over that key chunk alone, so
// two partials combine with the same correction the online softmax applies
// between key blocks ("Flash Attention" (karlkratz.de), "Tiling"): with
// m = max(LSE_a, LSE_b), w_x = exp(LSE_x - m),
//     O = (w_a O_a + w_b O_b) / (w_a + w_b),   LSE = m + ln(w_a + w_b).
// The running O is kept in fp32; gradients of a chunk summed over the ring are
// accumulated in fp32 as well.  All three kernels are bandwidth-bound: 8
// elements per thread, 16-byte loads and stores, grids of 16 CTAs per SM.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void unpack8(uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  u.x = pack_bf16x2(f[0], f[1]);
  u.y = pack_bf16x2(f[2], f[3]);
  u.z = pack_bf16x2(f[4], f[5]);
  u.w = pack_bf16x2(f[6], f[7]);
  return u;
}

// One thread per 8 features of one (b, n, h) row; the D / 8 threads of a row are
// consecutive lanes of one warp.  A warp takes kRows = 2 x 32 / (D / 8) rows per
// trip, issuing the loads of both halves before any arithmetic so twice the
// bytes are in flight.  Trips are per warp, so every lane runs the same number
// and the warp can meet at __syncwarp() between reading the rows' old LSE and
// writing the new one.  Idx is 32-bit whenever B N H d fits, so the
// row -> (b, n, h) split costs a few integer instructions rather than 64-bit
// divisions.
template <int D, typename Idx>
__global__ void __launch_bounds__(kThreads)
    merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc, const __nv_bfloat16* __restrict__ o_part,
                 const float* __restrict__ lse_part, __nv_bfloat16* __restrict__ o_out, int B, int H, int N,
                 int init) {
  constexpr int kPerRow = D / 8;
  constexpr int kRowsPerHalf = 32 / kPerRow;
  constexpr int kRows = 2 * kRowsPerHalf;
  const Idx rows = static_cast<Idx>(B) * N * H;
  const int lane = threadIdx.x & 31;
  const int part = lane % kPerRow;
  const Idx nwarps = static_cast<Idx>(gridDim.x) * (kThreads / 32);
  for (Idx r0 = (static_cast<Idx>(blockIdx.x) * (kThreads / 32) + threadIdx.x / 32) * kRows; r0 < rows;
       r0 += nwarps * kRows) {
    bool active[2];
    Idx li[2], oi[2];
    uint4 pb[2];
    float4 a0[2], a1[2];
    float la[2], lb[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const Idx row = r0 + u * kRowsPerHalf + lane / kPerRow;  // (b, n, h) in [B, N, H] order
      active[u] = row < rows;
      const Idx h = row % static_cast<Idx>(H);
      const Idx bn = row / static_cast<Idx>(H);
      const Idx n = bn % static_cast<Idx>(N);
      const Idx b = bn / static_cast<Idx>(N);
      li[u] = (b * H + h) * N + n;
      oi[u] = row * D + part * 8;
      la[u] = -INFINITY;
      lb[u] = -INFINITY;
      pb[u] = make_uint4(0u, 0u, 0u, 0u);
      a0[u] = a1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (active[u]) {
        pb[u] = *reinterpret_cast<const uint4*>(o_part + oi[u]);
        lb[u] = lse_part[li[u]];
        if (!init) {
          la[u] = lse_acc[li[u]];
          a0[u] = *reinterpret_cast<const float4*>(o_acc + oi[u]);
          a1[u] = *reinterpret_cast<const float4*>(o_acc + oi[u] + 4);
        }
      }
    }
    float l[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float o[8], ob[8];
      unpack8(pb[u], ob);
      const float oa[8] = {a0[u].x, a0[u].y, a0[u].z, a0[u].w, a1[u].x, a1[u].y, a1[u].z, a1[u].w};
      l[u] = -INFINITY;
      if (init) {
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = ob[i];
        l[u] = lb[u];
      } else {
        const float m = fmaxf(la[u], lb[u]);
        if (m == -INFINITY) {  // neither part saw a key
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = 0.f;
        } else {
          const float wa = expf(la[u] - m), wb = expf(lb[u] - m);
          const float inv = 1.f / (wa + wb);
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = (wa * oa[i] + wb * ob[i]) * inv;
          l[u] = m + logf(wa + wb);
        }
      }
      if (active[u]) {
        *reinterpret_cast<float4*>(o_acc + oi[u]) = make_float4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<float4*>(o_acc + oi[u] + 4) = make_float4(o[4], o[5], o[6], o[7]);
        if (o_out) *reinterpret_cast<uint4*>(o_out + oi[u]) = pack8(o);
      }
    }
    __syncwarp();  // every lane of the warp's rows has read lse_acc
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (active[u] && part == 0) lse_acc[li[u]] = l[u];
  }
}

__global__ void __launch_bounds__(kThreads)
    accumulate_kernel(float* __restrict__ acc, const __nv_bfloat16* __restrict__ part, long long n8, int init) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float p[8];
    unpack8(*reinterpret_cast<const uint4*>(part + 8 * i), p);
    float4* a = reinterpret_cast<float4*>(acc + 8 * i);
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
    if (!init) {
      a0 = a[0];
      a1 = a[1];
    }
    a[0] = make_float4(a0.x + p[0], a0.y + p[1], a0.z + p[2], a0.w + p[3]);
    a[1] = make_float4(a1.x + p[4], a1.y + p[5], a1.z + p[6], a1.w + p[7]);
  }
}

__global__ void __launch_bounds__(kThreads)
    cast_kernel(__nv_bfloat16* __restrict__ out, const float* __restrict__ in, long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 x0 = *reinterpret_cast<const float4*>(in + 8 * i);
    const float4 x1 = *reinterpret_cast<const float4*>(in + 8 * i + 4);
    const float f[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    *reinterpret_cast<uint4*>(out + 8 * i) = pack8(f);
  }
}

unsigned grid_for(long long items) {
  long long blocks = (items + kThreads - 1) / kThreads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return static_cast<unsigned>(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                         int H, int N, int d, int init, cudaStream_t s) {
  static_assert(kThreads % 32 == 0, "whole warps");
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  const long long rows = static_cast<long long>(B) * N * H;
  const unsigned grid = grid_for(rows * (d / 8));
  const bool narrow = rows * d < (1LL << 32);
  auto p = static_cast<const __nv_bfloat16*>(o_part);
  auto q = static_cast<__nv_bfloat16*>(o_out);
  if (d == 128) {
    if (narrow) merge_kernel<128, uint32_t><<<grid, kThreads, 0, s>>>(o_acc, lse_acc, p, lse_part, q, B, H, N, init);
    else merge_kernel<128, unsigned long long><<<grid, kThreads, 0, s>>>(o_acc, lse_acc, p, lse_part, q, B, H, N, init);
  } else {
    if (narrow) merge_kernel<64, uint32_t><<<grid, kThreads, 0, s>>>(o_acc, lse_acc, p, lse_part, q, B, H, N, init);
    else merge_kernel<64, unsigned long long><<<grid, kThreads, 0, s>>>(o_acc, lse_acc, p, lse_part, q, B, H, N, init);
  }
  return cudaGetLastError();
}

cudaError_t launch_accumulate(float* acc, const void* part, long long n, int init, cudaStream_t s) {
  accumulate_kernel<<<grid_for(n / 8), kThreads, 0, s>>>(acc, static_cast<const __nv_bfloat16*>(part), n / 8, init);
  return cudaGetLastError();
}

cudaError_t launch_cast(void* out, const float* in, long long n, cudaStream_t s) {
  cast_kernel<<<grid_for(n / 8), kThreads, 0, s>>>(static_cast<__nv_bfloat16*>(out), in, n / 8);
  return cudaGetLastError();
}

}  // namespace fa
