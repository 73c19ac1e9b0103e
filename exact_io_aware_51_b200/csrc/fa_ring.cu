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

// One thread per 8 features of one (b, n, h) row; the d / 8 threads of a row are
// consecutive lanes of one warp.  Every lane runs the same number of loop trips
// (inactive lanes are predicated off), so the warp can meet at __syncwarp()
// between reading the row's old LSE and its first lane writing the new one.
__global__ void __launch_bounds__(kThreads)
    merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc, const __nv_bfloat16* __restrict__ o_part,
                 const float* __restrict__ lse_part, __nv_bfloat16* __restrict__ o_out, int B, int H, int N, int d,
                 int init) {
  const int per_row = d / 8;
  const long long total = static_cast<long long>(B) * N * H * per_row;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long base = static_cast<long long>(blockIdx.x) * blockDim.x; base < total; base += stride) {
    const long long idx = base + threadIdx.x;
    const bool active = idx < total;
    const long long row = active ? idx / per_row : 0;  // (b, n, h) in [B, N, H] order
    const int part = static_cast<int>(idx % per_row);
    const int h = static_cast<int>(row % H);
    const long long bn = row / H;
    const int n = static_cast<int>(bn % N);
    const int b = static_cast<int>(bn / N);
    const size_t li = (static_cast<size_t>(b) * H + h) * N + n;
    const size_t oi = static_cast<size_t>(row) * d + part * 8;
    float o[8], l = -INFINITY;
    if (active) {
      float ob[8];
      unpack8(*reinterpret_cast<const uint4*>(o_part + oi), ob);
      const float lb = lse_part[li];
      if (init) {
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = ob[i];
        l = lb;
      } else {
        const float la = lse_acc[li];
        const float4 a0 = *reinterpret_cast<const float4*>(o_acc + oi);
        const float4 a1 = *reinterpret_cast<const float4*>(o_acc + oi + 4);
        const float oa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float m = fmaxf(la, lb);
        if (m == -INFINITY) {  // neither part saw a key
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = 0.f;
        } else {
          const float wa = expf(la - m), wb = expf(lb - m);
          const float inv = 1.f / (wa + wb);
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = (wa * oa[i] + wb * ob[i]) * inv;
          l = m + logf(wa + wb);
        }
      }
      *reinterpret_cast<float4*>(o_acc + oi) = make_float4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<float4*>(o_acc + oi + 4) = make_float4(o[4], o[5], o[6], o[7]);
      if (o_out) *reinterpret_cast<uint4*>(o_out + oi) = pack8(o);
    }
    __syncwarp();  // every lane of the row has read lse_acc[li]
    if (active && part == 0) lse_acc[li] = l;
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
  // per_row = d / 8 (8 or 16) divides 32, so the threads of one row are lanes of one warp
  static_assert(kThreads % 32 == 0, "whole warps");
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  const long long items = static_cast<long long>(B) * N * H * (d / 8);
  merge_kernel<<<grid_for(items), kThreads, 0, s>>>(o_acc, lse_acc, static_cast<const __nv_bfloat16*>(o_part), lse_part,
                                                    static_cast<__nv_bfloat16*>(o_out), B, H, N, d, init);
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
