// Attention forward in plain fp32 (FFMA on the CUDA cores, no TF32).
//
// Same online-softmax method as the bf16 kernel ("Flash Attention" (Ultralytics
// glossary), "Принцип работы Flash Attention"): key/value tiles stream
// through shared memory while each query row keeps its running maximum, running
// sum and unnormalised output in registers; the output is divided by the sum
// at the end and one log-sum-exp per row is written.  This path exists for
// problems whose inputs are fp32 and whose output must match the exact result
// to ~1e-5: the tensor cores' TF32 mode keeps only 10 mantissa bits and cannot.
//
// Layout: one CTA per 128 query rows of one (b, h); each row is owned by
// D / 64 threads (each holds 64 features of q and of the output accumulator);
// 32-key K/V tiles are staged in shared memory and read as broadcasts.  The
// CTA's 128 rows are exactly one block of a block-sparse mask, so a key tile
// whose 128-key block the mask drops is skipped by the whole CTA ("Flash
// Attention" (Ultralytics glossary), "Flash Attention и смежные понятия": the
// block-sparse form skips empty blocks).
#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kRows = 128;
constexpr int kKT = 32;  // keys per shared-memory tile

template <int D>
__global__ void __launch_bounds__(kRows * (D / 64))
    fwd_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V,
                   const FwdArgs a) {
  constexpr int TPR = D / 64;  // threads per query row
  constexpr int kThreads = kRows * TPR;
  __shared__ float sK[kKT][D];
  __shared__ float sV[kKT][D];

  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int hk = h / (a.H / a.Hkv);  // K/V head of this query head
  const int row0 = blockIdx.x * kRows;
  const int tid = threadIdx.x;
  const int part = tid % TPR;
  const int qrow = row0 + tid / TPR;
  const float sl2 = a.scale_log2;

  float q[64], o[64];
  const float* qp = Q + ((static_cast<size_t>(b) * a.N + min(qrow, a.N - 1)) * a.H + h) * D + part * 64;
#pragma unroll
  for (int i = 0; i < 64; i += 4) {
    const float4 x = *reinterpret_cast<const float4*>(qp + i);
    q[i] = x.x;
    q[i + 1] = x.y;
    q[i + 2] = x.z;
    q[i + 3] = x.w;
    o[i] = o[i + 1] = o[i + 2] = o[i + 3] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  // keys some row of this CTA may see: [first_key, last_key)
  const int first_key = max(0, row0 - a.wl) / kKT * kKT;
  const int last_key = min(a.N - 1, row0 + kRows - 1 + a.wr) + 1;
  // this query block's row of the block mask (null: every block kept)
  const uint8_t* mrow =
      a.block_mask ? a.block_mask + (static_cast<size_t>(a.mask_heads == 1 ? 0 : h) * a.nb + blockIdx.x) * a.nb
                   : nullptr;
  static_assert(kRows == 128 && 128 % kKT == 0, "a CTA's rows form one mask block; a key tile lies in one");
  for (int k0 = first_key; k0 < last_key; k0 += kKT) {
    if (mrow && mrow[k0 / 128] == 0) continue;  // the same for every thread of the CTA
    __syncthreads();
    for (int e = tid * 4; e < kKT * D; e += kThreads * 4) {
      const int kr = e / D, kc = e % D;
      const int key = k0 + kr;
      float4 kx = make_float4(0.f, 0.f, 0.f, 0.f), vx = kx;
      if (key < a.N) {
        const size_t off = ((static_cast<size_t>(b) * a.N + key) * a.Hkv + hk) * D + kc;
        kx = *reinterpret_cast<const float4*>(K + off);
        vx = *reinterpret_cast<const float4*>(V + off);
      }
      *reinterpret_cast<float4*>(&sK[kr][kc]) = kx;
      *reinterpret_cast<float4*>(&sV[kr][kc]) = vx;
    }
    __syncthreads();

    float s[kKT];
    float mx = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kKT; ++jj) {
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < 64; ++i) dot = fmaf(q[i], sK[jj][part * 64 + i], dot);
      if (TPR == 2) dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      const int key = k0 + jj;
      const bool visible = key < a.N && key <= qrow + a.wr && key >= qrow - a.wl;
      s[jj] = visible ? dot : -INFINITY;
      mx = fmaxf(mx, s[jj]);
    }
    const float m_new = fmaxf(m, mx * sl2);
    const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m - m_new);
    const float base = (m_new == -INFINITY) ? 0.f : m_new;
    l *= alpha;
#pragma unroll
    for (int i = 0; i < 64; ++i) o[i] *= alpha;
#pragma unroll
    for (int jj = 0; jj < kKT; ++jj) {
      const float p = exp2f(fmaf(s[jj], sl2, -base));
      l += p;
#pragma unroll
      for (int i = 0; i < 64; ++i) o[i] = fmaf(p, sV[jj][part * 64 + i], o[i]);
    }
    m = m_new;
  }

  if (qrow < a.N) {
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    float* op = reinterpret_cast<float*>(a.O) + ((static_cast<size_t>(b) * a.N + qrow) * a.H + h) * D + part * 64;
#pragma unroll
    for (int i = 0; i < 64; i += 4)
      *reinterpret_cast<float4*>(op + i) = make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
    if (part == 0)
      a.LSE[(static_cast<size_t>(b) * a.H + h) * a.N + qrow] =
          (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_fwd_f32(const float* Q, const float* K, const float* V, const FwdArgs& a, cudaStream_t s) {
  const dim3 grid((a.N + kRows - 1) / kRows, a.H, a.B);
  if (a.d == 128)
    fwd_f32_kernel<128><<<grid, kRows * 2, 0, s>>>(Q, K, V, a);
  else
    fwd_f32_kernel<64><<<grid, kRows, 0, s>>>(Q, K, V, a);
  return cudaGetLastError();
}

}  // namespace fa
