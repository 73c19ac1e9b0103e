// Attention backward by recomputation, bf16 inputs, fp32 accumulation, sm_100a.
//
// Method: "Flash Attention" (karlkratz.de), "Recomputation beim
// Rückwärtsdurchlauf", and "Flash Attention" (Ultralytics glossary), "Принцип
// работы Flash Attention": the N x N attention matrix is not stored; the
// backward pass recomputes the score blocks from Q, K and V.  With the saved
// per-row log-sum-exp L_i the probabilities are P_ij = exp(S_ij - L_i) without
// any renormalisation.  The gradients are calculus on the forward definition:
//   dV = P^T dO,  dP = dO V^T,  D_i = sum_k dO_ik O_ik,  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three kernels on one stream:
//   1. bwd_pre:  D_i = rowsum(dO * O) and L_i * log2(e) into [B, H, Npad]
//      fp32 rows, and zero the fp32 dQ accumulator (HBM-bound);
//   2. bwd_main: one CTA per 128-key tile j of one (b, h).  K_j and V_j stay in
//      shared memory; 64-row query tiles i stream past through a TMA ring.
//      Per tile, five tcgen05 MMAs with TMEM accumulators:
//        S^T  = K_j Q_i^T          (keys on TMEM lanes)
//        dP^T = V_j dO_i^T
//        dV_j += P^T dO_i          (P^T written by the softmax warps to smem)
//        dK_j += dS^T Q_i          (dS^T likewise)
//        dQ_i^T = K_j^T dS^T       (features on TMEM lanes, double buffered)
//      One warpgroup turns S^T / dP^T into P^T / dS^T (one key row per thread,
//      exp2 with the scale folded in), one warpgroup drains dQ_i^T from TMEM
//      into the fp32 accumulator with coalesced reductions, one warp loads and
//      one warp issues MMAs.  Causal: query tiles above the diagonal are skipped.
//   3. bwd_dq:   dQ = bf16(scale * dQacc).
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// 1. preprocess
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdArgs a) {
  constexpr int TPR = D / 8;  // threads per row, 8 bf16 (16 bytes) each
  constexpr int RPB = 256 / TPR;
  const long long row = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const long long total = static_cast<long long>(a.B) * a.H * a.Npad;
  if (row >= total) return;
  const int n = static_cast<int>(row % a.Npad);
  const long long bh = row / a.Npad;
  const int h = static_cast<int>(bh % a.H);
  const int b = static_cast<int>(bh / a.H);
  float acc = 0.f;
  if (n < a.N) {
    const size_t idx = ((static_cast<size_t>(b) * a.N + n) * a.H + h) * D + part * 8;
    const uint4 ov = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.O) + idx);
    const uint4 dv = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.dO) + idx);
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
    const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[i]));
      const float2 df = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dw[i]));
      acc = fmaf(of.x, df.x, acc);
      acc = fmaf(of.y, df.y, acc);
    }
    float4* z = reinterpret_cast<float4*>(a.dQacc + idx);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (part == 0) {
    a.Dvec[row] = acc;
    a.LSE2[row] = (n < a.N) ? a.LSE[bh * a.N + n] * kLog2e : 0.f;
  }
}

// ---------------------------------------------------------------------------
// 3. dQ convert
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_dq_kernel(const BwdArgs a, long long total) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x * 8;
  for (long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < total; i += stride) {
    const float4 x = *reinterpret_cast<const float4*>(a.dQacc + i);
    const float4 y = *reinterpret_cast<const float4*>(a.dQacc + i + 4);
    const float s = a.scale;
    uint4 out;
    out.x = pack_bf16x2(x.x * s, x.y * s);
    out.y = pack_bf16x2(x.z * s, x.w * s);
    out.z = pack_bf16x2(y.x * s, y.y * s);
    out.w = pack_bf16x2(y.z * s, y.w * s);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dQ) + i) = out;
  }
}

// ---------------------------------------------------------------------------
// 2. main kernel (D = 128)
// ---------------------------------------------------------------------------
constexpr int kBN = 128;       // keys per CTA (TMEM lanes of S^T, dP^T, dK, dV)
constexpr int kBMq = 64;       // query rows per streamed tile
constexpr int kThreads = 384;  // WG0 P/dS, WG1 dQ drain, WG2 loader + MMA
constexpr int kStages = 2;
// 384 x 168 at launch = 128 x 216 + 128 x 216 + 128 x 72.  A warpgroup above the
// launch count raises its share (setmaxnreg.inc), one below lowers it
// (setmaxnreg.dec); the other direction is an illegal instruction.
constexpr uint32_t kRegCompute = 216;
constexpr uint32_t kRegDq = 216;
constexpr uint32_t kRegOther = 72;
static_assert(kRegCompute >= 168 && kRegDq >= 168 && kRegOther <= 168, "setmaxnreg direction");
static_assert(kRegCompute + kRegDq + kRegOther == 3 * 168, "register split must match the launch");

struct BwdCfg {
  static constexpr int D = 128;
  static constexpr int kKVBytes = kBN * D * 2;    // 32 KB: two [128][64] sub-tiles
  static constexpr int kKVSub = kBN * 128;        // 16 KB
  static constexpr int kQBytes = kBMq * D * 2;    // 16 KB: two [64][64] sub-tiles
  static constexpr int kQSub = kBMq * 128;        // 8 KB
  static constexpr int kPBytes = kBN * kBMq * 2;  // 16 KB: one [128][64] tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffQ = kOffV + kKVBytes;
  static constexpr int kOffDO = kOffQ + kStages * kQBytes;
  static constexpr int kOffPt = kOffDO + kStages * kQBytes;
  static constexpr int kOffDSt = kOffPt + kPBytes;
  static constexpr int kOffL = kOffDSt + kPBytes;       // [stage][64] fp32 LSE2
  static constexpr int kOffDv = kOffL + kStages * 256;  // [stage][64] fp32 D
  static constexpr int kOffBar = kOffDv + kStages * 256;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
  // TMEM columns
  static constexpr uint32_t kColDV = 0, kColDK = 128, kColS = 256, kColDP = 320, kColDQ = 384;
  static constexpr uint32_t kIdescS = idesc_bf16(kBN, kBMq, 0, 0);   // S^T, dP^T
  static constexpr uint32_t kIdescKV = idesc_bf16(kBN, D, 0, 1);     // dV, dK
  static constexpr uint32_t kIdescQ = idesc_bf16(D, kBMq, 1, 1);     // dQ^T
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t q_full[kStages], q_empty[kStages];
  uint64_t s_full, dp_full, pt_ready, ds_ready;
  uint64_t dq_full[2], dq_free[2];
  uint64_t acc_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned long long limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
}

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// write one 64-value bf16 row (row r of a [128][64] SW128 tile)
__device__ __forceinline__ void store_row_sw128(uint32_t tile, int r, const float* v) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    st_shared_v4(tile + sw128_offset(r, u), pack_bf16x2(v[8 * u + 0], v[8 * u + 1]),
                 pack_bf16x2(v[8 * u + 2], v[8 * u + 3]), pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                 pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdArgs a, const DevCtl ctl) {
  using C = BwdCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::kOffBar);
  const int warp = warp_id();
  const int lane = lane_id();

  const int jt = blockIdx.x;  // key tile
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int key0 = jt * kBN;
  const int nq_total = (a.N + kBMq - 1) / kBMq;
  const int i0 = a.causal ? (key0 / kBMq) : 0;  // first query tile that sees these keys
  const int nq = max(0, nq_total - i0);
  const size_t bh = static_cast<size_t>(b) * a.H + h;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->pt_ready, 128);
    mbar_init(&bars->ds_ready, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->dq_full[s], 1);
      mbar_init(&bars->dq_free[s], 128);
    }
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = (*reinterpret_cast<volatile unsigned int*>(ctl.abort_epoch) == ctl.epoch) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(&bars->tmem_base, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl w{&bars->abort, ctl.status, ctl.abort_epoch, ctl.epoch, ctl.limit_ns};

  if (warp < 4) {
    // ===================== P^T / dS^T warpgroup =====================
    reg_alloc<kRegCompute>();
    if (bars->abort == 0) {
      const int r = warp * 32 + lane;  // key row within the tile = TMEM lane
      const int key = key0 + r;
      const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
      const uint32_t sPt = smem_u32(smem + C::kOffPt);
      const uint32_t sDSt = smem_u32(smem + C::kOffDSt);
      const float sl2 = a.scale_log2;
      bool ok = true;
      for (int it = 0; it < nq; ++it) {
        const int st = it % kStages;
        const int q0 = (i0 + it) * kBMq;
        ok = warp_all(wait_bar(&bars->q_full[st], (it / kStages) & 1, w, 20));
        if (!ok) break;
        ok = warp_all(wait_bar(&bars->s_full, it & 1, w, 21));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[kBMq];
        tmem_ld32(tmem + lane_bits + C::kColS, sr);
        tmem_ld32(tmem + lane_bits + C::kColS + 32, sr + 32);
        tmem_wait_ld();
        reg_fence32(sr);
        reg_fence32(sr + 32);
        const float* sL = reinterpret_cast<const float*>(smem + C::kOffL + st * 256);
        const float* sD = reinterpret_cast<const float*>(smem + C::kOffDv + st * 256);
        float p[kBMq];
        const bool need_mask = (q0 + kBMq > a.N) || (key0 + kBN > a.N) || (a.causal && q0 < key0 + kBN);
#pragma unroll
        for (int c = 0; c < kBMq; ++c) p[c] = ex2(fmaf(__uint_as_float(sr[c]), sl2, -sL[c]));
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < kBMq; ++c) {
            const int q = q0 + c;
            const bool vis = (q < a.N) && (key < a.N) && (!a.causal || q >= key);
            if (!vis) p[c] = 0.f;
          }
        }
        store_row_sw128(sPt, r, p);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->pt_ready);

        ok = warp_all(wait_bar(&bars->dp_full, it & 1, w, 22));
        if (!ok) break;
        tc_fence_after();
        uint32_t dr[kBMq];
        tmem_ld32(tmem + lane_bits + C::kColDP, dr);
        tmem_ld32(tmem + lane_bits + C::kColDP + 32, dr + 32);
        tmem_wait_ld();
        reg_fence32(dr);
        reg_fence32(dr + 32);
#pragma unroll
        for (int c = 0; c < kBMq; ++c) p[c] = p[c] * (__uint_as_float(dr[c]) - sD[c]);
        store_row_sw128(sDSt, r, p);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->ds_ready);
      }
      // ---- epilogue: dV and dK rows of this key ----
      if (ok) {
        if (nq > 0) ok = warp_all(wait_bar(&bars->acc_done, 0, w, 23));
        if (ok) {
          tc_fence_after();
          const size_t base = ((static_cast<size_t>(b) * a.N + key) * a.H + h) * D;
          __nv_bfloat16* dv = reinterpret_cast<__nv_bfloat16*>(a.dV) + base;
          __nv_bfloat16* dk = reinterpret_cast<__nv_bfloat16*>(a.dK) + base;
#pragma unroll
          for (int which = 0; which < 2; ++which) {
            const uint32_t col = which == 0 ? C::kColDV : C::kColDK;
            const float mul = which == 0 ? 1.f : a.scale;
            __nv_bfloat16* dst = which == 0 ? dv : dk;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t v[32];
              if (nq > 0) {
                tmem_ld32(tmem + lane_bits + col + c * 32, v);
                tmem_wait_ld();
                reg_fence32(v);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0u;
              }
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
              if (key < a.N) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  st_global_v4(dst + c * 32 + i * 8, pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
              }
            }
          }
        }
      }
    }
  } else if (warp < 8) {
    // ===================== dQ drain warpgroup =====================
    reg_alloc<kRegDq>();
    if (bars->abort == 0) {
      const int quarter = warp & 3;
      const int dd = quarter * 32 + lane;  // feature index = TMEM lane of dQ^T
      const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
      for (int it = 0; it < nq; ++it) {
        const int buf = it & 1;
        if (!warp_all(wait_bar(&bars->dq_full[buf], (it >> 1) & 1, w, 30))) break;
        tc_fence_after();
        uint32_t v[kBMq];
        tmem_ld32(tmem + lane_bits + C::kColDQ + buf * 64, v);
        tmem_ld32(tmem + lane_bits + C::kColDQ + buf * 64 + 32, v + 32);
        tmem_wait_ld();
        reg_fence32(v);
        reg_fence32(v + 32);
        tc_fence_before();
        mbar_arrive(&bars->dq_free[buf]);
        const int q0 = (i0 + it) * kBMq;
        float* dst = a.dQacc + ((static_cast<size_t>(b) * a.N + q0) * a.H + h) * D + dd;
        const size_t row_stride = static_cast<size_t>(a.H) * D;
        const int rows = min(kBMq, a.N - q0);
#pragma unroll
        for (int c = 0; c < kBMq; ++c)
          if (c < rows) red_add_f32(dst + c * row_stride, __uint_as_float(v[c]));
      }
    }
  } else {
    reg_dealloc<kRegOther>();
    if (bars->abort == 0 && warp == 8) {
      // ===================== TMA producer =====================
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmDO);
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kKVBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(smem + C::kOffK + c * C::kKVSub, &tmK, &bars->kv_full, c * 64, key0, h, b);
          tma_load_4d(smem + C::kOffV + c * C::kKVSub, &tmV, &bars->kv_full, c * 64, key0, h, b);
        }
        for (int it = 0; it < nq; ++it) {
          const int st = it % kStages;
          const int n = it / kStages;
          if (it >= kStages && !wait_bar(&bars->q_empty[st], (n - 1) & 1, w, 10)) break;
          const int q0 = (i0 + it) * kBMq;
          mbar_arrive_expect_tx(&bars->q_full[st], 2 * C::kQBytes + 512);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(smem + C::kOffQ + st * C::kQBytes + c * C::kQSub, &tmQ, &bars->q_full[st], c * 64, q0, h, b);
            tma_load_4d(smem + C::kOffDO + st * C::kQBytes + c * C::kQSub, &tmDO, &bars->q_full[st], c * 64, q0, h,
                        b);
          }
          bulk_load(smem + C::kOffL + st * 256, a.LSE2 + bh * a.Npad + q0, 256, &bars->q_full[st]);
          bulk_load(smem + C::kOffDv + st * 256, a.Dvec + bh * a.Npad + q0, 256, &bars->q_full[st]);
        }
      }
    } else if (bars->abort == 0 && warp == 9) {
      // ===================== MMA issuer =====================
      if (lane == 0 && nq > 0) {
        const uint32_t sK = smem_u32(smem + C::kOffK);
        const uint32_t sV = smem_u32(smem + C::kOffV);
        const uint32_t sQ = smem_u32(smem + C::kOffQ);
        const uint32_t sDO = smem_u32(smem + C::kOffDO);
        const uint32_t sPt = smem_u32(smem + C::kOffPt);
        const uint32_t sDSt = smem_u32(smem + C::kOffDSt);
        // S^T = K Q^T (or dP^T = V dO^T): A [128 keys][128 d] K-major, B [64 q][128 d] K-major
        auto issue_s = [&](uint32_t a_base, uint32_t b_base, uint32_t col) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ao = (kk >> 2) * C::kKVSub + (kk & 3) * 32;
            const uint32_t bo = (kk >> 2) * C::kQSub + (kk & 3) * 32;
            umma_ss(tmem + col, sw128_desc(a_base + ao, 16, 1024), sw128_desc(b_base + bo, 16, 1024), C::kIdescS,
                    kk > 0 ? 1u : 0u);
          }
        };
        // dV += P^T dO (or dK += dS^T Q): A [128 keys][64 q] K-major, B [64 q][128 d] MN-major
        auto issue_kv = [&](uint32_t a_base, uint32_t b_base, uint32_t col, bool acc) {
#pragma unroll
          for (int kk = 0; kk < kBMq / 16; ++kk) {
            umma_ss(tmem + col, sw128_desc(a_base + kk * 32, 16, 1024),
                    sw128_desc(b_base + kk * 2048, C::kQSub, 1024), C::kIdescKV, (acc || kk > 0) ? 1u : 0u);
          }
        };
        bool ok = wait_bar(&bars->kv_full, 0, w, 11) && wait_bar(&bars->q_full[0], 0, w, 12);
        if (ok) {
          tc_fence_after();
          issue_s(sK, sQ, C::kColS);
          umma_commit(&bars->s_full);
          issue_s(sV, sDO, C::kColDP);
          umma_commit(&bars->dp_full);
        }
        for (int it = 0; ok && it < nq; ++it) {
          const int st = it % kStages;
          const int st1 = (it + 1) % kStages;
          const bool more = it + 1 < nq;
          if (!(ok = wait_bar(&bars->pt_ready, it & 1, w, 13))) break;
          tc_fence_after();
          issue_kv(sPt, sDO + st * C::kQBytes, C::kColDV, it > 0);
          if (more) {
            if (!(ok = wait_bar(&bars->q_full[st1], ((it + 1) / kStages) & 1, w, 14))) break;
            tc_fence_after();
            issue_s(sK, sQ + st1 * C::kQBytes, C::kColS);
            umma_commit(&bars->s_full);
          }
          if (!(ok = wait_bar(&bars->ds_ready, it & 1, w, 15))) break;
          tc_fence_after();
          issue_kv(sDSt, sQ + st * C::kQBytes, C::kColDK, it > 0);
          umma_commit(&bars->q_empty[st]);
          const int buf = it & 1;
          if (it >= 2 && !(ok = wait_bar(&bars->dq_free[buf], ((it - 2) >> 1) & 1, w, 16))) break;
          tc_fence_after();
          // dQ^T = K^T dS^T: A = K as [128 d (M, contiguous)][128 keys], B = dS^T as [64 q (N, contiguous)][128 keys]
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            umma_ss(tmem + C::kColDQ + buf * 64, sw128_desc(sK + kk * 2048, C::kKVSub, 1024),
                    sw128_desc(sDSt + kk * 2048, C::kKVSub, 1024), C::kIdescQ, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars->dq_full[buf]);
          if (more) {
            issue_s(sV, sDO + st1 * C::kQBytes, C::kColDP);
            umma_commit(&bars->dp_full);
          }
        }
        if (ok) umma_commit(&bars->acc_done);
        umma_commit(&bars->drain);
        drain_wait(&bars->drain, 0, ctl.limit_ns);
      }
    }
  }

  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_bwd_pre(const BwdArgs& a, cudaStream_t s) {
  const long long rows = static_cast<long long>(a.B) * a.H * a.Npad;
  if (a.d == 128) {
    const long long blocks = (rows + 16 - 1) / 16;
    bwd_pre_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
  } else {
    const long long blocks = (rows + 32 - 1) / 32;
    bwd_pre_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_main(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdArgs& a, const DevCtl& c, cudaStream_t s) {
  constexpr int smem = BwdCfg::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(bwd_main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.N + kBN - 1) / kBN, a.H, a.B);
  bwd_main_kernel<<<grid, kThreads, smem, s>>>(tq, tk, tv, tdo, a, c);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const BwdArgs& a, cudaStream_t s) {
  const long long total = static_cast<long long>(a.B) * a.N * a.H * a.d;
  long long blocks = (total / 8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  bwd_dq_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a, total);
  return cudaGetLastError();
}

}  // namespace fa
