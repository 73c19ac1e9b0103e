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
// Three kernels on one stream (four more with a split walk, see below):
//   1. bwd_pre:  D_i = rowsum(dO * O) and L_i * log2(e) into [B, H, Npad]
//      fp32 rows, and zero the fp32 dQ accumulator (HBM-bound);
//   2. bwd_main: one CTA per 128-key tile j of one (b, K/V head).  K_j and V_j
//      stay in shared memory; 128-row query tiles i (of every query head of
//      the K/V head's group) stream past through a 2-stage TMA ring.  Per tile,
//      five tcgen05 MMAs with TMEM accumulators:
//        S^T  = K_j Q_i^T          (keys on TMEM lanes; both operands in smem)
//        dP^T = V_j dO_i^T
//        dV_j += P^T dO_i          (P^T written over S^T in TMEM as bf16 pairs)
//        dK_j += dS^T Q_i          (dS^T written over dP^T in TMEM likewise)
//        dQ_i^T = K_j^T dS^T       (features on TMEM lanes; dS^T also stored to
//                                   smem over dO_i as the B operand)
//      Two warpgroups turn S^T / dP^T into P^T / dS^T (one key row per thread,
//      64 query columns each, exp2 with the scale folded in); one warpgroup
//      reads dQ_i^T out of TMEM, stages 64 query rows at a time in shared
//      memory and adds them into the fp32 accumulator with TMA reduce-adds;
//      one warp loads and one warp issues MMAs.  Causal, window and
//      block-sparse masks: query tiles no key of the tile can see are skipped.
//      Small grids split each key tile's walk over several CTAs, whose fp32
//      dK, dV partial sums are added into workspace accumulators (zeroed before
//      and converted to bf16 after the main kernel).
//   3. bwd_dq:   dQ = bf16(scale * dQacc).
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
// When > 0, one float4 group of query columns in kPolyEvery takes its
// exponentials on the FMA pipe (exp2_poly2) instead of the MUFU unit.
constexpr int kPolyEvery = 0;

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
constexpr int kBN = 128;        // keys per CTA (TMEM lanes of S^T, dP^T, dK, dV)
constexpr int kBMq = 128;       // query rows per streamed tile
constexpr int kThreads = 512;   // WG0, WG1: P / dS for query columns 0-63 / 64-127; WG2: dQ drain; WG3: loader + MMA
constexpr int kStages = 2;      // Q/dO ring
// 512 x 128 at launch = 2 x 128 x 144 + 128 x 144 + 128 x 80.  A warpgroup above the
// launch count raises its share (setmaxnreg.inc), one below lowers it
// (setmaxnreg.dec); the other direction is an illegal instruction.
constexpr uint32_t kRegLaunch = 128;
constexpr uint32_t kRegCompute = 144;
constexpr uint32_t kRegDrain = 144;
constexpr uint32_t kRegCtrl = 80;
static_assert(kRegCompute >= kRegLaunch && kRegDrain >= kRegLaunch && kRegCtrl <= kRegLaunch,
              "setmaxnreg direction");
static_assert(2 * kRegCompute + kRegDrain + kRegCtrl == 4 * kRegLaunch, "register split must match the launch");

struct BwdCfg {
  static constexpr int D = 128;
  static constexpr int kSub = kBN * 128;          // one [128 rows][64] bf16 SW128 sub-tile: 16 KB
  static constexpr int kTile = 2 * kSub;          // one 128 x 128 bf16 tile: 32 KB
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;                 // [stage] Q_i
  static constexpr int kOffDO = kOffQ + kStages * kTile;      // [stage] dO_i, then dS^T_i
  static constexpr int kOffL = kOffDO + kStages * kTile;      // [stage][128] fp32 LSE * log2 e
  static constexpr int kOffDv = kOffL + kStages * 512;        // [stage][128] fp32 rowsum(dO * O)
  static constexpr int kOffDQS = kOffDv + kStages * 512;       // [64 q][128 d] fp32 dQ staging
  static constexpr int kOffBar = kOffDQS + 64 * 128 * 4;
  // no alignment slack: the dynamic shared memory is declared 1024-aligned and checked
  static constexpr int kSmemBytes = kOffBar + 256;
  // TMEM columns: dV | dK | R1 | R2.
  //   R1: S^T_i (fp32), then P^T_i as bf16 pairs in columns [0, 32) (query
  //       columns 0-63) and [64, 96) (query columns 64-127).
  //   R2: dP^T_i (fp32), then dS^T_i as bf16 pairs at the same places, then
  //       dQ_i^T (fp32, features on lanes) once dK_i has read dS^T_i.
  static constexpr uint32_t kColDV = 0, kColDK = 128, kColR1 = 256, kColR2 = 384;
  static constexpr uint32_t kIdescS = idesc_bf16(kBN, kBMq, 0, 0);   // S^T, dP^T: K-major A and B
  static constexpr uint32_t kIdescKV = idesc_bf16(kBN, D, 0, 1);     // dV, dK: A from TMEM, B MN-major
  static constexpr uint32_t kIdescQ = idesc_bf16(D, kBMq, 1, 1);     // dQ^T: both MN-major
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t q_full[kStages], q_empty[kStages];
  uint64_t s_full, dp_full, pt_ready, ds_ready, dv_done, dq_full, dq_free;
  uint64_t acc_done;
  uint64_t drain;
  uint64_t stage_sync;  // the dQ drain warpgroup's internal barrier
  uint32_t tmem_base;
  int abort;
  // block-sparse: first query row of tile i, in slot i % 4 (written by the
  // loader before it arms q_full for the tile; read by the compute warps after
  // their q_full wait)
  int info_q0[4];
  int sparse_nq;  // block-sparse: kept (query head, query tile) pairs of this key tile
  uint64_t epi_sync[2];  // split walks: a compute warpgroup's partial dV / dK is staged
};
static_assert(sizeof(BwdBars) <= 256, "barrier block");
static_assert(BwdCfg::kOffDQS % 1024 == 0 && BwdCfg::kSmemBytes <= 232448, "shared memory layout");

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }


// TMEM column of the bf16 pairs for reduction step kk (16 query columns) of a
// P^T / dS^T tile written by the two compute warpgroups.
__device__ __forceinline__ uint32_t ts_col(int kk) { return (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8; }

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                    const __grid_constant__ CUtensorMap tmDV, const BwdArgs a, const DevCtl ctl) {
  using C = BwdCfg;
  constexpr int D = C::D;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {  // the swizzled layouts need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicCAS(ctl.status, 0, kDevTimeout | 0xA1);
    return;
  }
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::kOffBar);
  const int warp = warp_id();
  const int lane = lane_id();

  // Key tile, K/V head, part of the key tile's walk, batch.  Causal: the
  // launch order (block x fastest, then y, then z) is longest first over every
  // (b, K/V head, part): the CTA's rank in it picks the key tile from the start
  // of the sequence (whose walks are longest), the rest vary fastest.
  int jt = static_cast<int>(blockIdx.x), y = static_cast<int>(blockIdx.y), b = static_cast<int>(blockIdx.z);
  if (a.causal) {
    const int yz = static_cast<int>(gridDim.y * gridDim.z);
    const int rank = static_cast<int>(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    jt = rank / yz;
    y = (rank % yz) % static_cast<int>(gridDim.y);
    b = (rank % yz) / static_cast<int>(gridDim.y);
  }
  const int hk = y / a.splits;  // K/V head
  const int sp = y % a.splits;  // part of this key tile's walk
  const int key0 = jt * kBN;
  const int nq_total = (a.N + kBMq - 1) / kBMq;
  // query tiles holding every query that sees one of these keys:
  // q in [key - wr, key + wl] for each key of the tile
  const int kmax = min(key0 + kBN - 1, a.N - 1);
  const int i0 = max(0, key0 - a.wr) / kBMq;
  const int i_end = min(a.N - 1, kmax + a.wl) / kBMq + 1;
  // Grouped-query attention: the G query heads of this K/V head all add into
  // this CTA's dK and dV, so the CTA walks (query head, query tile) pairs.
  const int G = a.H / a.Hkv;
  const int nq_head = max(0, min(nq_total, i_end) - i0);  // query tiles per query head
  int nq = G * nq_head;                       // iterations of this CTA
  // Iteration i works on query tile i0 + i % nq_head of query head hk G + i / nq_head;
  // the loops advance (qt, hq) by counters (a division per tile measurably slowed them).
  // Block-sparse: only the (query head, query tile) pairs the mask keeps for this key
  // tile, in the same order; the loader walks them and posts each tile's (q0, head).
  const int qt_end = i0 + nq_head;
  auto kept = [&](int hq, int qt) -> bool {
    return a.block_mask[(static_cast<size_t>(a.mask_heads == 1 ? 0 : hq) * a.nb + qt) * a.nb + jt] != 0;
  };
  if constexpr (kSparse) {
    // (a static __shared__ variable here would push the 1024-aligned dynamic
    // region past the shared-memory limit, so the count lives in the barrier block)
    int& s_nq = bars->sparse_nq;
    if (threadIdx.x == 0) s_nq = 0;
    __syncthreads();
    int cnt = 0;
    for (int c = static_cast<int>(threadIdx.x); c < nq; c += kThreads)
      cnt += kept(hk * G + c / nq_head, i0 + c % nq_head) ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0 && cnt) atomicAdd(&s_nq, cnt);
    __syncthreads();
    nq = s_nq;
  }
  // split walks: this CTA takes iterations [beg, beg + nq) of the key tile's walk
  const int beg = static_cast<int>((static_cast<long long>(nq) * sp) / a.splits);
  nq = static_cast<int>((static_cast<long long>(nq) * (sp + 1)) / a.splits) - beg;
  const int qt_beg = (nq_head > 0) ? i0 + beg % nq_head : i0;     // dense walk: first query tile
  const int hq_beg = hk * G + ((nq_head > 0) ? beg / nq_head : 0);  // and its query head

  if (threadIdx.x == 0) {
    mbar_init(&bars->epi_sync[0], 128);
    mbar_init(&bars->epi_sync[1], 128);
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->pt_ready, 256);
    mbar_init(&bars->ds_ready, 256);
    mbar_init(&bars->dv_done, 1);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, 128);
    mbar_init(&bars->acc_done, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->stage_sync, 128);
    bars->abort = (*reinterpret_cast<volatile unsigned int*>(ctl.abort_epoch) == ctl.epoch) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 13) tmem_alloc(&bars->tmem_base, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl w{&bars->abort, ctl.status, ctl.abort_epoch, ctl.epoch, ctl.limit_ns};

  if (warp < 8) {
    // ===================== P^T / dS^T warpgroups =====================
    // WG g owns query columns [64 g, 64 g + 64) of every tile.
    reg_alloc<kRegCompute>();
    if (bars->abort == 0) {
      const int g = warp >> 2;
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;  // key row within the tile = TMEM lane
      const int key = key0 + r;
      const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t tR1 = tmem + lane_bits + C::kColR1 + 64 * g;  // this WG's 64 fp32 columns
      const uint32_t tR2 = tmem + lane_bits + C::kColR2 + 64 * g;
      const float sl2 = a.scale_log2;
      bool ok = true;
      int qt = qt_beg;  // query tile of iteration i (the head does not matter here)
      for (int i = 0; i < nq; ++i) {
        const int st = i % kStages;
        const uint32_t par = i & 1;
        int q0 = qt * kBMq + 64 * g;  // first query column of this WG
        qt = (qt + 1 == qt_end) ? i0 : qt + 1;
        ok = warp_all(wait_bar(&bars->q_full[st], (i / kStages) & 1, w, 20));
        if (!ok) break;
        if constexpr (kSparse) q0 = *reinterpret_cast<volatile int*>(&bars->info_q0[i & 3]) + 64 * g;
        ok = warp_all(wait_bar(&bars->s_full, par, w, 21));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(tR1, sr);
        tmem_ld32(tR1 + 32, sr + 32);
        tmem_wait_ld();
        reg_fence32(sr);
        reg_fence32(sr + 32);
        const float4* sL = reinterpret_cast<const float4*>(smem + C::kOffL + st * 512 + 256 * g);
        const float4* sD = reinterpret_cast<const float4*>(smem + C::kOffDv + st * 512 + 256 * g);
        // every (query, key) pair of this WG's block visible: no mask
        const bool need_mask =
            (q0 + 64 > a.N) || (key0 + kBN > a.N) || (key0 + kBN - 1 > q0 + a.wr) || (key0 < q0 + 63 - a.wl);
        float p[64];
        // P = 2^(S^T * scale * log2 e - LSE * log2 e), 32 query columns at a time;
        // each half's P^T (bf16 pairs, 16 columns) goes to TMEM while the next half
        // is computed
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
          for (int c4 = 8 * hh; c4 < 8 * hh + 8; ++c4) {
            const float4 l4 = sL[c4];
            const float2 x0 = ffma2(make_float2(__uint_as_float(sr[4 * c4]), __uint_as_float(sr[4 * c4 + 1])),
                                    make_float2(sl2, sl2), make_float2(-l4.x, -l4.y));
            const float2 x1 = ffma2(make_float2(__uint_as_float(sr[4 * c4 + 2]), __uint_as_float(sr[4 * c4 + 3])),
                                    make_float2(sl2, sl2), make_float2(-l4.z, -l4.w));
            float2 y0, y1;
            if (kPolyEvery > 0 && (c4 % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1) {
              y0 = exp2_poly2(x0);
              y1 = exp2_poly2(x1);
            } else {
              y0 = make_float2(ex2(x0.x), ex2(x0.y));
              y1 = make_float2(ex2(x1.x), ex2(x1.y));
            }
            p[4 * c4 + 0] = y0.x;
            p[4 * c4 + 1] = y0.y;
            p[4 * c4 + 2] = y1.x;
            p[4 * c4 + 3] = y1.y;
          }
          if (need_mask) {
#pragma unroll
            for (int c = 32 * hh; c < 32 * hh + 32; ++c) {
              const int q = q0 + c;
              const bool vis = (q < a.N) && (key < a.N) && (key <= q + a.wr) && (key >= q - a.wl);
              if (!vis) p[c] = 0.f;
            }
          }
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(p[32 * hh + 2 * c], p[32 * hh + 2 * c + 1]);
          tmem_st16(tR1 + 16 * hh, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->pt_ready);

        ok = warp_all(wait_bar(&bars->dp_full, par, w, 22));
        if (!ok) break;
        // dS^T also goes to shared memory over dO_i, which dV_i must have read
        ok = warp_all(wait_bar(&bars->dv_done, par, w, 24));
        if (!ok) break;
        tc_fence_after();
        const uint32_t sDSt = smem_u32(smem + C::kOffDO + st * C::kTile + g * C::kSub);
        // dS = P (dP - D), 32 query columns at a time: to TMEM (A operand of dK)
        // and to shared memory (B operand of dQ^T)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t dr[32];
          tmem_ld32(tR2 + 32 * hh, dr);
          tmem_wait_ld();
          reg_fence32(dr);
          uint32_t pk[16];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 d4 = sD[8 * hh + c4];
            const int c = 32 * hh + 4 * c4;
            pk[2 * c4] = pack_bf16x2(p[c + 0] * (__uint_as_float(dr[4 * c4 + 0]) - d4.x),
                                     p[c + 1] * (__uint_as_float(dr[4 * c4 + 1]) - d4.y));
            pk[2 * c4 + 1] = pack_bf16x2(p[c + 2] * (__uint_as_float(dr[4 * c4 + 2]) - d4.z),
                                         p[c + 3] * (__uint_as_float(dr[4 * c4 + 3]) - d4.w));
          }
          tmem_st16(tR2 + 16 * hh, pk);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_shared_v4(sDSt + sw128_offset(r, 4 * hh + u), pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->ds_ready);
      }
      // ---- epilogue: WG0 writes the dV rows, WG1 the dK rows of its keys ----
      if (ok && nq > 0) ok = warp_all(wait_bar(&bars->acc_done, 0, w, 23));
      if (ok && a.splits > 1) {
        // a part of a split walk: add the fp32 partial sums into the accumulator.
        // The Q (WG0) or dO (WG1) stages, idle now, hold the [128 keys][128] fp32
        // rows; two TMA reduce-adds of 64 keys each carry them to global memory.
        tc_fence_after();
        float* stg = reinterpret_cast<float*>(smem + (g == 0 ? C::kOffQ : C::kOffDO));
        const uint32_t col = g == 0 ? C::kColDV : C::kColDK;
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
#pragma unroll
          for (int i = 0; i < 8; ++i)
            st_shared_v4(smem_u32(stg + r * D + c * 32 + 4 * i), v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars->epi_sync[g]);
        ok = warp_all(wait_bar(&bars->epi_sync[g], 0, w, 25));
        if (ok && r == 0) {
          const CUtensorMap* m = g == 0 ? &tmDV : &tmDK;
          tma_reduce_add_4d(m, stg, 0, key0, hk, b);
          tma_reduce_add_4d(m, stg + 64 * D, 0, key0 + 64, hk, b);
          bulk_commit();
          bulk_wait_all();
        }
      } else if (ok) {
        tc_fence_after();
        const size_t base = ((static_cast<size_t>(b) * a.N + key) * a.Hkv + hk) * D;
        const uint32_t col = g == 0 ? C::kColDV : C::kColDK;
        const float mul = g == 0 ? 1.f : a.scale;
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(g == 0 ? a.dV : a.dK) + base;
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
  } else if (warp < 12) {
    // ===================== dQ drain warpgroup =====================
    // dQ_i^T leaves TMEM as soon as it has been read (so dP_{i+1} can reuse
    // the columns); each 64-query half is then written to a shared-memory
    // staging tile [64 q][128 d] and added into the fp32 accumulator in global
    // memory by one TMA reduce-add (whole lines, no per-element atomics).
    reg_alloc<kRegDrain>();
    if (bars->abort == 0) {
      const int quarter = warp & 3;
      const int dd = quarter * 32 + lane;  // feature index = TMEM lane of dQ^T
      const uint32_t tQ = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + C::kColR2;
      float* stage = reinterpret_cast<float*>(smem + C::kOffDQS);
      const bool issuer = (dd == 0);
      uint32_t sync_phase = 0;
      bool ok = true;
      // all 128 drain threads meet here (bounded wait)
      auto drain_sync = [&]() -> bool {
        mbar_arrive(&bars->stage_sync);
        const bool r = warp_all(wait_bar(&bars->stage_sync, sync_phase & 1, w, 31));
        ++sync_phase;
        return r;
      };
      int qt = qt_beg, hq = hq_beg;
      if constexpr (kSparse) {
        // the first kept pair, then past the `beg` kept pairs of the earlier parts
        qt = i0;
        hq = hk * G;
        for (int skip = -1; skip < beg; ++skip) {
          if (skip >= 0 && ++qt == qt_end) {
            qt = i0;
            ++hq;
          }
          while (hq < hk * G + G && !kept(hq, qt)) {
            if (++qt == qt_end) {
              qt = i0;
              ++hq;
            }
          }
        }
      }
      for (int i = 0; ok && i < nq; ++i) {
        if (!(ok = warp_all(wait_bar(&bars->dq_full, i & 1, w, 30)))) break;
        tc_fence_after();
        const int q0 = qt * kBMq;
        uint32_t v[kBMq];
#pragma unroll
        for (int c = 0; c < kBMq / 32; ++c) tmem_ld32(tQ + 32 * c, v + 32 * c);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kBMq / 32; ++c) reg_fence32(v + 32 * c);
        tc_fence_before();
        mbar_arrive(&bars->dq_free);  // dP_{i+1} may overwrite the columns now
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (issuer) bulk_wait_read_all();  // the previous reduction has read the staging tile
          if (!(ok = drain_sync())) break;
#pragma unroll
          for (int c = 0; c < 64; ++c) stage[c * 128 + dd] = __uint_as_float(v[64 * half + c]);
          fence_proxy_async_smem();
          if (!(ok = drain_sync())) break;
          if (issuer) {
            if (fa_dbg(q0 >= 0 && q0 < a.N && hq < a.H, ctl.status, 0x14))
              tma_reduce_add_4d(&tmDQ, stage, 0, q0 + 64 * half, hq, b);
            bulk_commit();
          }
        }
        do {
          if (++qt == qt_end) {
            qt = i0;
            ++hq;
          }
        } while (kSparse && hq < hk * G + G && !kept(hq, qt));
      }
      if (issuer) bulk_wait_all();
    }
  } else {
    reg_dealloc<kRegCtrl>();
    if (bars->abort == 0 && warp == 12) {
      // ===================== TMA producer =====================
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmDO);
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kTile);
        const bool kv_ok = fa_dbg(key0 >= 0 && key0 < a.N && hk < a.Hkv && b < a.B, ctl.status, 0x11);
        for (int c = 0; kv_ok && c < D / 64; ++c) {
          tma_load_4d(smem + C::kOffK + c * C::kSub, &tmK, &bars->kv_full, c * 64, key0, hk, b);
          tma_load_4d(smem + C::kOffV + c * C::kSub, &tmV, &bars->kv_full, c * 64, key0, hk, b);
        }
        int qt = qt_beg, hq = hq_beg;
        if constexpr (kSparse) {
          // the first kept pair, then past the `beg` kept pairs of the earlier parts
          qt = i0;
          hq = hk * G;
          for (int skip = -1; skip < beg; ++skip) {
            if (skip >= 0 && ++qt == qt_end) {
              qt = i0;
              ++hq;
            }
            while (hq < hk * G + G && !kept(hq, qt)) {
              if (++qt == qt_end) {
                qt = i0;
                ++hq;
              }
            }
          }
        }
        int q_issued = 0;
        for (int i = 0; i < nq; ++i) {
          const int st = i % kStages;
          const int n = i / kStages;
          const int q0 = qt * kBMq;
          const int hq_i = hq;
          do {
            if (++qt == qt_end) {
              qt = i0;
              ++hq;
            }
          } while (kSparse && hq < hk * G + G && !kept(hq, qt));
          if (i >= kStages && !wait_bar(&bars->q_empty[st], (n - 1) & 1, w, 10)) break;
          if constexpr (kSparse) bars->info_q0[i & 3] = q0;
          const size_t bh = static_cast<size_t>(b) * a.H + hq_i;
          mbar_arrive_expect_tx(&bars->q_full[st], 2 * C::kTile + 1024);
          // the tile's rows and head exist, and its 128 LSE / D entries lie inside the [B, H, Npad] rows
          const bool q_ok = fa_dbg(q0 >= 0 && q0 < a.N && hq_i >= hk * G && hq_i < hk * G + G && hq_i < a.H,
                                   ctl.status, 0x12) &&
                            fa_dbg(bh * a.Npad + q0 + kBMq <= static_cast<size_t>(a.B) * a.H * a.Npad, ctl.status,
                                   0x13);
          for (int c = 0; q_ok && c < D / 64; ++c) {
            tma_load_4d(smem + C::kOffQ + st * C::kTile + c * C::kSub, &tmQ, &bars->q_full[st], c * 64, q0, hq_i,
                        b);
            tma_load_4d(smem + C::kOffDO + st * C::kTile + c * C::kSub, &tmDO, &bars->q_full[st], c * 64, q0, hq_i,
                        b);
          }
          if (q_ok) {
            bulk_load(smem + C::kOffL + st * 512, a.LSE2 + bh * a.Npad + q0, 512, &bars->q_full[st]);
            bulk_load(smem + C::kOffDv + st * 512, a.Dvec + bh * a.Npad + q0, 512, &bars->q_full[st]);
          }
          ++q_issued;
        }
        // teardown: no copy of this CTA may still be writing its shared memory
        drain_wait(&bars->kv_full, 0, ctl.limit_ns);
        drain_ring(bars->q_full, kStages, q_issued, ctl.limit_ns);
      }
    } else if (bars->abort == 0 && warp == 13) {
      // ===================== MMA issuer =====================
      if (lane == 0 && nq > 0) {
        const uint32_t sK = smem_u32(smem + C::kOffK);
        const uint32_t sV = smem_u32(smem + C::kOffV);
        const uint32_t sQ = smem_u32(smem + C::kOffQ);
        const uint32_t sDO = smem_u32(smem + C::kOffDO);
        // S^T = K Q^T (or dP^T = V dO^T): A [128 keys][128 d] K-major, B [128 q][128 d] K-major
        auto issue_s = [&](uint32_t a_base, uint32_t b_base, uint32_t col) {
          const uint64_t ad = sw128_desc(a_base, 16, 1024), bd = sw128_desc(b_base, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * C::kSub + (kk & 3) * 32) >> 4;
            umma_ss(tmem + col, ad + off, bd + off, C::kIdescS, kk > 0 ? 1u : 0u);
          }
        };
        // dV += P^T dO (or dK += dS^T Q): A from TMEM (bf16 pairs), B [128 q][128 d] MN-major
        auto issue_kv = [&](uint32_t a_col, uint32_t b_base, uint32_t d_col, bool acc) {
          const uint64_t bd = sw128_desc(b_base, C::kSub, 1024);
#pragma unroll
          for (int kk = 0; kk < kBMq / 16; ++kk)
            umma_ts(tmem + d_col, tmem + a_col + ts_col(kk), bd + static_cast<uint32_t>(kk * 2048 >> 4),
                    C::kIdescKV, (acc || kk > 0) ? 1u : 0u);
        };
        bool ok = wait_bar(&bars->kv_full, 0, w, 11) && wait_bar(&bars->q_full[0], 0, w, 12);
        if (ok) {
          tc_fence_after();
          issue_s(sK, sQ, C::kColR1);
          umma_commit(&bars->s_full);
          issue_s(sV, sDO, C::kColR2);
          umma_commit(&bars->dp_full);
        }
        // per tile: dV_i S_{i+1} dK_i dQ_i dP_{i+1}.  S_{i+1} goes right behind dV_i
        // (which reads P^T_i from the same columns; the tensor pipe keeps issue
        // order), so the softmax warps find it ready when they finish tile i.
        for (int i = 0; ok && i < nq; ++i) {
          const int st = i % kStages;
          const int st1 = (i + 1) % kStages;
          const uint32_t par = i & 1;
          const bool more = i + 1 < nq;
          if (!(ok = wait_bar(&bars->pt_ready, par, w, 13))) break;
          tc_fence_after();
          issue_kv(C::kColR1, sDO + st * C::kTile, C::kColDV, i > 0);
          umma_commit(&bars->dv_done);
          if (more) {
            if (!(ok = wait_bar(&bars->q_full[st1], ((i + 1) / kStages) & 1, w, 14))) break;
            tc_fence_after();
            issue_s(sK, sQ + st1 * C::kTile, C::kColR1);
            umma_commit(&bars->s_full);
          }
          if (!(ok = wait_bar(&bars->ds_ready, par, w, 15))) break;
          tc_fence_after();
          issue_kv(C::kColR2, sQ + st * C::kTile, C::kColDK, i > 0);
          // dQ^T = K^T dS^T over R2: A = K as [128 d (M, contiguous)][128 keys], B = dS^T as
          // [128 q (N, contiguous)][128 keys] in the dO stage buffer
          const uint32_t ds = sDO + st * C::kTile;
          const uint64_t kd = sw128_desc(sK, C::kSub, 1024), dsd = sw128_desc(ds, C::kSub, 1024);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            umma_ss(tmem + C::kColR2, kd + static_cast<uint32_t>(kk * 2048 >> 4),
                    dsd + static_cast<uint32_t>(kk * 2048 >> 4), C::kIdescQ, kk > 0 ? 1u : 0u);
          umma_commit(&bars->dq_full);
          umma_commit(&bars->q_empty[st]);
          if (more) {
            // dP_{i+1} overwrites dQ_i^T in R2: the drain must have read it
            if (!(ok = wait_bar(&bars->dq_free, par, w, 16))) break;
            tc_fence_after();
            issue_s(sV, sDO + st1 * C::kTile, C::kColR2);
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
  if (warp == 13) {
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
                            const CUtensorMap& tdo, const CUtensorMap& tdq, const CUtensorMap& tdk,
                            const CUtensorMap& tdv, const BwdArgs& a, const DevCtl& c, cudaStream_t s) {
  constexpr int smem = BwdCfg::kSmemBytes;
  const dim3 grid((a.N + kBN - 1) / kBN, a.Hkv * a.splits, a.B);
  auto run = [&](auto kernel) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, kThreads, smem, s>>>(tq, tk, tv, tdo, tdq, tdk, tdv, a, c);
    return cudaGetLastError();
  };
  return a.block_mask ? run(bwd_main_kernel<true>) : run(bwd_main_kernel<false>);
}

namespace {
__global__ void __launch_bounds__(256) kv_zero_kernel(float* __restrict__ p, long long n4) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    reinterpret_cast<float4*>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dK = bf16(scale * dKacc), dV = bf16(dVacc), 8 elements per thread
__global__ void __launch_bounds__(256) kv_convert_kernel(const BwdArgs a, long long total) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x * 8;
  for (long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < total; i += stride) {
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const float* src = which ? a.dKacc : a.dVacc;
      const float s = which ? a.scale : 1.f;
      const float4 x = *reinterpret_cast<const float4*>(src + i);
      const float4 y = *reinterpret_cast<const float4*>(src + i + 4);
      uint4 out;
      out.x = pack_bf16x2(x.x * s, x.y * s);
      out.y = pack_bf16x2(x.z * s, x.w * s);
      out.z = pack_bf16x2(y.x * s, y.y * s);
      out.w = pack_bf16x2(y.z * s, y.w * s);
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(which ? a.dK : a.dV) + i) = out;
    }
  }
}

unsigned blocks_for(long long items) {
  long long blocks = (items + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return static_cast<unsigned>(blocks < 1 ? 1 : blocks);
}
}  // namespace

cudaError_t launch_bwd_kv_zero(const BwdArgs& a, cudaStream_t s) {
  const long long n = static_cast<long long>(a.B) * a.N * a.Hkv * a.d;  // per accumulator, a multiple of 64
  kv_zero_kernel<<<blocks_for(n / 4), 256, 0, s>>>(a.dKacc, n / 4);
  kv_zero_kernel<<<blocks_for(n / 4), 256, 0, s>>>(a.dVacc, n / 4);
  return cudaGetLastError();
}

cudaError_t launch_bwd_kv_convert(const BwdArgs& a, cudaStream_t s) {
  const long long total = static_cast<long long>(a.B) * a.N * a.Hkv * a.d;
  kv_convert_kernel<<<blocks_for(total / 8), 256, 0, s>>>(a, total);
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
