// Backward main kernel for head dimension 64 (sm_100a).
//
// Same method as the d = 128 kernel ("Flash Attention" (karlkratz.de),
// "Recomputation beim Rückwärtsdurchlauf": the score tiles are recomputed
// from Q, K and the saved LSE), with the layout that d = 64 allows:
//   * K_j, V_j ([128 keys][64] bf16, 16 KB each) stay resident; Q_i, dO_i
//     stream through a 2-stage TMA ring;
//   * TMEM: dV (64 columns) | dK (64) | dQ_i (64, lanes = queries) | R1 (S^T,
//     then P^T) | R2 (dP^T, then dS^T).  dQ has columns of its own, so dP_(i+1)
//     never waits for the dQ drain (at d = 128 the four 128-column regions fill
//     TMEM and dQ^T must reuse R2);
//   * dQ_i = dS_i K_j is computed non-transposed (M = 128 queries, N = 64): A is
//     dS^T in shared memory read MN-major, B is K read MN-major; dS^T has two
//     32 KB buffers of its own (the dO tile is too small to hold it);
//   * the drain thread of query row q reads its 64 fp32 dQ values and writes
//     them into a 128-byte-swizzled staging tile with 16-byte stores; two TMA
//     reduce-adds (32 features each) add the tile into the fp32 accumulator.
// Masks (causal, window, block-sparse) and grouped K/V heads as at d = 128.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int D = 64;
constexpr int kBN = 128;       // keys per CTA (TMEM lanes of S^T, dP^T, dK, dV)
constexpr int kBMq = 128;      // query rows per streamed tile
constexpr int kThreads = 512;  // WG0, WG1: P / dS for query columns 0-63 / 64-127; WG2: dQ drain; WG3: loader + MMA
constexpr int kStages = 2;
constexpr uint32_t kRegLaunch = 128;
constexpr uint32_t kRegCompute = 144;
constexpr uint32_t kRegDrain = 144;
constexpr uint32_t kRegCtrl = 80;
static_assert(kRegCompute >= kRegLaunch && kRegDrain >= kRegLaunch && kRegCtrl <= kRegLaunch,
              "setmaxnreg direction");
static_assert(2 * kRegCompute + kRegDrain + kRegCtrl == 4 * kRegLaunch, "register split must match the launch");

struct Cfg {
  static constexpr int kTile = kBN * 128;                  // one [128 rows][64] bf16 SW128 tile: 16 KB
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;              // [stage] Q_i
  static constexpr int kOffDO = kOffQ + kStages * kTile;   // [stage] dO_i
  static constexpr int kOffDS = kOffDO + kStages * kTile;  // [2] dS^T_i: [128 keys][128 q] as 2 x [128][64]
  static constexpr int kOffDQS = kOffDS + 2 * 2 * kTile;   // dQ staging: [2 boxes][128 q][32 d] fp32, SW128
  static constexpr int kOffL = kOffDQS + 2 * 128 * 128;    // [stage][128] fp32 LSE * log2 e
  static constexpr int kOffDv = kOffL + kStages * 512;     // [stage][128] fp32 rowsum(dO * O)
  static constexpr int kOffBar = kOffDv + kStages * 512;
  static constexpr int kSmemBytes = kOffBar + 256;
  static constexpr uint32_t kColDV = 0, kColDK = 64, kColDQ = 128, kColR1 = 256, kColR2 = 384;
  static constexpr uint32_t kIdescS = idesc_bf16(kBN, kBMq, 0, 0);  // S^T, dP^T: K-major A and B
  static constexpr uint32_t kIdescKV = idesc_bf16(kBN, D, 0, 1);    // dV, dK: A from TMEM, B MN-major
  static constexpr uint32_t kIdescQ = idesc_bf16(kBMq, D, 1, 1);    // dQ: A (dS) and B (K) MN-major
};
static_assert(Cfg::kSmemBytes <= 232448, "shared memory layout");
static_assert(Cfg::kOffDS % 1024 == 0 && Cfg::kOffDQS % 1024 == 0, "swizzled tiles need 1024-byte alignment");

struct Bars {
  uint64_t kv_full;
  uint64_t q_full[kStages], q_empty[kStages];
  uint64_t s_full, dp_full, pt_ready, ds_ready, dq_full, dq_free;
  uint64_t ds_free[2];  // dQ_i has read dS^T buffer i % 2
  uint64_t acc_done;
  uint64_t drain;
  uint64_t stage_sync;
  uint32_t tmem_base;
  int abort;
  int info_q0[4];  // block-sparse: first query row of tile i in slot i % 4 (as at d = 128)
  int sparse_nq;
  uint64_t epi_sync[2];  // split walks: a compute warpgroup's partial dV / dK is staged
};
static_assert(sizeof(Bars) <= 256, "barrier block");

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }


// TMEM column of the bf16 pairs for reduction step kk (16 query columns) of a
// P^T / dS^T tile written by the two compute warpgroups.
__device__ __forceinline__ uint32_t ts_col(int kk) { return (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8; }

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    bwd64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                 const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                 const __grid_constant__ CUtensorMap tmDV, const BwdArgs a, const DevCtl ctl) {
  using C = Cfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(ctl.status, 0, kDevTimeout | 0xA2);
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
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
  const int kmax = min(key0 + kBN - 1, a.N - 1);
  const int i0 = max(0, key0 - a.wr) / kBMq;
  const int i_end = min(a.N - 1, kmax + a.wl) / kBMq + 1;
  const int G = a.H / a.Hkv;
  const int nq_head = max(0, min(nq_total, i_end) - i0);
  int nq = G * nq_head;
  const int qt_end = i0 + nq_head;
  auto kept = [&](int hq, int qt) -> bool {
    return a.block_mask[(static_cast<size_t>(a.mask_heads == 1 ? 0 : hq) * a.nb + qt) * a.nb + jt] != 0;
  };
  if constexpr (kSparse) {
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
  const int beg = static_cast<int>((static_cast<long long>(nq) * sp) / a.splits);
  nq = static_cast<int>((static_cast<long long>(nq) * (sp + 1)) / a.splits) - beg;
  const int qt_beg = (nq_head > 0) ? i0 + beg % nq_head : i0;
  const int hq_beg = hk * G + ((nq_head > 0) ? beg / nq_head : 0);

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
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, 128);
    mbar_init(&bars->ds_free[0], 1);
    mbar_init(&bars->ds_free[1], 1);
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
    reg_alloc<kRegCompute>();
    if (bars->abort == 0) {
      const int g = warp >> 2;
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;  // key row = TMEM lane
      const int key = key0 + r;
      const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t tR1 = tmem + lane_bits + C::kColR1 + 64 * g;
      const uint32_t tR2 = tmem + lane_bits + C::kColR2 + 64 * g;
      const float sl2 = a.scale_log2;
      bool ok = true;
      int qt = qt_beg;
      for (int i = 0; i < nq; ++i) {
        const int st = i % kStages;
        const uint32_t par = i & 1;
        int q0 = qt * kBMq + 64 * g;
        qt = (qt + 1 == qt_end) ? i0 : qt + 1;
        ok = warp_all(wait_bar(&bars->q_full[st], (i / kStages) & 1, w, 40));
        if (!ok) break;
        if constexpr (kSparse) q0 = *reinterpret_cast<volatile int*>(&bars->info_q0[i & 3]) + 64 * g;
        ok = warp_all(wait_bar(&bars->s_full, par, w, 41));
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
        const bool need_mask =
            (q0 + 64 > a.N) || (key0 + kBN > a.N) || (key0 + kBN - 1 > q0 + a.wr) || (key0 < q0 + 63 - a.wl);
        float p[64];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
          for (int c4 = 8 * hh; c4 < 8 * hh + 8; ++c4) {
            const float4 l4 = sL[c4];
            const float2 x0 = ffma2(make_float2(__uint_as_float(sr[4 * c4]), __uint_as_float(sr[4 * c4 + 1])),
                                    make_float2(sl2, sl2), make_float2(-l4.x, -l4.y));
            const float2 x1 = ffma2(make_float2(__uint_as_float(sr[4 * c4 + 2]), __uint_as_float(sr[4 * c4 + 3])),
                                    make_float2(sl2, sl2), make_float2(-l4.z, -l4.w));
            p[4 * c4 + 0] = ex2(x0.x);
            p[4 * c4 + 1] = ex2(x0.y);
            p[4 * c4 + 2] = ex2(x1.x);
            p[4 * c4 + 3] = ex2(x1.y);
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

        ok = warp_all(wait_bar(&bars->dp_full, par, w, 42));
        if (!ok) break;
        // dS^T buffer i % 2 was last read by dQ_(i-2)
        if (i >= 2) ok = warp_all(wait_bar(&bars->ds_free[i & 1], ((i >> 1) - 1) & 1, w, 43));
        if (!ok) break;
        tc_fence_after();
        const uint32_t sDSt = smem_u32(smem + C::kOffDS + (i & 1) * 2 * C::kTile + g * C::kTile);
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
            // packed pairs: the same subtract-then-multiply roundings, half the instructions
            const float2 lo = fmul2(make_float2(p[c + 0], p[c + 1]),
                                    fsub2(make_float2(__uint_as_float(dr[4 * c4 + 0]), __uint_as_float(dr[4 * c4 + 1])),
                                          make_float2(d4.x, d4.y)));
            const float2 hi = fmul2(make_float2(p[c + 2], p[c + 3]),
                                    fsub2(make_float2(__uint_as_float(dr[4 * c4 + 2]), __uint_as_float(dr[4 * c4 + 3])),
                                          make_float2(d4.z, d4.w)));
            pk[2 * c4] = pack_bf16x2(lo.x, lo.y);
            pk[2 * c4 + 1] = pack_bf16x2(hi.x, hi.y);
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
      if (ok && nq > 0) ok = warp_all(wait_bar(&bars->acc_done, 0, w, 44));
      if (ok && a.splits > 1) {
        // a part of a split walk: the Q (WG0) or dO (WG1) stages hold the
        // [128 keys][64] fp32 partial sums for one TMA reduce-add
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
        ok = warp_all(wait_bar(&bars->epi_sync[g], 0, w, 55));
        if (ok && r == 0) {
          tma_reduce_add_4d(g == 0 ? &tmDV : &tmDK, stg, 0, key0, hk, b);
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
    // Thread q (TMEM lane) owns query row q of dQ_i: 64 fp32 values, staged as
    // two [128 q][32 d] 128-byte-swizzled boxes and added into the fp32
    // accumulator by two TMA reduce-adds.
    reg_alloc<kRegDrain>();
    if (bars->abort == 0) {
      const int quarter = warp & 3;
      const int q = quarter * 32 + lane;
      const uint32_t tQ = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + C::kColDQ;
      uint8_t* stage = smem + C::kOffDQS;
      const bool issuer = (q == 0);
      uint32_t sync_phase = 0;
      bool ok = true;
      auto drain_sync = [&]() -> bool {
        mbar_arrive(&bars->stage_sync);
        const bool r = warp_all(wait_bar(&bars->stage_sync, sync_phase & 1, w, 45));
        ++sync_phase;
        return r;
      };
      int qt = qt_beg, hq = hq_beg;
      if constexpr (kSparse) {
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
        if (!(ok = warp_all(wait_bar(&bars->dq_full, i & 1, w, 46)))) break;
        tc_fence_after();
        const int q0 = qt * kBMq;
        uint32_t v[D];
        tmem_ld32(tQ, v);
        tmem_ld32(tQ + 32, v + 32);
        tmem_wait_ld();
        reg_fence32(v);
        reg_fence32(v + 32);
        tc_fence_before();
        mbar_arrive(&bars->dq_free);  // dQ_(i+1) may overwrite the columns now
        if (issuer) bulk_wait_read_all();  // the previous reduce-adds have read the staging tile
        if (!(ok = drain_sync())) break;
        const uint32_t row = smem_u32(stage) + q * 128;
#pragma unroll
        for (int bx = 0; bx < 2; ++bx) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(row + bx * 16384 + ((c ^ (q & 7)) << 4), v[32 * bx + 4 * c], v[32 * bx + 4 * c + 1],
                         v[32 * bx + 4 * c + 2], v[32 * bx + 4 * c + 3]);
        }
        fence_proxy_async_smem();
        if (!(ok = drain_sync())) break;
        if (issuer) {
          tma_reduce_add_4d(&tmDQ, stage, 0, q0, hq, b);
          tma_reduce_add_4d(&tmDQ, stage + 16384, 32, q0, hq, b);
          bulk_commit();
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
        if (fa_dbg(key0 >= 0 && key0 < a.N && hk < a.Hkv && b < a.B, ctl.status, 0x31)) {
          tma_load_4d(smem + C::kOffK, &tmK, &bars->kv_full, 0, key0, hk, b);
          tma_load_4d(smem + C::kOffV, &tmV, &bars->kv_full, 0, key0, hk, b);
        }
        int qt = qt_beg, hq = hq_beg;
        if constexpr (kSparse) {
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
          if (i >= kStages && !wait_bar(&bars->q_empty[st], (n - 1) & 1, w, 47)) break;
          if constexpr (kSparse) bars->info_q0[i & 3] = q0;
          const size_t bh = static_cast<size_t>(b) * a.H + hq_i;
          mbar_arrive_expect_tx(&bars->q_full[st], 2 * C::kTile + 1024);
          if (fa_dbg(q0 >= 0 && q0 < a.N && hq_i < a.H &&
                         bh * a.Npad + q0 + kBMq <= static_cast<size_t>(a.B) * a.H * a.Npad,
                     ctl.status, 0x32)) {
            tma_load_4d(smem + C::kOffQ + st * C::kTile, &tmQ, &bars->q_full[st], 0, q0, hq_i, b);
            tma_load_4d(smem + C::kOffDO + st * C::kTile, &tmDO, &bars->q_full[st], 0, q0, hq_i, b);
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
      // ===================== MMA issuer (one warp) =====================
      // The whole warp runs the loop (waits and descriptor arithmetic are
      // warp-uniform) and one lane elected by elect.sync issues each MMA and
      // commit: a lone lane-0 issuer loses its SMSP's issue slots to the
      // compute and drain warps there (measured on B200: B1 H32 N16384 7.46 ->
      // 6.20 ms, B4 H16 N1024 0.112 -> 0.102 ms).
      if (nq > 0) {
        const uint32_t sK = smem_u32(smem + C::kOffK);
        const uint32_t sV = smem_u32(smem + C::kOffV);
        const uint32_t sQ = smem_u32(smem + C::kOffQ);
        const uint32_t sDO = smem_u32(smem + C::kOffDO);
        const uint32_t sDS = smem_u32(smem + C::kOffDS);
        // S^T = K Q^T (dP^T = V dO^T): A [128 keys][64] and B [128 q][64], both K-major
        auto issue_s = [&](uint32_t a_base, uint32_t b_base, uint32_t col) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss_w(tmem + col, sw128_desc(a_base + kk * 32, 16, 1024), sw128_desc(b_base + kk * 32, 16, 1024),
                    C::kIdescS, kk > 0 ? 1u : 0u);
        };
        // dV += P^T dO (dK += dS^T Q): A from TMEM, B [128 q][64] MN-major
        auto issue_kv = [&](uint32_t a_col, uint32_t b_base, uint32_t d_col, bool acc) {
#pragma unroll
          for (int kk = 0; kk < kBMq / 16; ++kk)
            umma_ts_w(tmem + d_col, tmem + a_col + ts_col(kk), sw128_desc(b_base + kk * 2048, C::kTile, 1024),
                    C::kIdescKV, (acc || kk > 0) ? 1u : 0u);
        };
        bool ok = warp_all(wait_bar(&bars->kv_full, 0, w, 48)) && warp_all(wait_bar(&bars->q_full[0], 0, w, 49));
        if (ok) {
          tc_fence_after();
          issue_s(sK, sQ, C::kColR1);
          umma_commit_w(&bars->s_full);
          issue_s(sV, sDO, C::kColR2);
          umma_commit_w(&bars->dp_full);
        }
        // per tile: dV_i S_(i+1) dK_i dQ_i dP_(i+1); each overwrite of R1 / R2 comes
        // after the MMA that reads those columns (the tensor pipe keeps issue order)
        for (int i = 0; ok && i < nq; ++i) {
          const int st = i % kStages;
          const int st1 = (i + 1) % kStages;
          const uint32_t par = i & 1;
          const bool more = i + 1 < nq;
          if (!(ok = warp_all(wait_bar(&bars->pt_ready, par, w, 50)))) break;
          tc_fence_after();
          issue_kv(C::kColR1, sDO + st * C::kTile, C::kColDV, i > 0);
          if (more) {
            if (!(ok = warp_all(wait_bar(&bars->q_full[st1], ((i + 1) / kStages) & 1, w, 51)))) break;
            tc_fence_after();
            issue_s(sK, sQ + st1 * C::kTile, C::kColR1);
            umma_commit_w(&bars->s_full);
          }
          if (!(ok = warp_all(wait_bar(&bars->ds_ready, par, w, 52)))) break;
          tc_fence_after();
          issue_kv(C::kColR2, sQ + st * C::kTile, C::kColDK, i > 0);
          // dQ_i = dS_i K: A = dS (M = 128 queries contiguous in two 64-wide chunks,
          // K = keys on rows), B = K (N = 64 features contiguous, K = keys on rows)
          if (i > 0 && !(ok = warp_all(wait_bar(&bars->dq_free, (i - 1) & 1, w, 53)))) break;
          tc_fence_after();
          const uint32_t ds = sDS + (i & 1) * 2 * C::kTile;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            umma_ss_w(tmem + C::kColDQ, sw128_desc(ds + kk * 2048, C::kTile, 1024),
                    sw128_desc(sK + kk * 2048, C::kTile, 1024), C::kIdescQ, kk > 0 ? 1u : 0u);
          umma_commit_w(&bars->dq_full);
          umma_commit_w(&bars->ds_free[i & 1]);
          umma_commit_w(&bars->q_empty[st]);
          if (more) {
            // dO_(i+1) arrived with Q_(i+1) (same barrier, waited above); dK_i has
            // been issued, so it reads dS^T_i from R2 before dP_(i+1) overwrites it
            issue_s(sV, sDO + st1 * C::kTile, C::kColR2);
            umma_commit_w(&bars->dp_full);
          }
        }
        if (ok) umma_commit_w(&bars->acc_done);
        umma_commit_w(&bars->drain);
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

cudaError_t launch_bwd_main64(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& tdo, const CUtensorMap& tdq, const CUtensorMap& tdk,
                              const CUtensorMap& tdv, const BwdArgs& a, const DevCtl& c, cudaStream_t s) {
  constexpr int smem = Cfg::kSmemBytes;
  const dim3 grid((a.N + kBN - 1) / kBN, a.Hkv * a.splits, a.B);
  auto run = [&](auto kernel) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, kThreads, smem, s>>>(tq, tk, tv, tdo, tdq, tdk, tdv, a, c);
    return cudaGetLastError();
  };
  return a.block_mask ? run(bwd64_kernel<true>) : run(bwd64_kernel<false>);
}

}  // namespace fa
