// Fused attention forward with 8-bit (e4m3) Q, K, V, fp32 accumulation, sm_100a.
//
// The method is the one of the bf16 forward ("Flash Attention" (Ultralytics
// glossary), "Принцип работы Flash Attention"): key/value tiles stream past a
// resident query block, the running row maximum and sum are kept on chip, and
// only O and one log-sum-exp per row reach memory.  The FP8 form follows the
// pages' note that FlashAttention-3 runs attention with FP8 inputs
// ("Flash Attention" (karlkratz.de), "Versionen"; Ultralytics, "FlashAttention-2,
// -3 и -4").
//
// Numbers: Q, K, V are e4m3 with one fp32 scale per tensor (x = scale_x * code);
// S = Q K^T runs on the tensor cores in kind::f8f6f4 with fp32 accumulation and
// the three scales folded into the softmax's FFMA; P is written back to TMEM as
// e4m3 (the A operand of O += P V must have the same 8-bit kind as V).  Two
// choices keep P inside the e4m3 range with the most precision:
//   * P is scaled by 2^kPOff before rounding: p' = 2^(s - m + kPOff) with the
//     row's reference maximum m, so values down to 2^-(9 + kPOff) of the row's
//     maximum stay representable; the row sum l accumulates the same p' in fp32,
//     so the factor cancels in O = (sum p' v) / l and only enters the LSE;
//   * the lazy-rescale threshold is kTau = 4 (log2 units) so p' <= 2^(kTau +
//     kPOff) = 256 < 448, the largest finite e4m3.
// O is written in bf16 (scaled by V's scale), the LSE in fp32 natural log.
//
// Layout as in the bf16 kernel: one CTA owns two 128-row query tiles of one
// (b, h) and streams 128-key K/V tiles through a 4-stage TMA ring; a 128 x 128
// e4m3 tile is one 16 KB block of 128-byte swizzled rows (all 128 features of a
// row in one swizzle row).  TMEM: S_0 | S_1 | O_0 | O_1; P_t occupies the first
// 32 columns of S_t (four e4m3 per column).  V is the B operand of P V stored
// [keys][features], i.e. MN-major, which tcgen05 allows for 8-bit types.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int D = 128;
constexpr int kThreads = 384;
constexpr uint32_t kRegSoftmax = 216;
constexpr uint32_t kRegOther = 72;
static_assert(kRegSoftmax >= 168 && kRegOther <= 168, "setmaxnreg direction (launch count 168)");
static_assert(2 * kRegSoftmax + kRegOther == 3 * 168, "register split must match the launch");
constexpr float kTau = 4.0f;   // lazy-rescale threshold (log2 units)
constexpr float kPOff = 4.0f;  // P is stored as 2^(s - m + kPOff)
static_assert(kTau + kPOff <= 8.0f, "p' = 2^(kTau + kPOff) must stay below the e4m3 maximum 448");
// One score pair in kPolyEvery takes its exponentials on the FMA pipe
// (exp2_poly2: range reduction and a degree-3 polynomial, relative error
// 7.5e-5, far below e4m3's 2^-4) instead of the MUFU unit, which each score
// otherwise needs once while the 8-bit MMAs take half the bf16 time.  0: none.
constexpr int kPolyEvery = 8;

struct Cfg {
  static constexpr int kTile = kBM * 128;  // one [128][128] e4m3 tile: 16 KB
  static constexpr int kStages = 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffBar = kOffV + kStages * kTile;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
  static constexpr int kOffList = kOffBar + 512;  // block-sparse: the CTA's key-tile list
  static constexpr int kSmemBytesSparse = kOffList + 4 * kMaxSparseTiles + 1024;
  __device__ static constexpr uint32_t colS(int t) { return static_cast<uint32_t>(t) * 128u; }
  __device__ static constexpr uint32_t colO(int t) { return 256u + static_cast<uint32_t>(t) * D; }
  static constexpr uint32_t kIdescS = idesc_e4m3(kBM, kBN, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_e4m3(kBM, D, 0, 1);
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdArgs a, const float out_scale,
                   const DevCtl ctl) {
  using C = Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = warp_id();
  const int lane = lane_id();

  const int nqb = gridDim.x;
  // causal: longest first over every (b, h), as in the bf16 kernel
  int cb = static_cast<int>(blockIdx.x), h = static_cast<int>(blockIdx.y), b = static_cast<int>(blockIdx.z);
  if (a.causal) {
    const int hb = static_cast<int>(gridDim.y * gridDim.z);
    const int rank = static_cast<int>(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    cb = nqb - 1 - rank / hb;
    h = (rank % hb) % static_cast<int>(gridDim.y);
    b = (rank % hb) / static_cast<int>(gridDim.y);
  }
  const int hk = h / (a.H / a.Hkv);
  // key tiles [klo[t], klo[t] + nkt[t]) of query tile t; the CTA streams their union
  int q0[2], klo[2], nkt[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    q0[t] = cb * 2 * kBM + t * kBM;
    klo[t] = 0;
    nkt[t] = 0;
    if (q0[t] < a.N) {
      const int qmax = min(q0[t] + kBM - 1, a.N - 1);
      klo[t] = max(0, q0[t] - a.wl) / kBN;
      nkt[t] = min(a.N - 1, qmax + a.wr) / kBN + 1 - klo[t];
    }
  }
  const int kbase = klo[0];
  int nk = (nkt[1] > 0) ? max(klo[0] + nkt[0], klo[1] + nkt[1]) - kbase : nkt[0];

  // Block-sparse (as in the bf16 kernel): the key tiles of the window range
  // that the mask keeps for at least one of the two query tiles, ascending, as
  // (tile << 2 | bits) with bit t set when query tile t uses the tile; nkt[t]
  // becomes query tile t's count and nk the stream length.
  const uint32_t* klist = reinterpret_cast<const uint32_t*>(smem + C::kOffList);
  if constexpr (kSparse) {
    uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::kOffList);
    __shared__ int s_wcnt[kThreads / 32];
    __shared__ int s_cnt[3];
    const uint8_t* mrow0 = a.block_mask + (static_cast<size_t>(a.mask_heads == 1 ? 0 : h) * a.nb + q0[0] / kBM) * a.nb;
    const uint8_t* mrow1 = mrow0 + a.nb;
    if (threadIdx.x < 3) s_cnt[threadIdx.x] = 0;
    __syncthreads();
    for (int base = 0; base < nk; base += kThreads) {
      const int c = base + static_cast<int>(threadIdx.x);
      const int kt = kbase + c;
      uint32_t f = 0;
      if (c < nk) {
        if (kt >= klo[0] && kt < klo[0] + nkt[0] && mrow0[kt]) f |= 1u;
        if (kt >= klo[1] && kt < klo[1] + nkt[1] && mrow1[kt]) f |= 2u;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, f != 0);
      if (lane == 0) s_wcnt[warp] = __popc(bal);
      __syncthreads();
      int off = s_cnt[2];
      for (int w2 = 0; w2 < warp; ++w2) off += s_wcnt[w2];
      if (f) {
        list[off + __popc(bal & ((1u << lane) - 1u))] = (static_cast<uint32_t>(kt) << 2) | f;
        if (f & 1u) atomicAdd(&s_cnt[0], 1);
        if (f & 2u) atomicAdd(&s_cnt[1], 1);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int tot = 0;
        for (int w2 = 0; w2 < kThreads / 32; ++w2) tot += s_wcnt[w2];
        s_cnt[2] += tot;
      }
      __syncthreads();
    }
    nkt[0] = s_cnt[0];
    nkt[1] = s_cnt[1];
    nk = s_cnt[2];
  }
  // key tile of stream position j, and whether query tile t uses it (dense: the window ranges)
  auto stream_tile = [&](int j) -> int { return kSparse ? static_cast<int>(klist[j] >> 2) : kbase + j; };
  auto uses = [&](int t, int j) -> bool {
    return kSparse ? ((klist[j] >> t) & 1u) != 0 : (kbase + j >= klo[t] && kbase + j < klo[t] + nkt[t]);
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], kBM);
      mbar_init(&bars->o_done[t], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = (*reinterpret_cast<volatile unsigned int*>(ctl.abort_epoch) == ctl.epoch) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(&bars->tmem_base, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl w{&bars->abort, ctl.status, ctl.abort_epoch, ctl.epoch, ctl.limit_ns};

  if (warp < 8) {
    reg_alloc<kRegSoftmax>();
    if (bars->abort == 0) {
      // ===================== softmax warps =====================
      const int t = warp >> 2;
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;
      const int qrow = q0[t] + r;
      const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t tS = tmem + lane_bits + C::colS(t);
      const uint32_t tO = tmem + lane_bits + C::colO(t);
      const float sl2 = a.scale_log2;  // softmax scale * log2 e * scale_q * scale_k
      float m = -INFINITY;
      float l = 0.f;
      bool ok = true;
      int e = -1;  // stream position of this tile's j-th key tile
      for (int j = 0; j < nkt[t]; ++j) {
        if constexpr (kSparse) {
          do {
            ++e;
          } while (!uses(t, e));
        } else {
          e = klo[t] - kbase + j;
        }
        ok = warp_all(wait_bar(&bars->s_full[t], j & 1, w, 8));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) reg_fence32(sr + c * 32);

        const int k0 = stream_tile(e) * kBN;
        const bool need_mask = (k0 + kBN > a.N) || (k0 + kBN - 1 > q0[t] + a.wr) || (k0 < q0[t] + kBM - 1 - a.wl);
        if (need_mask) {
          const int hi = min(a.N - 1, qrow + a.wr);
          const int lo = qrow - a.wl;
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (k0 + c > hi || k0 + c < lo) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
        float mx2 = __uint_as_float(sr[2]), mx3 = __uint_as_float(sr[3]);
#pragma unroll
        for (int c = 4; c < kBN; c += 4) {
          mx0 = fmaxf(mx0, __uint_as_float(sr[c + 0]));
          mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
          mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
          mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
        }
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        const float m_new = fmaxf(m, mx * sl2);
        const bool need = m_new > m + kTau;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = (m_new == -INFINITY) ? 1.f : ex2(m - m_new);
          l *= alpha;
          if (j > 0) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + c * 32, o);
              tmem_wait_ld();
              reg_fence32(o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(tO + c * 32, o);
            }
          }
          m = m_new;
        }
        // p' = 2^(s * sl2 - m + kPOff); a row with no visible key so far has m = -inf
        // and only -inf scores, which give p' = 0 with any finite offset
        const float off = (m == -INFINITY) ? 0.f : kPOff - m;
        const float2 sl2v = make_float2(sl2, sl2);
        const float2 offv = make_float2(off, off);
        float2 rs = make_float2(0.f, 0.f);
        // P_t as e4m3 over the first 32 columns of S_t, 64 keys (16 columns) at a time
#pragma unroll
        for (int q = 0; q < kBN / 64; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = q * 64 + 4 * i;
            const float2 x0 = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2v, offv);
            const float2 x1 = ffma2(make_float2(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])), sl2v, offv);
            const bool poly0 = kPolyEvery > 0 && (2 * i) % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1;
            const bool poly1 = kPolyEvery > 0 && (2 * i + 1) % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1;
            const float2 p0 = poly0 ? exp2_poly2(x0) : make_float2(ex2(x0.x), ex2(x0.y));
            const float2 p1 = poly1 ? exp2_poly2(x1) : make_float2(ex2(x1.x), ex2(x1.y));
            rs = fadd2(rs, fadd2(p0, p1));
            pk[i] = pack_e4m3x4(p0.x, p0.y, p1.x, p1.y);
          }
          tmem_st16(tS + 16 * q, pk);
        }
        l += rs.x + rs.y;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[t]);
      }
      // ---- epilogue ----
      if (ok && nkt[t] == 0 && qrow < a.N) {
        // block-sparse: no key is visible to this row: O = 0, LSE = -inf
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.O) + ((static_cast<size_t>(b) * a.N + qrow) * a.H + h) * D;
#pragma unroll
        for (int c = 0; c < D; c += 8) st_global_v4(orow + c, 0u, 0u, 0u, 0u);
        a.LSE[(static_cast<size_t>(b) * a.H + h) * a.N + qrow] = -INFINITY;
      }
      if (ok && nkt[t] > 0) {
        ok = warp_all(wait_bar(&bars->o_done[t], (nkt[t] - 1) & 1, w, 9));
        if (ok) {
          tc_fence_after();
          const float inv = (l > 0.f) ? out_scale / l : 0.f;
          __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.O) +
                                ((static_cast<size_t>(b) * a.N + qrow) * a.H + h) * D;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
            reg_fence32(o);
            uint32_t pkd[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pkd[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            if (qrow < a.N) {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                st_global_v4(orow + c * 32 + i * 8, pkd[4 * i], pkd[4 * i + 1], pkd[4 * i + 2], pkd[4 * i + 3]);
            }
          }
          if (qrow < a.N) {
            const float lse = (l > 0.f) ? (m - kPOff + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            a.LSE[(static_cast<size_t>(b) * a.H + h) * a.N + qrow] = lse;
          }
        }
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
        uint32_t qbytes = 0;
        for (int t = 0; t < 2; ++t) qbytes += (nkt[t] > 0) ? C::kTile : 0;
        mbar_arrive_expect_tx(&bars->q_full, qbytes);
        for (int t = 0; t < 2; ++t)
          if (nkt[t] > 0 && fa_dbg(q0[t] >= 0 && q0[t] < a.N && h < a.H && b < a.B, ctl.status, 0x21))
            tma_load_4d(smem + C::kOffQ + t * C::kTile, &tmQ, &bars->q_full, 0, q0[t], h, b);
        int k_issued = 0, v_issued = 0;
        for (int j = 0; j < nk; ++j) {
          const int s = j % C::kStages;
          const int n = j / C::kStages;
          if (j >= C::kStages && !wait_bar(&bars->k_empty[s], (n - 1) & 1, w, 1)) break;
          mbar_arrive_expect_tx(&bars->k_full[s], C::kTile);
          const int krow = stream_tile(j) * kBN;
          const bool kv_ok = fa_dbg(krow >= 0 && krow < a.N && hk < a.Hkv && b < a.B, ctl.status, 0x22);
          if (kv_ok) tma_load_4d(smem + C::kOffK + s * C::kTile, &tmK, &bars->k_full[s], 0, krow, hk, b);
          ++k_issued;
          if (j >= C::kStages && !wait_bar(&bars->v_empty[s], (n - 1) & 1, w, 2)) break;
          mbar_arrive_expect_tx(&bars->v_full[s], C::kTile);
          if (kv_ok) tma_load_4d(smem + C::kOffV + s * C::kTile, &tmV, &bars->v_full[s], 0, krow, hk, b);
          ++v_issued;
        }
        // teardown: no copy of this CTA may still be writing its shared memory
        drain_wait(&bars->q_full, 0, ctl.limit_ns);
        drain_ring(bars->k_full, C::kStages, k_issued, ctl.limit_ns);
        drain_ring(bars->v_full, C::kStages, v_issued, ctl.limit_ns);
      }
    } else if (warp == 9) {
      // ===================== MMA issuer (one thread) =====================
      if (lane == 0) {
        const uint32_t sQ = smem_u32(smem + C::kOffQ);
        const uint32_t sK = smem_u32(smem + C::kOffK);
        const uint32_t sV = smem_u32(smem + C::kOffV);
        // S_t = Q_t K^T: K = 32 e4m3 (32 bytes of each swizzled row) per instruction
        auto issue_s = [&](int t, int s) {
          const uint32_t qa = sQ + t * C::kTile;
          const uint32_t kb = sK + s * C::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            umma_ss_f8(tmem + C::colS(t), sw128_desc(qa + kk * 32, 16, 1024), sw128_desc(kb + kk * 32, 16, 1024),
                       C::kIdescS, kk > 0 ? 1u : 0u);
          umma_commit(&bars->s_full[t]);
        };
        // O_t += P_t V: P_t from TMEM (8 columns = 32 keys per instruction), V
        // MN-major (32 key rows of 128 bytes = 4096 bytes per instruction)
        auto issue_pv = [&](int t, int s, bool acc) {
          const uint32_t vb = sV + s * C::kTile;
#pragma unroll
          for (int kk = 0; kk < kBN / 32; ++kk)
            umma_ts_f8(tmem + C::colO(t), tmem + C::colS(t) + kk * 8, sw128_desc(vb + kk * 4096, C::kTile, 1024),
                       C::kIdescPV, (acc || kk > 0) ? 1u : 0u);
          umma_commit(&bars->o_done[t]);
        };
        // jl[t]: how many of query tile t's key tiles have had their P V issued
        int jl[2] = {0, 0};
        // issue order as in the bf16 kernel: S_t(j+1) right behind PV_t(j), which
        // reads P_t(j) from the same columns (the tensor pipe keeps issue order)
        bool ok = nk > 0 && wait_bar(&bars->q_full, 0, w, 3) && wait_bar(&bars->k_full[0], 0, w, 4);
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (uses(t, 0)) issue_s(t, 0);
          umma_commit(&bars->k_empty[0]);
        }
        for (int j = 0; ok && j < nk; ++j) {
          const int s = j % C::kStages;
          const int sn = (j + 1) % C::kStages;
          if (!(ok = wait_bar(&bars->v_full[s], (j / C::kStages) & 1, w, 6))) break;
          bool next_k = false;
          for (int t = 0; t < 2; ++t) {
            if (uses(t, j)) {
              if (!(ok = wait_bar(&bars->p_full[t], jl[t] & 1, w, 7))) break;
              tc_fence_after();
              issue_pv(t, s, jl[t] > 0);
              ++jl[t];
            }
            if (j + 1 < nk && uses(t, j + 1)) {
              if (!next_k) {
                if (!(ok = wait_bar(&bars->k_full[sn], ((j + 1) / C::kStages) & 1, w, 5))) break;
                tc_fence_after();
                next_k = true;
              }
              issue_s(t, sn);
            }
          }
          if (!ok) break;
          umma_commit(&bars->v_empty[s]);
          if (next_k) umma_commit(&bars->k_empty[sn]);
        }
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

cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                           float out_scale, const DevCtl& c, cudaStream_t s) {
  const int nqb = (a.N + 2 * kBM - 1) / (2 * kBM);
  const dim3 grid(nqb, a.H, a.B);
  auto run = [&](auto kernel, int smem) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, kThreads, smem, s>>>(tq, tk, tv, a, out_scale, c);
    return cudaGetLastError();
  };
  return a.block_mask ? run(fwd_fp8_kernel<true>, Cfg::kSmemBytesSparse) : run(fwd_fp8_kernel<false>, Cfg::kSmemBytes);
}

}  // namespace fa
