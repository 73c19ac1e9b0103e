// Fused attention forward, bf16 inputs, fp32 accumulation, sm_100a.
//
// Method: "Flash Attention" (Ultralytics glossary), "Принцип работы Flash
// Attention" -- a block of queries stays on chip while key/value blocks stream
// past; per block the scores are formed, the running row maximum and sum are
// updated, the partial output is rescaled when the maximum grows, and the
// block's weighted values are added; only the output and one number per row
// (here the log-sum-exp) go back to HBM.  "Flash Attention" (karlkratz.de),
// "Tiling: Blockweise Berechnung im schnellen Speicher" gives the same per-row
// maximum / sum pair and the correction factor.
//
// B200 design (ours; the pages' A100/H100 tilings are prior art only):
//   * one CTA owns two 128-row query tiles (t = 0, 1) of one (b, h) and
//     streams 128-key K/V tiles through a TMA ring in shared memory
//     (128-byte swizzle, mbarrier completion);
//   * one warp issues all tcgen05 MMAs (converged, one lane elected per
//     instruction): S_t = Q_t K^T (both operands from
//     shared memory, accumulator in TMEM) and O_t += P_t V (P_t read straight
//     from TMEM where the softmax wrote it over S_t, V from shared memory);
//   * eight softmax warps (one TMEM lane = one query row per thread) read S_t,
//     mask, take the row max, form P = 2^(S*scale*log2e - m) with the scale
//     folded into one FFMA, add the row sum, and write P back as bf16;
//   * lazy rescale: the reference maximum m only moves when a row's maximum
//     grows by more than 2^12; numerator and denominator share m, so the result
//     is exact and the O rescale (a TMEM read-modify-write) is rare;
//   * causal and sliding-window masks: key tiles that no row of the query
//     tile can see are never loaded or multiplied ("Flash Attention"
//     (karlkratz.de), "Sliding Window Attention": blocks outside the window
//     are skipped); only the tiles that straddle the window's edge are masked;
//     under the causal mask the launch order is longest first over every
//     (b, h): the CTAs of the last query tiles of all heads go first;
//   * block-sparse masks (the kSparse instantiation): the CTA compacts the key
//     tiles either query tile keeps into a list in shared memory; the loader
//     streams only those, and each tile skips the ones it does not keep; a
//     row that keeps none gets O = 0, LSE = -inf;
//   * grouped-query attention: query head h reads K/V head h / (H / Hkv);
//   * epilogue: O / l -> bf16, staged in the query tile's shared memory (free
//     once its last S MMA is done) in the 128-byte swizzled layout and written
//     by TMA tile stores (whole coalesced lines); LSE = (m + log2 l) ln 2.
// The two query tiles ping-pong: while the softmax of one tile runs, the
// tensor pipe computes the other tile's products.  Short walks (a query row
// sees at most 768 keys) run one query tile per CTA and two CTAs per SM
// instead (half the tensor memory, under half the shared memory each), which
// ping-pong the same way and overlap each other's start and end.
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;        // query rows per tile = TMEM lanes
constexpr int kBN = 128;        // keys per K/V tile
// kT query tiles per CTA: 2 (one CTA per SM) or 1 (two CTAs per SM, each with
// half the tensor memory and under half the shared memory).  Warpgroups: kT
// softmax warpgroups, then one with the loader warp, the MMA warp and 2 spare.
template <int kT>
struct FwdShape {
  static constexpr int kThreads = 128 * (kT + 1);
  static constexpr int kMinBlocks = (kT == 1) ? 2 : 1;
  // Register split (per thread): kT = 2: 384 x 168 at launch = 256 x 216 + 128 x 72;
  // kT = 1: 256 x 128 = 128 x 208 + 128 x 48 (two CTAs share the register file;
  // 192 for the softmax warps left it spilling).
  static constexpr uint32_t kRegLaunch = (kT == 1) ? 128 : 168;
  static constexpr uint32_t kRegSoftmax = (kT == 1) ? 208 : 216;
  static constexpr uint32_t kRegOther = (kT == 1) ? 48 : 72;
  static constexpr uint32_t kTmemCols = (kT == 1) ? 256 : 512;
  static_assert(kRegSoftmax >= kRegLaunch && kRegOther <= kRegLaunch, "setmaxnreg direction");
  static_assert(kT * kRegSoftmax + kRegOther == (kT + 1) * kRegLaunch, "register split must match the launch");
  static_assert(kThreads * kRegLaunch * kMinBlocks <= 65536, "register file");
};
// Lazy-rescale threshold (log2 units).  A stale m leaves every p <= 2^kTau, so
// l <= 2^kTau * N and |O| <= 2^kTau * N * max|V| stay far inside fp32 for any
// N < 2^31; bf16 P keeps its relative precision at any scale.  12 rather than
// 8: inputs with a few large keys (the K-spike workload) otherwise move m on
// about a fifth of the (query tile, key tile) steps, each a stall of the
// softmax warps for a read-modify-write of O in TMEM.
constexpr float kTau = 12.0f;
// When > 0, one score pair in kPolyEvery<D, kT> takes its exponentials on the FMA
// pipe (exp2_poly2) instead of the MUFU unit.  Measured on B200 with the converged
// MMA warp: at d = 64 with two query tiles per CTA, one pair in 8 is 3.5% faster
// (B1 H32 N16384; 1% causal): the MMAs are half as long as at d = 128, so the two
// softmax warpgroups' exponentials overlap more.  At d = 128 the same share cost
// the bench step's forward 2%, and with one query tile per CTA (short walks) 13%,
// so those instantiations keep every exponential on the MUFU unit.
template <int D, int kT>
constexpr int kPolyEvery = (D == 64 && kT == 2) ? 8 : 0;

template <int D, int kT>
struct FwdCfg {
  static constexpr int kSub = D / 64;                 // 64-feature sub-tiles per row
  static constexpr int kSubBytes = kBM * 128;         // one [128][64] bf16 sub-tile
  static constexpr int kTileBytes = kSub * kSubBytes; // one 128 x D tile
  // K/V ring depth: two CTAs per SM (kT = 1) keep half as many stages each
  static constexpr int kStages = ((D == 128) ? 2 : 4) / (3 - kT);
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kT * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kOffList = kOffBar + 512;           // block-sparse: the CTA's key-tile list
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // barriers + base alignment slack
  static constexpr int kSmemBytesSparse = kOffList + 4 * kMaxSparseTiles + 1024;
  // TMEM columns: S_0 | S_1 | O_0 | O_1
  __device__ static constexpr uint32_t colS(int t) { return static_cast<uint32_t>(t) * 128u; }
  __device__ static constexpr uint32_t colO(int t) { return kT * 128u + static_cast<uint32_t>(t) * D; }
  static constexpr uint32_t kIdescS = idesc_bf16(kBM, kBN, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16(kBM, D, 0, 1);
};

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t drain;
  uint64_t epi[2];  // query tile t's O rows are staged in shared memory
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

template <int D, bool kSparse, int kT>
__global__ void __launch_bounds__(FwdShape<kT>::kThreads, FwdShape<kT>::kMinBlocks)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, const FwdArgs a,
                    const DevCtl ctl) {
  using C = FwdCfg<D, kT>;
  using W = FwdShape<kT>;
  static_assert(kT == 2 || !kSparse, "block-sparse walks pair two query tiles");
  constexpr int kThreads = W::kThreads;
  constexpr int kLoaderWarp = 4 * kT, kMmaWarp = 4 * kT + 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::kOffBar);
  const int warp = warp_id();
  const int lane = lane_id();

  // ---- work of this CTA ----
  // Causal: the launch order (block x fastest, then y, then z) is longest
  // first over every (b, h): the CTA's rank in that order picks the pair of
  // query tiles from the end of the sequence, the head and batch vary fastest.
  const int nqb = gridDim.x;
  int cb = static_cast<int>(blockIdx.x), h = static_cast<int>(blockIdx.y), b = static_cast<int>(blockIdx.z);
  if (a.causal) {
    const int hb = static_cast<int>(gridDim.y * gridDim.z);
    const int rank = static_cast<int>(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    cb = nqb - 1 - rank / hb;
    h = (rank % hb) % static_cast<int>(gridDim.y);
    b = (rank % hb) / static_cast<int>(gridDim.y);
  }
  const int hk = h / (a.H / a.Hkv);  // K/V head of this query head (grouped-query attention)
  // Key tiles [klo[t], klo[t] + nkt[t]) hold every key some row of query tile
  // t may see; the CTA streams their union, key tiles kbase .. kbase + nk - 1
  // (the two ranges overlap or touch, since each row sees its own key).
  int q0[2], klo[2], nkt[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    q0[t] = cb * kT * kBM + t * kBM;
    klo[t] = 0;
    nkt[t] = 0;
    if (t < kT && q0[t] < a.N) {
      const int qmax = min(q0[t] + kBM - 1, a.N - 1);
      klo[t] = max(0, q0[t] - a.wl) / kBN;
      nkt[t] = min(a.N - 1, qmax + a.wr) / kBN + 1 - klo[t];
    }
  }
  const int kbase = klo[0];
  int nk = (nkt[1] > 0) ? max(klo[0] + nkt[0], klo[1] + nkt[1]) - kbase : nkt[0];

  // Block-sparse: the key tiles of the window range that the mask keeps for at
  // least one of the two query tiles, in ascending order, as (tile << 2 | bits)
  // with bit t set when query tile t uses the tile.  All roles read this list;
  // nkt[t] becomes query tile t's count and nk the stream length.
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
      mbar_init(&bars->epi[t], kBM);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = (*reinterpret_cast<volatile unsigned int*>(ctl.abort_epoch) == ctl.epoch) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(&bars->tmem_base, W::kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl w{&bars->abort, ctl.status, ctl.abort_epoch, ctl.epoch, ctl.limit_ns};

  if (warp < 4 * kT) {
    reg_alloc<W::kRegSoftmax>();
    if (bars->abort == 0) {
      // ===================== softmax warps =====================
      const int t = warp >> 2;
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;
      const int qrow = q0[t] + r;
      const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t tS = tmem + lane_bits + C::colS(t);
      const uint32_t tO = tmem + lane_bits + C::colO(t);
      const float sl2 = a.scale_log2;
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
        // whole tile visible to every row of the query tile: no mask
        const bool need_mask = (k0 + kBN > a.N) || (k0 + kBN - 1 > q0[t] + a.wr) || (k0 < q0[t] + kBM - 1 - a.wl);
        if (need_mask) {
          const int hi = min(a.N - 1, qrow + a.wr);  // visible keys: [lo, hi]
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
            // O_t holds the sum over the previous key tiles: PV_t(j-1) was
            // issued before S_t(j), and s_full fired when S_t(j) completed.
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
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        const float2 sl2v = make_float2(sl2, sl2);
        const float2 negmv = make_float2(neg_m, neg_m);
        float2 rs = make_float2(0.f, 0.f);
        // P_t (bf16, two per column) over the first 64 columns of S_t, written
        // 16 columns (32 scores) at a time so the stores overlap the math
#pragma unroll
        for (int q = 0; q < kBN / 32; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = q * 32 + 2 * i;
            const float2 x = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2v, negmv);
            float2 p = make_float2(0.f, 0.f);
            bool poly = false;
            constexpr int kPoly = kPolyEvery<D, kT>;
            if constexpr (kPoly > 0) poly = (i % (kPoly > 0 ? kPoly : 1)) == kPoly - 1;
            if (poly) {
              p = exp2_poly2(x);
            } else {
              p.x = ex2(x.x);
              p.y = ex2(x.y);
            }
            rs = fadd2(rs, p);
            pk[i] = pack_bf16x2(p.x, p.y);
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
          // O_t / l as bf16 into Q_t's shared memory: every S_t MMA, issued
          // before the last P_t V, has completed when o_done fires.  Row r
          // writes its 16-byte units in the 128-byte swizzled [128][64]
          // sub-tiles (eight rows of a quarter-warp hit eight distinct bank
          // groups), then one thread stores the tile with TMA.
          tc_fence_after();
          const float inv = (l > 0.f) ? 1.f / l : 0.f;
          uint8_t* stage = smem + C::kOffQ + t * C::kTileBytes;
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
            const uint32_t sub = smem_u32(stage + (c >> 1) * C::kSubBytes);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              st_shared_v4(sub + sw128_offset(r, (c & 1) * 4 + i), pkd[4 * i], pkd[4 * i + 1], pkd[4 * i + 2],
                           pkd[4 * i + 3]);
          }
          fence_proxy_async_smem();
          if (qrow < a.N && fa_dbg(b < a.B && h < a.H, ctl.status, 0x04)) {
            const float lse = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            a.LSE[(static_cast<size_t>(b) * a.H + h) * a.N + qrow] = lse;
          }
          mbar_arrive(&bars->epi[t]);
          if (r == 0 && wait_bar(&bars->epi[t], 0, w, 10)) {
            // rows past N are outside the tensor and are not written
            if (fa_dbg(q0[t] >= 0 && q0[t] < a.N, ctl.status, 0x03))
              for (int c = 0; c < C::kSub; ++c) tma_store_4d(&tmO, stage + c * C::kSubBytes, c * 64, q0[t], h, b);
            bulk_commit();
            bulk_wait_read_all();  // the staging tile is read before the CTA's shared memory is released
          }
        }
      }
    }
  } else {
    reg_dealloc<W::kRegOther>();
    if (bars->abort == 0 && warp == kLoaderWarp) {
      // ===================== TMA producer =====================
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        uint32_t qbytes = 0;
        for (int t = 0; t < 2; ++t) qbytes += (nkt[t] > 0) ? C::kTileBytes : 0;
        mbar_arrive_expect_tx(&bars->q_full, qbytes);
        for (int t = 0; t < 2; ++t) {
          if (nkt[t] == 0) continue;
          if (!fa_dbg(q0[t] >= 0 && q0[t] < a.N && h < a.H && b < a.B, ctl.status, 0x01)) continue;
          for (int c = 0; c < C::kSub; ++c)
            tma_load_4d(smem + C::kOffQ + t * C::kTileBytes + c * C::kSubBytes, &tmQ, &bars->q_full, c * 64,
                        q0[t], h, b);
        }
        int k_issued = 0, v_issued = 0;
        for (int j = 0; j < nk; ++j) {
          const int s = j % C::kStages;
          const int n = j / C::kStages;
          if (j >= C::kStages && !wait_bar(&bars->k_empty[s], (n - 1) & 1, w, 1)) break;
          const uint32_t extra = (ctl.inject == 1 && j == 0) ? 16u : 0u;  // test-only: never completes
          int krow = stream_tile(j) * kBN;
#ifdef FA_DEBUG
          if (ctl.inject == 2 && j == 0) krow += a.N;  // test-only: a key row the check must refuse
#endif
          const bool kv_ok = fa_dbg(krow >= 0 && krow < a.N && hk < a.Hkv && b < a.B, ctl.status, 0x02);
          mbar_arrive_expect_tx(&bars->k_full[s], C::kTileBytes + extra);
          for (int c = 0; kv_ok && c < C::kSub; ++c)
            tma_load_4d(smem + C::kOffK + s * C::kTileBytes + c * C::kSubBytes, &tmK, &bars->k_full[s], c * 64,
                        krow, hk, b);
          ++k_issued;
          if (j >= C::kStages && !wait_bar(&bars->v_empty[s], (n - 1) & 1, w, 2)) break;
          mbar_arrive_expect_tx(&bars->v_full[s], C::kTileBytes);
          for (int c = 0; kv_ok && c < C::kSub; ++c)
            tma_load_4d(smem + C::kOffV + s * C::kTileBytes + c * C::kSubBytes, &tmV, &bars->v_full[s], c * 64,
                        krow, hk, b);
          ++v_issued;
        }
        // teardown: no copy of this CTA may still be writing its shared memory
        drain_wait(&bars->q_full, 0, ctl.limit_ns);
        drain_ring(bars->k_full, C::kStages, k_issued, ctl.limit_ns);
        drain_ring(bars->v_full, C::kStages, v_issued, ctl.limit_ns);
      }
    } else if (warp == kMmaWarp) {
      // ===================== MMA issuer (one warp) =====================
      // The whole warp runs the loop (waits and descriptor arithmetic are
      // warp-uniform) and one lane elected by elect.sync issues each MMA and
      // commit: a lone lane-0 issuer loses its SMSP's issue slots to the
      // ALU-bound softmax warps there and starves the tensor pipe.
      {
        const uint32_t sQ = smem_u32(smem + C::kOffQ);
        const uint32_t sK = smem_u32(smem + C::kOffK);
        const uint32_t sV = smem_u32(smem + C::kOffV);
        // S_t = Q_t K^T for key tile j (K from ring stage s)
        auto issue_s = [&](int t, int s) {
          const uint32_t qa = sQ + t * C::kTileBytes;
          const uint32_t kb = sK + s * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
            umma_ss_w(tmem + C::colS(t), sw128_desc(qa + off, 16, 1024), sw128_desc(kb + off, 16, 1024),
                    C::kIdescS, kk > 0 ? 1u : 0u);
          }
          umma_commit_w(&bars->s_full[t]);
        };
        // O_t += P_t V_j (P_t from TMEM over S_t, V from ring stage s)
        auto issue_pv = [&](int t, int s, bool acc) {
          const uint32_t vb = sV + s * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            umma_ts_w(tmem + C::colO(t), tmem + C::colS(t) + kk * 8, sw128_desc(vb + kk * 2048, C::kSubBytes, 1024),
                    C::kIdescPV, (acc || kk > 0) ? 1u : 0u);
          }
          umma_commit_w(&bars->o_done[t]);
        };
        // jl[t]: how many of query tile t's key tiles have had their P V issued
        int jl[2] = {0, 0};
        // Issue order: S_0(0) S_1(0) | PV_0(j) S_0(j+1) PV_1(j) S_1(j+1) | ...
        // S_t(j+1) overwrites the columns PV_t(j) reads P_t(j) from; the tensor
        // pipe executes one thread's MMAs in issue order, so PV_t(j) has read
        // P_t(j) before S_t(j+1) writes there.  A query tile whose first key
        // tile is a later stream tile gets its first S in the iteration before.
        bool ok = nk > 0 && warp_all(wait_bar(&bars->q_full, 0, w, 3)) && warp_all(wait_bar(&bars->k_full[0], 0, w, 4));
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (uses(t, 0)) issue_s(t, 0);
          umma_commit_w(&bars->k_empty[0]);
        }
        for (int j = 0; ok && j < nk; ++j) {
          const int s = j % C::kStages;
          const int sn = (j + 1) % C::kStages;
          if (!(ok = warp_all(wait_bar(&bars->v_full[s], (j / C::kStages) & 1, w, 6)))) break;
          bool next_k = false;
          for (int t = 0; t < 2; ++t) {
            if (uses(t, j)) {
              if (!(ok = warp_all(wait_bar(&bars->p_full[t], jl[t] & 1, w, 7)))) break;
              tc_fence_after();
              issue_pv(t, s, jl[t] > 0);
              ++jl[t];
            }
            if (j + 1 < nk && uses(t, j + 1)) {
              if (!next_k) {
                if (!(ok = warp_all(wait_bar(&bars->k_full[sn], ((j + 1) / C::kStages) & 1, w, 5)))) break;
                tc_fence_after();
                next_k = true;
              }
              issue_s(t, sn);
            }
          }
          if (!ok) break;
          umma_commit_w(&bars->v_empty[s]);
          if (next_k) umma_commit_w(&bars->k_empty[sn]);
        }
        // all MMAs of this CTA finish before TMEM is released
        umma_commit_w(&bars->drain);
        drain_wait(&bars->drain, 0, ctl.limit_ns);
      }
    }
  }

  // ---- teardown ----
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, W::kTmemCols);
  }
}

}  // namespace

// One query tile per CTA (two CTAs per SM) when a query row sees 768 keys or
// fewer on average (N <= 512, causal N <= 1536, short windows): there the
// CTAs' prologues, first loads and epilogues weigh on the few key tiles each
// CTA walks, and a second CTA on the SM overlaps them.  Longer walks keep two
// tiles per CTA, which load each K/V tile once for both.  Measured on B200,
// two tiles -> one tile per CTA: causal B4 H16 N1024 d64 0.035 -> 0.031 ms,
// causal B8 H16 N1024 d128 0.071 -> 0.063, B16 H16 N512 d64 0.051 -> 0.047 and
// causal 0.047 -> 0.040; but B4 H16 N1024 d64 0.042 -> 0.044, B4 H32 N2048
// d128 0.267 -> 0.283 and B1 H32 N16384 d128 3.54 -> 4.19.
bool one_tile_per_cta(const FwdArgs& a) {
  const long long n = a.N;
  const long long left = (a.wl >= a.N) ? n - 1 : a.wl;
  const long long right = (a.wr >= a.N) ? n - 1 : a.wr;
  // keys per query row, ignoring the sequence edges (causal: half the sequence on average)
  const long long seen = a.causal ? (n + 1) / 2 : ((left + right + 1 < n) ? left + right + 1 : n);
  return seen <= 768;
}

cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                            const FwdArgs& a, const DevCtl& c, cudaStream_t s) {
  const bool sparse = a.block_mask != nullptr;
  const bool one = !sparse && one_tile_per_cta(a);
  const int rows = (one ? 1 : 2) * kBM;
  const dim3 grid((a.N + rows - 1) / rows, a.H, a.B);
  auto run = [&](auto kernel, int smem, int threads) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, threads, smem, s>>>(tq, tk, tv, to, a, c);
    return cudaGetLastError();
  };
  constexpr int k1 = FwdShape<1>::kThreads, k2 = FwdShape<2>::kThreads;
  if (a.d == 128) {
    if (sparse) return run(fwd_bf16_kernel<128, true, 2>, FwdCfg<128, 2>::kSmemBytesSparse, k2);
    return one ? run(fwd_bf16_kernel<128, false, 1>, FwdCfg<128, 1>::kSmemBytes, k1)
               : run(fwd_bf16_kernel<128, false, 2>, FwdCfg<128, 2>::kSmemBytes, k2);
  }
  if (sparse) return run(fwd_bf16_kernel<64, true, 2>, FwdCfg<64, 2>::kSmemBytesSparse, k2);
  return one ? run(fwd_bf16_kernel<64, false, 1>, FwdCfg<64, 1>::kSmemBytes, k1)
             : run(fwd_bf16_kernel<64, false, 2>, FwdCfg<64, 2>::kSmemBytes, k2);
}

}  // namespace fa
