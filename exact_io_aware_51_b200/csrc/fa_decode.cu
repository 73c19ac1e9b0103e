// One decode step of attention over a paged KV cache, bf16, sm_100a.
//
// "Flash Attention" (Ultralytics glossary), "Flash Attention и смежные
// понятия" (PagedAttention): a serving system keeps the KV cache in pages of a
// fixed size, and the attention kernel reads keys and values from those pages.
// Position j of sequence b sits in slot j % page_size of page
// block_table[b][j / page_size]; the new query of each sequence attends to all
// seqlens[b] cached positions.  The arithmetic is the forward's online
// softmax ("Flash Attention" (karlkratz.de), "Tiling"): running row maximum
// and sum, the partial output rescaled when the maximum grows.
//
// The step is HBM-bound: each cached K/V row is read once per (sequence, K/V
// head) and feeds only H / Hkv query heads, 2 FLOP per byte at 8 heads.  The
// kernel is built around moving those bytes:
//   * grid (K/V head x head group, sequence, chunk); a CTA takes up to 16 query
//     heads of one K/V head and one chunk of the sequence's keys (long
//     sequences split into several chunks so small batches still fill the GPU);
//   * one producer thread walks the chunk 64 keys at a time and, per page
//     touched, issues 2-D TMA loads of the page's rows of this K/V head
//     (128-byte swizzle) into a 3- or 4-stage ring, completion on mbarriers;
//   * four consumer warps each take 16 keys of a tile.  The per-key
//     contraction is tiny (16 heads x d), so it runs on warp-level
//     mma.sync m16n8k16 (bf16 in, fp32 accumulate) straight from registers:
//     S = Q K^T with the query heads as the 16 rows, P = 2^(S*scale*log2e - m)
//     built in registers and reused as the A operand of O += P V (V read with
//     ldmatrix.trans).  No tensor-memory round trip, no block-wide sync per tile;
//   * each warp keeps its own running maximum, sum and output; the four are
//     merged through shared memory at the end of the chunk;
//   * keys past the sequence's end in its last tile get score -inf and their V
//     rows are zeroed in shared memory before the PV product, so whatever the
//     pool holds there (stale or non-finite) never reaches the output.
// With one chunk the kernel writes O (bf16) and LSE; with several it writes
// fp32 partials that decode_combine_kernel merges like ring-attention
// partials (LSE-weighted).
//
// Device-side data is checked before use: a sequence length outside
// [0, max_pages * page_size] or a page index outside [0, num_pages) sets the
// status word (kDevBadInput) and the affected CTA loads nothing and writes an
// empty result (O = 0, LSE = -inf).
#include <cuda_bf16.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kTileKeys = 64;               // keys per pipeline stage
constexpr int kHalfBytes = kTileKeys * 128;  // 64 keys x 64 features bf16
constexpr int kConsumers = 4;                // warps, 16 keys of each tile each
constexpr int kThreads = (kConsumers + 1) * 32;

template <int D>
struct DecCfg {
  static constexpr int kTileBytes = (D / 64) * kHalfBytes;  // K or V of one tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kOffML = kOffBar + 128;               // [2][4 warps][16 rows] fp32 max, sum
  static constexpr int kSmemBytes = kOffML + 2 * kConsumers * 16 * 4;
  static constexpr int kORow = D + 4;                        // merge buffer row stride (floats)
  static_assert(kConsumers * 16 * kORow * 4 <= kOffBar, "merge buffer fits in the stages");
};

struct DecBars {
  uint64_t full[4], empty[4];
  int bad;
};
static_assert(DecCfg<64>::kStages <= 4 && DecCfg<128>::kStages <= 4 && sizeof(DecBars) <= 128, "barrier block");

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// c += a b, m16n8k16, bf16 inputs, fp32 accumulate
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void named_sync_consumers() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
}

// Byte offset, inside one K or V tile, of the 16-byte unit `chunk` (8 features)
// of tile row `key`: halves of 64 features, each [64 rows][128 B] with the
// 128-byte swizzle the TMA applied.
__device__ __forceinline__ uint32_t tile_off(int key, int chunk) {
  return static_cast<uint32_t>((chunk >> 3) * kHalfBytes + key * 128 + (((chunk & 7) ^ (key & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const DecodeArgs a,
                  const DevCtl ctl) {
  using C = DecCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicCAS(ctl.status, 0, kDevTimeout | 0xC0);
    return;
  }
  DecBars* bars = reinterpret_cast<DecBars*>(smem + C::kOffBar);
  const int warp = warp_id();
  const int lane = lane_id();
  // chunk index slowest: the first CTAs to run take every sequence's first
  // chunk, the later ones the (shorter, often empty) chunks further out
  const int split = blockIdx.z;
  const int hkv = blockIdx.x / a.hgroups;
  const int hg = blockIdx.x % a.hgroups;
  const int b = blockIdx.y;
  const int G = a.H / a.Hkv;
  const int h0 = hkv * G + hg * 16;      // first query head of this CTA
  const int gv = min(16, G - hg * 16);   // query heads of this CTA
  const int P = a.page_size;
  const int* table = a.block_table + static_cast<size_t>(b) * a.max_pages;

  // ---- this CTA's keys [kbeg, kend), checked against the pool ----
  const int L = a.seqlens[b];
  const bool bad_len = L < 0 || L > a.max_pages * P;  // max_pages * P < 2^31 (host check)
  const int kbeg = split * a.chunk;
  int kend = bad_len ? kbeg : min(kbeg + a.chunk, L);
  if (threadIdx.x == 0) {
    bars->bad = bad_len ? 1 : 0;
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], kConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (kend > kbeg) {
    for (int p = kbeg / P + static_cast<int>(threadIdx.x); p <= (kend - 1) / P; p += kThreads) {
      const int pg = table[p];
      if (pg < 0 || pg >= a.num_pages) bars->bad = 1;
    }
  }
  __syncthreads();
  if (bars->bad) {
    if (threadIdx.x == 0) atomicCAS(ctl.status, 0, kDevBadInput | (bad_len ? 0xD1 : 0xD2));
    kend = kbeg;
  }
  const int ntiles = (kend > kbeg) ? (kend - kbeg + kTileKeys - 1) / kTileKeys : 0;
  volatile int abort_flag = 0;
  const WaitCtl w{&abort_flag, ctl.status, ctl.abort_epoch, ctl.epoch, ctl.limit_ns};

  if (warp == kConsumers) {
    // ===================== TMA producer =====================
    if (lane == 0 && ntiles > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int R = min(P, kTileKeys);  // rows per box (the maps' box height)
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % C::kStages;
        if (t >= C::kStages && !wait_bar(&bars->empty[st], ((t / C::kStages) - 1) & 1, w, 0xC1)) break;
        const int key0 = kbeg + t * kTileKeys;
        const int nval = min(kTileKeys, kend - key0);
        const int nbox = (nval + R - 1) / R;
        uint8_t* ks = smem + st * C::kStageBytes;
        uint8_t* vs = ks + C::kTileBytes;
        mbar_arrive_expect_tx(&bars->full[st], static_cast<uint32_t>(nbox * R * 128 * (D / 64) * 2));
        for (int bx = 0; bx < nbox; ++bx) {
          const int j = key0 + bx * R;  // first key of the box; the box stays inside one page
          const int row = table[j / P] * P + j % P;
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf) {
            tma_load_2d(ks + hf * kHalfBytes + bx * R * 128, &tmK, &bars->full[st], hkv * D + hf * 64, row);
            tma_load_2d(vs + hf * kHalfBytes + bx * R * 128, &tmV, &bars->full[st], hkv * D + hf * 64, row);
          }
        }
        ++issued;
      }
      // no copy of this CTA may still be writing its shared memory when it exits
      drain_ring(bars->full, C::kStages, issued, ctl.limit_ns);
    }
    return;  // the consumers' merge below syncs only the four consumer warps
  }

  // ===================== consumers =====================
  const int g = lane >> 2;  // fragment row group: query heads g and g + 8
  const int t4 = lane & 3;
  // Q as the A operand (16 heads x d), rows past this CTA's heads are zero
  uint32_t qa[D / 16][4];
  {
    const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(a.Q) + (static_cast<size_t>(b) * a.H + h0) * D;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int c0 = ks * 16 + 2 * t4;
      qa[ks][0] = (g < gv) ? *reinterpret_cast<const uint32_t*>(qb + g * D + c0) : 0u;
      qa[ks][1] = (g + 8 < gv) ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + c0) : 0u;
      qa[ks][2] = (g < gv) ? *reinterpret_cast<const uint32_t*>(qb + g * D + c0 + 8) : 0u;
      qa[ks][3] = (g + 8 < gv) ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + c0 + 8) : 0u;
    }
  }
  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY;  // running maxima (log2 units) of rows g, g + 8
  float l0 = 0.f, l1 = 0.f;              // this thread's share of the running sums
  const float sl2 = a.scale_log2;
  const int kw = warp * 16;              // this warp's 16 keys of every tile
  const int mi = lane >> 3, rr = lane & 7;

  for (int t = 0; t < ntiles; ++t) {
    const int st = t % C::kStages;
    if (!__all_sync(0xffffffffu, wait_bar(&bars->full[st], (t / C::kStages) & 1, w, 0xC2))) break;
    const int nval = min(kTileKeys, kend - (kbeg + t * kTileKeys));
    const uint32_t ks = smem_u32(smem + st * C::kStageBytes);
    const uint32_t vs = ks + C::kTileBytes;

    // S = Q K^T for this warp's 16 keys (two n-tiles of 8)
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t kb[4];
      ldsm_x4(ks + tile_off(kw + (mi >> 1) * 8 + rr, 2 * kk + (mi & 1)), kb);
      mma_bf16(s[0], qa[kk], kb[0], kb[1]);
      mma_bf16(s[1], qa[kk], kb[2], kb[3]);
    }
    // scores in log2 units; keys past the end of the sequence are hidden
    float x[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int key = kw + n * 8 + 2 * t4 + (i & 1);
        x[n][i] = (key < nval) ? s[n][i] * sl2 : -INFINITY;
      }
    float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
    float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    const float al0 = (n0 == -INFINITY) ? 1.f : ex2(m0 - n0);
    const float al1 = (n1 == -INFINITY) ? 1.f : ex2(m1 - n1);
    m0 = n0;
    m1 = n1;
    const float b0 = (n0 == -INFINITY) ? 0.f : n0;
    const float b1 = (n1 == -INFINITY) ? 0.f : n1;
    float p[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      p[n][0] = ex2(x[n][0] - b0);
      p[n][1] = ex2(x[n][1] - b0);
      p[n][2] = ex2(x[n][2] - b1);
      p[n][3] = ex2(x[n][3] - b1);
    }
    l0 = l0 * al0 + (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
    l1 = l1 * al1 + (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
    if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        o[j][0] *= al0;
        o[j][1] *= al0;
        o[j][2] *= al1;
        o[j][3] *= al1;
      }
    }
    const uint32_t pa[4] = {pack_bf16x2(p[0][0], p[0][1]), pack_bf16x2(p[0][2], p[0][3]),
                            pack_bf16x2(p[1][0], p[1][1]), pack_bf16x2(p[1][2], p[1][3])};
    // the last tile: zero this warp's V rows past the end (P is 0 there, but
    // 0 * a non-finite leftover would not be)
    const bool zeroed = kw + 16 > nval;
    if (zeroed) {
      for (int idx = lane; idx < 16 * (D / 8); idx += 32) {
        const int key = kw + idx / (D / 8);
        if (key >= nval) st_shared_v4(vs + tile_off(key, idx % (D / 8)), 0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }
    // O += P V: two 8-feature n-tiles per ldmatrix.trans
#pragma unroll
    for (int jj = 0; jj < D / 16; ++jj) {
      uint32_t vb[4];
      ldsm_x4_trans(vs + tile_off(kw + (mi & 1) * 8 + rr, 2 * jj + (mi >> 1)), vb);
      mma_bf16(o[2 * jj], pa, vb[0], vb[1]);
      mma_bf16(o[2 * jj + 1], pa, vb[2], vb[3]);
    }
    if (zeroed) fence_proxy_async_smem();  // the next TMA write of the stage follows these stores
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->empty[st]);
  }

  // ---- merge the four warps' (max, sum, output) ----
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* mw = reinterpret_cast<float*>(smem + C::kOffML);  // [4][16]
  float* lw = mw + kConsumers * 16;                       // [4][16]
  named_sync_consumers();  // every warp is done reading the stages
  if (t4 == 0) {
    mw[warp * 16 + g] = m0;
    mw[warp * 16 + g + 8] = m1;
    lw[warp * 16 + g] = l0;
    lw[warp * 16 + g + 8] = l1;
  }
  named_sync_consumers();
  auto row_max = [&](int row) {
    float mm = -INFINITY;
#pragma unroll
    for (int u = 0; u < kConsumers; ++u) mm = fmaxf(mm, mw[u * 16 + row]);
    return mm;
  };
  {
    const float M0 = row_max(g), M1 = row_max(g + 8);
    const float f0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M0);
    const float f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M1);
    float* ob = reinterpret_cast<float*>(smem) + warp * 16 * C::kORow;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      *reinterpret_cast<float2*>(ob + g * C::kORow + j * 8 + 2 * t4) = make_float2(o[j][0] * f0, o[j][1] * f0);
      *reinterpret_cast<float2*>(ob + (g + 8) * C::kORow + j * 8 + 2 * t4) = make_float2(o[j][2] * f1, o[j][3] * f1);
    }
  }
  named_sync_consumers();
  {
    const int tid = threadIdx.x;           // 0..127
    const int row = tid >> 3;              // query head row 0..15
    const int c0 = (tid & 7) * (D / 8);    // D / 8 features per thread
    if (row < gv) {
      const float M = row_max(row);
      float Lsum = 0.f;
#pragma unroll
      for (int u = 0; u < kConsumers; ++u) {
        const float mu = mw[u * 16 + row];
        if (mu != -INFINITY) Lsum += lw[u * 16 + row] * ex2(mu - M);
      }
      const float inv = (Lsum > 0.f) ? 1.f / Lsum : 0.f;
      const float lse = (Lsum > 0.f) ? (M + __log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
      float acc[D / 8];
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        float sum = 0.f;
#pragma unroll
        for (int u = 0; u < kConsumers; ++u) sum += reinterpret_cast<const float*>(smem)[(u * 16 + row) * C::kORow + c0 + c];
        acc[c] = sum * inv;
      }
      const int hq = h0 + row;
      if (a.splits == 1) {
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.O) + (static_cast<size_t>(b) * a.H + hq) * D + c0;
#pragma unroll
        for (int c = 0; c < D / 8; c += 8)
          st_global_v4(orow + c, pack_bf16x2(acc[c], acc[c + 1]), pack_bf16x2(acc[c + 2], acc[c + 3]),
                       pack_bf16x2(acc[c + 4], acc[c + 5]), pack_bf16x2(acc[c + 6], acc[c + 7]));
        if ((tid & 7) == 0) a.LSE[static_cast<size_t>(b) * a.H + hq] = lse;
      } else {
        const size_t ri = (static_cast<size_t>(split) * a.B + b) * a.H + hq;
        float* orow = a.Opart + ri * D + c0;
#pragma unroll
        for (int c = 0; c < D / 8; c += 4)
          *reinterpret_cast<float4*>(orow + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
        if ((tid & 7) == 0) a.LSEpart[ri] = lse;
      }
    }
  }
}

// Merge of the chunks' partial results, one CTA of four warps per (sequence,
// query head): with M = max_s LSE_s and w_s = exp(LSE_s - M),
//   O = sum_s w_s O_s / sum_s w_s,   LSE = M + ln sum_s w_s.
// The chunks are spread over the four warps (warp u takes s = u, u + 4, ...) and
// the loads of a warp's chunks are independent, so a long sequence's many
// partials are read with several loads in flight instead of one at a time.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeArgs a) {
  constexpr int kPer = D / 32;
  const long long rows = static_cast<long long>(a.B) * a.H;
  const long long row = blockIdx.x;
  const int warp = warp_id(), lane = lane_id();
  __shared__ float s_max[4], s_w[4];
  __shared__ float s_acc[4][D];
  float M = -INFINITY;
  for (int s = static_cast<int>(threadIdx.x); s < a.splits; s += 128) M = fmaxf(M, a.LSEpart[s * rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) s_max[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3]));
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int s = warp; s < a.splits; s += 4) {
      const float ls = a.LSEpart[s * rows + row];
      const float wgt = (ls == -INFINITY) ? 0.f : expf(ls - M);
      const float* op = a.Opart + (s * rows + row) * D + lane * kPer;
      float v[kPer];
      if constexpr (kPer == 4) {
        const float4 x = *reinterpret_cast<const float4*>(op);
        v[0] = x.x;
        v[1] = x.y;
        v[2] = x.z;
        v[3] = x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(op);
        v[0] = x.x;
        v[1] = x.y;
      }
      wsum += wgt;
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] += wgt * v[i];
    }
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) s_acc[warp][lane * kPer + i] = acc[i];
  if (lane == 0) s_w[warp] = wsum;
  __syncthreads();
  if (warp == 0) {
    const float W = (s_w[0] + s_w[1]) + (s_w[2] + s_w[3]);
    const float inv = (W > 0.f) ? 1.f / W : 0.f;
    float out[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int c = lane * kPer + i;
      out[i] = ((s_acc[0][c] + s_acc[1][c]) + (s_acc[2][c] + s_acc[3][c])) * inv;
    }
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.O) + row * D + lane * kPer;
    if constexpr (kPer == 4) {
      uint2 u;
      u.x = pack_bf16x2(out[0], out[1]);
      u.y = pack_bf16x2(out[2], out[3]);
      *reinterpret_cast<uint2*>(orow) = u;
    } else {
      *reinterpret_cast<uint32_t*>(orow) = pack_bf16x2(out[0], out[1]);
    }
    if (lane == 0) a.LSE[row] = (W > 0.f) ? M + logf(W) : -INFINITY;
  }
}

template <int D>
cudaError_t launch_decode_d(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, const DevCtl& c,
                            cudaStream_t s) {
  using C = DecCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.Hkv * a.hgroups, a.B, a.splits);
  decode_kernel<D><<<grid, kThreads, C::kSmemBytes, s>>>(tk, tv, a, c);
  if ((e = cudaGetLastError()) != cudaSuccess || a.splits == 1) return e;
  const long long rows = static_cast<long long>(a.B) * a.H;
  decode_combine_kernel<D><<<static_cast<unsigned>(rows), 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, const DevCtl& c,
                          cudaStream_t s) {
  if (a.d == 128) return launch_decode_d<128>(tk, tv, a, c, s);
  if (a.d == 64) return launch_decode_d<64>(tk, tv, a, c, s);
  return cudaErrorInvalidValue;
}

}  // namespace fa
