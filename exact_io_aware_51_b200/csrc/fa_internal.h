// Internal (not exported) declarations shared by the host library and the
// kernel translation units.  Nothing here is part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

// Device-side error reporting for one launch.
struct DevCtl {
  int* status;                  // device status word (0 = ok)
  unsigned int* abort_epoch;    // epoch of the last launch that hit a wait limit
  unsigned int epoch;           // epoch of this launch
  unsigned long long limit_ns;  // limit for any single wait
  int inject;                   // test-only fault injection (0 = off)
};

// Visibility mask of every pass: key k is visible to query q when
// q - wl <= k <= q + wr and k < N (wl, wr >= 0; a value >= N leaves that side
// unbounded).  (wl, wr) = (N, N) is unmasked attention, (N, 0) causal, and a
// finite wl a sliding window.  `causal` is set exactly for (N, 0); it only
// selects the order in which CTAs take their tiles.
struct FwdArgs {
  int B, H, N, d;
  int Hkv;           // K/V heads; query head h reads K/V head h / (H / Hkv)
  float scale_log2;  // softmax scale * log2(e)
  int causal;
  int wl, wr;        // window (see above)
  void* O;           // [B, N, H, d]
  float* LSE;        // [B, H, N], natural log
  // Block-sparse mask (nullptr: none): [mask_heads][nb][nb] bytes, nb = ceil(N / 128);
  // query tile i sees key tile j of query head h when mask[(mh * nb + i) * nb + j] != 0
  // with mh = (mask_heads == 1 ? 0 : h).
  const uint8_t* block_mask;
  int mask_heads, nb;
};

// Largest key-tile count (ceil(N / 128)) the block-sparse kernels accept.
constexpr int kMaxSparseTiles = 4096;

struct BwdArgs {
  int B, H, N, d, Npad;
  int Hkv;           // K/V heads (dK, dV are [B, N, Hkv, d])
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  int causal;
  int wl, wr;        // window (see FwdArgs)
  const void* O;
  const void* dO;
  const float* LSE;  // [B, H, N] natural log
  void* dQ;
  void* dK;
  void* dV;
  float* dQacc;      // [B, N, H, d] fp32 workspace
  float* Dvec;       // [B, H, Npad] rowsum(dO * O)
  float* LSE2;       // [B, H, Npad] LSE * log2(e)
  const uint8_t* block_mask;  // as in FwdArgs (nullptr: none)
  int mask_heads, nb;
  // Split of each key tile's (query head, query tile) walk over `splits` CTAs
  // (small grids): with splits > 1 the CTAs add their dK, dV partial sums into
  // these fp32 [B, N, Hkv, d] accumulators (zeroed first) instead of writing dK, dV.
  int splits;
  float* dKacc;
  float* dVacc;
};

// Bytes of backward workspace a call cannot do without (dQ accumulator and the two
// per-row arrays); the public size functions may add the split accumulators.
size_t bwd_workspace_base(int B, int H, int N, int d, int dtype);

// TMA descriptor for a [B, N, H, d] bf16 tensor with a box of `rows` sequence
// positions x 64 features of one (b, h); 128-byte swizzle.
CUresult make_tile_map(CUtensorMap* map, const void* base, int B, int N, int H, int d, int rows);

// TMA descriptor for a [B, N, H, d] e4m3 (byte) tensor with d = 128: a box of
// `rows` sequence positions x 128 features of one (b, h), 128-byte swizzle.
CUresult make_tile_map_e4m3(CUtensorMap* map, const void* base, int B, int N, int H, int d, int rows);

// TMA descriptor for the fp32 [B, N, H, d] dQ accumulator with a box of 64
// sequence positions x d features of one (b, h), no swizzle (for TMA reduce-add).
CUresult make_dq_accum_map(CUtensorMap* map, float* base, int B, int N, int H, int d);

// TMA descriptor for the fp32 dQ accumulator as the d = 64 backward adds into it:
// a box of 32 features x 128 sequence positions of one (b, h), 128-byte swizzle.
CUresult make_dq_accum_map_sw128(CUtensorMap* map, float* base, int B, int N, int H, int d);

// Status-word bit a kernel sets when device-side input data (a sequence length
// or a page index) is out of range; the low bits name the check.
constexpr int kDevBadInput = 0x2000;
constexpr int kDevCheck = 0x4000;    // | check id: a bounds check of the FA_DEBUG build failed

// Bounds and alignment checks of the checking build (compiled with FA_DEBUG):
// fa_dbg(cond, status, id) is true when the access may go ahead; when cond is
// false it records kDevCheck | id in the status word (first problem wins) and
// the caller skips the access, so nothing traps or faults.  Without FA_DEBUG
// it is the constant true and costs nothing.
#ifdef FA_DEBUG
__device__ __forceinline__ bool fa_dbg(bool cond, int* status, int id) {
  if (!cond) atomicCAS(status, 0, kDevCheck | id);
  return cond;
}
#else
__device__ __forceinline__ constexpr bool fa_dbg(bool, int*, int) { return true; }
#endif

// One decode step over a paged KV cache: Q [B, H, d] (one query per sequence),
// K, V pools [num_pages, page_size, Hkv, d], block_table [B, max_pages],
// seqlens [B]; both int32 arrays live on the device.
struct DecodeArgs {
  int B, H, Hkv, d;
  int page_size, num_pages, max_pages;
  int hgroups;       // CTAs per K/V head: ceil((H / Hkv) / 16) groups of <= 16 query heads
  int splits;        // key chunks per (sequence, head group)
  int chunk;         // keys per chunk (a multiple of 64)
  float scale_log2;  // softmax scale * log2(e)
  const void* Q;
  const int* block_table;
  const int* seqlens;
  void* O;           // [B, H, d] bf16
  float* LSE;        // [B, H] natural log
  float* Opart;      // splits > 1: [splits, B, H, d] fp32, normalised per chunk
  float* LSEpart;    // splits > 1: [splits, B, H] natural log (-inf: no key in the chunk)
};

// TMA descriptor for a paged K or V pool [num_pages, page_size, Hkv, d] bf16 viewed
// as [num_pages * page_size rows][Hkv * d]: a box of min(page_size, 64) rows x 64
// features, 128-byte swizzle.
CUresult make_paged_map(CUtensorMap* map, const void* base, int num_pages, int page_size, int Hkv, int d);
cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, const DevCtl& c,
                          cudaStream_t s);

// Kernel launchers (each returns the cudaError_t of the launch).
cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const FwdArgs& a, const DevCtl& c, cudaStream_t s);
cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                           float out_scale, const DevCtl& c, cudaStream_t s);
cudaError_t launch_fwd_f32(const float* Q, const float* K, const float* V, const FwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_pre(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_main(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdq, const CUtensorMap& tdk,
                            const CUtensorMap& tdv, const BwdArgs& a, const DevCtl& c, cudaStream_t s);
// zero the split accumulators before, and write bf16 dK (x scale), dV from them after, the main kernel
cudaError_t launch_bwd_kv_zero(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_kv_convert(const BwdArgs& a, cudaStream_t s);
// TMA descriptor for an fp32 [B, N, Hkv, d] dK / dV accumulator: a box of d features x
// 64 (d = 128) or 128 (d = 64) keys of one (b, head), no swizzle (for TMA reduce-add).
CUresult make_kv_accum_map(CUtensorMap* map, float* base, int B, int N, int Hkv, int d);
cudaError_t launch_bwd_main64(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& tdo, const CUtensorMap& tdq, const CUtensorMap& tdk,
                              const CUtensorMap& tdv, const BwdArgs& a, const DevCtl& c, cudaStream_t s);
cudaError_t launch_bwd_dq(const BwdArgs& a, cudaStream_t s);

// Chunked-sequence (ring) helpers: merge of partial results, fp32 accumulation, cast.
cudaError_t launch_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                         int H, int N, int d, int init, cudaStream_t s);
cudaError_t launch_accumulate(float* acc, const void* part, long long n, int init, cudaStream_t s);
cudaError_t launch_cast(void* out, const float* in, long long n, cudaStream_t s);

}  // namespace fa
