/*
 * Exact IO-aware attention on B200 (sm_100a): the C ABI.
 *
 * What the library computes (per batch b and head h):
 *
 *     S = scale * Q K^T  (+ causal mask: key j hidden from query i when j > i)
 *     O = softmax_rows(S) V,      LSE_i = log sum_j exp(S_ij)   (natural log)
 *
 * exactly as standard attention does, without ever writing the N x N score
 * matrix to device memory.  Sources (web pages on FlashAttention, cited by
 * title and section):
 *   "Flash Attention" (karlkratz.de): "Tiling: Blockweise Berechnung im
 *     schnellen Speicher" (block-wise computation with a running maximum and
 *     sum per row), "Speicherbedarf und Laufzeitverhalten" (O(N) extra memory,
 *     exactly the same result), "Recomputation beim Rückwärtsdurchlauf"
 *     (the backward pass recomputes the attention values).
 *   "Flash Attention" (Ultralytics glossary): "Принцип работы Flash Attention"
 *     (query block resident, key/value blocks streamed, only the output and
 *     per-row statistics return to HBM; backward recomputes score blocks).
 *   "Beschleunigte Transformer: FlashAttention, effiziente Kernel und kluge
 *     Speicherlayouts": "Layout-Entscheidungen für Q, K und V" (the
 *     [batch, sequence, heads, features] layout used here).
 *
 * Conventions shared by every entry point
 *   Layout: Q, K, V, O, dO, dQ, dK, dV are dense, contiguous [B, N, H, d]
 *     tensors (element (b, n, h, k) at ((b*N + n)*H + h)*d + k) of the call's
 *     dtype.  LSE is a dense [B, H, N] fp32 tensor in natural-log units.
 *   Pointers: all tensor pointers are DEVICE pointers of the current CUDA
 *     device and must be 16-byte aligned.  The caller allocates and owns every
 *     buffer, including the backward workspace.  The library allocates no
 *     device memory, copies nothing between host and device and never
 *     synchronises, except where an entry point says so.
 *   Stream: `stream` is a cudaStream_t (NULL = the legacy default stream).
 *     All work is enqueued asynchronously on it.
 *   Sizes: B, H, N >= 0; B*H*N == 0 is a valid empty problem (returns FA_OK,
 *     writes nothing).  d must be 64 or 128.  N <= 2^22, H <= 65535,
 *     B <= 65535.
 *   Errors: every entry point returns 0 (FA_OK) or a negative FA_ERR_* code;
 *     on a validation error nothing is enqueued and no output is written.
 *     An unsupported shape is refused rather than computed wrongly (a wrongly
 *     configured block size "leads to errors": "Flash Attention"
 *     (karlkratz.de), "Grenzen und Einschränkungen").
 *   Threads: entry points are safe to call from several host threads.
 */
#ifndef EXACT_IO_AWARE_FA_H
#define EXACT_IO_AWARE_FA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of Q, K, V, O, dO, dQ, dK, dV. */
typedef enum { FA_BF16 = 0, FA_FP32 = 1 } fa_dtype;

enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1,     /* null pointer, negative size, bad scale or dtype */
  FA_ERR_UNSUPPORTED = -2,     /* d not 64/128, or a dtype/d the pass does not implement */
  FA_ERR_MISALIGNED = -3,      /* a tensor pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = -4,       /* backward workspace missing, too small or misaligned */
  FA_ERR_ARCH = -5,            /* current device is not compute capability 10.0 */
  FA_ERR_LAUNCH = -6,          /* a CUDA call failed; see fa_last_cuda_error() */
  FA_ERR_DEVICE_TIMEOUT = -7,  /* a kernel's bounded wait expired (see fa_last_device_status) */
  FA_ERR_TOO_LARGE = -8,       /* a size limit above is exceeded */
  FA_ERR_DEVICE_INPUT = -9,    /* a kernel found device-side input out of range (see fa_last_device_status) */
  FA_ERR_DEVICE_CHECK = -10    /* a debug build's device-side bounds check failed (see fa_last_device_status) */
};

/*
 * Forward pass.
 *   Q, K, V  [B, N, H, d] inputs (dtype).
 *   O        [B, N, H, d] output (dtype), written completely.
 *   LSE      [B, H, N] fp32 output, natural log of the softmax denominator
 *            of each row (the one per-row statistic the backward needs).
 *   scale    softmax scale, finite and > 0 (usually 1/sqrt(d)).
 *   causal   0 = bidirectional, 1 = key j hidden from query i when j > i.
 *   dtype    FA_BF16: tcgen05 tensor-core kernel, fp32 accumulation, O in bf16.
 *            FA_FP32: fp32 CUDA-core kernel (no TF32), O in fp32.
 * Online softmax over streamed key/value tiles ("Flash Attention" (Ultralytics
 * glossary), "Принцип работы Flash Attention"); only O and LSE reach memory.
 */
int fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
           float scale, int causal, int dtype, void* stream);

/*
 * Forward pass with grouped-query attention ("Flash Attention"
 * (karlkratz.de), "Grouped Query Attention"): Hkv key/value heads, each
 * shared by H / Hkv consecutive query heads; query head h attends with K/V
 * head h / (H / Hkv).  Hkv = H is fa_fwd; Hkv = 1 is multi-query attention.
 *   Q, O     [B, N, H, d];  K, V  [B, N, Hkv, d];  LSE  [B, H, N].
 *   Hkv      1 <= Hkv <= H and H % Hkv == 0 (FA_ERR_INVALID_ARG otherwise;
 *            Hkv = 0 only with H = 0).
 * Other arguments, results and errors as fa_fwd.
 */
int fa_fwd_gqa(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv, int N,
               int d, float scale, int causal, int dtype, void* stream);

/*
 * Forward pass with a sliding-window mask ("Flash Attention" (karlkratz.de),
 * "Sliding Window Attention": each position attends to a fixed neighbourhood,
 * and blocks outside the window are neither loaded nor computed).
 *   Key j is visible to query i when
 *     i - window_left <= j <= i + window_right   (and j < N);
 *   a bound of -1 leaves that side open.  (-1, -1) is fa_fwd_gqa without the
 *   causal mask, (-1, 0) with it; a window of W tokens ending at the query
 *   (Mistral-style) is (W - 1, 0).  Bounds below -1 are FA_ERR_INVALID_ARG.
 *   Every row sees at least its own key, so no row is empty.
 * Other arguments (grouped K/V heads included), results and errors as fa_fwd_gqa.
 */
int fa_fwd_window(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv, int N,
                  int d, float scale, int window_left, int window_right, int dtype, void* stream);

/*
 * Forward pass with a block-sparse mask ("Flash Attention" (Ultralytics
 * glossary), "Flash Attention и смежные понятия": sparse attention scores only
 * chosen query/key pairs; the block-sparse form skips empty blocks).
 *   block_mask  device array of bytes [mask_heads][nb][nb], nb = ceil(N / 128):
 *               query block i (rows 128 i .. 128 i + 127) sees key block j of
 *               query head h when block_mask[(mh * nb + i) * nb + j] != 0, with
 *               mh = 0 if mask_heads == 1 (one mask for every head), else h.
 *               Shared by every batch entry.  Must not be null.
 *   mask_heads  1 or H (FA_ERR_INVALID_ARG otherwise).
 *   window_left, window_right  as fa_fwd_window; both masks apply.
 * Key blocks a query block does not see are neither loaded nor multiplied.  A
 * row that sees no key gets O = 0 and LSE = -inf.  FA_BF16 (tensor cores) and
 * FA_FP32 (the exact fp32 kernel); nb <= 4096, i.e. N <= 524288
 * (FA_ERR_TOO_LARGE otherwise).  Other arguments as fa_fwd_window.
 */
int fa_fwd_blocksparse(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv,
                       int N, int d, float scale, int window_left, int window_right, const void* block_mask,
                       int mask_heads, int dtype, void* stream);

/*
 * Forward pass with 8-bit inputs (FP8 attention as FlashAttention-3 runs it:
 * "Flash Attention" (karlkratz.de), "Versionen").
 *   Q        [B, N, H, d] e4m3 codes (one byte each); the value is scale_q * code.
 *   K, V     [B, N, Hkv, d] e4m3 codes with scales scale_k, scale_v.
 *   O        [B, N, H, d] bf16 output; LSE [B, H, N] fp32 natural log.
 *   scale    softmax scale (finite, > 0); scale_q, scale_k, scale_v finite, > 0.
 *   Hkv, window_left, window_right as fa_fwd_window (-1, -1: no mask; -1, 0: causal).
 *   d        128 only (FA_ERR_UNSUPPORTED otherwise).
 * S = Q K^T accumulates the 8-bit products in fp32 on the tensor cores; the
 * probabilities are rounded to e4m3 (after scaling by 2^4, so the largest is at
 * most 256) before P V, and the row sums use the unrounded fp32 values.  The
 * result is the exact attention of the dequantised inputs up to those
 * roundings (see the design notes for the bound the tests use).
 */
int fa_fwd_fp8(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv, int N,
               int d, float scale, float scale_q, float scale_k, float scale_v, int window_left, int window_right,
               void* stream);

/*
 * The 8-bit forward under a block-sparse mask: block_mask and mask_heads as
 * fa_fwd_blocksparse (NULL: no mask, which is fa_fwd_fp8), the other arguments
 * as fa_fwd_fp8.  Key blocks a query block does not see are neither loaded nor
 * multiplied; a row that sees no key gets O = 0 and LSE = -inf.
 */
int fa_fwd_fp8_blocksparse(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv,
                           int N, int d, float scale, float scale_q, float scale_k, float scale_v, int window_left,
                           int window_right, const void* block_mask, int mask_heads, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for this problem: an fp32 dQ
 * accumulator [B, N, H, d] plus two fp32 [B, H, roundup(N, 128)] rows
 * (rowsum(dO * O) and LSE * log2 e), each region 256-byte aligned.  This is
 * the O(N) extra memory of the method ("Flash Attention" (karlkratz.de),
 * "Speicherbedarf und Laufzeitverhalten").
 * For small problems (fewer than three waves of key-tile CTAs on the GPU's 148
 * SMs) the size also covers two fp32 [B, N, Hkv, d] dK / dV accumulators: with
 * them the backward splits each key tile's work over several CTAs and sums
 * their partial dK, dV.  A workspace of only the first three regions is still
 * accepted (no split).  Returns 0 for invalid or empty problems.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d, int dtype);

/* The same for Hkv K/V heads (fa_bwd_gqa, fa_bwd_window, fa_bwd_blocksparse). */
size_t fa_bwd_workspace_size_gqa(int B, int H, int Hkv, int N, int d, int dtype);

/*
 * Backward pass by recomputation ("Flash Attention" (karlkratz.de),
 * "Recomputation beim Rückwärtsdurchlauf"): score tiles are rebuilt from Q, K
 * and the saved LSE, and
 *   dV = P^T dO, dP = dO V^T, D_i = sum_k dO_ik O_ik, dS = P * (dP - D),
 *   dQ = scale * dS K, dK = scale * dS^T Q.
 *   Q, K, V, O, dO  [B, N, H, d] inputs; O and LSE as written by fa_fwd.
 *   dQ, dK, dV      [B, N, H, d] outputs, written completely.
 *   workspace       device buffer of at least fa_bwd_workspace_size() bytes,
 *                   256-byte aligned; overwritten.
 * dtype FA_BF16 with d = 64 or 128 (FA_ERR_UNSUPPORTED for FA_FP32).
 * dQ is summed over key tiles by fp32 reduce-adds in L2 whose order varies
 * from run to run, so it is not bitwise deterministic.
 */
int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE, void* dQ,
           void* dK, void* dV, int B, int H, int N, int d, float scale, int causal, int dtype, void* workspace,
           size_t workspace_bytes, void* stream);

/*
 * Backward pass with grouped-query attention (see fa_fwd_gqa).  The gradient
 * of a shared K/V head is the sum over its H / Hkv query heads:
 *   dK[:, :, g] = sum over h in group g of scale * dS_h^T Q_h,
 *   dV[:, :, g] = sum over h in group g of P_h^T dO_h,
 * accumulated in fp32 inside one CTA per (key tile, K/V head) and written once.
 *   Q, O, dO, dQ  [B, N, H, d];  K, V, dK, dV  [B, N, Hkv, d];  LSE  [B, H, N].
 *   workspace     as fa_bwd: fa_bwd_workspace_size(B, H, N, d, dtype) bytes
 *                 (it depends on the query heads only).
 * Other arguments, results and errors as fa_bwd.
 */
int fa_bwd_gqa(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
               void* dQ, void* dK, void* dV, int B, int H, int Hkv, int N, int d, float scale, int causal, int dtype,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass under the sliding-window mask of fa_fwd_window (same
 * window_left / window_right meaning); the forward's O and LSE must come from
 * the same window.  Each key tile visits only the query tiles inside its
 * window.  Other arguments, results and errors as fa_bwd_gqa.
 */
int fa_bwd_window(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                  void* dQ, void* dK, void* dV, int B, int H, int Hkv, int N, int d, float scale, int window_left,
                  int window_right, int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass under the block-sparse mask of fa_fwd_blocksparse (same mask,
 * window and heads as the forward that produced O and LSE).  Each key block
 * visits only the query blocks that see it; a key that no query sees gets
 * dK = dV = 0.  Other arguments, results and errors as fa_bwd_window.
 */
int fa_bwd_blocksparse(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                       const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int Hkv, int N, int d,
                       float scale, int window_left, int window_right, const void* block_mask, int mask_heads,
                       int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd for callers that cannot allocate device memory when they run the
 * backward pass (runtimes whose device memory is laid out once at start-up,
 * or code that must not call cudaMalloc mid-run because it can synchronise
 * the device or fail under memory pressure).  The pages have no counterpart
 * to this entry point; it is a service of this library.
 *   Same arguments and results as fa_bwd, minus the workspace: the scratch is
 *   a 64 MiB array compiled into the library, which every GPU that loads the
 *   library holds until the process exits.  The call allocates nothing.
 *   A problem whose base workspace (the fp32 dQ accumulator and the two
 *   per-row arrays, i.e. fa_bwd_workspace_size() without the split-walk dK /
 *   dV accumulators) exceeds 64 MiB is refused with FA_ERR_TOO_LARGE.  When
 *   the base fits but the split-walk accumulators do not, the walks run
 *   unsplit: the same gradients, without the small-grid speed-up.
 *   All calls share that one array.  Each call's first kernel rewrites what
 *   the later ones read, so results never depend on an earlier call, but
 *   calls whose kernels overlap on the GPU (other streams, or other host
 *   threads without ordering) race on it and give wrong gradients.
 *   The first call on a device looks up the array's device address with that
 *   device current; make it before any stream capture.
 */
int fa_bwd_static_scratch(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                          const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d, float scale,
                          int causal, int dtype, void* stream);

/*
 * Helpers for attention over a sequence split into chunks, as ring attention
 * runs it ("Flash Attention" (Ultralytics glossary), "Flash Attention и
 * смежные понятия": each device computes blockwise attention for its part of
 * the sequence while the key/value blocks travel around a ring of devices).
 *
 * fa_merge_partial: combine a query chunk's running result with the partial
 * result of one more key chunk.  Each partial is exact attention over its keys
 * (as fa_fwd returns it), so with m = max(LSE_acc, LSE_part) and
 * w_x = exp(LSE_x - m):
 *     O_acc = (w_acc O_acc + w_part O_part) / (w_acc + w_part),
 *     LSE_acc = m + ln(w_acc + w_part)
 * (the online softmax's correction between key blocks, "Flash Attention"
 * (karlkratz.de), "Tiling").  A row where both sides saw no key stays O = 0,
 * LSE = -inf.
 *   O_acc     [B, N, H, d] fp32, in/out;  LSE_acc [B, H, N] fp32, in/out.
 *   O_part    [B, N, H, d] bf16;          LSE_part [B, H, N] fp32.
 *   O_out     [B, N, H, d] bf16 copy of the merged O, or NULL.
 *   init      nonzero: O_acc, LSE_acc := the partial (their old contents unread).
 *   d         64 or 128.
 */
int fa_merge_partial(float* O_acc, float* LSE_acc, const void* O_part, const float* LSE_part, void* O_out, int B,
                     int H, int N, int d, int init, void* stream);

/*
 * acc[i] += part[i] (fp32 += bf16) for i < n, or acc[i] = part[i] when init is
 * nonzero: the fp32 sum of one chunk's gradient contributions.  n a multiple
 * of 8, both pointers 16-byte aligned.
 */
int fa_accumulate_bf16(float* acc, const void* part, long long n, int init, void* stream);

/* out[i] = bf16(in[i]) (round to nearest even) for i < n; n a multiple of 8. */
int fa_cast_bf16(void* out, const float* in, long long n, void* stream);

/*
 * One decode step of attention over a paged KV cache ("Flash Attention"
 * (Ultralytics glossary), "Flash Attention и смежные понятия", PagedAttention:
 * the KV cache is kept in fixed-size pages and the attention kernel reads keys
 * and values from those pages).
 *   Q            [B, H, d] bf16: the one new query of each sequence.
 *   K_cache,     [num_pages, page_size, Hkv, d] bf16 page pools; position j of
 *   V_cache      sequence b is slot j % page_size of page
 *                block_table[b * max_pages + j / page_size].
 *   block_table  [B, max_pages] int32 device array of page indices; only the
 *                first ceil(seqlens[b] / page_size) entries of a row are read.
 *   seqlens      [B] int32 device array: cached positions of each sequence,
 *                0 <= seqlens[b] <= max_pages * page_size.
 *   O            [B, H, d] bf16 output;  LSE  [B, H] fp32 output (natural log).
 *   H, Hkv       query and K/V heads, H % Hkv == 0; query head h reads K/V head
 *                h / (H / Hkv) (as fa_fwd_gqa).
 *   d            64 or 128;  page_size  a power of two from 8 to 4096
 *                (FA_ERR_UNSUPPORTED otherwise).
 *   scale        softmax scale, finite and > 0.
 *   workspace    device buffer of workspace_bytes (16-byte aligned) or NULL.
 *                With at least fa_decode_workspace_size() bytes, long sequences
 *                are split into key chunks processed by separate CTAs and merged
 *                (fp32 partials); with less, the call splits no further than the
 *                buffer holds (NULL: one chunk per sequence).
 * Each query attends to all seqlens[b] cached positions (the caller appends the
 * new token's K, V before the call); a sequence with seqlens[b] == 0 gets O = 0
 * and LSE = -inf.  Q, the pools and O must be 16-byte aligned; LSE, block_table
 * and seqlens 4-byte aligned.  num_pages * page_size and max_pages * page_size
 * must stay below 2^31, B <= 65535 (FA_ERR_TOO_LARGE otherwise).  Because
 * seqlens and block_table are device data, the kernel checks them: a length
 * out of range or a page index outside [0, num_pages) leaves the affected
 * sequence's rows empty (O = 0, LSE = -inf), loads nothing from the pool, and
 * makes the next fa_last_device_status() return FA_ERR_DEVICE_INPUT.
 */
int fa_decode_paged(const void* Q, const void* K_cache, const void* V_cache, const int* block_table,
                    const int* seqlens, void* O, float* LSE, int B, int H, int Hkv, int d, int page_size,
                    int num_pages, int max_pages, float scale, void* workspace, size_t workspace_bytes,
                    void* stream);

/* Workspace bytes with which fa_decode_paged splits as it would unconstrained:
 * the fp32 partials of each key chunk (0 when one chunk suffices or the
 * arguments are invalid). */
size_t fa_decode_workspace_size(int B, int H, int Hkv, int d, int page_size, int max_pages);

/* Static English text for a status code. */
const char* fa_status_string(int status);

/* The cudaError_t of the last failed CUDA call on this host thread (0 if none);
 * 100000 + CUresult when encoding a TMA descriptor failed. */
int fa_last_cuda_error(void);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word.  Returns FA_OK if no kernel reported a problem since the last call,
 * FA_ERR_DEVICE_INPUT if a kernel found device-side input out of range
 * (fa_decode_paged), FA_ERR_DEVICE_TIMEOUT if a bounded wait expired (the
 * affected launch's outputs are then undefined), FA_ERR_DEVICE_CHECK if a
 * kernel of the checking build (libfa_debug.so, compiled with FA_DEBUG) found
 * an index, coordinate or tensor-memory column outside its buffer (it skipped
 * that access; the launch's outputs are undefined), or FA_ERR_LAUNCH.  *detail
 * (if not NULL) receives the raw word: 0x1000 | the id of the wait that
 * expired, 0x2000 | the id of the failed input check (0xD1 a sequence
 * length, 0xD2 a page index), or 0x4000 | the id of the failed bounds check.
 * The first problem recorded wins.
 */
int fa_last_device_status(void* stream, int* detail);

/*
 * Diagnostics knob (process-wide): the limit for any single wait inside a
 * kernel (default 2000 ms, or the FA_TIMEOUT_MS environment variable); after
 * it the launch gives up and reports FA_ERR_DEVICE_TIMEOUT.
 */
void fa_set_wait_limit_ms(int ms);

/*
 * Diagnostics: while set, each fa_fwd / fa_bwd call made on this host thread
 * records the cudaEvent_t `start` on its stream right before its tensor-core
 * kernel (the fused forward, or the backward main kernel) and `stop` right
 * after it, so a caller can time that one kernel with cudaEventElapsedTime.
 * Pass NULL, NULL to turn it off.  The events stay owned by the caller.
 */
void fa_set_kernel_events(void* start, void* stop);

/* Library version: major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_IO_AWARE_FA_H */
