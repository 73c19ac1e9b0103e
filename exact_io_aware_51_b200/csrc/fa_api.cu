// Host side of the C ABI: argument validation, TMA descriptors, per-device
// state and kernel launches.  See include/fa.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"
#include "fa_testing.h"

namespace fa {

// Device status word and the epoch of the last launch that hit a wait limit.
__device__ int g_status;
__device__ unsigned int g_abort_epoch;

namespace {

constexpr int kMaxDevices = 64;
constexpr long long kMaxN = 1LL << 22;

thread_local int t_last_cuda_error = 0;
thread_local int t_bound_device = -1;  // device whose primary context this thread has made current
thread_local cudaEvent_t t_ev_start = nullptr;
thread_local cudaEvent_t t_ev_stop = nullptr;
std::atomic<unsigned int> g_epoch{1};
std::atomic<unsigned long long> g_limit_ns{0};
std::atomic<int> g_inject{0};

struct DeviceState {
  std::once_flag once;
  int arch_ok = 0;
  int init_err = 0;
  int* status = nullptr;
  unsigned int* abort_epoch = nullptr;
};
DeviceState g_dev[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

unsigned long long wait_limit_ns() {
  unsigned long long v = g_limit_ns.load();
  if (v == 0) {
    const char* e = std::getenv("FA_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 2000;
    if (ms <= 0) ms = 2000;
    v = static_cast<unsigned long long>(ms) * 1000000ull;
    g_limit_ns.store(v);
  }
  return v;
}

int fail_cuda(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return FA_ERR_LAUNCH;
}

// A failed TMA descriptor encode is reported as 100000 + the CUresult.
int fail_encode(CUresult r) {
  t_last_cuda_error = 100000 + static_cast<int>(r);
  return FA_ERR_LAUNCH;
}

// Per-device one-time set-up: architecture check and the device addresses of
// the status word and abort epoch (done with that device current).
int device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_ARCH;
  // A thread that has not yet made a CUDA runtime call that needs a context
  // (for example an autograd worker thread) has none current; the driver's TMA
  // descriptor encoder needs one, so bind the device's primary context once.
  if (t_bound_device != dev) {
    e = cudaSetDevice(dev);
    if (e != cudaSuccess) return fail_cuda(e);
    t_bound_device = dev;
  }
  DeviceState& st = g_dev[dev];
  std::call_once(st.once, [&] {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      st.init_err = FA_ERR_ARCH;
      return;
    }
    st.arch_ok = (major == 10 && minor == 0);
    void* p = nullptr;
    cudaError_t e1 = cudaGetSymbolAddress(&p, g_status);
    if (e1 != cudaSuccess) {
      st.init_err = fail_cuda(e1);
      return;
    }
    st.status = static_cast<int*>(p);
    cudaError_t e2 = cudaGetSymbolAddress(&p, g_abort_epoch);
    if (e2 != cudaSuccess) {
      st.init_err = fail_cuda(e2);
      return;
    }
    st.abort_epoch = static_cast<unsigned int*>(p);
  });
  if (st.init_err) return st.init_err;
  if (!st.arch_ok) return FA_ERR_ARCH;
  *out = &st;
  return FA_OK;
}

DevCtl make_ctl(const DeviceState& st) {
  DevCtl c;
  c.status = st.status;
  c.abort_epoch = st.abort_epoch;
  unsigned int ep = g_epoch.fetch_add(1);
  if (ep == 0) ep = g_epoch.fetch_add(1);  // 0 never names a launch
  c.epoch = ep;
  c.limit_ns = wait_limit_ns();
  c.inject = g_inject.load();
  return c;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int check_shape(int B, int H, int N, int d, int dtype) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (N > kMaxN || H > 65535 || B > 65535) return FA_ERR_TOO_LARGE;
  const double elems = static_cast<double>(B) * N * H * d;
  if (elems >= 1099511627776.0) return FA_ERR_TOO_LARGE;  // 2^40
  return FA_OK;
}

// K/V heads: each of the Hkv heads serves H / Hkv query heads.
int check_kv_heads(int H, int Hkv) {
  if (Hkv < 0 || Hkv > H) return FA_ERR_INVALID_ARG;
  if (H > 0 && (Hkv == 0 || H % Hkv != 0)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// Window bounds: -1 leaves a side unbounded, otherwise 0 <= bound.
int check_window(int left, int right) {
  if (left < -1 || right < -1) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// Kernel form of a window: a side with no bound gets kUnbounded, which is
// above any sequence length the library accepts, so q - wl and q + wr never
// clip a visible key and never overflow an int.
constexpr int kUnbounded = 1 << 30;
static_assert(kMaxN < kUnbounded / 2, "window sentinel must exceed every sequence length");

void set_window(int left, int right, int* wl, int* wr, int* causal) {
  // a bound at or above the longest sequence hides nothing: same as no bound
  *wl = (left < 0 || left >= kMaxN) ? kUnbounded : left;
  *wr = (right < 0 || right >= kMaxN) ? kUnbounded : right;
  *causal = (*wl == kUnbounded && *wr == 0) ? 1 : 0;
}

// Parts each key tile's (query head, query tile) walk is split into (1, 2, 4 or
// 8; each part keeps at least 8 query tiles, non-causal count).  One CTA runs
// per SM (148 SMs).
//   * Unmasked walks are equally long: the launch takes ceil(CTAs / 148) waves
//     of whole walks, so parts = p costs ceil(p CTAs / 148) / p waves, plus the
//     partial sums (zeroing, reduce-adds, convert), taken as the time of 4 query
//     tiles per part: a factor 1 + 4 p / (query tiles per walk).  The cheapest p
//     wins (ties: fewer parts).  Measured on B200: +16% at B1 H64 Hkv8 N8192
//     d128 (2 parts), and the factor keeps d = 64 walks of 32 tiles unsplit.
//   * Causal and windowed walks differ in length from one key tile to the next,
//     so a grid of fewer than three waves is split until it has three.
int bwd_splits(int B, int H, int Hkv, int N, bool masked) {
  const long long nkt = (static_cast<long long>(N) + 127) / 128;
  const long long ctas = nkt * Hkv * B;
  const long long per_cta = (H / (Hkv > 0 ? Hkv : 1)) * nkt;
  int parts = 1;
  if (masked) {
    while (parts < 8 && ctas * parts < 3 * 148 && per_cta / (2 * parts) >= 8) parts *= 2;
    return parts;
  }
  double best = static_cast<double>((ctas + 147) / 148);
  for (int p = 2; p <= 8 && per_cta / p >= 8; p *= 2) {
    const double cost = static_cast<double>((ctas * p + 147) / 148) / p * (1.0 + 4.0 * p / per_cta);
    if (cost < best - 1e-9) {
      best = cost;
      parts = p;
    }
  }
  return parts;
}

int check_scale(float scale) {
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

}  // namespace

namespace {
// The driver's TMA descriptor encoder, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}
}  // namespace

CUresult make_tile_map(CUtensorMap* map, const void* base, int B, int N, int H, int d, int rows) {
  if (!encoder()) return CUDA_ERROR_NOT_FOUND;
  // dims innermost first: feature, sequence, head, batch
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(H) * d * 2, static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * H * d * 2};
  const cuuint32_t box[4] = {64u, static_cast<cuuint32_t>(rows), 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult make_paged_map(CUtensorMap* map, const void* base, int num_pages, int page_size, int Hkv, int d) {
  if (!encoder()) return CUDA_ERROR_NOT_FOUND;
  // dims innermost first: (K/V head, feature), pool row = page * page_size + slot
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(Hkv) * d,
                              static_cast<cuuint64_t>(num_pages) * static_cast<cuuint64_t>(page_size)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(Hkv) * d * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(page_size < 64 ? page_size : 64)};
  const cuuint32_t estr[2] = {1u, 1u};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult make_tile_map_e4m3(CUtensorMap* map, const void* base, int B, int N, int H, int d, int rows) {
  if (!encoder()) return CUDA_ERROR_NOT_FOUND;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(H) * d, static_cast<cuuint64_t>(d),
                                 static_cast<cuuint64_t>(N) * H * d};
  const cuuint32_t box[4] = {128u, static_cast<cuuint32_t>(rows), 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

size_t bwd_workspace_base(int B, int H, int N, int d, int dtype) {
  if (check_shape(B, H, N, d, dtype) != FA_OK) return 0;
  if (static_cast<long long>(B) * H * N == 0) return 0;
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  const size_t dq = align256(static_cast<size_t>(B) * N * H * d * sizeof(float));
  const size_t rows = align256(static_cast<size_t>(B) * H * npad * sizeof(float));
  return dq + 2 * rows;
}

CUresult make_kv_accum_map(CUtensorMap* map, float* base, int B, int N, int Hkv, int d) {
  if (!encoder()) return CUDA_ERROR_NOT_FOUND;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(Hkv) * d * 4, static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(N) * Hkv * d * 4};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(d), d == 128 ? 64u : 128u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult make_dq_accum_map_sw128(CUtensorMap* map, float* base, int B, int N, int H, int d) {
  if (!encoder()) return CUDA_ERROR_NOT_FOUND;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(H) * d * 4, static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(N) * H * d * 4};
  const cuuint32_t box[4] = {32u, 128u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult make_dq_accum_map(CUtensorMap* map, float* base, int B, int N, int H, int d) {
  if (!encoder()) return CUDA_ERROR_NOT_FOUND;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(H) * d * 4, static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(N) * H * d * 4};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(d), 64u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace fa

using namespace fa;

extern "C" {

int fa_version(void) { return 100; }

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size, bad scale or dtype)";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration (head dim, dtype or pass)";
    case FA_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "backward workspace missing, too small or misaligned";
    case FA_ERR_ARCH: return "current CUDA device is not an sm_100 (B200-class) GPU";
    case FA_ERR_LAUNCH: return "CUDA call failed (see fa_last_cuda_error)";
    case FA_ERR_DEVICE_TIMEOUT: return "a kernel wait exceeded its limit; outputs of that launch are undefined";
    case FA_ERR_TOO_LARGE: return "problem exceeds a size limit";
    case FA_ERR_DEVICE_INPUT: return "device-side input out of range (sequence length or page index)";
    case FA_ERR_DEVICE_CHECK: return "a device-side bounds check of the checking build failed";
    default: return "unknown status";
  }
}

int fa_last_cuda_error(void) { return t_last_cuda_error; }

void fa_set_wait_limit_ms(int ms) {
  g_limit_ns.store(ms > 0 ? static_cast<unsigned long long>(ms) * 1000000ull : 0ull);
}

void fa_debug_inject(int mode) { g_inject.store(mode); }

void fa_set_kernel_events(void* start, void* stop) {
  t_ev_start = static_cast<cudaEvent_t>(start);
  t_ev_stop = static_cast<cudaEvent_t>(stop);
}

int fa_last_device_status(void* stream, int* detail) {
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  int v = 0;
  e = cudaMemcpy(&v, st->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_cuda(e);
  const int zero = 0;
  e = cudaMemcpy(st->status, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return fail_cuda(e);
  if (detail) *detail = v;
  if (v & kDevCheck) return FA_ERR_DEVICE_CHECK;
  if (v & kDevBadInput) return FA_ERR_DEVICE_INPUT;
  return v ? FA_ERR_DEVICE_TIMEOUT : FA_OK;
}

}  // extern "C"

namespace {
// Block-sparse mask checks: mask_heads is 1 or H and the key-tile count fits the
// kernels' per-CTA list.  A null mask means no mask.  (Both dtypes take a mask in
// the forward; the backward refuses fp32 on its own.)
int check_mask(const uint8_t* mask, int mask_heads, int H, int N, int dtype) {
  (void)dtype;
  if (!mask) return FA_OK;
  if (mask_heads != 1 && mask_heads != H) return FA_ERR_INVALID_ARG;
  if ((N + 127) / 128 > kMaxSparseTiles) return FA_ERR_TOO_LARGE;
  return FA_OK;
}

int fwd_common(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv, int N, int d,
               float scale, int window_left, int window_right, const uint8_t* mask, int mask_heads, int dtype,
               void* stream) {
  int rc = check_shape(B, H, N, d, dtype);
  if (rc) return rc;
  if ((rc = check_kv_heads(H, Hkv))) return rc;
  if ((rc = check_window(window_left, window_right))) return rc;
  if ((rc = check_mask(mask, mask_heads, H, N, dtype))) return rc;
  if ((rc = check_scale(scale))) return rc;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FA_ERR_MISALIGNED;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  FwdArgs a;
  a.B = B;
  a.H = H;
  a.Hkv = Hkv;
  a.N = N;
  a.d = d;
  a.scale_log2 = scale * 1.4426950408889634f;
  set_window(window_left, window_right, &a.wl, &a.wr, &a.causal);
  a.O = O;
  a.LSE = LSE;
  a.block_mask = mask;
  a.mask_heads = mask_heads;
  a.nb = (N + 127) / 128;
  cudaError_t e;
  if (dtype == FA_FP32) {
    e = launch_fwd_f32(static_cast<const float*>(Q), static_cast<const float*>(K), static_cast<const float*>(V), a, s);
  } else {
    CUtensorMap tq, tk, tv, to;
    CUresult r;
    if ((r = make_tile_map(&tq, Q, B, N, H, d, 128)) != CUDA_SUCCESS ||
        (r = make_tile_map(&tk, K, B, N, Hkv, d, 128)) != CUDA_SUCCESS ||
        (r = make_tile_map(&tv, V, B, N, Hkv, d, 128)) != CUDA_SUCCESS ||
        (r = make_tile_map(&to, O, B, N, H, d, 128)) != CUDA_SUCCESS)
      return fail_encode(r);
    if (t_ev_start) cudaEventRecord(t_ev_start, s);
    e = launch_fwd_bf16(tq, tk, tv, to, a, make_ctl(*st), s);
    if (t_ev_stop && e == cudaSuccess) cudaEventRecord(t_ev_stop, s);
  }
  if (e != cudaSuccess) return fail_cuda(e);
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_fwd_window(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv, int N,
                  int d, float scale, int window_left, int window_right, int dtype, void* stream) {
  return fwd_common(Q, K, V, O, LSE, B, H, Hkv, N, d, scale, window_left, window_right, nullptr, 0, dtype, stream);
}

int fa_fwd_blocksparse(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv, int N,
                       int d, float scale, int window_left, int window_right, const void* block_mask,
                       int mask_heads, int dtype, void* stream) {
  if (!block_mask && static_cast<long long>(B) * H * N > 0) return FA_ERR_INVALID_ARG;
  return fwd_common(Q, K, V, O, LSE, B, H, Hkv, N, d, scale, window_left, window_right,
                    static_cast<const uint8_t*>(block_mask), mask_heads, dtype, stream);
}

int fa_fwd_gqa(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv, int N, int d,
               float scale, int causal, int dtype, void* stream) {
  return fa_fwd_window(Q, K, V, O, LSE, B, H, Hkv, N, d, scale, -1, causal ? 0 : -1, dtype, stream);
}

int fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d, float scale,
           int causal, int dtype, void* stream) {
  return fa_fwd_window(Q, K, V, O, LSE, B, H, H, N, d, scale, -1, causal ? 0 : -1, dtype, stream);
}

int fa_fwd_fp8_blocksparse(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv,
                           int N, int d, float scale, float scale_q, float scale_k, float scale_v, int window_left,
                           int window_right, const void* block_mask, int mask_heads, void* stream) {
  int rc = check_shape(B, H, N, d, FA_BF16);
  if (rc) return rc;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if ((rc = check_kv_heads(H, Hkv))) return rc;
  if ((rc = check_window(window_left, window_right))) return rc;
  const uint8_t* mask = static_cast<const uint8_t*>(block_mask);
  if ((rc = check_mask(mask, mask_heads, H, N, FA_BF16))) return rc;
  if ((rc = check_scale(scale)) || (rc = check_scale(scale_q)) || (rc = check_scale(scale_k)) ||
      (rc = check_scale(scale_v)))
    return rc;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FA_ERR_MISALIGNED;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FwdArgs a;
  a.B = B;
  a.H = H;
  a.Hkv = Hkv;
  a.N = N;
  a.d = d;
  // the per-tensor scales of Q and K fold into the softmax's exponent scale
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * scale_q * scale_k * 1.4426950408889634);
  set_window(window_left, window_right, &a.wl, &a.wr, &a.causal);
  a.O = O;
  a.LSE = LSE;
  a.block_mask = mask;
  a.mask_heads = mask ? mask_heads : 0;
  a.nb = (N + 127) / 128;
  CUtensorMap tq, tk, tv;
  CUresult r;
  if ((r = make_tile_map_e4m3(&tq, Q, B, N, H, d, 128)) != CUDA_SUCCESS ||
      (r = make_tile_map_e4m3(&tk, K, B, N, Hkv, d, 128)) != CUDA_SUCCESS ||
      (r = make_tile_map_e4m3(&tv, V, B, N, Hkv, d, 128)) != CUDA_SUCCESS)
    return fail_encode(r);
  if (t_ev_start) cudaEventRecord(t_ev_start, s);
  cudaError_t e = launch_fwd_fp8(tq, tk, tv, a, scale_v, make_ctl(*st), s);
  if (e != cudaSuccess) return fail_cuda(e);
  if (t_ev_stop) cudaEventRecord(t_ev_stop, s);
  return FA_OK;
}

int fa_fwd_fp8(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Hkv, int N, int d,
               float scale, float scale_q, float scale_k, float scale_v, int window_left, int window_right,
               void* stream) {
  return fa_fwd_fp8_blocksparse(Q, K, V, O, LSE, B, H, Hkv, N, d, scale, scale_q, scale_k, scale_v, window_left,
                                window_right, nullptr, 0, stream);
}

size_t fa_bwd_workspace_size_gqa(int B, int H, int Hkv, int N, int d, int dtype) {
  if (check_kv_heads(H, Hkv) != FA_OK) return 0;
  const size_t base = fa::bwd_workspace_base(B, H, N, d, dtype);
  if (base == 0) return 0;
  // the accumulators whenever masked or unmasked walks of this shape would split
  const bool split = bwd_splits(B, H, Hkv, N, true) > 1 || bwd_splits(B, H, Hkv, N, false) > 1;
  const size_t kv = split ? 2 * align256(static_cast<size_t>(B) * N * Hkv * d * sizeof(float)) : 0;
  return base + kv;
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d, int dtype) {
  return fa_bwd_workspace_size_gqa(B, H, H, N, d, dtype);
}

}  // extern "C"

namespace {
int bwd_common(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
               void* dQ, void* dK, void* dV, int B, int H, int Hkv, int N, int d, float scale, int window_left,
               int window_right, const uint8_t* mask, int mask_heads, int dtype, void* workspace,
               size_t workspace_bytes, void* stream) {
  int rc = check_shape(B, H, N, d, dtype);
  if (rc) return rc;
  if ((rc = check_kv_heads(H, Hkv))) return rc;
  if ((rc = check_window(window_left, window_right))) return rc;
  if ((rc = check_mask(mask, mask_heads, H, N, dtype))) return rc;
  if ((rc = check_scale(scale))) return rc;
  if (dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return FA_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV};
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_MISALIGNED;
  const size_t need = bwd_workspace_base(B, H, N, d, dtype);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_WORKSPACE;
  // split the walks when the grid is small and the workspace holds the fp32 dK / dV sums
  const bool masked = window_left >= 0 || window_right >= 0 || mask != nullptr;
  const int parts = (workspace_bytes >= fa_bwd_workspace_size_gqa(B, H, Hkv, N, d, dtype))
                        ? bwd_splits(B, H, Hkv, N, masked)
                        : 1;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const int npad = (N + 127) / 128 * 128;
  BwdArgs a;
  a.B = B;
  a.H = H;
  a.Hkv = Hkv;
  a.N = N;
  a.d = d;
  a.Npad = npad;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  set_window(window_left, window_right, &a.wl, &a.wr, &a.causal);
  a.block_mask = mask;
  a.mask_heads = mask_heads;
  a.nb = (N + 127) / 128;
  a.O = O;
  a.dO = dO;
  a.LSE = LSE;
  a.dQ = dQ;
  a.dK = dK;
  a.dV = dV;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.dQacc = reinterpret_cast<float*>(ws);
  ws += align256(static_cast<size_t>(B) * N * H * d * sizeof(float));
  a.Dvec = reinterpret_cast<float*>(ws);
  ws += align256(static_cast<size_t>(B) * H * npad * sizeof(float));
  a.LSE2 = reinterpret_cast<float*>(ws);
  ws += align256(static_cast<size_t>(B) * H * npad * sizeof(float));
  a.splits = parts;
  a.dKacc = parts > 1 ? reinterpret_cast<float*>(ws) : nullptr;
  a.dVacc = parts > 1 ? reinterpret_cast<float*>(ws + align256(static_cast<size_t>(B) * N * Hkv * d * sizeof(float)))
                      : nullptr;

  CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
  CUresult r;
  if ((r = make_tile_map(&tq, Q, B, N, H, d, 128)) != CUDA_SUCCESS ||
      (r = make_tile_map(&tdo, dO, B, N, H, d, 128)) != CUDA_SUCCESS ||
      (r = make_tile_map(&tk, K, B, N, Hkv, d, 128)) != CUDA_SUCCESS ||
      (r = make_tile_map(&tv, V, B, N, Hkv, d, 128)) != CUDA_SUCCESS ||
      (r = (d == 128 ? make_dq_accum_map(&tdq, a.dQacc, B, N, H, d)
                     : make_dq_accum_map_sw128(&tdq, a.dQacc, B, N, H, d))) != CUDA_SUCCESS)
    return fail_encode(r);
  if (parts > 1) {
    if ((r = make_kv_accum_map(&tdk, a.dKacc, B, N, Hkv, d)) != CUDA_SUCCESS ||
        (r = make_kv_accum_map(&tdv, a.dVacc, B, N, Hkv, d)) != CUDA_SUCCESS)
      return fail_encode(r);
  } else {
    tdk = tdq;  // not read by the kernels without a split
    tdv = tdq;
  }
  cudaError_t e = launch_bwd_pre(a, s);
  if (e == cudaSuccess && parts > 1) e = launch_bwd_kv_zero(a, s);
  if (e != cudaSuccess) return fail_cuda(e);
  if (t_ev_start) cudaEventRecord(t_ev_start, s);
  e = (d == 128) ? launch_bwd_main(tq, tk, tv, tdo, tdq, tdk, tdv, a, make_ctl(*st), s)
                 : launch_bwd_main64(tq, tk, tv, tdo, tdq, tdk, tdv, a, make_ctl(*st), s);
  if (e != cudaSuccess) return fail_cuda(e);
  if (t_ev_stop) cudaEventRecord(t_ev_stop, s);
  e = launch_bwd_dq(a, s);
  if (e == cudaSuccess && parts > 1) e = launch_bwd_kv_convert(a, s);
  if (e != cudaSuccess) return fail_cuda(e);
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_bwd_window(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                  void* dQ, void* dK, void* dV, int B, int H, int Hkv, int N, int d, float scale, int window_left,
                  int window_right, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Hkv, N, d, scale, window_left, window_right, nullptr, 0,
                    dtype, workspace, workspace_bytes, stream);
}

int fa_bwd_blocksparse(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                       void* dQ, void* dK, void* dV, int B, int H, int Hkv, int N, int d, float scale,
                       int window_left, int window_right, const void* block_mask, int mask_heads, int dtype,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!block_mask && static_cast<long long>(B) * H * N > 0) return FA_ERR_INVALID_ARG;
  return bwd_common(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Hkv, N, d, scale, window_left, window_right,
                    static_cast<const uint8_t*>(block_mask), mask_heads, dtype, workspace, workspace_bytes, stream);
}

int fa_bwd_gqa(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
               void* dQ, void* dK, void* dV, int B, int H, int Hkv, int N, int d, float scale, int causal, int dtype,
               void* workspace, size_t workspace_bytes, void* stream) {
  return fa_bwd_window(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, Hkv, N, d, scale, -1, causal ? 0 : -1, dtype,
                       workspace, workspace_bytes, stream);
}

int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE, void* dQ,
           void* dK, void* dV, int B, int H, int N, int d, float scale, int causal, int dtype, void* workspace,
           size_t workspace_bytes, void* stream) {
  return fa_bwd_window(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, H, N, d, scale, -1, causal ? 0 : -1, dtype,
                       workspace, workspace_bytes, stream);
}

int fa_merge_partial(float* O_acc, float* LSE_acc, const void* O_part, const float* LSE_part, void* O_out, int B,
                     int H, int N, int d, int init, void* stream) {
  int rc = check_shape(B, H, N, d, FA_BF16);
  if (rc) return rc;
  if (static_cast<long long>(B) * H * N == 0) return FA_OK;
  if (!O_acc || !LSE_acc || !O_part || !LSE_part) return FA_ERR_INVALID_ARG;
  if (!aligned16(O_acc) || !aligned16(O_part) || (O_out && !aligned16(O_out)) ||
      (reinterpret_cast<uintptr_t>(LSE_acc) & 3u) || (reinterpret_cast<uintptr_t>(LSE_part) & 3u))
    return FA_ERR_MISALIGNED;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  cudaError_t e = launch_merge(O_acc, LSE_acc, O_part, LSE_part, O_out, B, H, N, d, init ? 1 : 0,
                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  return FA_OK;
}

int fa_accumulate_bf16(float* acc, const void* part, long long n, int init, void* stream) {
  if (n < 0 || n % 8 != 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!acc || !part) return FA_ERR_INVALID_ARG;
  if (!aligned16(acc) || !aligned16(part)) return FA_ERR_MISALIGNED;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  cudaError_t e = launch_accumulate(acc, part, n, init ? 1 : 0, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  return FA_OK;
}

int fa_cast_bf16(void* out, const float* in, long long n, void* stream) {
  if (n < 0 || n % 8 != 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!out || !in) return FA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(in)) return FA_ERR_MISALIGNED;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  cudaError_t e = launch_cast(out, in, n, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e);
  return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// One decode step over a paged KV cache
// ---------------------------------------------------------------------------
namespace {

struct DecodePlan {
  int hgroups, splits, chunk;
  size_t ws;  // workspace bytes the plan needs (0 with one chunk)
};

bool pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

int check_decode(int B, int H, int Hkv, int d, int page_size, int num_pages, int max_pages, float scale) {
  if (B < 0 || H < 1 || num_pages < 1 || max_pages < 1) return FA_ERR_INVALID_ARG;
  int rc = check_kv_heads(H, Hkv);
  if (rc) return rc;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!pow2_in(page_size, 8, 4096)) return FA_ERR_UNSUPPORTED;
  if ((rc = check_scale(scale))) return rc;
  const long long hg = (H / Hkv + 15) / 16;
  if (static_cast<long long>(num_pages) * page_size > 0x7fffffffLL ||
      static_cast<long long>(max_pages) * page_size > 0x7fffffffLL || B > 65535 || Hkv * hg > 65535)
    return FA_ERR_TOO_LARGE;
  return FA_OK;
}

size_t decode_ws_bytes(int B, int H, int d, int splits) {
  if (splits <= 1) return 0;
  const size_t rows = static_cast<size_t>(splits) * B * H;
  return align256(rows * d * sizeof(float)) + align256(rows * sizeof(float));
}

// Chunks per (sequence, head group).  Each CTA pays a fixed start (length and
// page checks, the first loads in flight) and end (merge of its warps), so chunks
// hold at least 512 KB of K/V (16 tiles at d = 128, 32 at d = 64).  A batch with
// fewer (sequence, head group) pairs than CTA slots (148 SMs x 2) is split into
// about two waves of CTAs; a larger batch into about four, the later waves'
// chunks being the short or empty ends of the sequences.  No more chunks than
// the workspace holds.
DecodePlan decode_plan(int B, int H, int Hkv, int d, int page_size, int max_pages, size_t ws_cap) {
  DecodePlan p;
  p.hgroups = (H / Hkv + 15) / 16;
  const long long max_keys = static_cast<long long>(max_pages) * page_size;
  const long long tiles = (max_keys + 63) / 64;
  const long long ctas = static_cast<long long>(B) * Hkv * p.hgroups;
  const long long slots = 2 * 148;
  const long long waves = 4;  // for batches that fill the slots
  const long long min_tiles = d == 128 ? 16 : 32;
  // a small batch: two waves (one wave suits equal lengths best, but a long
  // sequence among shorter ones then runs alone at the end)
  const long long w = ctas < slots ? 2 : waves;
  long long want = ctas <= 0 ? 1 : (w * slots + ctas - 1) / ctas;
  want = std::max(1LL, std::min({want, tiles / min_tiles, 65535LL}));
  for (;;) {
    const long long chunk_tiles = (tiles + want - 1) / want;
    p.splits = static_cast<int>((tiles + chunk_tiles - 1) / chunk_tiles);
    p.chunk = static_cast<int>(chunk_tiles * 64);
    p.ws = decode_ws_bytes(B, H, d, p.splits);
    if (p.splits == 1 || p.ws <= ws_cap) break;
    want = p.splits - 1;
  }
  return p;
}

}  // namespace

extern "C" {

size_t fa_decode_workspace_size(int B, int H, int Hkv, int d, int page_size, int max_pages) {
  if (check_decode(B, H, Hkv, d, page_size, 1, max_pages, 1.0f) != FA_OK) return 0;
  return decode_plan(B, H, Hkv, d, page_size, max_pages, SIZE_MAX).ws;
}

int fa_decode_paged(const void* Q, const void* K_cache, const void* V_cache, const int* block_table,
                    const int* seqlens, void* O, float* LSE, int B, int H, int Hkv, int d, int page_size,
                    int num_pages, int max_pages, float scale, void* workspace, size_t workspace_bytes,
                    void* stream) {
  int rc = check_decode(B, H, Hkv, d, page_size, num_pages, max_pages, scale);
  if (rc) return rc;
  if (B == 0) return FA_OK;
  if (!Q || !K_cache || !V_cache || !block_table || !seqlens || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K_cache) || !aligned16(V_cache) || !aligned16(O) ||
      (reinterpret_cast<uintptr_t>(LSE) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return FA_ERR_MISALIGNED;
  if (workspace && !aligned16(workspace)) return FA_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  if ((rc = device_state(&st))) return rc;
  const DecodePlan plan = decode_plan(B, H, Hkv, d, page_size, max_pages, workspace ? workspace_bytes : 0);
  DecodeArgs a;
  a.B = B;
  a.H = H;
  a.Hkv = Hkv;
  a.d = d;
  a.page_size = page_size;
  a.num_pages = num_pages;
  a.max_pages = max_pages;
  a.hgroups = plan.hgroups;
  a.splits = plan.splits;
  a.chunk = plan.chunk;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.Q = Q;
  a.block_table = block_table;
  a.seqlens = seqlens;
  a.O = O;
  a.LSE = LSE;
  const size_t rows = static_cast<size_t>(plan.splits) * B * H;
  a.Opart = plan.splits > 1 ? static_cast<float*>(workspace) : nullptr;
  a.LSEpart = plan.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(rows * d * 4))
                              : nullptr;
  CUtensorMap tk, tv;
  CUresult r;
  if ((r = make_paged_map(&tk, K_cache, num_pages, page_size, Hkv, d)) != CUDA_SUCCESS ||
      (r = make_paged_map(&tv, V_cache, num_pages, page_size, Hkv, d)) != CUDA_SUCCESS)
    return fail_encode(r);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (t_ev_start) cudaEventRecord(t_ev_start, s);
  cudaError_t e = launch_decode(tk, tv, a, make_ctl(*st), s);
  if (t_ev_stop && e == cudaSuccess) cudaEventRecord(t_ev_stop, s);
  if (e != cudaSuccess) return fail_cuda(e);
  return FA_OK;
}

}  // extern "C"
