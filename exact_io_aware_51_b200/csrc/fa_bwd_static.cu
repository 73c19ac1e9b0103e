// Backward pass whose scratch memory lives inside the library.
//
// fa_bwd needs device scratch (the fp32 dQ accumulator and two per-row arrays)
// that the caller allocates and passes in.  Some callers cannot allocate at the
// point where they run the backward pass: runtimes that lay out all device
// memory once at start-up and hand kernels fixed buffers afterwards, or code
// that must not call cudaMalloc mid-run because it can synchronise the device
// or fail under memory pressure.  fa_bwd_static_scratch serves them: it runs
// the same kernels as fa_bwd, but on a fixed-size scratch array compiled into
// this library, so the call itself allocates nothing.
//
// Cost and limits:
//   * the array is kStaticScratchBytes (64 MiB) of device memory on every GPU
//     that loads the library, held until the process exits;
//   * problems whose base workspace (the fp32 dQ accumulator and the two
//     per-row arrays) exceeds it are refused with FA_ERR_TOO_LARGE; a problem
//     whose base fits but whose split-walk dK / dV accumulators do not (so
//     fa_bwd_workspace_size is larger than the array) runs with unsplit walks,
//     which gives the same gradients, only without the small-grid speed-up;
//   * every call shares the array and leaves its contents behind; the
//     backward's preprocess kernel rewrites everything the later kernels read
//     (it zeroes the dQ accumulator and fills both per-row arrays), so nothing
//     carries over between calls, but calls whose kernels overlap on the GPU
//     (different streams, or different host threads without ordering) race
//     on the array and produce wrong gradients;
//   * the first call on each device looks up the array's device address with
//     that device current (cudaGetSymbolAddress); make that first call before
//     any stream capture.
#include <cuda_runtime.h>

#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace fa {
namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;
constexpr int kMaxScratchDevices = 64;

// In host code this name is only a stand-in for the device copy; the device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_bwd_scratch[kStaticScratchBytes];

struct ScratchSlot {
  std::mutex mu;
  void* ptr = nullptr;
};
ScratchSlot g_slots[kMaxScratchDevices];

// Device address of the scratch array on the current device, looked up with
// that device current.  Only a successful lookup is kept; after a failure the
// next call tries again.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_LAUNCH;
  if (dev < 0 || dev >= kMaxScratchDevices) return FA_ERR_ARCH;
  ScratchSlot& s = g_slots[dev];
  std::lock_guard<std::mutex> lock(s.mu);
  if (s.ptr == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return FA_ERR_LAUNCH;
    s.ptr = p;
  }
  *out = s.ptr;
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" int fa_bwd_static_scratch(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                     const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d,
                                     float scale, int causal, int dtype, void* stream) {
  const size_t need = fa::bwd_workspace_base(B, H, N, d, dtype);
  if (need > fa::kStaticScratchBytes) return FA_ERR_TOO_LARGE;
  if (need == 0) {
    // invalid or empty problem: fa_bwd reports which, without touching scratch
    return fa_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal, dtype, nullptr, 0, stream);
  }
  void* scratch = nullptr;
  const int rc = fa::scratch_address(&scratch);
  if (rc != FA_OK) return rc;
  return fa_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal, dtype, scratch,
                fa::kStaticScratchBytes, stream);
}
