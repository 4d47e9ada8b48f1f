// falqon_linear_bwd_noalloc: the backward call for callers that cannot
// allocate device memory.
//
// Some callers have no way to call cudaMalloc on the hot path: a host
// application that hands the library only the device pointers of its own
// tensors and runs with a fixed memory budget, a plugin inside another
// runtime that owns every allocation, or code that must not allocate
// between steps.  This entry point takes the same inputs and outputs as
// falqon_linear_bwd but no workspace: the adapter products keep their
// intermediates (T and U as bf16 hi/lo pairs, split-K partial sums) in one
// scratch array compiled into the library.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds kScratchBytes of it until the process exits.  Host code may
// not pass its name to a kernel (on the host it is a stand-in, not a device
// address); its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made
// on that device.  That first call must therefore come before any stream
// capture on that device.
//
// Every call shares the array and it keeps whatever the last call left in
// it; nothing in it needs to start at zero (each kernel writes every
// scratch element it later reads).  Calls that overlap on the GPU (on
// different streams, or from different threads without ordering) race on
// the array and produce garbage; serialise them.
#include <mutex>

#include "../../include/falqon.h"
#include "internal.h"

namespace falqon {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_bwd_scratch[kScratchBytes];

std::once_flag g_once[kMaxDevices];
void* g_addr[kMaxDevices];
cudaError_t g_err[kMaxDevices];

// Device address of the scratch array for the current device (set-up on first use).
void* scratch_address(cudaError_t* err) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
    return nullptr;
  }
  std::call_once(g_once[dev], [dev]() {
    void* p = nullptr;
    g_err[dev] = cudaGetSymbolAddress(&p, g_bwd_scratch);
    g_addr[dev] = g_err[dev] == cudaSuccess ? p : nullptr;
  });
  *err = g_err[dev];
  return g_addr[dev];
}

}  // namespace
}  // namespace falqon

extern "C" FALQON_API falqon_status falqon_linear_bwd_noalloc(
    const uint8_t* dyq, const float* s_dy, const uint8_t* wq, const float* s_w,
    const uint8_t* xq, const float* s_x, const void* A, const void* B, int64_t M, int64_t N,
    int64_t K, int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status, void* stream) {
  using namespace falqon;
  if (dA || dB) {
    // refuse problems whose intermediates would not fit the built-in scratch
    if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return FALQON_ERR_INVALID_ARG;
    if (adapter_workspace_bytes(M, N, K, r, dA != nullptr) > kScratchBytes)
      return FALQON_ERR_WORKSPACE;
  }
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_address(&err);
  if (!scratch) return FALQON_ERR_CUDA;
  return falqon_linear_bwd(dyq, s_dy, wq, s_w, xq, s_x, A, B, M, N, K, r, dx, dA, dB, dev_status,
                           scratch, kScratchBytes, stream);
}
