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
// address); its device address is looked up with cudaGetSymbolAddress, with
// that device current, by the first call on that device that needs scratch
// (one asking for dA or dB) and cached.  A failed lookup is not cached: the
// next such call tries again.  That first call must come before any stream
// capture on that device.  A dX-only call needs no scratch and does no
// lookup.
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

std::mutex g_mu;
void* g_addr[kMaxDevices];  // cached after a successful lookup only

// Device address of the scratch array for the current device (looked up on
// the first call that needs it; a failure is returned and not remembered).
void* scratch_address(cudaError_t* err) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess) {
      *err = e;
      return nullptr;
    }
    g_addr[dev] = p;
  }
  *err = cudaSuccess;
  return g_addr[dev];
}

}  // namespace
}  // namespace falqon

extern "C" FALQON_API falqon_status falqon_linear_bwd_noalloc(
    const uint8_t* dyq, const float* s_dy, const uint8_t* wq, const float* s_w,
    const uint8_t* xq, const float* s_x, const void* A, const void* B, int64_t M, int64_t N,
    int64_t K, int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status, void* stream) {
  using namespace falqon;
  // the same argument checks, in the same order, as falqon_linear_bwd
  const falqon_status s = linear_bwd_validate(dyq, s_dy, wq, s_w, xq, s_x, A, B, M, N, K, r, dx, dA, dB);
  if (s != FALQON_OK) return s;
  if (!dA && !dB)  // dX alone needs no scratch
    return falqon_linear_bwd(dyq, s_dy, wq, s_w, xq, s_x, A, B, M, N, K, r, dx, dA, dB, dev_status, nullptr, 0,
                             stream);
  // refuse problems whose intermediates would not fit the built-in scratch
  if (adapter_workspace_bytes(M, N, K, r, dA != nullptr) > kScratchBytes) return FALQON_ERR_WORKSPACE;
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_address(&err);
  if (!scratch) return FALQON_ERR_CUDA;
  return falqon_linear_bwd(dyq, s_dy, wq, s_w, xq, s_x, A, B, M, N, K, r, dx, dA, dB, dev_status,
                           scratch, kScratchBytes, stream);
}
