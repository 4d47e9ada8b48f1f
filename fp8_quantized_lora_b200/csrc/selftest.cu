// Self-test of the failure detection: the bounded waits give up and report.
//
// Every wait in the library's kernels is bounded (about one second of clock
// cycles); on expiry the waiting role sets FALQON_DEV_TIMEOUT in the status
// word and the kernel returns, so that the context stays usable.  This
// one-CTA kernel runs the two kinds of wait on things that never complete:
//   warp 0  the mbarrier wait of the tcgen05 and quantize kernels
//           (warp_wait / mbar_wait) on a phase that nothing arrives on;
//   warp 1  a poll of a global word, bounded like the quantize kernel's
//           grid exchange, on a flag the caller leaves at zero (or sets, to
//           see the poll succeed).
#include "../../include/falqon.h"
#include "internal.h"
#include "tc_common.cuh"

namespace falqon {
namespace {

__global__ void __launch_bounds__(64) selftest_wait_kernel(const int32_t* __restrict__ flag,
                                                           int32_t* __restrict__ dev_status,
                                                           int32_t* __restrict__ which) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival completes phase 0; none comes
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    const bool ok = warp_wait(&bar, 0, &abort_flag);
    if (!ok && lane == 0) {
      raise_status(dev_status, kDevTimeout);
      atomicOr(which, 1);
    }
  } else if (lane == 0) {
    const long long t0 = clock64();
    bool ok = false;
    while (true) {
      int32_t v;
      asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(flag));
      if (v != 0) {
        ok = true;
        break;
      }
      if (clock64() - t0 > kWaitBudget) break;
    }
    if (!ok) {
      raise_status(dev_status, kDevTimeout);
      atomicOr(which, 2);
    }
  }
}

}  // namespace
}  // namespace falqon

using namespace falqon;

extern "C" {

falqon_status falqon_selftest_bounded_waits(const int32_t* flag, int32_t* dev_status, int32_t* which,
                                            void* stream) {
  if (!flag || !dev_status || !which) return FALQON_ERR_INVALID_ARG;
  if (!current_device_info()) return FALQON_ERR_CUDA;
  const cudaError_t e = launch_pdl(selftest_wait_kernel, dim3(1), dim3(64), 0, static_cast<cudaStream_t>(stream),
                                   1u, flag, dev_status, which);
  return e == cudaSuccess ? FALQON_OK : FALQON_ERR_CUDA;
}

}  // extern "C"
