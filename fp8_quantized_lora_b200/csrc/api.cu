// C ABI of libfalqon: argument validation, workspace layout, dispatch.
#include <mutex>

#include "../../include/falqon.h"
#include "internal.h"

namespace falqon {

namespace {

constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::once_flag g_info_once[kMaxDevices];
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

falqon_status from_cuda(cudaError_t e) {
  return e == cudaSuccess ? FALQON_OK
         : e == cudaErrorInvalidValue ? FALQON_ERR_UNSUPPORTED
                                      : FALQON_ERR_CUDA;
}

falqon_status check_ws(size_t need, const void* ws, size_t have) {
  if (need == 0) return FALQON_OK;
  if (!ws || have < need || !aligned256(ws)) return FALQON_ERR_WORKSPACE;
  return FALQON_OK;
}

}  // namespace

const DeviceInfo* current_device_info() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_info_once[dev], [dev]() {
    DeviceInfo d;
    d.device = dev;
    cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&d.coop_launch, cudaDevAttrCooperativeLaunch, dev);
    g_info[dev] = d;
  });
  return g_info[dev].sm_count > 0 ? &g_info[dev] : nullptr;
}

falqon_status linear_bwd_validate(const uint8_t* dyq, const float* s_dy, const uint8_t* wq, const float* s_w,
                                  const uint8_t* xq, const float* s_x, const void* A, const void* B, int64_t M,
                                  int64_t N, int64_t K, int64_t r, const void* dx, const void* dA,
                                  const void* dB) {
  if (!dx && !dA && !dB) return FALQON_ERR_INVALID_ARG;
  if (!dyq || !s_dy) return FALQON_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return FALQON_ERR_INVALID_ARG;
  if (N % 16 != 0 || K % 16 != 0) return FALQON_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 256 || N > (int64_t(1) << 31) - 256 || K > (int64_t(1) << 31) - 256)
    return FALQON_ERR_UNSUPPORTED;
  if (!aligned16(dyq)) return FALQON_ERR_UNSUPPORTED;
  if (dx) {
    if (!wq || !s_w) return FALQON_ERR_INVALID_ARG;
    if (!aligned16(wq) || !aligned16(dx)) return FALQON_ERR_UNSUPPORTED;
  }
  if (dA || dB) {
    if (r <= 0 || !xq || !s_x || !A) return FALQON_ERR_INVALID_ARG;
    if (dA && !B) return FALQON_ERR_INVALID_ARG;
    if (r % 16 != 0 || r > 65536) return FALQON_ERR_UNSUPPORTED;
    if (!aligned16(xq) || !aligned16(A) || (B && !aligned16(B)) || (dA && !aligned16(dA)) ||
        (dB && !aligned16(dB)))
      return FALQON_ERR_UNSUPPORTED;
  }
  return FALQON_OK;
}

EncodeTiledFn encode_tiled_fn() {
  std::call_once(g_encode_once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, size_t elem_bytes,
                  const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                  uint32_t box_outer, bool swizzle128, uint64_t ld) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {(ld ? ld : inner) * elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d_sw64(CUtensorMap* map, CUtensorMapDataType dtype, size_t elem_bytes, const void* base,
                       uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc || box_inner * elem_bytes != 64) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace falqon

using namespace falqon;

extern "C" {

const char* falqon_version(void) { return "falqon-b200 0.1.0 (sm_100a)"; }

const char* falqon_status_string(falqon_status s) {
  switch (s) {
    case FALQON_OK: return "ok";
    case FALQON_ERR_INVALID_ARG: return "invalid argument";
    case FALQON_ERR_UNSUPPORTED: return "unsupported shape or alignment";
    case FALQON_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case FALQON_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

falqon_status falqon_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes == 0) return FALQON_ERR_INVALID_ARG;
  if (!aligned256(workspace)) return FALQON_ERR_WORKSPACE;
  return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FALQON_OK
             : FALQON_ERR_CUDA;
}

size_t falqon_workspace_size(falqon_op op, int64_t M, int64_t N, int64_t K, int64_t r) {
  switch (op) {
    case FALQON_OP_QUANTIZE: return quantize_workspace_bytes(M * N);
    case FALQON_OP_LINEAR_FWD: return 0;
    case FALQON_OP_LINEAR_BWD:
      if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return 0;
      return adapter_workspace_bytes(M, N, K, r, true);
    case FALQON_OP_PROXY_UPDATE:
      if (N <= 0 || K <= 0) return 0;
      return proxy_workspace_bytes(N, K);
    case FALQON_OP_PROXY_UPDATE_TOPK:
      if (N <= 0 || K <= 0 || r <= 0) return 0;
      return proxy_topk_workspace_bytes(N, K, r);
    case FALQON_OP_FOLDED_T:
    case FALQON_OP_LINEAR_BWD_FOLDED:
      if (M <= 0 || r <= 0) return 0;
      return 2 * adapter_plane_bytes(M, r);
    case FALQON_OP_SEPARATE_SAVED_BF16:
    case FALQON_OP_SEPARATE_SAVED_FP8:
      if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return 0;
      return separate_saved_bytes(op == FALQON_OP_SEPARATE_SAVED_FP8, M, N, K, r);
    case FALQON_OP_SEPARATE_FWD_FP8:
      return separate_fwd_workspace_bytes(true, M, N, K, r);
    case FALQON_OP_SEPARATE_BWD_BF16:
    case FALQON_OP_SEPARATE_BWD_FP8:
      if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return 0;
      return separate_bwd_workspace_bytes(op == FALQON_OP_SEPARATE_BWD_FP8, M, N, K, r);
  }
  return 0;
}

}  // extern "C"

namespace {

falqon_status quantize_call(const void* x, falqon_dtype dtype, int64_t rows, int64_t cols, uint8_t* codes,
                            float* scale, float* amax, float* residual, int32_t* dev_status, void* workspace,
                            size_t workspace_bytes, void* stream, bool e5m2) {
  if (!x || !codes || !scale) return FALQON_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0) return FALQON_ERR_INVALID_ARG;
  if (dtype != FALQON_DTYPE_BF16 && dtype != FALQON_DTYPE_F32) return FALQON_ERR_INVALID_ARG;
  if (cols % 16 != 0) return FALQON_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(codes) || (residual && !aligned16(residual)))
    return FALQON_ERR_UNSUPPORTED;
  const int64_t n = rows * cols;
  falqon_status s = check_ws(quantize_workspace_bytes(n), workspace, workspace_bytes);
  if (s != FALQON_OK) return s;
  if (!current_device_info()) return FALQON_ERR_CUDA;
  return from_cuda(launch_quantize(x, dtype == FALQON_DTYPE_BF16, n, codes, scale, amax, residual,
                                   dev_status, workspace, static_cast<cudaStream_t>(stream), e5m2));
}

}  // namespace

extern "C" {

falqon_status falqon_quantize(const void* x, falqon_dtype dtype, int64_t rows, int64_t cols,
                              uint8_t* codes, float* scale, float* amax, float* residual,
                              int32_t* dev_status, void* workspace, size_t workspace_bytes,
                              void* stream) {
  return quantize_call(x, dtype, rows, cols, codes, scale, amax, residual, dev_status, workspace,
                       workspace_bytes, stream, false);
}

falqon_status falqon_quantize_e5m2(const void* x, falqon_dtype dtype, int64_t rows, int64_t cols,
                                   uint8_t* codes, float* scale, float* amax, int32_t* dev_status,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  return quantize_call(x, dtype, rows, cols, codes, scale, amax, nullptr, dev_status, workspace,
                       workspace_bytes, stream, true);
}

falqon_status falqon_linear_fwd(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                const float* s_w, int64_t M, int64_t N, int64_t K, void* y,
                                int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!xq || !s_x || !wq || !s_w || !y) return FALQON_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return FALQON_ERR_INVALID_ARG;
  if (N % 16 != 0 || K % 16 != 0) return FALQON_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 256 || N > (int64_t(1) << 31) - 256 || K > (int64_t(1) << 31) - 256)
    return FALQON_ERR_UNSUPPORTED;
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(y)) return FALQON_ERR_UNSUPPORTED;
  if (!current_device_info()) return FALQON_ERR_CUDA;
  return from_cuda(launch_fp8_gemm_fwd(xq, s_x, wq, s_w, M, N, K, y, dev_status,
                                       static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

falqon_status linear_bwd_call(const uint8_t* dyq, const float* s_dy, const uint8_t* wq, const float* s_w,
                              const uint8_t* xq, const float* s_x, const void* A, const void* B, int64_t M,
                              int64_t N, int64_t K, int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status,
                              void* workspace, size_t workspace_bytes, void* stream, bool dy_e5m2) {
  falqon_status s0 = linear_bwd_validate(dyq, s_dy, wq, s_w, xq, s_x, A, B, M, N, K, r, dx, dA, dB);
  if (s0 != FALQON_OK) return s0;
  const bool adapters = dA || dB;
  if (adapters) {
    falqon_status s =
        check_ws(adapter_workspace_bytes(M, N, K, r, dA != nullptr), workspace, workspace_bytes);
    if (s != FALQON_OK) return s;
  }
  if (!current_device_info()) return FALQON_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (adapters) {
    cudaError_t e = launch_adapter_grads(dyq, s_dy, xq, s_x, A, B, M, N, K, r, dA, dB,
                                         dev_status, workspace, st, dy_e5m2);
    if (e != cudaSuccess) return from_cuda(e);
  }
  if (dx) return from_cuda(launch_fp8_gemm_dx(dyq, s_dy, wq, s_w, M, N, K, dx, dev_status, st, dy_e5m2));
  return FALQON_OK;
}

}  // namespace

extern "C" {

falqon_status falqon_linear_bwd(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                                const float* s_w, const uint8_t* xq, const float* s_x,
                                const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                                int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return linear_bwd_call(dyq, s_dy, wq, s_w, xq, s_x, A, B, M, N, K, r, dx, dA, dB, dev_status, workspace,
                         workspace_bytes, stream, false);
}

falqon_status falqon_linear_bwd_e5m2(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                                     const float* s_w, const uint8_t* xq, const float* s_x,
                                     const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                                     int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  return linear_bwd_call(dyq, s_dy, wq, s_w, xq, s_x, A, B, M, N, K, r, dx, dA, dB, dev_status, workspace,
                         workspace_bytes, stream, true);
}

falqon_status falqon_proxy_update(uint8_t* wq, const float* s_w, float* proxy,
                                  const void* dB_inc, const void* A, int64_t N, int64_t K,
                                  int64_t r, uint32_t flags, uint8_t* row_mask,
                                  int32_t* n_selected, int32_t* dev_status, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  const uint32_t known = FALQON_PROXY_ACCUMULATE | FALQON_PROXY_SELECT | FALQON_PROXY_KEEP_RESIDUAL |
                         FALQON_PROXY_STRICT | FALQON_PROXY_TENSOR | FALQON_PROXY_DEFER_CLEAR;
  if ((flags & (FALQON_PROXY_ACCUMULATE | FALQON_PROXY_SELECT)) == 0 || (flags & ~known)) return FALQON_ERR_INVALID_ARG;
  // a deferred clear needs a call that rewrites every row's proxy (ACCUMULATE) and the mask (SELECT)
  if ((flags & FALQON_PROXY_DEFER_CLEAR) &&
      ((flags & (FALQON_PROXY_ACCUMULATE | FALQON_PROXY_SELECT)) != (FALQON_PROXY_ACCUMULATE | FALQON_PROXY_SELECT) ||
       (flags & (FALQON_PROXY_KEEP_RESIDUAL | FALQON_PROXY_TENSOR)) || !row_mask))
    return FALQON_ERR_INVALID_ARG;
  if ((flags & FALQON_PROXY_KEEP_RESIDUAL) && !(flags & FALQON_PROXY_SELECT)) return FALQON_ERR_INVALID_ARG;
  if ((flags & FALQON_PROXY_TENSOR) &&
      (!(flags & FALQON_PROXY_ACCUMULATE) || (flags & FALQON_PROXY_STRICT)))
    return FALQON_ERR_INVALID_ARG;
  if (!proxy || N <= 0 || K <= 0) return FALQON_ERR_INVALID_ARG;
  if (K % 16 != 0) return FALQON_ERR_UNSUPPORTED;
  if (!aligned16(proxy)) return FALQON_ERR_UNSUPPORTED;
  if (flags & FALQON_PROXY_ACCUMULATE) {
    if (!dB_inc || !A || r <= 0) return FALQON_ERR_INVALID_ARG;
  }
  if (flags & FALQON_PROXY_TENSOR) {
    if (r % 8 != 0 || N > (int64_t(1) << 31) - 256 || K > (int64_t(1) << 31) - 256) return FALQON_ERR_UNSUPPORTED;
    if (!aligned16(dB_inc) || !aligned16(A)) return FALQON_ERR_UNSUPPORTED;
  }
  if (flags & FALQON_PROXY_SELECT) {
    if (!wq || !s_w) return FALQON_ERR_INVALID_ARG;
    if (!aligned16(wq)) return FALQON_ERR_UNSUPPORTED;
    falqon_status s = check_ws(proxy_workspace_bytes(N, K), workspace, workspace_bytes);
    if (s != FALQON_OK) return s;
  }
  if (!current_device_info()) return FALQON_ERR_CUDA;
  return from_cuda(launch_proxy_update(wq, s_w, proxy, dB_inc, A, N, K, r, flags, row_mask,
                                       n_selected, dev_status, workspace,
                                       static_cast<cudaStream_t>(stream)));
}

falqon_status falqon_proxy_update_topk(uint8_t* wq, const float* s_w, float* proxy_q,
                                       const void* dB_inc, const void* A, int64_t N, int64_t K,
                                       int64_t r, int64_t k, uint32_t flags, uint8_t* comp_mask,
                                       int32_t* n_selected, int32_t* dev_status, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  const uint32_t known = FALQON_PROXY_ACCUMULATE | FALQON_PROXY_SELECT | FALQON_PROXY_STRICT;
  if ((flags & (FALQON_PROXY_ACCUMULATE | FALQON_PROXY_SELECT)) == 0 || (flags & ~known))
    return FALQON_ERR_INVALID_ARG;
  if (!proxy_q || N <= 0 || K <= 0 || r <= 0 || k < 0) return FALQON_ERR_INVALID_ARG;
  if ((flags & FALQON_PROXY_ACCUMULATE) && !dB_inc) return FALQON_ERR_INVALID_ARG;
  const bool select = flags & FALQON_PROXY_SELECT;
  if (select && (!wq || !s_w || !A)) return FALQON_ERR_INVALID_ARG;
  if (K % 16 != 0 || N > INT32_MAX || r > kTopkMaxRank) return FALQON_ERR_UNSUPPORTED;
  if (select && (!aligned16(wq) || !aligned16(A))) return FALQON_ERR_UNSUPPORTED;
  if (select) {
    falqon_status s = check_ws(proxy_topk_workspace_bytes(N, K, r), workspace, workspace_bytes);
    if (s != FALQON_OK) return s;
  }
  if (!current_device_info()) return FALQON_ERR_CUDA;
  return from_cuda(launch_proxy_update_topk(wq, s_w, proxy_q, dB_inc, A, N, K, r, k, flags, comp_mask,
                                            n_selected, dev_status, workspace,
                                            static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Shape checks shared by the folded calls: the backbone's, plus r.
falqon_status folded_shape(int64_t M, int64_t N, int64_t K, int64_t r) {
  if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return FALQON_ERR_INVALID_ARG;
  if (N % 16 != 0 || K % 16 != 0 || r % 16 != 0 || r > 65536) return FALQON_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 256 || N > (int64_t(1) << 31) - 256 || K > (int64_t(1) << 31) - 256)
    return FALQON_ERR_UNSUPPORTED;
  return FALQON_OK;
}

}  // namespace

extern "C" {

falqon_status falqon_linear_fwd_folded(const uint8_t* xq, const float* s_x, const uint8_t* wq, const float* s_w,
                                       const uint8_t* aq, const float* s_a, int64_t M, int64_t N, int64_t K,
                                       int64_t r, void* y, void* t_saved, size_t t_saved_bytes,
                                       int32_t* dev_status, void* stream) {
  if (!xq || !s_x || !wq || !s_w || !aq || !s_a || !y) return FALQON_ERR_INVALID_ARG;
  falqon_status s = folded_shape(M, N, K, r);
  if (s != FALQON_OK) return s;
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(aq) || !aligned16(y)) return FALQON_ERR_UNSUPPORTED;
  const size_t plane = adapter_plane_bytes(M, r);
  s = check_ws(2 * plane, t_saved, t_saved_bytes);
  if (s != FALQON_OK) return s;
  if (!current_device_info()) return FALQON_ERR_CUDA;
  uint8_t* t = static_cast<uint8_t*>(t_saved);
  return from_cuda(launch_fp8_gemm_fwd_folded(xq, s_x, wq, s_w, aq, s_a, M, N, K, r, y, t, t + plane,
                                              adapter_tu_ld(M), dev_status, static_cast<cudaStream_t>(stream)));
}

falqon_status falqon_linear_bwd_folded(const uint8_t* dyq, const float* s_dy, const uint8_t* wq, const float* s_w,
                                       const uint8_t* bq, const float* s_b, const uint8_t* xq, const float* s_x,
                                       const void* t_saved, size_t t_saved_bytes, int64_t M, int64_t N, int64_t K,
                                       int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!dx && !dA && !dB) return FALQON_ERR_INVALID_ARG;
  if (!dyq || !s_dy) return FALQON_ERR_INVALID_ARG;
  falqon_status s = folded_shape(M, N, K, r);
  if (s != FALQON_OK) return s;
  if (!aligned16(dyq)) return FALQON_ERR_UNSUPPORTED;
  if (dx) {
    if (!wq || !s_w) return FALQON_ERR_INVALID_ARG;
    if (!aligned16(wq) || !aligned16(dx)) return FALQON_ERR_UNSUPPORTED;
  }
  const size_t plane = adapter_plane_bytes(M, r);
  if (dB) {
    if (!aligned16(dB)) return FALQON_ERR_UNSUPPORTED;
    if (!t_saved) return FALQON_ERR_INVALID_ARG;
    s = check_ws(2 * plane, t_saved, t_saved_bytes);
    if (s != FALQON_OK) return s;
  }
  if (dA) {
    if (!bq || !s_b || !xq || !s_x) return FALQON_ERR_INVALID_ARG;
    if (!aligned16(bq) || !aligned16(xq) || !aligned16(dA)) return FALQON_ERR_UNSUPPORTED;
    s = check_ws(2 * plane, workspace, workspace_bytes);
    if (s != FALQON_OK) return s;
  }
  if (!current_device_info()) return FALQON_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* u = static_cast<uint8_t*>(workspace);
  const int64_t ld = adapter_tu_ld(M);
  if (dx || dA) {
    cudaError_t e = launch_fp8_gemm_dx_folded(dyq, s_dy, wq, s_w, dA ? bq : nullptr, s_b, M, N, K, r, dx,
                                              dA ? u : nullptr, dA ? u + plane : nullptr, ld, dev_status, st);
    if (e != cudaSuccess) return from_cuda(e);
  }
  if (!dA && !dB) return FALQON_OK;
  const uint8_t* t = static_cast<const uint8_t*>(t_saved);
  return from_cuda(launch_adapter_stage2(dyq, s_dy, xq, s_x, dB ? t : nullptr, dB ? t + plane : nullptr,
                                         dA ? u : nullptr, dA ? u + plane : nullptr, ld, M, N, K, r, dA, dB,
                                         dev_status, st));
}

}  // extern "C"

namespace {

falqon_status separate_shape(int precision, int64_t M, int64_t N, int64_t K, int64_t r) {
  if (precision != FALQON_SEPARATE_BF16 && precision != FALQON_SEPARATE_FP8) return FALQON_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return FALQON_ERR_INVALID_ARG;
  if (N % 16 != 0 || K % 16 != 0 || r % 16 != 0 || r > 65536) return FALQON_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 256 || N > (int64_t(1) << 31) - 256 || K > (int64_t(1) << 31) - 256 ||
      (M + 31) / 32 > 65535)
    return FALQON_ERR_UNSUPPORTED;
  return FALQON_OK;
}

}  // namespace

extern "C" {

falqon_status falqon_lora_separate_fwd(int precision, const uint8_t* xq, const float* s_x, const void* x,
                                       const uint8_t* wq, const float* s_w, const void* A, const void* B, int64_t M,
                                       int64_t N, int64_t K, int64_t r, void* y, void* saved, size_t saved_bytes,
                                       int32_t* dev_status, void* workspace, size_t workspace_bytes, void* stream) {
  falqon_status s = separate_shape(precision, M, N, K, r);
  if (s != FALQON_OK) return s;
  const bool fp8 = precision == FALQON_SEPARATE_FP8;
  if (!xq || !s_x || !wq || !s_w || !A || !B || !y || !saved) return FALQON_ERR_INVALID_ARG;
  if (!fp8 && !x) return FALQON_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(A) || !aligned16(B) || !aligned16(y) ||
      (x && !aligned16(x)))
    return FALQON_ERR_UNSUPPORTED;
  s = check_ws(separate_saved_bytes(fp8, M, N, K, r), saved, saved_bytes);
  if (s != FALQON_OK) return s;
  s = check_ws(separate_fwd_workspace_bytes(fp8, M, N, K, r), workspace, workspace_bytes);
  if (s != FALQON_OK) return s;
  if (!current_device_info()) return FALQON_ERR_CUDA;
  return from_cuda(launch_separate_fwd(fp8, xq, s_x, x, wq, s_w, A, B, M, N, K, r, y, saved, dev_status, workspace,
                                       static_cast<cudaStream_t>(stream)));
}

falqon_status falqon_lora_separate_bwd(int precision, const uint8_t* dyq, const float* s_dy, const void* dy,
                                       const uint8_t* wq, const float* s_w, const uint8_t* xq, const float* s_x,
                                       const void* x, const void* A, const void* B, const void* saved,
                                       size_t saved_bytes, int64_t M, int64_t N, int64_t K, int64_t r, void* dx,
                                       void* dA, void* dB, int32_t* dev_status, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  falqon_status s = separate_shape(precision, M, N, K, r);
  if (s != FALQON_OK) return s;
  const bool fp8 = precision == FALQON_SEPARATE_FP8;
  if (!dx && !dA && !dB) return FALQON_ERR_INVALID_ARG;
  if (!dyq || !s_dy || !A || !B || !saved) return FALQON_ERR_INVALID_ARG;
  if (dx && (!wq || !s_w)) return FALQON_ERR_INVALID_ARG;
  if (!fp8 && !dy) return FALQON_ERR_INVALID_ARG;
  if (dA && (fp8 ? (!xq || !s_x) : !x)) return FALQON_ERR_INVALID_ARG;
  if (!aligned16(dyq) || !aligned16(A) || !aligned16(B) || (dy && !aligned16(dy)) || (wq && !aligned16(wq)) ||
      (xq && !aligned16(xq)) || (x && !aligned16(x)) || (dx && !aligned16(dx)) || (dA && !aligned16(dA)) ||
      (dB && !aligned16(dB)))
    return FALQON_ERR_UNSUPPORTED;
  s = check_ws(separate_saved_bytes(fp8, M, N, K, r), saved, saved_bytes);
  if (s != FALQON_OK) return s;
  s = check_ws(separate_bwd_workspace_bytes(fp8, M, N, K, r), workspace, workspace_bytes);
  if (s != FALQON_OK) return s;
  if (!current_device_info()) return FALQON_ERR_CUDA;
  return from_cuda(launch_separate_bwd(fp8, dyq, s_dy, dy, wq, s_w, xq, s_x, x, A, B, saved, M, N, K, r, dx, dA, dB,
                                       dev_status, workspace, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

extern "C" {

falqon_status falqon_linear_fwd_grouped(const uint8_t* xq, const float* s_x, int nseg, const uint8_t* const* wq,
                                        const float* const* s_w, const int64_t* N, void* const* y, int64_t M,
                                        int64_t K, int32_t* dev_status, void* stream) {
  if (!xq || !s_x || !wq || !s_w || !N || !y) return FALQON_ERR_INVALID_ARG;
  if (nseg < 1 || nseg > 3 || M <= 0 || K <= 0) return FALQON_ERR_INVALID_ARG;
  if (K % 16 != 0 || M > (int64_t(1) << 31) - 256 || K > (int64_t(1) << 31) - 256) return FALQON_ERR_UNSUPPORTED;
  if (!aligned16(xq)) return FALQON_ERR_UNSUPPORTED;
  int64_t tiles = 0;
  for (int s = 0; s < nseg; ++s) {
    if (!wq[s] || !s_w[s] || !y[s] || N[s] <= 0) return FALQON_ERR_INVALID_ARG;
    if (N[s] % 16 != 0 || N[s] > (int64_t(1) << 31) - 256) return FALQON_ERR_UNSUPPORTED;
    if (!aligned16(wq[s]) || !aligned16(y[s])) return FALQON_ERR_UNSUPPORTED;
    tiles += (N[s] + 255) / 256;
  }
  if (tiles * ((M + 127) / 128) > (int64_t(1) << 30)) return FALQON_ERR_UNSUPPORTED;
  if (!current_device_info()) return FALQON_ERR_CUDA;
  return from_cuda(launch_fp8_gemm_fwd_grouped(xq, s_x, nseg, wq, s_w, N, y, M, K, dev_status,
                                               static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
