// Host-side declarations shared by the C-ABI layer and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "../../include/falqon.h"

namespace falqon {

struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int max_smem_optin = 0;
  int cc_major = 0;
  int cc_minor = 0;
  int coop_launch = 0;  // cooperative launches supported
};

// Cached per device; returns nullptr if the current device cannot be queried.
const DeviceInfo* current_device_info();

// Driver entry point for cuTensorMapEncodeTiled (resolved once).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// 2-D tensor map over a row-major [outer, inner] tensor whose rows are `ld`
// elements apart (0: ld = inner).
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, size_t elem_bytes,
                  const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                  uint32_t box_outer, bool swizzle128, uint64_t ld = 0);
// The same with the 64-byte swizzle (box_inner * elem_bytes == 64).
bool make_tmap_2d_sw64(CUtensorMap* map, CUtensorMapDataType dtype, size_t elem_bytes, const void* base,
                       uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer);

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Launches `kernel` with programmatic dependent launch allowed, so that its
// CTAs may start while the previous kernel in the stream drains; every
// kernel of the library calls pdl_wait() before it touches global memory.
// cluster_x > 1 also sets the cluster shape.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster_x > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster_x;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- quantize
size_t quantize_workspace_bytes(int64_t n);
cudaError_t launch_quantize(const void* x, bool is_bf16, int64_t n, uint8_t* codes,
                            float* scale, float* amax, float* residual, int32_t* dev_status,
                            void* workspace, cudaStream_t stream, bool e5m2 = false);

// ---------------------------------------------------------------- GEMMs
// Y[M,N] = bf16( Xq . Wq^T / (s_x s_w) )
cudaError_t launch_fp8_gemm_fwd(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                const float* s_w, int64_t M, int64_t N, int64_t K, void* y,
                                int32_t* dev_status, cudaStream_t stream);
// Y_s[M, N_s] = bf16( Xq . Wq_s^T / (s_x s_w_s) ), s < nseg <= 3: one launch over
// the concatenated output tiles of backbones that read the same Xq.
cudaError_t launch_fp8_gemm_fwd_grouped(const uint8_t* xq, const float* s_x, int nseg, const uint8_t* const* wq,
                                        const float* const* s_w, const int64_t* n, void* const* y, int64_t M,
                                        int64_t K, int32_t* dev_status, cudaStream_t stream);
// dX[M,K] = bf16( dYq . Wq / (s_dy s_w) )
cudaError_t launch_fp8_gemm_dx(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                               const float* s_w, int64_t M, int64_t N, int64_t K, void* dx,
                               int32_t* dev_status, cudaStream_t stream, bool dy_e5m2 = false);

// The same two products on pairs of SMs (tcgen05 cta_group::2, 256 x 256
// tiles); launch_fp8_gemm_fwd / _dx route here.
cudaError_t launch_fp8_gemm_fwd_pair(const uint8_t* xq, const float* s_x, const uint8_t* wq, const float* s_w,
                                     int64_t M, int64_t N, int64_t K, void* y, int32_t* dev_status,
                                     cudaStream_t stream);
cudaError_t launch_fp8_gemm_dx_pair(const uint8_t* dyq, const float* s_dy, const uint8_t* wq, const float* s_w,
                                    int64_t M, int64_t N, int64_t K, void* dx, int32_t* dev_status,
                                    cudaStream_t stream, bool dy_e5m2);

// Plain products on the tcgen05 GEMM: C[M, Ncols] = bf16(A . op(B) / (sa sb)),
// then, when addend is not null, bf16(fl32(C + addend)) (bf16 tensors adding).
// A [M, Kc] K-major.  _nt: B [Ncols, Kc] (K-major);  _nn: B [Kc, Ncols] (MN-major).
// bf16: operands are bf16 (kind::f16) and the scales may be null; else E4M3 codes.
cudaError_t launch_gemm_nt(bool bf16, const void* a, const float* sa, const void* b, const float* sb, int64_t M,
                           int64_t Ncols, int64_t Kc, void* out, const void* addend, int32_t* dev_status,
                           cudaStream_t stream);
// lda: elements between rows of A (0: Kc); a multiple of 16 bytes.
cudaError_t launch_gemm_nn(bool bf16, const void* a, const float* sa, const void* b, const float* sb, int64_t M,
                           int64_t Ncols, int64_t Kc, void* out, const void* addend, int32_t* dev_status,
                           cudaStream_t stream, int64_t lda = 0);

// out[M, Ncols] (float32) = fl32(out + A . B): A [M, Kc] and B [Kc, Ncols]
// bf16, float32 accumulation on the tensor cores (kind::f16).
// out [M, Ncols] float32 = fl32(product / *sb) (sb nullable: 1), bf16 operands:
// A [M, Kc] K-major (rows lda elements apart, 0: Kc); B [Ncols, Kc] K-major or,
// with b_mn, [Kc, Ncols].
cudaError_t launch_gemm_bf16_f32out(bool b_mn, const void* a, int64_t lda, const void* b, const float* sb, int64_t M,
                                    int64_t Ncols, int64_t Kc, float* out, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_gemm_nn_f32acc(const void* a, const void* b, int64_t M, int64_t Ncols, int64_t Kc, float* out,
                                  int32_t* dev_status, cudaStream_t stream);

size_t adapter_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, bool want_da);
// Every argument check of falqon_linear_bwd except the workspace's (returns
// the status that call would return before launching, or FALQON_OK).
falqon_status linear_bwd_validate(const uint8_t* dyq, const float* s_dy, const uint8_t* wq, const float* s_w,
                                  const uint8_t* xq, const float* s_x, const void* A, const void* B, int64_t M,
                                  int64_t N, int64_t K, int64_t r, const void* dx, const void* dA,
                                  const void* dB);
cudaError_t launch_adapter_grads(const uint8_t* dyq, const float* s_dy, const uint8_t* xq,
                                 const float* s_x, const void* A, const void* B, int64_t M,
                                 int64_t N, int64_t K, int64_t r, void* dA, void* dB,
                                 int32_t* dev_status, void* workspace, cudaStream_t stream, bool dy_e5m2 = false);
// dB / dA from T and U held as transposed bf16 hi/lo planes [r][ld]
cudaError_t launch_adapter_stage2(const uint8_t* dyq, const float* s_dy, const uint8_t* xq, const float* s_x,
                                  const void* T_hi, const void* T_lo, const void* U_hi, const void* U_lo,
                                  int64_t ld, int64_t M, int64_t N, int64_t K, int64_t r, void* dA, void* dB,
                                  int32_t* dev_status, cudaStream_t stream, bool dy_e5m2 = false);
// Large ranks (adapter_gemm.cu): the adapter products on the bf16 GEMM, with
// the codes expanded once; used by launch_adapter_grads when adapter_gemm_path.
bool adapter_gemm_path(int64_t M, int64_t r);
size_t adapter_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r);
cudaError_t launch_adapter_grads_gemm(const uint8_t* dyq, const float* s_dy, const uint8_t* xq, const float* s_x,
                                      const void* A, const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                                      void* dA, void* dB, int32_t* dev_status, void* workspace, cudaStream_t stream,
                                      bool dy_e5m2);
// Row stride (elements) of a transposed T / U plane: M rounded up to 8.
inline int64_t adapter_tu_ld(int64_t M) { return (M + 7) / 8 * 8; }
// Bytes of one [r][ld] bf16 plane, padded to 256.
inline size_t adapter_plane_bytes(int64_t M, int64_t r) {
  return align_up(static_cast<size_t>(adapter_tu_ld(M)) * static_cast<size_t>(r) * 2, 256);
}

// Folded quantized adapters: the backbone GEMMs with the adapter columns
// appended (T = Xq . A~q^T / (s_x s_a), U = dYq . B~q / (s_dy s_b)), written
// transposed as bf16 hi/lo planes [r][ld].  y / dx may be null (adapter
// columns only); bq may be null in the dX launch (no U).
cudaError_t launch_fp8_gemm_fwd_folded(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                       const float* s_w, const uint8_t* aq, const float* s_a, int64_t M,
                                       int64_t N, int64_t K, int64_t r, void* y, void* t_hi, void* t_lo,
                                       int64_t ld, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_fp8_gemm_dx_folded(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                                      const float* s_w, const uint8_t* bq, const float* s_b, int64_t M,
                                      int64_t N, int64_t K, int64_t r, void* dx, void* u_hi, void* u_lo,
                                      int64_t ld, int32_t* dev_status, cudaStream_t stream);

// ---------------------------------------------------------------- separate LoRA paths
size_t separate_saved_bytes(bool fp8, int64_t M, int64_t N, int64_t K, int64_t r);
size_t separate_fwd_workspace_bytes(bool fp8, int64_t M, int64_t N, int64_t K, int64_t r);
size_t separate_bwd_workspace_bytes(bool fp8, int64_t M, int64_t N, int64_t K, int64_t r);
cudaError_t launch_separate_fwd(bool fp8, const uint8_t* xq, const float* s_x, const void* x, const uint8_t* wq,
                                const float* s_w, const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                                int64_t r, void* y, void* saved, int32_t* dev_status, void* workspace,
                                cudaStream_t stream);
cudaError_t launch_separate_bwd(bool fp8, const uint8_t* dyq, const float* s_dy, const void* dy, const uint8_t* wq,
                                const float* s_w, const uint8_t* xq, const float* s_x, const void* x,
                                const void* A, const void* B, const void* saved, int64_t M, int64_t N, int64_t K,
                                int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status, void* workspace,
                                cudaStream_t stream);

// ---------------------------------------------------------------- proxy
size_t proxy_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_proxy_update(uint8_t* wq, const float* s_w, float* proxy, const void* dB_inc,
                                const void* A, int64_t N, int64_t K, int64_t r, uint32_t flags,
                                uint8_t* row_mask, int32_t* n_selected, int32_t* dev_status,
                                void* workspace, cudaStream_t stream);
// Top-k over the r rank components: Q [r, N] float32 (row i: the unmerged
// part of B's column i).  flags: 1 accumulate, 2 select / merge / clear.
constexpr int64_t kTopkMaxRank = 16384;  // the select kernel keeps r 8-byte keys in shared memory
size_t proxy_topk_workspace_bytes(int64_t N, int64_t K, int64_t r);
cudaError_t launch_proxy_update_topk(uint8_t* wq, const float* s_w, float* Q, const void* dB_inc,
                                     const void* A, int64_t N, int64_t K, int64_t r, int64_t k,
                                     uint32_t flags, uint8_t* comp_mask, int32_t* n_selected,
                                     int32_t* dev_status, void* workspace, cudaStream_t stream);

}  // namespace falqon
