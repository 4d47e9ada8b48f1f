// Separate LoRA paths beside the FP8 backbone: the comparison FALQON is set
// against, not FALQON's own path.
//
// The paper's introduction sets FALQON against LoRA kept as a separate path
// beside an FP8 backbone, where every small adapter product pays its own
// quantization; the OpenReview rebuttals compare FP8 and FP16 adapters
// across ranks (reviewer 2, W4, Table R1; reviewer 3, Q3, Table R6).  Here
// the adapter branch is a separate layer of four products, each rounded to
// bf16, added to the backbone's bf16 output as bf16 tensors add:
//   forward   S = X A^T,  Y = Ybb + S B^T
//   backward  G = dY B,   dX = dXbb + G A,  dB = dY^T S,  dA = G^T X
// in bf16 (kind::f16 on the same tcgen05 GEMM) or with every operand
// quantized to E4M3 right before its product (X and dY reuse the backbone's
// codes; A and B are quantized each call, S and G once formed).  The
// branch's sum with the backbone output is fused into the epilogue of the
// GEMM that forms the branch (the backbone output is its addend).  The
// products over the token dimension (dB, dA) read S^T and G^T, which one
// small transpose kernel forms; dB^T is transposed back to [N, r].
#include "../../include/falqon.h"
#include "internal.h"
#include "ptx.cuh"

namespace falqon {
namespace {

constexpr int kTr = 32;  // transpose tile

// out[c][r] = in[r][c] for an [rows, cols] row-major tensor of T; the rows of
// out are ld_out elements apart.
template <typename T>
__global__ void __launch_bounds__(kTr * 8)
    transpose_kernel(const T* __restrict__ in, T* __restrict__ out, int64_t rows, int64_t cols, int64_t ld_out) {
  pdl_trigger();
  pdl_wait();
  __shared__ T tile[kTr][kTr + 1];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTr, c0 = static_cast<int64_t>(blockIdx.x) * kTr;
  for (int j = threadIdx.y; j < kTr; j += 8) {
    const int64_t r = r0 + j, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[j][threadIdx.x] = in[r * cols + c];
  }
  __syncthreads();
  for (int j = threadIdx.y; j < kTr; j += 8) {
    const int64_t c = c0 + j, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[c * ld_out + r] = tile[threadIdx.x][j];
  }
}

template <typename T>
cudaError_t transpose(const void* in, void* out, int64_t rows, int64_t cols, int64_t ld_out, cudaStream_t stream) {
  const int64_t gy = (rows + kTr - 1) / kTr, gx = (cols + kTr - 1) / kTr;
  if (gy > 65535 || gx > (int64_t(1) << 31) - 1) return cudaErrorInvalidValue;
  return launch_pdl(transpose_kernel<T>, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                    dim3(kTr, 8), 0, stream, 1u, static_cast<const T*>(in), static_cast<T*>(out), rows, cols,
                    ld_out);
}

// Row stride (elements) of the transposed [r][M] operands: M rounded up to 16,
// so that every row starts on a 16-byte boundary (a TMA stride).
int64_t ldt(int64_t M) { return (M + 15) / 16 * 16; }

size_t a256(size_t v) { return align_up(v, 256); }

// Regions of the forward's saved buffer (kept for the backward).
struct Saved {
  size_t s, sq, aq, bq, scales, total;  // byte offsets; scales: s_S, s_A, s_B
};
Saved saved_layout(bool fp8, int64_t M, int64_t N, int64_t K, int64_t r) {
  Saved L{};
  size_t o = 0;
  L.s = o;
  o += a256(static_cast<size_t>(M) * r * 2);
  if (fp8) {
    L.sq = o;
    o += a256(static_cast<size_t>(M) * r);
    L.aq = o;
    o += a256(static_cast<size_t>(r) * K);
    L.bq = o;
    o += a256(static_cast<size_t>(N) * r);
    L.scales = o;
    o += 256;
  }
  L.total = o;
  return L;
}

// Regions of the backward's workspace; the quantize workspace comes first
// (it must be initialised once, as falqon.h says of quantize workspaces).
struct Bwd {
  size_t qws, g, gq, st, gt, dbt, scales, total;  // scales: s_G
};
Bwd bwd_layout(bool fp8, int64_t M, int64_t N, int64_t r) {
  Bwd L{};
  size_t o = 0;
  L.qws = o;
  o += a256(quantize_workspace_bytes(M * r));
  L.g = o;
  o += a256(static_cast<size_t>(M) * r * 2);
  L.gq = o;
  if (fp8) o += a256(static_cast<size_t>(M) * r);
  L.st = o;  // S^T (bf16) or Sq^T (codes), [r][ldt(M)]
  o += a256(static_cast<size_t>(ldt(M)) * r * (fp8 ? 1 : 2));
  L.gt = o;  // G^T or Gq^T
  o += a256(static_cast<size_t>(ldt(M)) * r * (fp8 ? 1 : 2));
  L.dbt = o;
  o += a256(static_cast<size_t>(N) * r * 2);
  L.scales = o;
  o += 256;
  L.total = o;
  return L;
}

}  // namespace

size_t separate_saved_bytes(bool fp8, int64_t M, int64_t N, int64_t K, int64_t r) {
  return saved_layout(fp8, M, N, K, r).total;
}
size_t separate_fwd_workspace_bytes(bool fp8, int64_t M, int64_t N, int64_t K, int64_t r) {
  (void)M, (void)N, (void)K, (void)r;
  return fp8 ? a256(quantize_workspace_bytes(0)) : 0;
}
size_t separate_bwd_workspace_bytes(bool fp8, int64_t M, int64_t N, int64_t K, int64_t r) {
  (void)K;
  return bwd_layout(fp8, M, N, r).total;
}

cudaError_t launch_separate_fwd(bool fp8, const uint8_t* xq, const float* s_x, const void* x, const uint8_t* wq,
                                const float* s_w, const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                                int64_t r, void* y, void* saved, int32_t* dev_status, void* workspace,
                                cudaStream_t st) {
  const Saved L = saved_layout(fp8, M, N, K, r);
  uint8_t* sv = static_cast<uint8_t*>(saved);
  void* S = sv + L.s;
  // backbone: Y = bf16(Xq . Wq^T / (s_X s_W)); the adapter branch is added onto it
  cudaError_t e = launch_fp8_gemm_fwd(xq, s_x, wq, s_w, M, N, K, y, dev_status, st);
  if (e != cudaSuccess) return e;
  if (!fp8) {
    e = launch_gemm_nt(true, x, nullptr, A, nullptr, M, r, K, S, nullptr, dev_status, st);  // S = bf16(X A^T)
    if (e != cudaSuccess) return e;
    return launch_gemm_nt(true, S, nullptr, B, nullptr, M, N, r, y, y, dev_status, st);   // Y += bf16(S B^T)
  }
  uint8_t* sq = sv + L.sq;
  uint8_t* aq = sv + L.aq;
  uint8_t* bq = sv + L.bq;
  float* scales = reinterpret_cast<float*>(sv + L.scales);  // s_S, s_A, s_B
  e = launch_quantize(A, true, r * K, aq, scales + 1, nullptr, nullptr, dev_status, workspace, st);
  if (e != cudaSuccess) return e;
  e = launch_quantize(B, true, N * r, bq, scales + 2, nullptr, nullptr, dev_status, workspace, st);
  if (e != cudaSuccess) return e;
  e = launch_gemm_nt(false, xq, s_x, aq, scales + 1, M, r, K, S, nullptr, dev_status, st);  // S
  if (e != cudaSuccess) return e;
  e = launch_quantize(S, true, M * r, sq, scales, nullptr, nullptr, dev_status, workspace, st);  // Sq
  if (e != cudaSuccess) return e;
  return launch_gemm_nt(false, sq, scales, bq, scales + 2, M, N, r, y, y, dev_status, st);  // Y += bf16(Sq Bq^T)
}

cudaError_t launch_separate_bwd(bool fp8, const uint8_t* dyq, const float* s_dy, const void* dy, const uint8_t* wq,
                                const float* s_w, const uint8_t* xq, const float* s_x, const void* x,
                                const void* A, const void* B, const void* saved, int64_t M, int64_t N, int64_t K,
                                int64_t r, void* dx, void* dA, void* dB, int32_t* dev_status, void* workspace,
                                cudaStream_t st) {
  const Saved S = saved_layout(fp8, M, N, K, r);
  const Bwd W = bwd_layout(fp8, M, N, r);
  const uint8_t* sv = static_cast<const uint8_t*>(saved);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* G = ws + W.g;
  void* ST = ws + W.st;
  void* GT = ws + W.gt;
  void* dBT = ws + W.dbt;
  cudaError_t e;
  if (dx) {  // backbone: dX = bf16(dYq . Wq / (s_dY s_W)); the branch is added onto it
    e = launch_fp8_gemm_dx(dyq, s_dy, wq, s_w, M, N, K, dx, dev_status, st);
    if (e != cudaSuccess) return e;
  }
  if (!fp8) {
    e = launch_gemm_nn(true, dy, nullptr, B, nullptr, M, r, N, G, nullptr, dev_status, st);  // G = bf16(dY B)
    if (e != cudaSuccess) return e;
    if (dx) {
      e = launch_gemm_nn(true, G, nullptr, A, nullptr, M, K, r, dx, dx, dev_status, st);  // dX += bf16(G A)
      if (e != cudaSuccess) return e;
    }
    if (dB) {
      e = transpose<uint16_t>(sv + S.s, ST, M, r, ldt(M), st);
      if (e != cudaSuccess) return e;
      e = launch_gemm_nn(true, ST, nullptr, dy, nullptr, r, N, M, dBT, nullptr, dev_status, st, ldt(M));  // (dY^T S)^T
      if (e != cudaSuccess) return e;
      e = transpose<uint16_t>(dBT, dB, r, N, r, st);
      if (e != cudaSuccess) return e;
    }
    if (dA) {
      e = transpose<uint16_t>(G, GT, M, r, ldt(M), st);
      if (e != cudaSuccess) return e;
      e = launch_gemm_nn(true, GT, nullptr, x, nullptr, r, K, M, dA, nullptr, dev_status, st, ldt(M));  // G^T X
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  const uint8_t* sq = sv + S.sq;
  const uint8_t* aq = sv + S.aq;
  const uint8_t* bq = sv + S.bq;
  const float* fs = reinterpret_cast<const float*>(sv + S.scales);  // s_S, s_A, s_B
  uint8_t* gq = ws + W.gq;
  float* s_g = reinterpret_cast<float*>(ws + W.scales);
  e = launch_gemm_nn(false, dyq, s_dy, bq, fs + 2, M, r, N, G, nullptr, dev_status, st);  // G
  if (e != cudaSuccess) return e;
  e = launch_quantize(G, true, M * r, gq, s_g, nullptr, nullptr, dev_status, ws + W.qws, st);  // Gq
  if (e != cudaSuccess) return e;
  if (dx) {
    e = launch_gemm_nn(false, gq, s_g, aq, fs + 1, M, K, r, dx, dx, dev_status, st);  // dX += bf16(Gq Aq)
    if (e != cudaSuccess) return e;
  }
  if (dB) {
    e = transpose<uint8_t>(sq, ST, M, r, ldt(M), st);
    if (e != cudaSuccess) return e;
    e = launch_gemm_nn(false, ST, fs, dyq, s_dy, r, N, M, dBT, nullptr, dev_status, st, ldt(M));  // (dYq^T Sq)^T
    if (e != cudaSuccess) return e;
    e = transpose<uint16_t>(dBT, dB, r, N, r, st);
    if (e != cudaSuccess) return e;
  }
  if (dA) {
    e = transpose<uint8_t>(gq, GT, M, r, ldt(M), st);
    if (e != cudaSuccess) return e;
    e = launch_gemm_nn(false, GT, s_g, xq, s_x, r, K, M, dA, nullptr, dev_status, st, ldt(M));  // Gq^T Xq
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace falqon
