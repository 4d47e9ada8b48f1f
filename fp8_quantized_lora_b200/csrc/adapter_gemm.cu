// Adapter products of the melded FP8 linear backward at large rank, on the
// bf16 tcgen05 GEMM (sm_100a):
//   T  = Xq . A^T / s_X      dB = dYq^T . T / s_dY
//   U  = dYq . B / s_dY      dA = U^T . Xq / s_X
// FALQON, OpenReview rebuttal (reviewer 4, Q1): B's gradient comes from the
// precomputable product A x; A's from B^T dL/dO.  The products read the
// E4M3 codes the quantize step produced (exact as bf16 values).
//
// The rank-on-M kernel of skinny.cu expands every code once per 128-rank
// tile, r / 128 times over; past a few hundred ranks the four products are
// plain large GEMMs.  Here the codes are expanded to bf16 once, T and U are
// formed in float32 (exact bf16 products summed in float32), split into bf16
// hi + lo planes (about 16 significant bits), and dB and dA take the hi and lo
// planes stacked along M in one GEMM each, whose two halves are added in
// float32 and rounded once to bf16.  Nine launches for dB and dA together.
#include "internal.h"
#include "tc_common.cuh"

namespace falqon {
namespace {

constexpr int kAgThreads = 256;

// codes [n] -> bf16 values [n], 16 codes per step (n % 16 == 0); a batch of 16
// holding a NaN code (an E5M2 infinity or NaN) takes the hardware conversion.
template <bool kE5>
__global__ void __launch_bounds__(kAgThreads)
    expand_codes_kernel(const uint8_t* __restrict__ codes, __nv_bfloat16* __restrict__ out, int64_t n16) {
  pdl_trigger();
  pdl_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n16; u += stride) {
    const uint4 q = reinterpret_cast<const uint4*>(codes)[u];
    const uint32_t fold = kE5 ? special5_fold(0u, q) : nan_fold(0u, q);
    uint32_t o[8];
    if (kE5) e5m2x16_to_bf16(q, nan_found(fold), o);
    else e4m3x16_to_bf16(q, nan_found(fold), o);
    uint4* dst = reinterpret_cast<uint4*>(out) + 2 * u;
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(v);
  lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

// in [R][C] float32 (rows ldi apart) -> hi [R][ldo], lo [R][ldo] bf16 with hi + lo ~ in.
__global__ void __launch_bounds__(kAgThreads)
    split_rows_kernel(const float* __restrict__ in, int64_t ldi, __nv_bfloat16* __restrict__ hi,
                      __nv_bfloat16* __restrict__ lo, int64_t ldo, int64_t R, int64_t C) {
  pdl_trigger();
  pdl_wait();
  const int64_t total = R * C, stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += stride) {
    const int64_t i = e / C, c = e % C;
    split_bf16(in[i * ldi + c], hi[i * ldo + c], lo[i * ldo + c]);
  }
}

constexpr int kAgTile = 32;

// in [Rin][Cin] float32 -> hi/lo [Cin][ldo] bf16, transposed: out[c][r] = in[r][c].
__global__ void __launch_bounds__(kAgTile * 8)
    transpose_split_kernel(const float* __restrict__ in, int64_t Rin, int64_t Cin, __nv_bfloat16* __restrict__ hi,
                           __nv_bfloat16* __restrict__ lo, int64_t ldo) {
  pdl_trigger();
  pdl_wait();
  __shared__ float tile[kAgTile][kAgTile + 1];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kAgTile, c0 = static_cast<int64_t>(blockIdx.x) * kAgTile;
  for (int j = threadIdx.y; j < kAgTile; j += 8) {
    const int64_t r = r0 + j, c = c0 + threadIdx.x;
    if (r < Rin && c < Cin) tile[j][threadIdx.x] = in[r * Cin + c];
  }
  __syncthreads();
  for (int j = threadIdx.y; j < kAgTile; j += 8) {
    const int64_t c = c0 + j, r = r0 + threadIdx.x;
    if (r < Rin && c < Cin) split_bf16(tile[threadIdx.x][j], hi[c * ldo + r], lo[c * ldo + r]);
  }
}

// in [2R][C] float32 (the hi rows, then the lo rows) -> out bf16 of
// fl32(in[i][c] + in[R + i][c]): [R][C] rows ldo apart, or transposed [C][ldo].
template <bool kTranspose>
__global__ void __launch_bounds__(kAgTile * 8)
    sum_halves_kernel(const float* __restrict__ in, int64_t R, int64_t C, __nv_bfloat16* __restrict__ out,
                      int64_t ldo) {
  pdl_trigger();
  pdl_wait();
  __shared__ float tile[kAgTile][kAgTile + 1];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kAgTile, c0 = static_cast<int64_t>(blockIdx.x) * kAgTile;
  for (int j = threadIdx.y; j < kAgTile; j += 8) {
    const int64_t r = r0 + j, c = c0 + threadIdx.x;
    if (r < R && c < C) {
      const float v = __fadd_rn(in[r * C + c], in[(R + r) * C + c]);
      if constexpr (kTranspose) tile[j][threadIdx.x] = v;
      else out[r * ldo + c] = __float2bfloat16_rn(v);
    }
  }
  if constexpr (kTranspose) {
    __syncthreads();
    for (int j = threadIdx.y; j < kAgTile; j += 8) {
      const int64_t c = c0 + j, r = r0 + threadIdx.x;
      if (r < R && c < C) out[c * ldo + r] = __float2bfloat16_rn(tile[threadIdx.x][j]);
    }
  }
}

int grid_for(int64_t items, const DeviceInfo* di) {
  int64_t g = (items + kAgThreads - 1) / kAgThreads;
  const int64_t cap = static_cast<int64_t>(di->sm_count) * 8;
  return static_cast<int>(g < cap ? (g > 0 ? g : 1) : cap);
}

cudaError_t expand(const uint8_t* codes, int64_t n, __nv_bfloat16* out, bool e5, const DeviceInfo* di,
                   cudaStream_t stream) {
  const int64_t n16 = n / 16;
  return e5 ? launch_pdl(expand_codes_kernel<true>, dim3(grid_for(n16, di)), dim3(kAgThreads), 0, stream, 1u, codes,
                         out, n16)
            : launch_pdl(expand_codes_kernel<false>, dim3(grid_for(n16, di)), dim3(kAgThreads), 0, stream, 1u, codes,
                         out, n16);
}

dim3 tile_grid(int64_t rows, int64_t cols) {
  return dim3(static_cast<unsigned>((cols + kAgTile - 1) / kAgTile), static_cast<unsigned>((rows + kAgTile - 1) / kAgTile));
}

struct AgLayout {
  size_t xe, dye, f32a, planes, f32b, total;
  int64_t ld;
};

AgLayout ag_layout(int64_t M, int64_t N, int64_t K, int64_t r) {
  AgLayout L{};
  L.ld = adapter_tu_ld(M);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes, 256);
    return at;
  };
  L.xe = take(static_cast<size_t>(M) * K * 2);
  L.dye = take(static_cast<size_t>(M) * N * 2);
  L.f32a = take(static_cast<size_t>(r) * M * 4);                        // T [r][M], then U [M][r]
  L.planes = take(static_cast<size_t>(2 * r) * L.ld * 2);               // hi rows, then lo rows
  L.f32b = take(static_cast<size_t>(2 * r) * (N > K ? N : K) * 4);      // stacked dB^T, then dA
  L.total = off;
  return L;
}

}  // namespace

// Measured on the 4096-cube (M = N = K = 4096): the two launches of the
// rank-on-M kernel took 0.113 ms at r = 256 and 0.395 ms at r = 1024, this
// path 0.167 and 0.255 ms.
bool adapter_gemm_path(int64_t M, int64_t r) { return r >= 512 && M % 8 == 0; }

size_t adapter_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r) {
  return ag_layout(M, N, K, r).total;
}

cudaError_t launch_adapter_grads_gemm(const uint8_t* dyq, const float* s_dy, const uint8_t* xq, const float* s_x,
                                      const void* A, const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                                      void* dA, void* dB, int32_t* dev_status, void* workspace, cudaStream_t stream,
                                      bool dy_e5m2) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  if (!dA && !dB) return cudaSuccess;
  if ((2 * r + kAgTile - 1) / kAgTile > 65535 || (M + kAgTile - 1) / kAgTile > 65535) return cudaErrorInvalidValue;
  const AgLayout L = ag_layout(M, N, K, r);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto* xe = reinterpret_cast<__nv_bfloat16*>(ws + L.xe);
  auto* dye = reinterpret_cast<__nv_bfloat16*>(ws + L.dye);
  auto* f32a = reinterpret_cast<float*>(ws + L.f32a);
  auto* planes = reinterpret_cast<__nv_bfloat16*>(ws + L.planes);
  auto* f32b = reinterpret_cast<float*>(ws + L.f32b);
  __nv_bfloat16* lo_planes = planes + r * L.ld;
  const dim3 tb(kAgTile, 8);
  cudaError_t e = expand(xq, M * K, xe, false, di, stream);
  if (e == cudaSuccess) e = expand(dyq, M * N, dye, dy_e5m2, di, stream);
  if (e != cudaSuccess) return e;
  if (dB) {
    // T^T [r][M] = A . Xe^T / s_X, then its hi / lo planes
    e = launch_gemm_bf16_f32out(false, A, 0, xe, s_x, r, M, K, f32a, dev_status, stream);
    if (e == cudaSuccess)
      e = launch_pdl(split_rows_kernel, dim3(grid_for(r * M, di)), dim3(kAgThreads), 0, stream, 1u,
                     static_cast<const float*>(f32a), M, planes, lo_planes, L.ld, r, M);
    // [dB^T from hi; from lo] [2r][N] = [T_hi; T_lo] . dYe / s_dY, then dB [N][r] = bf16(hi + lo)
    if (e == cudaSuccess)
      e = launch_gemm_bf16_f32out(true, planes, L.ld, dye, s_dy, 2 * r, N, M, f32b, dev_status, stream);
    if (e == cudaSuccess)
      e = launch_pdl(sum_halves_kernel<true>, tile_grid(r, N), tb, 0, stream, 1u, static_cast<const float*>(f32b), r,
                     N, static_cast<__nv_bfloat16*>(dB), r);
    if (e != cudaSuccess) return e;
  }
  if (dA) {
    // U [M][r] = dYe . B / s_dY, then U^T's hi / lo planes
    e = launch_gemm_bf16_f32out(true, dye, 0, B, s_dy, M, r, N, f32a, dev_status, stream);
    if (e == cudaSuccess)
      e = launch_pdl(transpose_split_kernel, tile_grid(M, r), tb, 0, stream, 1u, static_cast<const float*>(f32a), M, r,
                     planes, lo_planes, L.ld);
    // [dA from hi; from lo] [2r][K] = [U_hi^T; U_lo^T] . Xe / s_X, then dA [r][K] = bf16(hi + lo)
    if (e == cudaSuccess)
      e = launch_gemm_bf16_f32out(true, planes, L.ld, xe, s_x, 2 * r, K, M, f32b, dev_status, stream);
    if (e == cudaSuccess)
      e = launch_pdl(sum_halves_kernel<false>, tile_grid(r, K), tb, 0, stream, 1u, static_cast<const float*>(f32b), r,
                     K, static_cast<__nv_bfloat16*>(dA), K);
  }
  return e;
}

}  // namespace falqon
