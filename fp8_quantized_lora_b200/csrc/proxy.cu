// Row-wise proxy update of the FP8 backbone.
//
// FALQON (abstract and introduction): a row-wise proxy accumulates the
// adapter updates and only the substantial ones are applied to the quantized
// backbone; updates that would vanish under quantization are skipped.
//
// This implementation:
//   accumulate_flag_kernel  (grid over 32 x 256 tiles of P)
//     D = dB_inc . A as a float32 fused-multiply-add chain in index order
//     i = 0..r-1 starting from +0 (each thread keeps an 8 x 4 register tile;
//     A and dB_inc are staged through shared memory in chunks of 32 i), then
//     P' = P + D.  With SELECT it also forms t = dec(Wq) + s_W * P' and
//     c' = E4M3(t) and records, per (row, column tile), whether any code
//     changes value.  Writes P' back (ACCUMULATE).
//   select_rows_kernel  (grid over rows)
//     ORs a row's column-tile flags; selected rows get Wq = c' (recomputed
//     from P' exactly as above) and P = +0.  Writes the row mask and adds to
//     the selected-row count (zeroed by the first kernel).
// The float32 chain is what the hardware FMA computes, so the result is
// reproducible bit-for-bit.
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace falqon {
namespace {

constexpr int kTileRows = 32;
constexpr int kTileCols = 256;
constexpr int kIChunk = 32;
constexpr int kThreads = 256;  // 4 row groups of 8 rows x 64 column groups of 4 columns

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Exact value of one E4M3 code (hardware conversion through f16).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h2;
  const uint16_t c = static_cast<uint16_t>(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

__device__ __forceinline__ uint32_t e4m3_code(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// Two codes hold the same value: identical non-NaN codes, or both zero.
__device__ __forceinline__ bool same_value(uint32_t a, uint32_t b) {
  const bool nan = ((a & 0x7Fu) == 0x7Fu) || ((b & 0x7Fu) == 0x7Fu);
  return !nan && (a == b || ((a & 0x7Fu) == 0u && (b & 0x7Fu) == 0u));
}

// New code for one element: E4M3( dec(c) + s_w * p ), no fused multiply-add.
__device__ __forceinline__ uint32_t requantized(uint32_t c, float s_w, float p) {
  return e4m3_code(__fadd_rn(e4m3_value(c), __fmul_rn(s_w, p)));
}

template <bool kAccumulate, bool kSelect>
__global__ void __launch_bounds__(kThreads)
    accumulate_flag_kernel(const uint8_t* __restrict__ wq, const float* __restrict__ s_w_ptr,
                           float* __restrict__ proxy, const uint16_t* __restrict__ dB_inc,
                           const uint16_t* __restrict__ A, int64_t N, int64_t K, int64_t r,
                           uint8_t* __restrict__ flags, int n_ct, int32_t* n_selected,
                           int32_t* dev_status) {
  __shared__ __align__(16) float As[kIChunk][kTileCols];
  __shared__ __align__(16) float Bs[kIChunk][kTileRows];
  __shared__ int row_changed[kTileRows];

  const int ct = blockIdx.x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTileRows;
  const int64_t c0 = static_cast<int64_t>(ct) * kTileCols;
  const int tc = threadIdx.x & 63;  // column group: columns c0 + 4*tc .. +3
  const int tr = threadIdx.x >> 6;  // row group: rows r0 + 8*tr .. +7
  if (kSelect && threadIdx.x < kTileRows) row_changed[threadIdx.x] = 0;
  if (kSelect && n_selected && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
    *n_selected = 0;

  float acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[j][c] = 0.0f;

  if constexpr (kAccumulate) {
    for (int64_t i0 = 0; i0 < r; i0 += kIChunk) {
      const int ni = static_cast<int>(r - i0 < kIChunk ? r - i0 : kIChunk);
      __syncthreads();
      // stage A[i0 : i0+ni, c0 : c0+256] and dB_inc[r0 : r0+32, i0 : i0+ni] as float32
      for (int e = threadIdx.x; e < kIChunk * kTileCols; e += kThreads) {
        const int i = e / kTileCols, c = e % kTileCols;
        const int64_t gc = c0 + c;
        As[i][c] = (i < ni && gc < K) ? bf16_bits_to_f32(A[(i0 + i) * K + gc]) : 0.0f;
      }
      for (int e = threadIdx.x; e < kIChunk * kTileRows; e += kThreads) {
        const int i = e / kTileRows, rr = e % kTileRows;
        const int64_t gr = r0 + rr;
        Bs[i][rr] = (i < ni && gr < N) ? bf16_bits_to_f32(dB_inc[gr * r + i0 + i]) : 0.0f;
      }
      __syncthreads();
      for (int i = 0; i < ni; ++i) {
        const float4 a = *reinterpret_cast<const float4*>(&As[i][4 * tc]);
        const float4 b0 = *reinterpret_cast<const float4*>(&Bs[i][8 * tr]);
        const float4 b1 = *reinterpret_cast<const float4*>(&Bs[i][8 * tr + 4]);
        const float av[4] = {a.x, a.y, a.z, a.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[j][c] = __fmaf_rn(bv[j], av[c], acc[j][c]);
      }
    }
  }
  if (kSelect) __syncthreads();  // row_changed initialised before anyone sets it

  const float s_w = kSelect ? *s_w_ptr : 1.0f;
  const int64_t col = c0 + 4 * tc;
  bool nonfinite = false;
  if (col < K) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t row = r0 + 8 * tr + j;
      if (row >= N) break;
      float4* pp = reinterpret_cast<float4*>(proxy + row * K + col);
      float4 p = *pp;
      if constexpr (kAccumulate) {
        p.x = __fadd_rn(p.x, acc[j][0]);
        p.y = __fadd_rn(p.y, acc[j][1]);
        p.z = __fadd_rn(p.z, acc[j][2]);
        p.w = __fadd_rn(p.w, acc[j][3]);
        *pp = p;
      }
      nonfinite |= !(isfinite(p.x) && isfinite(p.y) && isfinite(p.z) && isfinite(p.w));
      if constexpr (kSelect) {
        const uint32_t w4 = *reinterpret_cast<const uint32_t*>(wq + row * K + col);
        const float pv[4] = {p.x, p.y, p.z, p.w};
        bool changed = false;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t old = (w4 >> (8 * c)) & 0xFFu;
          changed |= !same_value(requantized(old, s_w, pv[c]), old);
        }
        if (changed) row_changed[8 * tr + j] = 1;
      }
    }
  }
  if (__any_sync(0xFFFFFFFFu, nonfinite) && (threadIdx.x & 31) == 0 && dev_status)
    atomicOr(dev_status, kDevNonfinite);
  if constexpr (kSelect) {
    __syncthreads();
    if (threadIdx.x < kTileRows) {
      const int64_t row = r0 + threadIdx.x;
      if (row < N) flags[row * n_ct + ct] = static_cast<uint8_t>(row_changed[threadIdx.x]);
    }
  }
}

constexpr int kSelThreads = 256;

__global__ void __launch_bounds__(kSelThreads)
    select_rows_kernel(uint8_t* __restrict__ wq, const float* __restrict__ s_w_ptr,
                       float* __restrict__ proxy, int64_t N, int64_t K,
                       const uint8_t* __restrict__ flags, int n_ct, uint8_t* row_mask,
                       int32_t* n_selected) {
  const float s_w = *s_w_ptr;
  int my_count = 0;
  for (int64_t row = blockIdx.x; row < N; row += gridDim.x) {
    int f = 0;
    for (int t = threadIdx.x; t < n_ct; t += kSelThreads) f |= flags[row * n_ct + t];
    const int sel = __syncthreads_or(f);
    if (threadIdx.x == 0) {
      if (row_mask) row_mask[row] = static_cast<uint8_t>(sel ? 1 : 0);
      my_count += sel ? 1 : 0;
    }
    if (!sel) continue;
    for (int64_t c = 4 * static_cast<int64_t>(threadIdx.x); c < K; c += 4 * kSelThreads) {
      float4* pp = reinterpret_cast<float4*>(proxy + row * K + c);
      const float4 p = *pp;
      uint32_t* wp = reinterpret_cast<uint32_t*>(wq + row * K + c);
      const uint32_t w4 = *wp;
      const float pv[4] = {p.x, p.y, p.z, p.w};
      uint32_t out = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) out |= requantized((w4 >> (8 * j)) & 0xFFu, s_w, pv[j]) << (8 * j);
      *wp = out;
      *pp = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
  }
  if (threadIdx.x == 0 && my_count && n_selected) atomicAdd(n_selected, my_count);
}

}  // namespace

size_t proxy_workspace_bytes(int64_t N, int64_t K) {
  const int64_t n_ct = (K + kTileCols - 1) / kTileCols;
  return align_up(static_cast<size_t>(N * n_ct), 256);
}

cudaError_t launch_proxy_update(uint8_t* wq, const float* s_w, float* proxy, const void* dB_inc,
                                const void* A, int64_t N, int64_t K, int64_t r, uint32_t flags,
                                uint8_t* row_mask, int32_t* n_selected, int32_t* dev_status,
                                void* workspace, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  const bool acc = flags & 1u, sel = flags & 2u;
  const int n_ct = static_cast<int>((K + kTileCols - 1) / kTileCols);
  const dim3 grid(n_ct, static_cast<unsigned>((N + kTileRows - 1) / kTileRows));
  uint8_t* fl = static_cast<uint8_t*>(workspace);
  const uint16_t* dB = static_cast<const uint16_t*>(dB_inc);
  const uint16_t* Am = static_cast<const uint16_t*>(A);
  if (acc && sel)
    accumulate_flag_kernel<true, true><<<grid, kThreads, 0, stream>>>(
        wq, s_w, proxy, dB, Am, N, K, r, fl, n_ct, n_selected, dev_status);
  else if (acc)
    accumulate_flag_kernel<true, false><<<grid, kThreads, 0, stream>>>(
        wq, s_w, proxy, dB, Am, N, K, r, fl, n_ct, n_selected, dev_status);
  else
    accumulate_flag_kernel<false, true><<<grid, kThreads, 0, stream>>>(
        wq, s_w, proxy, dB, Am, N, K, r, fl, n_ct, n_selected, dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !sel) return e;
  int64_t blocks = N < static_cast<int64_t>(di->sm_count) * 8 ? N : static_cast<int64_t>(di->sm_count) * 8;
  select_rows_kernel<<<static_cast<int>(blocks), kSelThreads, 0, stream>>>(
      wq, s_w, proxy, N, K, fl, n_ct, row_mask, n_selected);
  return cudaGetLastError();
}

}  // namespace falqon
