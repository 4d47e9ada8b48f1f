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

// Values of the two codes in the low 16 bits of `c2` (hardware conversion via f16).
__device__ __forceinline__ float2 e4m3x2_values(uint32_t c2) {
  uint32_t h2;
  const uint16_t c = static_cast<uint16_t>(c2);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  __half2 h;
  memcpy(&h, &h2, 4);
  return __half22float2(h);
}

// Four codes (bytes of w4) -> four new codes E4M3(dec(c) + s_w * p), no FMA.
__device__ __forceinline__ uint32_t requantized4(uint32_t w4, float s_w, float4 p) {
  const float2 d01 = e4m3x2_values(w4);
  const float2 d23 = e4m3x2_values(w4 >> 16);
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
      : "=h"(lo)
      : "f"(__fadd_rn(d01.y, __fmul_rn(s_w, p.y))), "f"(__fadd_rn(d01.x, __fmul_rn(s_w, p.x))));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
      : "=h"(hi)
      : "f"(__fadd_rn(d23.y, __fmul_rn(s_w, p.w))), "f"(__fadd_rn(d23.x, __fmul_rn(s_w, p.z))));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Does any of the four byte pairs differ in value (+0 == -0; a NaN code differs)?
__device__ __forceinline__ bool codes_changed4(uint32_t a, uint32_t b) {
  bool changed = false;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    changed |= !same_value((a >> (8 * c)) & 0xFFu, (b >> (8 * c)) & 0xFFu);
  return changed;
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

// ---------------------------------------------------------------- single pass
// One cluster of `cs` CTAs owns a row group of `rb` rows at a time; CTA q of
// the cluster owns the column slice [q*wc, (q+1)*wc) for the whole kernel and
// keeps A[:, slice] resident in shared memory (bf16, converted exactly to
// float32 at use).  Each thread holds kRT rows x 4 columns of P' = P + D in
// registers; the per-row "some code changes" bits are OR-ed inside the CTA,
// published in shared memory and OR-ed across the cluster through DSMEM
// after one cluster barrier per row group.  Then every element is written
// once: P' (row kept) or +0 and the new codes (row selected).  Traffic per
// element: read P and Wq, write P, and write Wq only for selected rows.
constexpr int kRT = 8;  // rows per thread

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

__device__ __forceinline__ uint32_t dsmem_load_u32(const uint32_t* local, uint32_t rank) {
  uint32_t remote, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

// 4-byte store into cluster CTA `rank`'s shared memory at the same offset as
// `local_dst`, counted as 4 transaction bytes on that CTA's mbarrier at the
// offset of `local_bar`.
__device__ __forceinline__ void st_async_u32(uint32_t* local_dst, uint64_t* local_bar,
                                             uint32_t rank, uint32_t value) {
  uint32_t rdst, rbar;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rdst) : "r"(smem_u32(local_dst)), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(smem_u32(local_bar)), "r"(rank));
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(rdst),
               "r"(value), "r"(rbar)
               : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

struct ProxyGeom {
  int cs, wc, cg, rs, rb, threads;
  size_t smem;
};

template <bool kAcc, bool kSel>
__global__ void __launch_bounds__(256, 2)
    proxy_cluster_kernel(uint8_t* __restrict__ wq, const float* __restrict__ s_w_ptr,
                         float* __restrict__ proxy, const uint16_t* __restrict__ dB_inc,
                         const uint16_t* __restrict__ A, int64_t N, int64_t K, int r,
                         ProxyGeom geo, int n_groups, uint8_t* row_mask, int32_t* n_selected,
                         int32_t* dev_status) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int wc = geo.wc, cg = geo.cg, rb = geo.rb, cs = geo.cs;
  uint16_t* As = reinterpret_cast<uint16_t*>(sm);                       // [r][wc] bf16
  const size_t as_bytes = align_up(static_cast<size_t>(r) * wc * 2, 16);
  // [2][r][rb] pairs (b, b): the FFMA2 operand comes straight from a broadcast load
  float2* Bs0 = reinterpret_cast<float2*>(sm + as_bytes);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(Bs0 + 2 * static_cast<size_t>(r) * rb);  // [2]
  uint32_t* xbuf = reinterpret_cast<uint32_t*>(mbar + 2);  // [2] this CTA's row bits
  uint32_t* inbox = xbuf + 2;                              // [2][16] row bits from each CTA
  __shared__ int abort_flag;

  const uint32_t crank = cs > 1 ? cluster_ctarank() : 0u;
  const int n_clusters = gridDim.x / cs;
  const int tid = threadIdx.x;
  const int tcg = tid % cg;
  const int trs = tid / cg;
  const bool active = trs < geo.rs;
  const int64_t c0 = static_cast<int64_t>(crank) * wc;
  const int64_t col = c0 + 4 * tcg;
  const bool col_ok = active && (4 * tcg < wc) && col < K;

  // A[:, slice] -> shared memory, once (16-byte chunks; K % 8 == 0 keeps them aligned)
  if constexpr (kAcc) {
    const int chunks = wc / 8;
    for (int e = tid; e < r * chunks; e += blockDim.x) {
      const int i = e / chunks, c8 = e % chunks;
      const int64_t gc = c0 + 8 * c8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (gc < K) v = *reinterpret_cast<const uint4*>(A + static_cast<int64_t>(i) * K + gc);
      *reinterpret_cast<uint4*>(As + static_cast<size_t>(i) * wc + 8 * c8) = v;
    }
  }
  if (tid < 2) xbuf[tid] = 0u;
  if (tid == 0) {
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  const float s_w = kSel ? *s_w_ptr : 1.0f;

  // dB_inc rows of a group -> (registers) -> Bs[buffer] as float32, [i][row]
  constexpr int kMaxB = 8;  // rb * r <= 32 * 1024 elements over >= 32 threads... bounded below
  const int per_thread_b = (rb * r + blockDim.x - 1) / blockDim.x;
  auto load_b = [&](int g, uint16_t (&v)[kMaxB], int k0) {
#pragma unroll
    for (int k = 0; k < kMaxB; ++k) {
      const int e = tid + (k0 + k) * blockDim.x;
      v[k] = 0;
      if (k0 + k < per_thread_b && e < rb * r) {
        const int row = e / r, i = e % r;
        const int64_t n = static_cast<int64_t>(g) * rb + row;
        if (n < N) v[k] = dB_inc[n * r + i];
      }
    }
  };
  auto store_b = [&](const uint16_t (&v)[kMaxB], int k0, float2* dst) {
#pragma unroll
    for (int k = 0; k < kMaxB; ++k) {
      const int e = tid + (k0 + k) * blockDim.x;
      if (k0 + k < per_thread_b && e < rb * r) {
        const int row = e / r, i = e % r;
        const float f = bf16_bits_to_f32(v[k]);
        dst[static_cast<size_t>(i) * rb + row] = make_float2(f, f);
      }
    }
  };
  auto stage_b = [&](int g, float2* dst) {
    for (int k0 = 0; k0 < per_thread_b; k0 += kMaxB) {
      uint16_t v[kMaxB];
      load_b(g, v, k0);
      store_b(v, k0, dst);
    }
  };
  int g = blockIdx.x / cs;
  if (kAcc && g < n_groups) stage_b(g, Bs0);
  __syncthreads();
  int local_count = 0;
  bool nonfinite = false;
  for (int it = 0; g < n_groups; g += n_clusters, ++it) {
    const int64_t n0 = static_cast<int64_t>(g) * rb;
    const int b = it & 1;
    float2* Bs = Bs0 + b * static_cast<size_t>(r) * rb;

    // this group's P and Wq: pulled from HBM into L2 now (no registers held),
    // read from L2 after the FMA chain
#pragma unroll
    for (int j = 0; j < kRT; ++j) {
      const int64_t n = n0 + trs * kRT + j;
      if (col_ok && n < N) {
        prefetch_l2(proxy + n * K + col);
        if (kSel && (tcg & 3) == 0) prefetch_l2(wq + n * K + col);
      }
    }
    // next group's dB_inc, also in flight during the FMA chain (first kMaxB per thread)
    const int g_next = g + n_clusters;
    uint16_t bnext[kMaxB];
    if (kAcc && g_next < n_groups) load_b(g_next, bnext, 0);

    float2 acc[kRT][2];
#pragma unroll
    for (int j = 0; j < kRT; ++j) acc[j][0] = acc[j][1] = make_float2(0.0f, 0.0f);
    if constexpr (kAcc) {
      if (active) {
        const uint16_t* arow = As + 4 * tcg;
        const float2* brow = Bs + trs * kRT;
#pragma unroll 4
        for (int i = 0; i < r; ++i) {
          const uint2 a2 = *reinterpret_cast<const uint2*>(arow);
          const float2 a01 = make_float2(__uint_as_float(a2.x << 16), __uint_as_float(a2.x & 0xFFFF0000u));
          const float2 a23 = make_float2(__uint_as_float(a2.y << 16), __uint_as_float(a2.y & 0xFFFF0000u));
          float2 bb[kRT];
#pragma unroll
          for (int j = 0; j < kRT; j += 2) {
            const float4 q = *reinterpret_cast<const float4*>(brow + j);
            bb[j] = make_float2(q.x, q.y);
            bb[j + 1] = make_float2(q.z, q.w);
          }
#pragma unroll
          for (int j = 0; j < kRT; ++j) {
            acc[j][0] = __ffma2_rn(bb[j], a01, acc[j][0]);
            acc[j][1] = __ffma2_rn(bb[j], a23, acc[j][1]);
          }
          arow += wc;
          brow += rb;
        }
      }
    }

    // next group's dB_inc into the other buffer (its readers finished a group ago)
    if (kAcc && g_next < n_groups) {
      float2* dst = Bs0 + (b ^ 1) * static_cast<size_t>(r) * rb;
      store_b(bnext, 0, dst);
      for (int k0 = kMaxB; k0 < per_thread_b; k0 += kMaxB) {
        uint16_t v[kMaxB];
        load_b(g_next, v, k0);
        store_b(v, k0, dst);
      }
    }

    float4 p[kRT];
    uint32_t w[kRT];
#pragma unroll
    for (int j = 0; j < kRT; ++j) {
      const int64_t n = n0 + trs * kRT + j;
      if (col_ok && n < N) {
        p[j] = *reinterpret_cast<const float4*>(proxy + n * K + col);
        if (kSel) w[j] = *reinterpret_cast<const uint32_t*>(wq + n * K + col);
      }
    }

    // P' = P + D, new codes, per-row change bits
    uint32_t cnew[kRT];
    uint32_t mymask = 0;
#pragma unroll
    for (int j = 0; j < kRT; ++j) {
      const int64_t n = n0 + trs * kRT + j;
      cnew[j] = 0;
      if (col_ok && n < N) {
        if constexpr (kAcc) {
          p[j].x = __fadd_rn(p[j].x, acc[j][0].x);
          p[j].y = __fadd_rn(p[j].y, acc[j][0].y);
          p[j].z = __fadd_rn(p[j].z, acc[j][1].x);
          p[j].w = __fadd_rn(p[j].w, acc[j][1].y);
        }
        nonfinite |= !(isfinite(p[j].x) && isfinite(p[j].y) && isfinite(p[j].z) && isfinite(p[j].w));
        if constexpr (kSel) {
          cnew[j] = requantized4(w[j], s_w, p[j]);
          if (codes_changed4(w[j], cnew[j])) mymask |= 1u << (trs * kRT + j);
        }
      }
    }

    uint32_t rowsel = 0;
    if constexpr (kSel) {
      uint32_t* xb = xbuf + b;
      const uint32_t m = __reduce_or_sync(0xFFFFFFFFu, mymask);
      if ((tid & 31) == 0 && m) atomicOr(xb, m);
      __syncthreads();  // this CTA's bits are complete in xb
      uint32_t* box = inbox + 16 * b;
      if (cs > 1) {
        // all-gather of the row bits: push this CTA's word into every CTA's
        // inbox (slot = own rank), each push counted on that CTA's mbarrier
        if (tid == 0) {
          mbar_arrive_expect_tx(&mbar[b], 4u * static_cast<uint32_t>(cs));
          const uint32_t mine = *xb;
          for (int q = 0; q < cs; ++q) st_async_u32(box + crank, &mbar[b], static_cast<uint32_t>(q), mine);
        }
        // phase of mbar[b] used by group `it` is (it >> 1) & 1; one warp polls,
        // the others sleep in the barrier below instead of spinning
        if (tid < 32) {
          const bool ok = mbar_wait(&mbar[b], static_cast<uint32_t>((it >> 1) & 1), &abort_flag);
          if (!__all_sync(0xFFFFFFFFu, ok) && tid == 0) {
            abort_flag = 1;
            if (dev_status) atomicOr(dev_status, kDevTimeout);
          }
        }
        __syncthreads();
        for (int q = 0; q < cs; ++q) rowsel |= box[q];
      } else {
        rowsel = *xb;
      }
    }
    __syncthreads();  // everyone has rowsel; next Bs staged
    if (kSel && tid == 0) xbuf[b] = 0u;  // reused two groups from now, after another barrier
    if (abort_flag) break;

#pragma unroll
    for (int j = 0; j < kRT; ++j) {
      const int64_t n = n0 + trs * kRT + j;
      if (col_ok && n < N) {
        const bool sel = kSel && ((rowsel >> (trs * kRT + j)) & 1u);
        float4* pp = reinterpret_cast<float4*>(proxy + n * K + col);
        if (sel) {
          *reinterpret_cast<uint32_t*>(wq + n * K + col) = cnew[j];
          *pp = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        } else if (kAcc) {
          *pp = p[j];
        }
      }
    }
    if (kSel && crank == 0 && tid < rb && n0 + tid < N) {
      const uint32_t sel = (rowsel >> tid) & 1u;
      if (row_mask) row_mask[n0 + tid] = static_cast<uint8_t>(sel);
      local_count += static_cast<int>(sel);
    }
  }
  if (__any_sync(0xFFFFFFFFu, nonfinite) && (tid & 31) == 0 && dev_status)
    atomicOr(dev_status, kDevNonfinite);
  if (kSel && n_selected && local_count) atomicAdd(n_selected, local_count);
  if (cs > 1) cluster_sync_all();  // no CTA leaves while a peer may still push into it
}

// Picks the cluster split of K; returns false when A's slice does not fit.
bool plan_proxy(int64_t K, int64_t r, ProxyGeom* geo) {
  // about 512 columns per CTA; clusters of up to 8 (portable) or 16 CTAs
  int cs = static_cast<int>((K + 511) / 512);
  if (cs < 1) cs = 1;
  if (cs > 8) cs = 16;
  int wc = static_cast<int>((K + cs - 1) / cs);
  wc = (wc + 7) / 8 * 8;
  const int cg = wc / 4;
  if (cg > 256) return false;
  int rs = 256 / cg;
  if (rs > 4) rs = 4;
  if (rs < 1) rs = 1;
  const int rb = kRT * rs;  // <= 32 rows: one bit each in a 32-bit mask
  const int threads = (cg * rs + 31) / 32 * 32;
  const size_t smem = align_up(static_cast<size_t>(r) * wc * 2, 16) +
                      2 * static_cast<size_t>(r) * rb * sizeof(float2) + 16 + 8 + 128;
  if (smem > 200 * 1024) return false;
  *geo = ProxyGeom{cs, wc, cg, rs, rb, threads, smem};
  return true;
}

template <bool kAcc, bool kSel>
cudaError_t launch_proxy_cluster(const ProxyGeom& geo, uint8_t* wq, const float* s_w, float* proxy,
                                 const void* dB_inc, const void* A, int64_t N, int64_t K, int r,
                                 uint8_t* row_mask, int32_t* n_selected, int32_t* dev_status,
                                 cudaStream_t stream) {
  auto kern = proxy_cluster_kernel<kAcc, kSel>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(geo.smem));
  if (e != cudaSuccess) return e;
  if (geo.cs > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = geo.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(geo.threads);
  cfg.dynamicSmemBytes = geo.smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters = 0;
  cfg.gridDim = dim3(geo.cs);
  e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
  if (e != cudaSuccess) return e;
  if (max_clusters < 1) return cudaErrorInvalidConfiguration;
  const int n_groups = static_cast<int>((N + geo.rb - 1) / geo.rb);
  int clusters = max_clusters < n_groups ? max_clusters : n_groups;
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * geo.cs));
  return cudaLaunchKernelEx(&cfg, kern, wq, s_w, proxy, static_cast<const uint16_t*>(dB_inc),
                            static_cast<const uint16_t*>(A), N, K, r, geo, n_groups, row_mask,
                            n_selected, dev_status);
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
  const DeviceInfo* di0 = current_device_info();
  if (!di0) return cudaErrorInvalidDevice;
  ProxyGeom geo;
  const bool acc0 = flags & 1u, sel0 = flags & 2u;
  if (r <= 1024 && plan_proxy(K, acc0 ? r : 0, &geo)) {
    if (sel0 && n_selected) {
      cudaError_t e0 = cudaMemsetAsync(n_selected, 0, sizeof(int32_t), stream);
      if (e0 != cudaSuccess) return e0;
    }
    const int rr = acc0 ? static_cast<int>(r) : 0;
    cudaError_t e1;
    if (acc0 && sel0)
      e1 = launch_proxy_cluster<true, true>(geo, wq, s_w, proxy, dB_inc, A, N, K, rr, row_mask,
                                            n_selected, dev_status, stream);
    else if (acc0)
      e1 = launch_proxy_cluster<true, false>(geo, wq, s_w, proxy, dB_inc, A, N, K, rr, row_mask,
                                             n_selected, dev_status, stream);
    else
      e1 = launch_proxy_cluster<false, true>(geo, wq, s_w, proxy, dB_inc, A, N, K, rr, row_mask,
                                             n_selected, dev_status, stream);
    if (e1 == cudaSuccess) return cudaSuccess;
    if (e1 != cudaErrorInvalidConfiguration) return e1;
    (void)cudaGetLastError();  // no cluster fits: fall through to the two-kernel path
  }

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
