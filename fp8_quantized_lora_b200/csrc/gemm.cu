// tcgen05 GEMMs of the melded FP8 linear layer (sm_100a).
//
// One persistent, warp-specialised kernel template serves every product of
// the step:
//   forward    Y  = Xq  . Wq^T           kind::f8f6f4, A K-major, B K-major
//   dX         dX = dYq . Wq             kind::f8f6f4, A K-major, B MN-major
//   adapter T  T  = Xq  . A^T            kind::f16 (bf16), codes expanded in smem
//   adapter U  U  = dYq . B              kind::f16, B MN-major
//   dB         dB = dYq^T . T            kind::f16, A and B MN-major
//   dA^T       dA^T = Xq^T . U           kind::f16, A and B MN-major
// FALQON's point (paper introduction) is that the forward and dX run on the
// FP8 backbone alone; the adapter products only see the codes that the
// quantize step already produced, so no extra quantization happens here.
//
// Roles (one CTA per SM, persistent over output tiles / K splits):
//   warp 0      TMA producer (one lane): fills a `kStages`-deep smem ring.
//   warp 1      TMEM owner and UMMA issuer (one lane issues, the warp waits).
//   warps 2-5   epilogue: tcgen05.ld of the accumulator, scale, store.
//   warps 6-9   (bf16 kinds only) converters: E4M3 codes -> bf16 in the
//               128-byte-swizzled operand layout, exact (every E4M3 value is
//               a bf16 value).
// The accumulator lives in TMEM, double-buffered (2 x BN fp32 columns), so
// the epilogue of one tile overlaps the MMAs of the next.
//
// Every operand tile in smem is a stack of 128-byte rows in the SWIZZLE_128B
// layout TMA writes: K-major tiles are [rows][128 B of K]; MN-major tiles are
// 128-byte-wide column blocks of [K rows][128 B of M/N], LBO apart.
#include <algorithm>
#include <cfloat>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace falqon {
namespace {

constexpr int kBM = 128;       // UMMA M (cta_group::1)
constexpr int kRowBytes = 128;  // every smem operand row is one 128-byte swizzle row

struct GemmArgs {
  int32_t m_tiles, n_tiles, splits, kb_total, kb_per_split;
  int64_t M, N;            // output extent (rows = UMMA M side, cols = UMMA N side)
  void* out;               // bf16 [M, N] (ld = ldo) or fp32 partials [splits][m_pad][n_pad]
  int64_t ldo;
  int64_t m_pad, n_pad;    // partial-buffer extents
  const float* scale_a;    // alpha = 1 / (scale_a * scale_b); either may be null (= 1)
  const float* scale_b;
  int32_t* dev_status;
};

template <bool kF8, bool kAMn, bool kBMn, bool kAConv, int kBN, int kStages, bool kPartial,
          bool kBSplit = false>
struct Cfg {
  static constexpr bool F8 = kF8;
  static constexpr bool AMn = kAMn;
  static constexpr bool BMn = kBMn;
  static constexpr bool AConv = kAConv;
  static constexpr int BN = kBN;
  static constexpr int Stages = kStages;
  static constexpr bool Partial = kPartial;
  static constexpr bool BSplit = kBSplit;  // B = B_hi + B_lo: two bf16 tiles, two MMAs per k-step
  static constexpr int ElemBytes = kF8 ? 1 : 2;
  static constexpr int BK = kRowBytes / ElemBytes;       // K per stage (128 fp8 / 64 bf16)
  static constexpr int UmmaK = 32 / ElemBytes;           // K per UMMA instruction
  static constexpr int KSteps = BK / UmmaK;              // 4
  static constexpr int ABytes = kBM * BK * ElemBytes;     // operand A tile (16 KB)
  static constexpr int BBytes = kBN * BK * ElemBytes;     // operand B tile
  static constexpr int B2Bytes = kBSplit ? BBytes : 0;   // low half of a split B operand
  static constexpr int RawBytes = kAConv ? kBM * BK : 0;  // fp8 codes of A before expansion
  static constexpr int StageBytes = ABytes + BBytes + B2Bytes + RawBytes;
  static constexpr int TmaBytes = (kAConv ? RawBytes : ABytes) + BBytes + B2Bytes;
  static constexpr int NumConvWarps = kAConv ? 4 : 0;
  static constexpr int Threads = 32 * (6 + NumConvWarps);
  static constexpr uint32_t TmemCols = 2 * kBN < 32 ? 32 : 2 * kBN;
  static constexpr int BarBytes = 8 * (3 * kStages + 5) + 16;
  static constexpr int SmemBytes = kStages * StageBytes + BarBytes + 1024;
  static constexpr uint32_t IDesc =
      idesc_f32acc(kF8 ? 0u : 1u, kF8 ? 0u : 1u, kAMn ? 1u : 0u, kBMn ? 1u : 0u, kBM, kBN);
  static_assert(kBN % 16 == 0 && kBN >= 16 && kBN <= 256, "UMMA N");
  static_assert(!kBMn || (kBN * ElemBytes) % kRowBytes == 0, "MN-major B needs 128-byte blocks");
  static_assert(!kAConv || !kF8, "expansion feeds the bf16 kind only");
  static_assert(SmemBytes <= 232448, "shared memory per CTA");
};

// Descriptor of operand tile `base` for UMMA k-step `ks`.
template <bool kMn, int kElemBytes, int kKRows>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int ks) {
  if constexpr (kMn) {
    // k-step = (32 / elem) K-rows of 128 bytes; column blocks are kKRows rows apart
    return sdesc_sw128(base + ks * (32 / kElemBytes) * kRowBytes, kKRows * kRowBytes, 1024);
  } else {
    // k-step = 32 bytes along the swizzled 128-byte row
    return sdesc_sw128(base + ks * 32, 16, 1024);
  }
}

// Expands `kRows x kCols` E4M3 codes (row-major, unswizzled) into bf16 in the
// SWIZZLE_128B layout: 64-element column blocks of [kRows][128 B], each
// 16-byte unit of a row XOR-ed with (row % 8).
template <int kRows, int kCols>
__device__ __forceinline__ void expand_codes(const uint8_t* raw, uint8_t* dst, int t,
                                             int nthreads) {
  constexpr int kGroups = kRows * kCols / 8;
  for (int g = t; g < kGroups; g += nthreads) {
    const int row = g / (kCols / 8);
    const int col = (g % (kCols / 8)) * 8;
    const uint2 c = *reinterpret_cast<const uint2*>(raw + row * kCols + col);
    uint32_t out[4];
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint16_t pair = static_cast<uint16_t>(w[j >> 1] >> (16 * (j & 1)));
      uint32_t h2;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
      __half2 h;
      memcpy(&h, &h2, 4);
      const float2 f = __half22float2(h);
      const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
      memcpy(&out[j], &b, 4);
    }
    const int blk = col / 64;
    const int unit = (col % 64) / 8;
    uint8_t* p = dst + blk * (kRows * kRowBytes) + row * kRowBytes + ((unit ^ (row & 7)) << 4);
    *reinterpret_cast<uint4*>(p) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// All lanes wait; the warp agrees on the outcome so it never diverges on a timeout.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity,
                                          const volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ void raise_status(int32_t* st, int32_t bits) {
  if (st) atomicOr(st, bits);
}

template <class C>
__global__ void __launch_bounds__(C::Threads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const GemmArgs g) {
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::Stages * C::StageBytes);
  uint64_t* full = bars;                      // TMA landed
  uint64_t* conv = bars + C::Stages;          // codes expanded (bf16 kinds)
  uint64_t* empty = bars + 2 * C::Stages;     // MMAs done reading the stage
  uint64_t* acc_full = bars + 3 * C::Stages;  // [2] accumulator ready
  uint64_t* acc_empty = acc_full + 2;         // [2] accumulator drained
  uint64_t* drain = acc_empty + 2;            // all issued MMAs retired (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total = g.m_tiles * g.n_tiles * g.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&conv[s], C::NumConvWarps > 0 ? C::NumConvWarps : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if constexpr (C::BSplit) tma_prefetch_desc(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    raise_status(g.dev_status, kDevTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;  // per-stage: ever loaded / parity of last load
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int split = w % g.splits;
        const int nt = (w / g.splits) % g.n_tiles;
        const int mt = w / (g.splits * g.n_tiles);
        const int kb0 = split * g.kb_per_split;
        const int kb1 = min(g.kb_total, kb0 + g.kb_per_split);
        const int m0 = mt * kBM, n0 = nt * C::BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { fail(); ok = false; break; }
          uint8_t* sA = smem + stage * C::StageBytes;
          uint8_t* sB = sA + C::ABytes;
          uint8_t* sB2 = sB + C::BBytes;
          uint8_t* sRaw = sB2 + C::B2Bytes;
          mbar_arrive_expect_tx(&full[stage], C::TmaBytes);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          // operand A: rows m0.., K block kb
          if constexpr (C::AConv) {
            if constexpr (C::AMn) {
              tma_load_2d(sRaw, &tmA, &full[stage], m0, kb * C::BK);  // [BK rows][128 codes]
            } else {
              tma_load_2d(sRaw, &tmA, &full[stage], kb * C::BK, m0);  // [128 rows][BK codes]
            }
          } else if constexpr (C::AMn) {
#pragma unroll
            for (int c = 0; c < kBM * C::ElemBytes / kRowBytes; ++c)
              tma_load_2d(sA + c * C::BK * kRowBytes, &tmA, &full[stage],
                          m0 + c * (kRowBytes / C::ElemBytes), kb * C::BK);
          } else {
            tma_load_2d(sA, &tmA, &full[stage], kb * C::BK, m0);
          }
          // operand B: cols n0.., K block kb
          if constexpr (C::BMn) {
#pragma unroll
            for (int c = 0; c < C::BN * C::ElemBytes / kRowBytes; ++c) {
              tma_load_2d(sB + c * C::BK * kRowBytes, &tmB, &full[stage],
                          n0 + c * (kRowBytes / C::ElemBytes), kb * C::BK);
              if constexpr (C::BSplit)
                tma_load_2d(sB2 + c * C::BK * kRowBytes, &tmB2, &full[stage],
                            n0 + c * (kRowBytes / C::ElemBytes), kb * C::BK);
            }
          } else {
            tma_load_2d(sB, &tmB, &full[stage], kb * C::BK, n0);
            if constexpr (C::BSplit) tma_load_2d(sB2, &tmB2, &full[stage], kb * C::BK, n0);
          }
          if (++stage == C::Stages) { stage = 0; phase ^= 1; }
        }
      }
      // every load this lane issued must land before the CTA exits (matters
      // only after an abort; otherwise the MMA warp already consumed them)
      for (int s = 0; s < C::Stages; ++s)
        if (issued & (1u << s)) mbar_wait_budget(&full[s], (issued_parity >> s) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const int split = w % g.splits;
      const int kb0 = split * g.kb_per_split;
      const int kb1 = min(g.kb_total, kb0 + g.kb_per_split);
      if (!warp_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
      tc_fence_after();
      const uint32_t tmem_d = tmem_base + acc * C::BN;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!warp_wait(&full[stage], phase, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
        if constexpr (C::AConv) {
          if (!warp_wait(&conv[stage], phase, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_base = smem_u32(smem + stage * C::StageBytes);
          const uint32_t b_base = a_base + C::ABytes;
#pragma unroll
          for (int ks = 0; ks < C::KSteps; ++ks) {
            const uint64_t ad = operand_desc<C::AMn, C::ElemBytes, C::BK>(a_base, ks);
            const uint64_t bd = operand_desc<C::BMn, C::ElemBytes, C::BK>(b_base, ks);
            const uint32_t accum = (kb > kb0 || ks > 0) ? 1u : 0u;
            if constexpr (C::F8) umma_f8(tmem_d, ad, bd, C::IDesc, accum);
            else umma_bf16(tmem_d, ad, bd, C::IDesc, accum);
            if constexpr (C::BSplit) {
              const uint64_t bd2 = operand_desc<C::BMn, C::ElemBytes, C::BK>(b_base + C::BBytes, ks);
              umma_bf16(tmem_d, ad, bd2, C::IDesc, 1u);
            }
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::Stages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&acc_full[acc]);
      __syncwarp();
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    // drain the tensor pipe before TMEM is released
    if (lane == 0) {
      umma_commit(drain);
      mbar_wait_budget(drain, 0);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    float alpha = 1.0f;
    {
      double den = 1.0;
      if (g.scale_a) den *= static_cast<double>(*g.scale_a);
      if (g.scale_b) den *= static_cast<double>(*g.scale_b);
      alpha = static_cast<float>(1.0 / den);
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const int split = w % g.splits;
      const int nt = (w / g.splits) % g.n_tiles;
      const int mt = w / (g.splits * g.n_tiles);
      if (!warp_wait(&acc_full[acc], acc_phase, abort_flag)) { if (lane == 0) fail(); break; }
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mt) * kBM + q * 32 + lane;
      const int64_t col_base = static_cast<int64_t>(nt) * C::BN;
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::BN + c * 32, r);
        tmem_ld_wait();
        const int64_t col0 = col_base + c * 32;
        if constexpr (C::Partial) {
          float* dst = static_cast<float*>(g.out) +
                       (static_cast<int64_t>(split) * g.m_pad + row) * g.n_pad + col0;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            reinterpret_cast<float4*>(dst)[j] =
                make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                            __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
        } else {
          if (row < g.M) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.out) + row * g.ldo;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int64_t col = col0 + 8 * j;
              if (col < g.N) {
                uint32_t pk[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  const __nv_bfloat162 b = __floats2bfloat162_rn(
                      __uint_as_float(r[8 * j + 2 * h]) * alpha,
                      __uint_as_float(r[8 * j + 2 * h + 1]) * alpha);
                  memcpy(&pk[h], &b, 4);
                }
                *reinterpret_cast<uint4*>(dst + col) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  } else if constexpr (C::AConv) {
    // ------------------------------------------------------------ converters
    const int t = threadIdx.x - 6 * 32;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const int split = w % g.splits;
      const int kb0 = split * g.kb_per_split;
      const int kb1 = min(g.kb_total, kb0 + g.kb_per_split);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!warp_wait(&full[stage], phase, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
        uint8_t* sA = smem + stage * C::StageBytes;
        const uint8_t* sRaw = sA + C::ABytes + C::BBytes + C::B2Bytes;
        if constexpr (C::AMn) expand_codes<C::BK, kBM>(sRaw, sA, t, 128);
        else expand_codes<kBM, C::BK>(sRaw, sA, t, 128);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv[stage]);
        if (++stage == C::Stages) { stage = 0; phase ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TmemCols);
  }
}

// ---------------------------------------------------------------- reduce
// v = alpha * sum_s part[s] over [rows, cols] (fixed order s = 0..splits-1);
// out = bf16(v), and when `out_lo` is given out_lo = bf16(v - out), so that
// out + out_lo carries v to about 16 significant bits.  Transposed store
// (out[col][row]) when `transpose`.
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int splits, int64_t m_pad,
                                     int64_t n_pad, int64_t rows, int64_t cols,
                                     const float* scale_a, const float* scale_b, int transpose,
                                     __nv_bfloat16* __restrict__ out,
                                     __nv_bfloat16* __restrict__ out_lo) {
  double den = 1.0;
  if (scale_a) den *= static_cast<double>(*scale_a);
  if (scale_b) den *= static_cast<double>(*scale_b);
  const float alpha = static_cast<float>(1.0 / den);
  const int64_t n = rows * cols;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t r, c;
    if (transpose) {  // consecutive threads walk consecutive output elements out[c][r]
      c = i / rows;
      r = i % rows;
    } else {
      r = i / cols;
      c = i % cols;
    }
    float acc = 0.0f;
    for (int s = 0; s < splits; ++s) acc += part[(s * m_pad + r) * n_pad + c];
    const float v = acc * alpha;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    out[i] = hi;
    if (out_lo) out_lo[i] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

// ---------------------------------------------------------------- host side
template <class C>
cudaError_t launch_gemm(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tB2,
                        const GemmArgs& g, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  static int configured_mask = 0;  // one bit per device ordinal < 31
  const int bit = di->device < 31 ? (1 << di->device) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SmemBytes);
    if (e != cudaSuccess) return e;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_ACQ_REL);
  }
  const int total = g.m_tiles * g.n_tiles * g.splits;
  const int grid = total < di->sm_count ? total : di->sm_count;
  tc_gemm_kernel<C><<<grid, C::Threads, C::SmemBytes, stream>>>(tA, tB, tB2, g);
  return cudaGetLastError();
}

inline int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

using FwdCfg = Cfg<true, false, false, false, 256, 4, false>;
using DxCfg = Cfg<true, false, true, false, 256, 4, false>;

template <int BN> using TCfg = Cfg<false, false, false, true, BN, 4, true>;   // Xq . A^T
template <int BN> using UCfg = Cfg<false, false, true, true, BN, 4, true>;    // dYq . B
// dYq^T . (T_hi + T_lo), Xq^T . (U_hi + U_lo): fewer stages at BN = 256 to fit smem
template <int BN> using MnCfg = Cfg<false, true, true, true, BN, (BN >= 256 ? 2 : (BN >= 128 ? 3 : 4)), true, true>;

// Split count that fills the SMs with whole K blocks per split.
int choose_splits(int tiles, int kb_total, int sm_count) {
  int s = (sm_count + tiles - 1) / tiles;
  if (s > kb_total) s = kb_total;
  if (s < 1) s = 1;
  return s;
}

// Skinny product out[rows_out, r] (fp32 partials) then bf16 reduce.
// kind: 0 = T (A K-major conv, B K-major), 1 = U (A K-major conv, B MN-major),
//       2 = dB/dA^T (A MN-major conv, B MN-major).
template <template <int> class CF>
cudaError_t skinny_dispatch(int bn, const CUtensorMap& tA, const CUtensorMap& tB,
                            const CUtensorMap& tB2, GemmArgs& g, cudaStream_t stream) {
  switch (bn) {
    case 64: return launch_gemm<CF<64>>(tA, tB, tB2, g, stream);
    case 128: return launch_gemm<CF<128>>(tA, tB, tB2, g, stream);
    default: return launch_gemm<CF<256>>(tA, tB, tB2, g, stream);
  }
}

int skinny_bn(int64_t r) { return r <= 64 ? 64 : (r <= 128 ? 128 : 256); }

struct SkinnyPlan {
  int bn, m_tiles, n_tiles, kb_total, splits, kb_per_split;
  int64_t m_pad, n_pad;
};

SkinnyPlan plan_skinny(int64_t rows_out, int64_t r, int64_t kc, int sm_count) {
  SkinnyPlan p;
  p.bn = skinny_bn(r);
  p.m_tiles = ceil_div(rows_out, kBM);
  p.n_tiles = ceil_div(r, p.bn);
  p.kb_total = ceil_div(kc, 64);
  p.splits = choose_splits(p.m_tiles * p.n_tiles, p.kb_total, sm_count);
  p.kb_per_split = ceil_div(p.kb_total, p.splits);
  p.splits = ceil_div(p.kb_total, p.kb_per_split);  // no empty split
  p.m_pad = static_cast<int64_t>(p.m_tiles) * kBM;
  p.n_pad = static_cast<int64_t>(p.n_tiles) * p.bn;
  return p;
}

size_t plan_partial_bytes(const SkinnyPlan& p) {
  return static_cast<size_t>(p.splits) * p.m_pad * p.n_pad * sizeof(float);
}

cudaError_t launch_reduce(const float* part, const SkinnyPlan& p, int64_t rows, int64_t cols,
                          const float* sa, const float* sb, bool transpose, void* out,
                          void* out_lo, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  const int64_t n = rows * cols;
  int64_t blocks = (n + 255) / 256;
  if (blocks > di->sm_count * 8) blocks = di->sm_count * 8;
  splitk_reduce_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
      part, p.splits, p.m_pad, p.n_pad, rows, cols, sa, sb, transpose ? 1 : 0,
      static_cast<__nv_bfloat16*>(out), static_cast<__nv_bfloat16*>(out_lo));
  return cudaGetLastError();
}

}  // namespace

// ------------------------------------------------------------------ big GEMMs
cudaError_t launch_fp8_gemm_fwd(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                const float* s_w, int64_t M, int64_t N, int64_t K, void* y,
                                int32_t* dev_status, cudaStream_t stream) {
  CUtensorMap tA, tB;
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, K, M, 128, kBM, true) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq, K, N, 128, FwdCfg::BN, true))
    return cudaErrorInvalidValue;
  GemmArgs g{};
  g.m_tiles = ceil_div(M, kBM);
  g.n_tiles = ceil_div(N, FwdCfg::BN);
  g.splits = 1;
  g.kb_total = ceil_div(K, FwdCfg::BK);
  g.kb_per_split = g.kb_total;
  g.M = M;
  g.N = N;
  g.out = y;
  g.ldo = N;
  g.scale_a = s_x;
  g.scale_b = s_w;
  g.dev_status = dev_status;
  return launch_gemm<FwdCfg>(tA, tB, tB, g, stream);
}

cudaError_t launch_fp8_gemm_dx(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                               const float* s_w, int64_t M, int64_t N, int64_t K, void* dx,
                               int32_t* dev_status, cudaStream_t stream) {
  // contraction over N: A = dYq [M, N] K-major; B = Wq [N, K] read MN-major (K contiguous)
  CUtensorMap tA, tB;
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, dyq, N, M, 128, kBM, true) ||
      !make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq, K, N, 128, DxCfg::BK, true))
    return cudaErrorInvalidValue;
  GemmArgs g{};
  g.m_tiles = ceil_div(M, kBM);
  g.n_tiles = ceil_div(K, DxCfg::BN);
  g.splits = 1;
  g.kb_total = ceil_div(N, DxCfg::BK);
  g.kb_per_split = g.kb_total;
  g.M = M;
  g.N = K;
  g.out = dx;
  g.ldo = K;
  g.scale_a = s_dy;
  g.scale_b = s_w;
  g.dev_status = dev_status;
  return launch_gemm<DxCfg>(tA, tB, tB, g, stream);
}

// ------------------------------------------------------------------ adapter products
// Workspace: T_hi, T_lo, U_hi, U_lo bf16 [M, r] | fp32 partials (largest plan).
// T and U are carried as bf16 hi/lo pairs (about 16 significant bits): a
// single bf16 rounding of T would move small dB entries by more than one bf16
// ulp of the tensor's scale.
size_t adapter_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, bool want_da) {
  const DeviceInfo* di = current_device_info();
  const int sms = di ? di->sm_count : 148;
  const size_t tu = align_up(static_cast<size_t>(M) * r * 2, 256);
  size_t part = plan_partial_bytes(plan_skinny(M, r, K, sms));            // T
  part = std::max(part, plan_partial_bytes(plan_skinny(N, r, M, sms)));   // dB
  if (want_da) {
    part = std::max(part, plan_partial_bytes(plan_skinny(M, r, N, sms)));  // U
    part = std::max(part, plan_partial_bytes(plan_skinny(K, r, M, sms)));  // dA^T
  }
  return 4 * tu + align_up(part, 256);
}

namespace {

GemmArgs skinny_args(const SkinnyPlan& p, int64_t rows, int64_t r, float* part, int32_t* st) {
  GemmArgs g{};
  g.m_tiles = p.m_tiles;
  g.n_tiles = p.n_tiles;
  g.splits = p.splits;
  g.kb_total = p.kb_total;
  g.kb_per_split = p.kb_per_split;
  g.M = rows;
  g.N = r;
  g.out = part;
  g.m_pad = p.m_pad;
  g.n_pad = p.n_pad;
  g.dev_status = st;
  return g;
}

}  // namespace

cudaError_t launch_adapter_grads(const uint8_t* dyq, const float* s_dy, const uint8_t* xq,
                                 const float* s_x, const void* A, const void* B, int64_t M,
                                 int64_t N, int64_t K, int64_t r, void* dA, void* dB,
                                 int32_t* dev_status, void* workspace, cudaStream_t stream) {
  const DeviceInfo* di = current_device_info();
  if (!di) return cudaErrorInvalidDevice;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t tu = align_up(static_cast<size_t>(M) * r * 2, 256);
  void* T_hi = ws;
  void* T_lo = ws + tu;
  void* U_hi = ws + 2 * tu;
  void* U_lo = ws + 3 * tu;
  float* part = reinterpret_cast<float*>(ws + 4 * tu);
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cudaError_t e;
  CUtensorMap tA, tB, tB2;

  if (dB) {
    // T = Xq . A^T / s_x: A-op Xq [M, K] K-major (expanded), B-op A [r, K] K-major
    SkinnyPlan p = plan_skinny(M, r, K, di->sm_count);
    if (!make_tmap_2d(&tA, U8, 1, xq, K, M, 64, kBM, false) ||
        !make_tmap_2d(&tB, BF, 2, A, K, r, 64, p.bn, true))
      return cudaErrorInvalidValue;
    GemmArgs g = skinny_args(p, M, r, part, dev_status);
    if ((e = skinny_dispatch<TCfg>(p.bn, tA, tB, tB, g, stream)) != cudaSuccess) return e;
    if ((e = launch_reduce(part, p, M, r, s_x, nullptr, false, T_hi, T_lo, stream)) != cudaSuccess)
      return e;
    // dB = dYq^T . (T_hi + T_lo) / s_dy: A-op dYq^T (MN-major, expanded), B-op T [M, r] MN-major
    SkinnyPlan q = plan_skinny(N, r, M, di->sm_count);
    if (!make_tmap_2d(&tA, U8, 1, dyq, N, M, 128, 64, false) ||
        !make_tmap_2d(&tB, BF, 2, T_hi, r, M, 64, 64, true) ||
        !make_tmap_2d(&tB2, BF, 2, T_lo, r, M, 64, 64, true))
      return cudaErrorInvalidValue;
    GemmArgs h = skinny_args(q, N, r, part, dev_status);
    if ((e = skinny_dispatch<MnCfg>(q.bn, tA, tB, tB2, h, stream)) != cudaSuccess) return e;
    if ((e = launch_reduce(part, q, N, r, s_dy, nullptr, false, dB, nullptr, stream)) != cudaSuccess)
      return e;
  }
  if (dA) {
    // U = dYq . B / s_dy: A-op dYq [M, N] K-major (expanded), B-op B [N, r] MN-major
    SkinnyPlan p = plan_skinny(M, r, N, di->sm_count);
    if (!make_tmap_2d(&tA, U8, 1, dyq, N, M, 64, kBM, false) ||
        !make_tmap_2d(&tB, BF, 2, B, r, N, 64, 64, true))
      return cudaErrorInvalidValue;
    GemmArgs g = skinny_args(p, M, r, part, dev_status);
    if ((e = skinny_dispatch<UCfg>(p.bn, tA, tB, tB, g, stream)) != cudaSuccess) return e;
    if ((e = launch_reduce(part, p, M, r, s_dy, nullptr, false, U_hi, U_lo, stream)) != cudaSuccess)
      return e;
    // dA^T = Xq^T . (U_hi + U_lo) / s_x, stored transposed into dA [r, K]
    SkinnyPlan q = plan_skinny(K, r, M, di->sm_count);
    if (!make_tmap_2d(&tA, U8, 1, xq, K, M, 128, 64, false) ||
        !make_tmap_2d(&tB, BF, 2, U_hi, r, M, 64, 64, true) ||
        !make_tmap_2d(&tB2, BF, 2, U_lo, r, M, 64, 64, true))
      return cudaErrorInvalidValue;
    GemmArgs h = skinny_args(q, K, r, part, dev_status);
    if ((e = skinny_dispatch<MnCfg>(q.bn, tA, tB, tB2, h, stream)) != cudaSuccess) return e;
    if ((e = launch_reduce(part, q, K, r, s_x, nullptr, true, dA, nullptr, stream)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

}  // namespace falqon
