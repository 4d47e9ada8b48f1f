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
  void* out;               // bf16 output, row-major [M][ldo] (or [N][ldo] when transposed)
  void* out_lo;            // optional low half: out + out_lo carries ~16 significant bits
  int64_t ldo;
  int transpose;           // store out[col * ldo + row]
  const float* scale_a;    // alpha = 1 / (scale_a * scale_b); either may be null (= 1)
  const float* scale_b;
  int32_t* dev_status;
};

constexpr int kMaxSplits = 8;  // split-K partners: at most the portable cluster size

template <bool kF8, bool kAMn, bool kBMn, bool kAConv, int kBN, int kStages, bool kClusterK,
          bool kBSplit = false, int kRawStages = 0, int kBStages = kStages>
struct Cfg {
  static constexpr bool F8 = kF8;
  static constexpr bool AMn = kAMn;
  static constexpr bool BMn = kBMn;
  static constexpr bool AConv = kAConv;
  static constexpr int BN = kBN;
  static constexpr int Stages = kStages;
  // split-K across the CTAs of a cluster: each parks its fp32 tile in shared
  // memory and the cluster sums the tiles through DSMEM in rank order
  static constexpr bool ClusterK = kClusterK;
  static constexpr bool BSplit = kBSplit;  // B = B_hi + B_lo: two bf16 tiles, two MMAs per k-step
  static constexpr int ElemBytes = kF8 ? 1 : 2;
  static constexpr int BK = kRowBytes / ElemBytes;       // K per stage (128 fp8 / 64 bf16)
  static constexpr int UmmaK = 32 / ElemBytes;           // K per UMMA instruction
  static constexpr int KSteps = BK / UmmaK;              // 4
  static constexpr int ABytes = kBM * BK * ElemBytes;     // operand A tile (16 KB)
  static constexpr int BBytes = kBN * BK * ElemBytes;     // operand B tile
  static constexpr int B2Bytes = kBSplit ? BBytes : 0;   // low half of a split B operand
  // TMA ring (B, plus A when A comes by TMA) and, with expansion, a separate
  // ring of expanded A tiles so that B loads run ahead independently
  static constexpr int BStages = kAConv ? kBStages : kStages;
  static constexpr int BSlotBytes = (kAConv ? 0 : ABytes) + BBytes + B2Bytes;
  static constexpr int ARingBytes = kAConv ? kStages * ABytes : 0;
  static constexpr int BRingBytes = BStages * BSlotBytes;
  static constexpr int TmaBytes = BSlotBytes;
  static constexpr int NumConvWarps = kAConv ? 16 : 0;
  // ring of raw E4M3 A tiles (one k-block each, unswizzled, row-major), filled
  // by TMA from a warp of its own kRawStages k-blocks ahead of the converters
  static constexpr int RawStages = kAConv ? kRawStages : 0;
  static constexpr int RawSlotBytes = kAConv ? kBM * BK : 0;  // 8 KB of codes
  static_assert(!kAConv || kRawStages >= 2, "raw ring depth");
  static_assert(!kAConv || RawSlotBytes == 16 * 32 * NumConvWarps, "one 16-byte chunk per converter thread");
  static constexpr int RawWarp = 6 + NumConvWarps;  // raw-code producer (expansion only)
  static constexpr int Threads = 32 * (6 + NumConvWarps + (kAConv ? 1 : 0));
  static constexpr uint32_t TmemCols = 2 * kBN < 32 ? 32 : 2 * kBN;
  static constexpr int BarBytes = 8 * (2 * kStages + 2 * BStages + 2 * RawStages + 5) + 16;
  static constexpr int SmemBytes = ARingBytes + BRingBytes + RawStages * RawSlotBytes + BarBytes + 1024;
  static constexpr int RedStride = kBN + 4;  // fp32 words per row of the reduction tile (16-byte rows)
  static_assert(!kClusterK || kBM * RedStride * 4 <= ARingBytes + BRingBytes, "reduction tile");
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

// Two E4M3 codes, in bytes 0 and 2 of x (bytes 1 and 3 zero), to a bf16x2
// word, exactly.  Shifted left by 4, a code's exponent and mantissa fields
// land on the bf16 exponent and the top of the bf16 mantissa, so the word
// reads as the code's value times 2^-120 (E4M3 bias 7 against bf16 bias 127;
// E4M3 subnormals land on bf16 subnormals, which scale the same way).  The
// sign, left at bit 11, moves to bit 15 by adding 15 * 2^11 (= 2^15 - 2^11),
// and one bf16 multiply by 2^120 (plus -0) restores the value with no
// rounding.  NaN codes (0x7F, 0xFF) are not handled here.
__device__ __forceinline__ uint32_t e4m3_pair_to_bf16x2(uint32_t x) {
  uint32_t h = x << 4;
  h += 15u * (h & 0x08000800u);
  uint32_t out;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(out) : "r"(h), "r"(0x7B807B80u), "r"(0x80008000u));
  return out;
}

// Nonzero iff one of the 16 codes is a NaN code (magnitude bits all ones).
__device__ __forceinline__ uint32_t has_nan_code(uint4 q) {
  const uint32_t m = 0x7F7F7F7Fu, one = 0x01010101u;
  return (((q.x & m) + one) | ((q.y & m) + one) | ((q.z & m) + one) | ((q.w & m) + one)) &
         0x80808080u;
}

// Four codes -> four bf16 (two words) through the hardware conversion; exact
// for every code, NaN included.
__device__ __forceinline__ void e4m3x4_to_bf16_hw(uint32_t w, uint32_t& lo, uint32_t& hi) {
  uint32_t o[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const uint16_t pair = static_cast<uint16_t>(w >> (16 * j));
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
    __half2 hh;
    memcpy(&hh, &h2, 4);
    const float2 f = __half22float2(hh);
    const __nv_bfloat162 bb = __floats2bfloat162_rn(f.x, f.y);
    memcpy(&o[j], &bb, 4);
  }
  lo = o[0];
  hi = o[1];
}


__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

// Address of `local` (this CTA's shared memory) in the shared window of cluster CTA `rank`.
__device__ __forceinline__ uint32_t dsmem_addr(const void* local, int rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  return remote;
}

// Peer tiles are stable between the two cluster barriers around the
// reduction, so these loads may be reordered and overlapped freely.
__device__ __forceinline__ float4 dsmem_load_f32x4(uint32_t addr) {
  float4 v;
  asm("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
      : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
      : "r"(addr));
  return v;
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
  uint8_t* a_ring = smem;                                // expanded A tiles (expansion only)
  uint8_t* b_ring = smem + C::ARingBytes;                // TMA-fed tiles
  uint8_t* raw_ring = b_ring + C::BRingBytes;            // converters' raw codes
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw_ring + C::RawStages * C::RawSlotBytes);
  uint64_t* full = bars;                                 // [BStages] TMA landed
  uint64_t* empty = full + C::BStages;                   // [BStages] MMAs done with the TMA slot
  uint64_t* conv = empty + C::BStages;                   // [Stages] codes expanded
  uint64_t* aempty = conv + C::Stages;                   // [Stages] MMAs done with the A slot
  uint64_t* rawfull = aempty + C::Stages;                // [RawStages] raw codes landed
  uint64_t* rawempty = rawfull + C::RawStages;           // [RawStages] converters done reading
  uint64_t* acc_full = rawempty + C::RawStages;          // [2] accumulator ready
  uint64_t* acc_empty = acc_full + 2;         // [2] accumulator drained
  uint64_t* drain = acc_empty + 2;            // all issued MMAs retired (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total = g.m_tiles * g.n_tiles * g.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::BStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::Stages; ++s) {
      mbar_init(&conv[s], C::NumConvWarps > 0 ? C::NumConvWarps : 1);
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < C::RawStages; ++s) {
      mbar_init(&rawfull[s], 1);
      mbar_init(&rawempty[s], C::NumConvWarps);
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
          uint8_t* sA = b_ring + stage * C::BSlotBytes;  // A by TMA only when not expanded
          uint8_t* sB = sA + (C::AConv ? 0 : C::ABytes);
          uint8_t* sB2 = sB + C::BBytes;
          mbar_arrive_expect_tx(&full[stage], C::TmaBytes);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          // operand A: rows m0.., K block kb
          if constexpr (C::AConv) {
            // A arrives through the converter warps (global loads, expanded in place)
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
          if (++stage == C::BStages) { stage = 0; phase ^= 1; }
        }
      }
      // every load this lane issued must land before the CTA exits (matters
      // only after an abort; otherwise the MMA warp already consumed them)
      for (int s = 0; s < C::BStages; ++s)
        if (issued & (1u << s)) mbar_wait_budget(&full[s], (issued_parity >> s) & 1u);
    }
    __syncwarp();  // the warp reaches the CTA barriers below together
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0, astage = 0;
    uint32_t phase = 0, aphase = 0;
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
        if constexpr (C::AConv) {
          if (!warp_wait(&conv[astage], aphase, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
        }
        if (!warp_wait(&full[stage], phase, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t slot = smem_u32(b_ring + stage * C::BSlotBytes);
          const uint32_t a_base = C::AConv ? smem_u32(a_ring + astage * C::ABytes) : slot;
          const uint32_t b_base = slot + (C::AConv ? 0 : C::ABytes);
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
          if constexpr (C::AConv) umma_commit(&aempty[astage]);
        }
        __syncwarp();
        if (++stage == C::BStages) { stage = 0; phase ^= 1; }
        if constexpr (C::AConv) {
          if (++astage == C::Stages) { astage = 0; aphase ^= 1; }
        }
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
      (void)split;
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::BN + c * 32, r);
        tmem_ld_wait();
        const int64_t col0 = col_base + c * 32;
        (void)col0;
        if constexpr (C::ClusterK) {
          // this CTA's fp32 tile, reusing the (drained) stage buffers
          float4* red = reinterpret_cast<float4*>(reinterpret_cast<float*>(smem) +
                                                  (q * 32 + lane) * C::RedStride + c * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            red[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
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
    constexpr int kTileRows = C::AMn ? C::BK : kBM;        // rows of the A tile (and of its raw box)
    constexpr int kTileCols = C::AMn ? kBM : C::BK;        // codes per row
    if (warp == C::RawWarp) {
      // ---------------------------------------------------------- raw-code producer
      // One TMA box per k-block: K-major A = codes[m0 .. +128, kb*64 .. +64];
      // MN-major A = codes[kb*64 .. +64, m0 .. +128] (rows of the code matrix are K).
      if (lane == 0) {
        int rs = 0;
        uint32_t rphase = 0;
        uint32_t issued = 0, issued_parity = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
          const int split = w % g.splits;
          const int mt = w / (g.splits * g.n_tiles);
          const int kb0 = split * g.kb_per_split;
          const int kb1 = min(g.kb_total, kb0 + g.kb_per_split);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(&rawempty[rs], rphase ^ 1, abort_flag)) { fail(); ok = false; break; }
            mbar_arrive_expect_tx(&rawfull[rs], C::RawSlotBytes);
            issued |= 1u << rs;
            issued_parity = (issued_parity & ~(1u << rs)) | (rphase << rs);
            if constexpr (C::AMn)
              tma_load_2d(raw_ring + rs * C::RawSlotBytes, &tmA, &rawfull[rs], mt * kBM, kb * C::BK);
            else
              tma_load_2d(raw_ring + rs * C::RawSlotBytes, &tmA, &rawfull[rs], kb * C::BK, mt * kBM);
            if (++rs == C::RawStages) { rs = 0; rphase ^= 1; }
          }
        }
        for (int s2 = 0; s2 < C::RawStages; ++s2)
          if (issued & (1u << s2)) mbar_wait_budget(&rawfull[s2], (issued_parity >> s2) & 1u);
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------------- converters
      // 512 threads; each expands one 16-byte chunk (16 codes) of every A tile:
      //   K-major  [128 rows][64 codes]: row = t / 4,  columns (t % 4) * 16 ..
      //   MN-major [64 rows][128 codes]: row = t / 8,  columns (t % 8) * 16 ..
      constexpr int kThrPerRow = kTileCols / 16;
      const int t = threadIdx.x - 6 * 32;
      const int trow = t / kThrPerRow;
      const int tcol = (t % kThrPerRow) * 16;
      const uint32_t raw_off = trow * kTileCols + tcol;
      // destinations of the two 16-byte units (8 bf16 each) in the swizzled tile
      const int blk = tcol / 64;
      const int unit0 = (tcol % 64) / 8;
      const uint32_t dst_off0 = blk * (kTileRows * kRowBytes) + trow * kRowBytes + ((unit0 ^ (trow & 7)) << 4);
      const uint32_t dst_off1 = blk * (kTileRows * kRowBytes) + trow * kRowBytes + (((unit0 + 1) ^ (trow & 7)) << 4);
      // Two k-blocks per iteration: their expansions are independent, so the
      // two dependency chains overlap within the warp.
      auto expand = [&](const uint4& q, uint8_t* sA) {
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
        uint32_t o[8];
        if (!has_nan_code(q)) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            o[2 * j] = e4m3_pair_to_bf16x2(__byte_perm(words[j], 0u, 0x4140));
            o[2 * j + 1] = e4m3_pair_to_bf16x2(__byte_perm(words[j], 0u, 0x4342));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) e4m3x4_to_bf16_hw(words[j], o[2 * j], o[2 * j + 1]);
        }
        *reinterpret_cast<uint4*>(sA + dst_off0) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(sA + dst_off1) = make_uint4(o[4], o[5], o[6], o[7]);
      };
      int stage = 0, rs = 0;
      uint32_t phase = 0, rphase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int split = w % g.splits;
        const int kb0 = split * g.kb_per_split;
        const int kb1 = min(g.kb_total, kb0 + g.kb_per_split);
        for (int kb = kb0; kb < kb1; kb += 2) {
          const bool two = kb + 1 < kb1;
          // raw codes of k-blocks kb (and kb + 1)
          const int rs1 = rs + 1 == C::RawStages ? 0 : rs + 1;
          const uint32_t rphase1 = rs + 1 == C::RawStages ? rphase ^ 1 : rphase;
          if (!warp_wait(&rawfull[rs], rphase, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
          const uint4 q0 = *reinterpret_cast<const uint4*>(raw_ring + rs * C::RawSlotBytes + raw_off);
          uint4 q1 = make_uint4(0u, 0u, 0u, 0u);
          if (two) {
            if (!warp_wait(&rawfull[rs1], rphase1, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
            q1 = *reinterpret_cast<const uint4*>(raw_ring + rs1 * C::RawSlotBytes + raw_off);
          }
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&rawempty[rs]);
            if (two) mbar_arrive(&rawempty[rs1]);
          }
          rs = two ? (rs1 + 1 == C::RawStages ? 0 : rs1 + 1) : rs1;
          rphase = two ? (rs1 + 1 == C::RawStages ? rphase1 ^ 1 : rphase1) : rphase1;
          // expanded-A stages for kb (and kb + 1)
          const int st1 = stage + 1 == C::Stages ? 0 : stage + 1;
          const uint32_t phase1 = stage + 1 == C::Stages ? phase ^ 1 : phase;
          if (!warp_wait(&aempty[stage], phase ^ 1, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
          if (two && !warp_wait(&aempty[st1], phase1 ^ 1, abort_flag)) { if (lane == 0) fail(); ok = false; break; }
          expand(q0, a_ring + stage * C::ABytes);
          if (two) expand(q1, a_ring + st1 * C::ABytes);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&conv[stage]);
            if (two) mbar_arrive(&conv[st1]);
          }
          stage = two ? (st1 + 1 == C::Stages ? 0 : st1 + 1) : st1;
          phase = two ? (st1 + 1 == C::Stages ? phase1 ^ 1 : phase1) : phase1;
        }
      }
    }
  }

  if constexpr (C::ClusterK) {
    // One work item per CTA: rank = split.  Sum the cluster's tiles row slice by
    // row slice (this CTA owns rows [q0, q1) of the tile), in rank order.
    __syncthreads();
    cluster_sync_all();
    const int S = g.splits;
    const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
    const int w = blockIdx.x;
    const int nt = (w / S) % g.n_tiles;
    const int mt = w / (S * g.n_tiles);
    const int rows_per = (kBM + S - 1) / S;
    const int q0 = static_cast<int>(rank) * rows_per;
    const int q1 = min(kBM, q0 + rows_per);
    const float* red = reinterpret_cast<const float*>(smem);
    uint32_t peer[kMaxSplits];
#pragma unroll
    for (int sidx = 0; sidx < kMaxSplits; ++sidx) peer[sidx] = dsmem_addr(red, sidx < S ? sidx : 0);
    double den = 1.0;
    if (g.scale_a) den *= static_cast<double>(*g.scale_a);
    if (g.scale_b) den *= static_cast<double>(*g.scale_b);
    const float alpha = static_cast<float>(1.0 / den);
    const int nrows = q1 - q0;
    constexpr int G = C::BN / 4;  // float4 groups per row
    const int ngroups = nrows > 0 ? nrows * G : 0;
    for (int e = threadIdx.x; e < ngroups; e += blockDim.x) {
      int lr, lg;
      if (g.transpose) { lr = q0 + e % nrows; lg = e / nrows; }  // walk rows: coalesced out[col][row]
      else { lr = q0 + e / G; lg = e % G; }
      const uint32_t off = static_cast<uint32_t>((lr * C::RedStride + 4 * lg) * 4);
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int s0 = 0; s0 < kMaxSplits; s0 += 4) {  // fixed order: rank 0, 1, ...
        float4 part[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (s0 + k < S) part[k] = dsmem_load_f32x4(peer[s0 + k] + off);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (s0 + k < S) {
            acc.x += part[k].x;
            acc.y += part[k].y;
            acc.z += part[k].z;
            acc.w += part[k].w;
          }
        }
      }
      const int64_t grow = static_cast<int64_t>(mt) * kBM + lr;
      const int64_t gcol0 = static_cast<int64_t>(nt) * C::BN + 4 * lg;
      if (grow >= g.M || gcol0 >= g.N) continue;  // N % 16 == 0: groups of 4 in or out
      const float vals[4] = {acc.x * alpha, acc.y * alpha, acc.z * alpha, acc.w * alpha};
      __nv_bfloat16 hi[4], lo[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        hi[k] = __float2bfloat16_rn(vals[k]);
        lo[k] = __float2bfloat16_rn(vals[k] - __bfloat162float(hi[k]));
      }
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
      __nv_bfloat16* out_lo = static_cast<__nv_bfloat16*>(g.out_lo);
      if (g.transpose) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          out[(gcol0 + k) * g.ldo + grow] = hi[k];
          if (out_lo) out_lo[(gcol0 + k) * g.ldo + grow] = lo[k];
        }
      } else {
        uint2 ph, pl;
        memcpy(&ph, hi, 8);
        memcpy(&pl, lo, 8);
        *reinterpret_cast<uint2*>(out + grow * g.ldo + gcol0) = ph;
        if (out_lo) *reinterpret_cast<uint2*>(out_lo + grow * g.ldo + gcol0) = pl;
      }
    }
    cluster_sync_all();  // no CTA leaves while a peer still reads its tile
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TmemCols);
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
  if constexpr (C::ClusterK) {
    // one work item per CTA; the `splits` CTAs of an output tile form one cluster
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(g.splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(total));
    cfg.blockDim = dim3(C::Threads);
    cfg.dynamicSmemBytes = C::SmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tc_gemm_kernel<C>, tA, tB, tB2, g);
  } else {
    const int grid = total < di->sm_count ? total : di->sm_count;
    tc_gemm_kernel<C><<<grid, C::Threads, C::SmemBytes, stream>>>(tA, tB, tB2, g);
    return cudaGetLastError();
  }
}

inline int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

using FwdCfg = Cfg<true, false, false, false, 256, 4, false>;
using DxCfg = Cfg<true, false, true, false, 256, 4, false>;

// Stage counts <A (expanded), raw codes, B> sized to about 224 KB of shared
// memory.  The expanded-A ring is the deep one: a stage is released only when
// the MMAs that read it have completed, so its depth has to cover the MMA
// completion latency; the raw ring needs only to cover HBM latency.
template <int BN> using TCfg = Cfg<false, false, false, true, BN, (BN >= 256 ? 3 : (BN >= 128 ? 4 : 6)), true, false,
                                   (BN >= 256 ? 4 : 8), (BN >= 256 ? 3 : (BN >= 128 ? 4 : 8))>;  // Xq . A^T
template <int BN> using UCfg = Cfg<false, false, true, true, BN, (BN >= 256 ? 3 : (BN >= 128 ? 4 : 6)), true, false,
                                   (BN >= 256 ? 4 : 8), (BN >= 256 ? 3 : (BN >= 128 ? 4 : 8))>;  // dYq . B
// dYq^T . (T_hi + T_lo), Xq^T . (U_hi + U_lo): B is split hi/lo, so fewer stages
template <int BN> using MnCfg = Cfg<false, true, true, true, BN, (BN >= 256 ? 2 : (BN >= 128 ? 3 : 5)), true, true,
                                    (BN >= 256 ? 4 : 8), (BN >= 256 ? 2 : (BN >= 128 ? 3 : 5))>;

// Split count: as many K splits as fit beside the tiles in one wave, at most 8
// (the portable cluster size), never more than there are K blocks.
int choose_splits(int tiles, int kb_total, int sm_count) {
  int s = sm_count / (tiles > 0 ? tiles : 1);
  if (s > kMaxSplits) s = kMaxSplits;
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
  return p;
}

}  // namespace

// ------------------------------------------------------------------ big GEMMs
namespace {

template <class C>
cudaError_t fp8_gemm(const uint8_t* a, const float* sa, const uint8_t* b, const float* sb,
                     int64_t M, int64_t Ncols, int64_t Kc, bool b_mn, void* out,
                     int32_t* dev_status, cudaStream_t stream) {
  CUtensorMap tA, tB;
  // A [M, Kc] K-major; B K-major [Ncols, Kc] or MN-major [Kc, Ncols]
  if (!make_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a, Kc, M, 128, kBM, true))
    return cudaErrorInvalidValue;
  const bool okb = b_mn ? make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, b, Ncols, Kc, 128, C::BK, true)
                        : make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, b, Kc, Ncols, 128, C::BN, true);
  if (!okb) return cudaErrorInvalidValue;
  GemmArgs g{};
  g.m_tiles = ceil_div(M, kBM);
  g.n_tiles = ceil_div(Ncols, C::BN);
  g.splits = 1;
  g.kb_total = ceil_div(Kc, C::BK);
  g.kb_per_split = g.kb_total;
  g.M = M;
  g.N = Ncols;
  g.out = out;
  g.ldo = Ncols;
  g.scale_a = sa;
  g.scale_b = sb;
  g.dev_status = dev_status;
  return launch_gemm<C>(tA, tB, tB, g, stream);
}

}  // namespace

cudaError_t launch_fp8_gemm_fwd(const uint8_t* xq, const float* s_x, const uint8_t* wq,
                                const float* s_w, int64_t M, int64_t N, int64_t K, void* y,
                                int32_t* dev_status, cudaStream_t stream) {
  return fp8_gemm<FwdCfg>(xq, s_x, wq, s_w, M, N, K, false, y, dev_status, stream);
}

cudaError_t launch_fp8_gemm_dx(const uint8_t* dyq, const float* s_dy, const uint8_t* wq,
                               const float* s_w, int64_t M, int64_t N, int64_t K, void* dx,
                               int32_t* dev_status, cudaStream_t stream) {
  // contraction over N: A = dYq [M, N] K-major; B = Wq [N, K] read MN-major (K contiguous)
  return fp8_gemm<DxCfg>(dyq, s_dy, wq, s_w, M, K, N, true, dx, dev_status, stream);
}

// ------------------------------------------------------------------ adapter products
// Workspace: T_hi, T_lo, U_hi, U_lo, each bf16 [M, r].  T and U are carried
// as bf16 hi/lo pairs (about 16 significant bits): a single bf16 rounding of
// T would move small dB entries by more than one bf16 ulp of the tensor's
// scale.  The split-K sums never leave the chip (cluster reduction).
size_t adapter_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, bool want_da) {
  (void)N;
  (void)K;
  (void)want_da;
  const size_t tu = align_up(static_cast<size_t>(M) * r * 2, 256);
  return 4 * tu;
}

namespace {

GemmArgs skinny_args(const SkinnyPlan& p, int64_t rows, int64_t r, void* out, void* out_lo,
                     int64_t ldo, bool transpose, const float* scale, int32_t* st) {
  GemmArgs g{};
  g.m_tiles = p.m_tiles;
  g.n_tiles = p.n_tiles;
  g.splits = p.splits;
  g.kb_total = p.kb_total;
  g.kb_per_split = p.kb_per_split;
  g.M = rows;
  g.N = r;
  g.out = out;
  g.out_lo = out_lo;
  g.ldo = ldo;
  g.transpose = transpose ? 1 : 0;
  g.scale_a = scale;
  g.scale_b = nullptr;
  g.dev_status = st;
  return g;
}

// Tensor map over an E4M3 code matrix [rows, cols] for the raw-code ring of an
// expanded A operand, unswizzled: K-major (contraction along cols) boxes are
// 128 rows x 64 codes; MN-major (contraction along rows) boxes are 64 rows x 128 codes.
bool codes_tmap(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t cols, bool mn_major) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, codes, static_cast<uint64_t>(cols),
                      static_cast<uint64_t>(rows), mn_major ? 128 : 64, mn_major ? 64 : 128, false);
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
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cudaError_t e;
  CUtensorMap tA, tB, tB2;

  if (dB) {
    // T = Xq . A^T / s_x -> (T_hi, T_lo): A-op Xq [M, K] K-major (expanded), B-op A [r, K] K-major
    SkinnyPlan p = plan_skinny(M, r, K, di->sm_count);
    if (!make_tmap_2d(&tB, BF, 2, A, K, r, 64, p.bn, true) || !codes_tmap(&tA, xq, M, K, false))
      return cudaErrorInvalidValue;
    GemmArgs g = skinny_args(p, M, r, T_hi, T_lo, r, false, s_x, dev_status);
    if ((e = skinny_dispatch<TCfg>(p.bn, tA, tB, tB, g, stream)) != cudaSuccess) return e;
    // dB = dYq^T . (T_hi + T_lo) / s_dy: A-op dYq^T (MN-major, expanded), B-op T [M, r] MN-major
    SkinnyPlan q = plan_skinny(N, r, M, di->sm_count);
    if (!make_tmap_2d(&tB, BF, 2, T_hi, r, M, 64, 64, true) ||
        !make_tmap_2d(&tB2, BF, 2, T_lo, r, M, 64, 64, true) || !codes_tmap(&tA, dyq, M, N, true))
      return cudaErrorInvalidValue;
    GemmArgs h = skinny_args(q, N, r, dB, nullptr, r, false, s_dy, dev_status);
    if ((e = skinny_dispatch<MnCfg>(q.bn, tA, tB, tB2, h, stream)) != cudaSuccess) return e;
  }
  if (dA) {
    // U = dYq . B / s_dy -> (U_hi, U_lo): A-op dYq [M, N] K-major (expanded), B-op B [N, r] MN-major
    SkinnyPlan p = plan_skinny(M, r, N, di->sm_count);
    if (!make_tmap_2d(&tB, BF, 2, B, r, N, 64, 64, true) || !codes_tmap(&tA, dyq, M, N, false))
      return cudaErrorInvalidValue;
    GemmArgs g = skinny_args(p, M, r, U_hi, U_lo, r, false, s_dy, dev_status);
    if ((e = skinny_dispatch<UCfg>(p.bn, tA, tB, tB, g, stream)) != cudaSuccess) return e;
    // dA^T = Xq^T . (U_hi + U_lo) / s_x, stored transposed into dA [r, K]
    SkinnyPlan q = plan_skinny(K, r, M, di->sm_count);
    if (!make_tmap_2d(&tB, BF, 2, U_hi, r, M, 64, 64, true) ||
        !make_tmap_2d(&tB2, BF, 2, U_lo, r, M, 64, 64, true) || !codes_tmap(&tA, xq, M, K, true))
      return cudaErrorInvalidValue;
    GemmArgs h = skinny_args(q, K, r, dA, nullptr, K, true, s_x, dev_status);
    if ((e = skinny_dispatch<MnCfg>(q.bn, tA, tB, tB2, h, stream)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace falqon
