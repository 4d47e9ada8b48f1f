// Device helpers shared by the tcgen05 GEMM kernels (gemm.cu, skinny.cu):
// UMMA shared-memory descriptors for 128-byte-swizzled operand tiles, the
// exact E4M3 -> bf16 expansion used to feed E4M3 codes to the bf16 kind,
// cluster / DSMEM primitives and warp-uniform bounded waits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <cstring>

#include "ptx.cuh"

namespace falqon {

constexpr int kBM = 128;        // UMMA M (cta_group::1)
constexpr int kRowBytes = 128;  // every smem operand row is one 128-byte swizzle row
constexpr int kMaxSplits = 8;   // split-K partners: at most the portable cluster size

// Descriptor of operand tile `base` for UMMA k-step `ks`.  K-major tiles are
// [rows][128 B of K]; MN-major tiles are 128-byte-wide column blocks of
// [kKRows K rows][128 B of M/N], kKRows * 128 bytes apart.
template <int kElemBytes, int kKRows>
__device__ __forceinline__ uint64_t operand_desc_rt(bool mn, uint32_t base, int ks) {
  if (mn) {
    // k-step = (32 / elem) K-rows of 128 bytes; column blocks are kKRows rows apart
    return sdesc_sw128(base + ks * (32 / kElemBytes) * kRowBytes, kKRows * kRowBytes, 1024);
  }
  // k-step = 32 bytes along the swizzled 128-byte row
  return sdesc_sw128(base + ks * 32, 16, 1024);
}

template <bool kMn, int kElemBytes, int kKRows>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int ks) {
  return operand_desc_rt<kElemBytes, kKRows>(kMn, base, ks);
}

// Two E4M3 codes (bytes `sel` picks from w) to a bf16x2 word, exactly.  The
// byte permute puts each code in the low byte of its 16-bit lane and its sign
// bit, replicated, in the high byte.  Shifted left by 4 and masked, the
// lane holds the sign at bit 15 and the code's exponent and mantissa fields
// on the low four bits of the bf16 exponent and the top of the bf16
// mantissa: it reads as the code's value times 2^-120 (E4M3 bias 7 against
// bf16 bias 127; E4M3 subnormals land on bf16 subnormals, which scale the
// same way).  One bf16 multiply by 2^120 (plus -0) restores the value with no
// rounding.  NaN codes (0x7F, 0xFF) are not handled here.
template <uint32_t kSel>
__device__ __forceinline__ uint32_t e4m3_pair_to_bf16x2(uint32_t w) {
  uint32_t y, out;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(y) : "r"(w), "n"(kSel));
  const uint32_t h = (y << 4) & 0x87F087F0u;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(out) : "r"(h), "r"(0x7B807B80u), "r"(0x80008000u));
  return out;
}

// Accumulates NaN evidence over code words: bit 7 of a byte of the result of
// nan_fold ends up set iff that byte of some folded word had all seven
// magnitude bits set (a NaN code); test with nan_found.
__device__ __forceinline__ uint32_t nan_fold(uint32_t acc, uint4 q) {
  const uint32_t m = 0x7F7F7F7Fu, one = 0x01010101u;
  return acc | ((q.x & m) + one) | ((q.y & m) + one) | ((q.z & m) + one) | ((q.w & m) + one);
}
__device__ __forceinline__ bool nan_found(uint32_t acc) { return (acc & 0x80808080u) != 0u; }

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

// Sixteen codes -> sixteen bf16 (eight words, in code order); `nan` selects
// the hardware conversion, which also carries NaN codes.
__device__ __forceinline__ void e4m3x16_to_bf16(uint4 q, bool nan, uint32_t (&o)[8]) {
  const uint32_t words[4] = {q.x, q.y, q.z, q.w};
  if (!nan) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      o[2 * j] = e4m3_pair_to_bf16x2<0x9180u>(words[j]);      // codes 0, 1 of the word
      o[2 * j + 1] = e4m3_pair_to_bf16x2<0xB3A2u>(words[j]);  // codes 2, 3
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) e4m3x4_to_bf16_hw(words[j], o[2 * j], o[2 * j + 1]);
  }
}

// E5M2 codes (sign, 5 exponent bits of bias 15, 2 mantissa bits) to bf16,
// the same way: the byte permute replicates each code's sign into the high
// byte, a shift by 5 and a mask put the exponent on the low five bits of the
// bf16 exponent and the mantissa on the top of the bf16 mantissa, and one
// exact bf16 multiply by 2^112 (the bias difference 127 - 15) restores the
// value; subnormals land on bf16 subnormals and scale the same way.  Codes
// with an all-ones exponent (infinity, NaN) are not handled here.
template <uint32_t kSel>
__device__ __forceinline__ uint32_t e5m2_pair_to_bf16x2(uint32_t w) {
  uint32_t y, out;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(y) : "r"(w), "n"(kSel));
  const uint32_t h = (y << 5) & 0x8FE08FE0u;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(out) : "r"(h), "r"(0x77807780u), "r"(0x80008000u));
  return out;
}

// Evidence of E5M2 codes with an all-ones exponent (infinity or NaN): bit 7
// of a byte of the fold ends up set iff that byte of some folded word has it.
__device__ __forceinline__ uint32_t special5_fold(uint32_t acc, uint4 q) {
  const uint32_t m = 0x7C7C7C7Cu, one = 0x04040404u;
  return acc | ((q.x & m) + one) | ((q.y & m) + one) | ((q.z & m) + one) | ((q.w & m) + one);
}

// Four E5M2 codes -> four bf16 (two words) through the hardware conversion;
// exact for every code, infinity and NaN included.
__device__ __forceinline__ void e5m2x4_to_bf16_hw(uint32_t w, uint32_t& lo, uint32_t& hi) {
  uint32_t o[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const uint16_t pair = static_cast<uint16_t>(w >> (16 * j));
    uint32_t h2;
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"(pair));
    __half2 hh;
    memcpy(&hh, &h2, 4);
    const float2 f = __half22float2(hh);
    const __nv_bfloat162 bb = __floats2bfloat162_rn(f.x, f.y);
    memcpy(&o[j], &bb, 4);
  }
  lo = o[0];
  hi = o[1];
}

// Sixteen E5M2 codes -> sixteen bf16 (eight words, in code order); `special`
// selects the hardware conversion.
__device__ __forceinline__ void e5m2x16_to_bf16(uint4 q, bool special, uint32_t (&o)[8]) {
  const uint32_t words[4] = {q.x, q.y, q.z, q.w};
  if (!special) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      o[2 * j] = e5m2_pair_to_bf16x2<0x9180u>(words[j]);
      o[2 * j + 1] = e5m2_pair_to_bf16x2<0xB3A2u>(words[j]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) e5m2x4_to_bf16_hw(words[j], o[2 * j], o[2 * j + 1]);
  }
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

// Named barrier `id` over `nthreads` threads (whole warps) that also ORs a
// predicate across them: every participant gets true iff one passed true.
// Unlike an mbarrier wait, it does not hold back the tcgen05.mma stream of an
// issuing thread that takes part, so an MMA issuer can be released stage by
// stage through it by a warp that does the mbarrier waits.
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0u;
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

// Split count: as many K splits as fit beside the tiles in `slots` CTAs, at
// most kMaxSplits (the portable cluster size), never more than K blocks.
inline int choose_splits(int tiles, int kb_total, int slots) {
  int s = slots / (tiles > 0 ? tiles : 1);
  if (s > kMaxSplits) s = kMaxSplits;
  if (s > kb_total) s = kb_total;
  if (s < 1) s = 1;
  return s;
}

inline int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

}  // namespace falqon
