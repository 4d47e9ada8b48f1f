// Device helpers shared by the proxy kernels: cp.async staging and the
// E4M3 arithmetic of the requantization (decode by the hardware conversion,
// one separately rounded multiply and add, re-encode with satfinite), plus
// byte-parallel comparisons of packed codes.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>
#include <cstring>

#include "ptx.cuh"

namespace falqon {
namespace codes {

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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

// Four codes (bytes of w4) -> the four codes E4M3(dec(c) + s_w * p), no FMA.
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

// 0x80 in every byte of x that is zero, 0x00 elsewhere (exact per byte: the
// masked add cannot carry across bytes).
__device__ __forceinline__ uint32_t zero_bytes(uint32_t x) {
  const uint32_t t = (x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu;  // bit 7 set iff the low 7 bits are not all 0
  return ~(t | x) & 0x80808080u;
}

// 0xFF in every byte of `a` that holds a NaN code.
__device__ __forceinline__ uint32_t nan_bytes(uint32_t a) {
  const uint32_t mag = 0x7F7F7F7Fu;
  return (zero_bytes((a & mag) ^ mag) >> 7) * 0xFFu;
}

// Byte mask (0xFF per byte) of the codes whose value changes from `a` to `b`.
// Two codes hold the same value when they are identical non-NaN codes or
// both zero (either sign); a NaN code never holds the same value.
__device__ __forceinline__ uint32_t changed_bytes(uint32_t a, uint32_t b) {
  const uint32_t mag = 0x7F7F7F7Fu;
  const uint32_t same_bits = zero_bytes(a ^ b);
  const uint32_t both_zero = zero_bytes((a | b) & mag);
  const uint32_t nan = zero_bytes((a & mag) ^ mag) | zero_bytes((b & mag) ^ mag);
  const uint32_t changed = ~((same_bits | both_zero) & ~nan) & 0x80808080u;
  return (changed >> 7) * 0xFFu;
}

}  // namespace codes
}  // namespace falqon
