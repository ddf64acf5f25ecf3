// Packed two-float arithmetic (f32x2) and the nibble-to-float trick shared by
// the attention kernels.
//
// An f32x2 value travels in one 64-bit register from the instruction that
// makes it to the instruction that uses it, so no register-pair moves are
// needed around the packed operations.  Low half = first float.
#pragma once
#include <cstdint>

namespace kvq {

typedef unsigned long long u64;

__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
  u64 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ u64 add2(u64 a, u64 b) {
  u64 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ u64 pack2(float lo, float hi) {
  u64 d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}

__device__ __forceinline__ float lo_f(u64 x) { return __uint_as_float(static_cast<uint32_t>(x)); }
__device__ __forceinline__ float hi_f(u64 x) { return __uint_as_float(static_cast<uint32_t>(x >> 32)); }

// The two 4-bit codes of one byte after a shift that puts them at bits
// 15..18 and 19..22, masked into the mantissa of 1.0:
// (1 + n_even 2^-8, 1 + n_odd 2^-4) as one f32x2 value.
__device__ __forceinline__ u64 nibble_pair(uint32_t a) {
  u64 x;
  asm("{.reg .b32 t0, t1;\n\t"
      "lop3.b32 t0, %1, 0x00078000, 0x3F800000, 0xEA;\n\t"
      "lop3.b32 t1, %1, 0x00780000, 0x3F800000, 0xEA;\n\t"
      "mov.b64 %0, {t0, t1};}"
      : "=l"(x)
      : "r"(a));
  return x;
}

// Byte r (0..3) of w shifted so its two nibbles sit at bits 15..22.
__device__ __forceinline__ uint32_t byte_at15(uint32_t w, int r) {
  return r == 0 ? (w << 15) : r == 1 ? (w << 7) : r == 2 ? (w >> 1) : (w >> 9);
}

// Two 8-bit codes (bytes r, r + 1 of w) in the low mantissa bits of 2^23:
// (2^23 + c_r, 2^23 + c_{r+1}) as one f32x2 value.
__device__ __forceinline__ u64 byte_pair(uint32_t w, int r) {
  const uint32_t lo = __byte_perm(w, 0x4B000000u, 0x7540u + r);
  const uint32_t hi = __byte_perm(w, 0x4B000000u, 0x7540u + r + 1);
  return (static_cast<u64>(hi) << 32) | lo;
}

}  // namespace kvq
