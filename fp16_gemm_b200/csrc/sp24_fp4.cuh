// NVFP4 decoding into 16-bit MMA operands, shared by the skinny / decode kernels and the
// routed-expert tensor-core kernel.
//
// An E2M1 code's three magnitude bits, shifted into place, form the 16-bit pattern of
// E2M1(code) * 2^-126 (bf16) or E2M1(code) * 2^-14 (f16): code 0 and 1 land on zero and the
// smallest subnormals, the rest on normal values with the right mantissa bit.  Multiplying by
// the block scale E4M3 * 2^118 (bf16) or E4M3 * 2^6 (f16) in the same 16-bit type is exact (at
// most 7 significant bits), which leaves every product 2^-8 times its true value; the epilogue
// multiplies by 256 * tensor scale.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

namespace sp24 {
namespace {

template <typename T>
struct P2;
template <>
struct P2<__nv_bfloat16> {  // 16-bit pattern of E2M1(code) * 2^-126
  static constexpr uint32_t MAG = 0x01C001C0u;
  static constexpr int MAGPOS = 6;
  static constexpr float FOLD = 0x1p118f;
};
template <>
struct P2<__half> {  // 16-bit pattern of E2M1(code) * 2^-14
  static constexpr uint32_t MAG = 0x0E000E00u;
  static constexpr int MAGPOS = 9;
  static constexpr float FOLD = 0x1p6f;
};

__device__ __forceinline__ uint32_t shl2(uint32_t x, int n) { return n >= 0 ? x << n : x >> (-n); }

// Nibbles i and i+4 of w -> 16-bit pair of E2M1 patterns.
template <typename T>
__device__ __forceinline__ uint32_t fp4_pair_i4(uint32_t w, int i) {
  return (shl2(w, P2<T>::MAGPOS - 4 * i) & P2<T>::MAG) | (shl2(w, 12 - 4 * i) & 0x80008000u);
}

// The byte at bits [8bb, 8bb+8) of w (two consecutive codes) -> 16-bit pair (lo, hi).  With the
// byte alone in x, x * (2^P + 2^(P+12)) is x << P plus x << (P + 12), two copies whose bits do
// not overlap, so the product places the low code's magnitude bits at P and the high code's at
// P + 16 at once; x * (2^12 + 2^24) likewise moves the two sign bits (3, 7) to 15 and 31.  Two
// integer multiplies and two masks instead of four shift-and-mask terms.
template <typename T>
__device__ __forceinline__ uint32_t fp4_pair_byte(uint32_t w, int bb) {
  const uint32_t x = __byte_perm(w, 0u, 0x4440u | (uint32_t)bb);  // byte bb, upper bytes zero
  constexpr int P = P2<T>::MAGPOS;
  const uint32_t mag = (x * ((1u << P) | (1u << (P + 12)))) & P2<T>::MAG;
  return mag | ((x * 0x01001000u) & 0x80008000u);
}

// Four bytes of E2M1 codes -> four f16 pairs (byte i -> ri; the low code of a byte in the low
// half), by the sm_100a conversion instruction: every E2M1 value is exact in f16.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "mov.b32 {q0, q1, q2, q3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, q1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, q2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, q3;\n\t}"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(w));
}

// The two low bytes of w -> two f16 pairs (byte 0 -> r0, byte 1 -> r1).
__device__ __forceinline__ void e2m1x4_to_f16x2(uint32_t w, uint32_t& r0, uint32_t& r1) {
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "mov.b32 {q0, q1, q2, q3}, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, q1;\n\t}"
      : "=r"(r0), "=r"(r1)
      : "r"(w));
}

// Two E4M3 codes (low bytes of code2) -> f16 pair (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t code2) {
  uint32_t h2;
  const uint16_t c = (uint16_t)code2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return h2;
}

template <typename T>
__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  } else {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
}

template <typename T>
__device__ __forceinline__ uint16_t to_bits16(float f) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    __nv_bfloat16 v = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&v);
  } else {
    __half v = __float2half_rn(f);
    return *reinterpret_cast<uint16_t*>(&v);
  }
}

// Two E4M3 block scales (low bytes of code2) -> two packed multipliers E4M3 * FOLD (exact).
template <typename T>
__device__ __forceinline__ void scale_pair(uint32_t code2, uint32_t& s0, uint32_t& s1) {
  uint32_t h2;
  const uint16_t c = (uint16_t)code2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  const uint32_t a = to_bits16<T>(__half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu))) * P2<T>::FOLD);
  const uint32_t b = to_bits16<T>(__half2float(__ushort_as_half((unsigned short)(h2 >> 16))) * P2<T>::FOLD);
  s0 = a | (a << 16);
  s1 = b | (b << 16);
}

}  // namespace
}  // namespace sp24
