// Exact decoding of FP8 E4M3 weight codes with power-of-two block scales to
// bf16, shared by the FP8 expert-FFN kernel (which decodes straight into
// tensor memory) and the stand-alone dequantization kernel.
//
// Format (the FP8 counterpart of the BF16 expert weights the GLM-5.2 model
// pages name): each weight w = e4m3(code) * 2^e, where code is an OCP E4M3
// (float8_e4m3fn) byte and e an int8 exponent shared by a 128 x 128 block of
// the [rows, K] matrix.  Every such value has at most 4 significant bits, so
// it is exactly a bf16 value whenever it lies in bf16's normal range; the
// kernels accept e in [kMinExp, kMaxExp], which guarantees that, and flag
// other exponents.  The two NaN codes (0x7F, 0xFF) are outside the format.
#pragma once

#include <cstdint>

namespace moe {
namespace fp8 {

constexpr int kBlock = 128;
constexpr int kMinExp = -117;   // 2^-9 * 2^-117 = 2^-126, the smallest normal bf16
constexpr int kMaxExp = 7;      // 2^(120 + 7) = 2^127, the largest bf16 power of two

__device__ __forceinline__ bool exp_ok(int e) { return e >= kMinExp && e <= kMaxExp; }

// bf16x2 holding 2^(120 + e) twice.
__device__ __forceinline__ uint32_t scale_pair(int e) {
  const uint32_t b = static_cast<uint32_t>(247 + e) << 7;
  return b | (b << 16);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Two codes -> bf16x2 of their values times 2^e.  `sel` picks the byte pair of
// `w` (0x1404: bytes 0 and 1, 0x3424: bytes 2 and 3) and places code j at bits
// 8..15 of half j.  Shifting right by 4 moves the code's exponent and
// mantissa fields (7 bits) to bf16 bits 4..10 and leaves its sign at bit 15,
// which reads as a bf16 whose value is exactly the code's value times 2^-120
// (E4M3 and bf16 exponent biases are 7 and 127; E4M3 subnormals become bf16
// subnormals with the same ratio, zero stays zero).  The multiplication by
// 2^(120 + e) is exact because the product is a normal bf16.
__device__ __forceinline__ uint32_t decode_pair(uint32_t w, uint32_t sel, uint32_t s2) {
  const uint32_t p = __byte_perm(w, 0u, sel);
  const uint32_t t = ((p >> 4) & 0x07F007F0u) | (p & 0x80008000u);
  return bf16x2_mul(t, s2);
}

// Four codes (bytes of w, lowest first) -> two bf16x2 words.
__device__ __forceinline__ void decode4(uint32_t w, uint32_t s2, uint32_t& lo, uint32_t& hi) {
  lo = decode_pair(w, 0x1404u, s2);
  hi = decode_pair(w, 0x3424u, s2);
}

}  // namespace fp8
}  // namespace moe
