// Element arithmetic shared by every kernel that quantises to E4M3 or applies
// SwiGLU, so that fused and standalone paths give identical bytes.  Each step
// uses an explicitly rounded fp32 intrinsic: no contraction into FMAs can
// make two call sites differ.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace moe {

constexpr float kE4M3Max = 448.0f;
constexpr float kQuantEps = 1e-4f;

// Dequantisation multiplier of a tile with max |x| = amax ("Online
// Quantization": s = Q_max / max(A_max, eps); stored as its inverse).
__device__ __forceinline__ float quant_scale(float amax) {
  return __fdiv_rn(fmaxf(amax, kQuantEps), kE4M3Max);
}

// Smallest power of two >= s for a positive normal fp32 s: a non-zero
// mantissa moves the exponent up by one and is cleared.
__device__ __forceinline__ float pow2_ceil(float s) {
  uint32_t b = __float_as_uint(s);
  if (b & 0x007FFFFFu) b = (b & 0x7F800000u) + 0x00800000u;
  return __uint_as_float(b);
}

// x / s rounded to nearest even, given r = RN(1/s): Markstein's correction
// step (P. W. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): y = RN(x r),
// e = x - s y (exact by FMA), q = RN(y + e r).  A zero residual returns y
// itself, which keeps the sign of a zero quotient.  For a bf16 x and a scale
// s from a bf16 tile maximum (the activation and weight quantisers) the tests
// check it against IEEE division on every such (x, s) pair; the SwiGLU
// requantisation applies it to fp32 h, where the tests bound the E4M3 bytes
// against the fp64 reference.
__device__ __forceinline__ float div_by_scale(float x, float s, float r) {
  const float y = __fmul_rn(x, r);
  const float e = __fmaf_rn(-y, s, x);
  return e == 0.0f ? y : __fmaf_rn(e, r, y);
}

// Two fp32 values -> two E4M3 bytes (lo in the low byte), round to nearest
// even, saturating to +-448 (hardware cvt.rn.satfinite.e4m3x2).
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  return static_cast<uint32_t>(e4m3x2(a, b)) | (static_cast<uint32_t>(e4m3x2(c, d)) << 16);
}

// SiLU(g) * u with Swish beta = 1, g / (1 + e^-g) evaluated with the
// hardware exponential and reciprocal approximations (a few fp32 ulps; the
// result is quantised to E4M3, whose step is 2^20 fp32 ulps).  For g < -87,
// e^-g overflows and the quotient is a signed zero.
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float den = __fadd_rn(1.0f, __expf(-g));
  return __fmul_rn(__fdividef(g, den), u);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

}  // namespace moe
