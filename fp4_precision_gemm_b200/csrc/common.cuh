// Device helpers shared by the quantize kernels: BF16 unpacking, E4M3 / E2M1 encoding,
// the MX exponent rule, Philox4x32-10 and small reductions.  sm_100a only.
#pragma once
#include <cfloat>
#include <cstdint>
#include <cuda_runtime.h>

namespace fp8q {

// Status word codes written by kernels (match fp8q_status).
constexpr uint32_t kDevTimeout = 6;
constexpr uint32_t kDevBadArg = 7;

// ------------------------------------------------------------------ BF16
// A 32-bit word holds two BF16 values, the lower-addressed one in bits 0..15.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Packed |x| of two BF16 values (sign bits cleared): non-negative BF16 bit patterns order
// like their values, so a SIMD unsigned 16-bit max gives the larger magnitude exactly.
__device__ __forceinline__ uint32_t abs2(uint32_t w) { return w & 0x7FFF7FFFu; }
__device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b) { return __vmaxu2(a, b); }
__device__ __forceinline__ uint32_t hmax(uint32_t w) { return max(w & 0xFFFFu, w >> 16); }
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// ------------------------------------------------------------------ E4M3
// Two FP32 values -> two E4M3 codes, round to nearest even, saturating to +-448
// ("satfinite"); `lo` lands in bits 0..7.  The PTX instruction puts its first source
// operand in the upper byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}

// Two FP32 values to E5M2 (round to nearest even, saturating at +-57344): lo in bits 0-7.
__device__ __forceinline__ uint32_t cvt_e5m2x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}

// Tile scale: sf = 448 / amax (IEEE division); amax == 0 -> 1; overflow -> FLT_MAX.
__device__ __forceinline__ float e4m3_sf(float amax) {
  if (amax == 0.0f) return 1.0f;
  float sf = __fdiv_rn(448.0f, amax);
  return (sf > FLT_MAX) ? FLT_MAX : sf;
}

// E4M3 code -> FP32 (codes 0x7F/0xFF never occur here: the encoder saturates).
__device__ __forceinline__ float e4m3_to_float(uint32_t c) {
  uint32_t e = (c >> 3) & 0xF, m = c & 7;
  float mag = (e == 0) ? (float)m * 0.001953125f                      // m * 2^-9
                       : __uint_as_float(((e + 120u) << 23) | (m << 20));  // 2^(e-7)(1+m/8)
  return (c & 0x80) ? -mag : mag;
}

// ------------------------------------------------------------------ MX (E8M0)
// Smallest e with amax <= 448 * 2^e from the FP32 bits of amax (amax = 1.f * 2^E:
// e = E - 8, plus one when the 23-bit fraction exceeds 0x600000 = 0.75); amax == 0 ->
// -127; clamped to [-127, 127].
__device__ __forceinline__ int mx_exponent(float amax) {
  uint32_t b = __float_as_uint(amax) & 0x7FFFFFFFu;
  if (b == 0) return -127;
  int E;
  uint32_t mant;
  uint32_t ef = b >> 23;
  if (ef == 0) {                       // FP32 subnormal: normalise
    int lz = __clz(b);                 // most significant set bit at 31 - lz (< 23)
    E = (31 - lz) - 149;
    mant = (b << (lz - 8)) & 0x7FFFFFu;
  } else {
    E = (int)ef - 127;
    mant = b & 0x7FFFFFu;
  }
  int e = E - 8 + (mant > 0x600000u ? 1 : 0);
  return max(-127, min(127, e));
}

// 2^-e as an exact FP32 value for e in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2_neg(int e) {
  int k = -e;
  return (k >= -126) ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// ------------------------------------------------------------------ E2M1
// Magnitude grid {0, 0.5, 1, 1.5, 2, 3, 4, 6}; code index = grid index, bit 3 = sign.
// Stochastic rounding with one 32-bit random word: up iff (word >> 8) * 2^-24 < p,
// p = (|y| - lo) / (hi - lo).  The gaps of the E2M1 grid are powers of two, so p is a
// fixed-point fraction of |y|'s own mantissa bits and the decision is exact in integers:
//   |y| in [1, 6):   lo keeps |y|'s exponent and top mantissa bit, p = (low 22 bits) / 2^22,
//                    and "up" is the carry out of those 22 bits when 2^22 - 1 - (u24 >> 2)
//                    is added to them; the code is then (bits >> 22) - 252, capped at 7
//                    (|y| >= 6 saturates, no rounding);
//   |y| < 1:         the grid step is 0.5 throughout, so with F = |y| * 2^25 (exact) the
//                    floor code is F >> 24 and "up" is u24 < F mod 2^24; both are the carry
//                    of ceil(F) + (2^24 - 1 - u24) into bit 24 (u24 < F <=> u24 < ceil(F)).
// (u < p with u = u24 / 2^24 and p = L / 2^22 is u24 < 4L, i.e. (u24 >> 2) < L.)
__device__ __forceinline__ uint32_t e2m1_sr(float y, uint32_t word) {
  const uint32_t b = __float_as_uint(y), ab = b & 0x7FFFFFFFu;
  const uint32_t c_hi = min((ab + (0x3FFFFFu - (word >> 10)) - (252u << 22)) >> 22, 7u);
  const uint32_t c_lo = (__float2uint_ru(__fmul_rn(__uint_as_float(ab), 33554432.0f)) + (0xFFFFFFu - (word >> 8))) >> 24;
  return (ab >= 0x3F800000u ? c_hi : c_lo) | ((b >> 28) & 8u);
}

// Two values to E2M1 by round-to-nearest-even with saturation at 6 (hardware conversion):
// returns (code(hi) << 4) | code(lo).
__device__ __forceinline__ uint32_t e2m1x2_rne(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// ------------------------------------------------------------------ Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11).
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    // 32 x 32 -> 64-bit products (one wide multiply each): high and low words
    const uint64_t p0 = (uint64_t)c.x * 0xD2511F53u, p1 = (uint64_t)c.z * 0xCD9E8D57u;
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// The same generator with the key schedule precomputed: rk[2r], rk[2r + 1] are the key words
// of round r (k0 + r * 0x9E3779B9, k1 + r * 0xBB67AE85), e.g. kernel parameters, so a round is
// two wide multiplies and two three-way xors.
__device__ __forceinline__ uint4 philox4x32_10_rk(uint4 c, const uint32_t (&rk)[20]) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)c.x * 0xD2511F53u, p1 = (uint64_t)c.z * 0xCD9E8D57u;
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    c = make_uint4(hi1 ^ c.y ^ rk[2 * r], lo1, hi0 ^ c.w ^ rk[2 * r + 1], lo0);
  }
  return c;
}

// ------------------------------------------------------------------ MMA-tiled scale layout
// Byte offset of scale (row r, scale column c) with `s4` = ceil(scale columns / 4) atoms
// per 128-row band.
__device__ __forceinline__ int64_t sf_tiled_offset(int64_t r, int64_t c, int64_t s4) {
  return (((r >> 7) * s4 + (c >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (c & 3);
}

}  // namespace fp8q
