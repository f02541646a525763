// NVFP4 element and scale conversions on the device (sm_100a).
//
// Format (BiLoCo README, section "Kernel": FP4 activation and residual with
// block scales): E2M1 codes on {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}, one
// E4M3 scale per 16 elements along K.  Rounding: FP32 quotient v/S rounded to
// nearest, then E2M1 to nearest with ties to the even code and saturation
// (the hardware cvt.rn.satfinite.e2m1x2.f32); E4M3 scales to nearest-even with
// saturation at 448 (cvt.rn.satfinite.e4m3x2.f32).  Zero magnitudes are stored
// as code 0, never as negative zero.
#pragma once

#include <cstdint>

namespace biloco {

// FP32 -> E4M3 byte, nearest-even, clamped to +-448.
__device__ __forceinline__ uint32_t e4m3_from_f32(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
  return r & 0xFFu;
}

// Exact value of a non-negative E4M3 byte (sign bit ignored; 0x7F never occurs).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (e == 0) return static_cast<float>(m) * 0x1p-9f;          // subnormal: m/8 * 2^-6
  return __uint_as_float(((e + 120u) << 23) | (m << 20));     // (1+m/8) * 2^(e-7)
}

// Two FP32 values -> one byte of E2M1 codes, `lo` in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  uint32_t b = r & 0xFFu;
  if ((b & 0x07u) == 0) b &= 0xF0u;     // -0 -> +0 in the low nibble
  if ((b & 0x70u) == 0) b &= 0x0Fu;     // and in the high nibble
  return b;
}

// 16 values and their block scale S (FP32) -> 8 bytes of packed codes.
__device__ __forceinline__ uint2 encode_block16(const float (&v)[16], float S) {
  uint2 out = make_uint2(0u, 0u);
  if (S != 0.0f) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      out.x |= e2m1x2(__fdiv_rn(v[2 * j], S), __fdiv_rn(v[2 * j + 1], S)) << (8 * j);
      out.y |= e2m1x2(__fdiv_rn(v[8 + 2 * j], S), __fdiv_rn(v[8 + 2 * j + 1], S)) << (8 * j);
    }
  }
  return out;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ float amax16(const float (&v)[16]) {
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) a = fmaxf(a, fabsf(v[j]));
  return a;
}

// E2M1 code of a BF16 value v under block scale S, without dividing.
//
// The format asks for E2M1_RNE(RN_fp32(v / S)).  S is an E4M3 value (at most 4
// significant bits) and every E2M1 rounding boundary t in {.25, .75, 1.25, 1.75,
// 2.5, 3.5, 5} has at most 3, so t * S is exact in FP32.  A BF16 |v| has at most 8
// significant bits, so it is either equal to t * S or at least one BF16 step
// (relative 2^-8) away from it, far outside the FP32 rounding of the quotient.
// Hence RN(|v| / S) > t  <=>  |v| > t * S  and  RN(|v| / S) == t  <=>  |v| == t * S,
// and comparing |v| with the seven exact products gives the same code as the
// division.  At an exact boundary the even code wins (ties to even), i.e. the
// boundaries .75, 1.75 and 3.5 round up and the others round down.
struct E2M1Thresholds {
  float t[7];
};
__device__ __forceinline__ E2M1Thresholds e2m1_thresholds(float S) {
  E2M1Thresholds th;
  th.t[0] = 0.25f * S; th.t[1] = 0.75f * S; th.t[2] = 1.25f * S; th.t[3] = 1.75f * S;
  th.t[4] = 2.5f * S;  th.t[5] = 3.5f * S;  th.t[6] = 5.0f * S;
  return th;
}
__device__ __forceinline__ uint32_t e2m1_code_bf16(float v, const E2M1Thresholds& th, bool zero_scale) {
  const float a = fabsf(v);
  uint32_t c = (a > th.t[0]) + (a >= th.t[1]) + (a > th.t[2]) + (a >= th.t[3]) + (a > th.t[4]) +
               (a >= th.t[5]) + (a > th.t[6]);
  if (zero_scale) c = 0;
  return (c != 0 && v < 0.0f) ? (c | 8u) : c;
}

// RN_FP32(v / S) without a division instruction, by Markstein's correction of a
// reciprocal-based quotient (P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990, Thm. 8):
// with y = RN(1/S), q0 = RN(v y) and the exact remainder r = v - S q0 (one FMA),
// RN(q0 + r y) equals RN(v / S) in round-to-nearest when y is correctly rounded
// and nothing overflows or underflows.  Here |v| < 2^16 and S >= 2^-9.
__device__ __forceinline__ float div_rn_by(float v, float S, float y) {
  const float q0 = __fmul_rn(v, y);
  const float r = __fmaf_rn(-S, q0, v);
  return __fmaf_rn(r, y, q0);
}

// Activation block (no tensor scale), quotient by Markstein's correction and the
// hardware E2M1 conversion (nearest, ties to even, saturating): the same codes as
// the definition E2M1(RN(x / s)).
__device__ __forceinline__ uint32_t quant_act_block_fast(const float (&v)[16], uint2& codes) {
  const float t = __fdiv_rn(amax16(v), 6.0f);
  const uint32_t s = e4m3_from_f32(t);
  const float S = e4m3_to_f32(s);
  codes = make_uint2(0u, 0u);
  if (S != 0.0f) {
    const float y = __frcp_rn(S);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      codes.x |= e2m1x2(div_rn_by(v[2 * j], S, y), div_rn_by(v[2 * j + 1], S, y)) << (8 * j);
      codes.y |= e2m1x2(div_rn_by(v[8 + 2 * j], S, y), div_rn_by(v[8 + 2 * j + 1], S, y)) << (8 * j);
    }
  }
  return s;
}

// 16 BF16 values from 32 bytes (16-byte aligned) of shared or global memory.
__device__ __forceinline__ void bf16x16_to_f32(const uint4& a, const uint4& b, float (&v)[16]) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFFu);
    v[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
  }
}

// Byte offset of the scale of row `row` (< 128 within its 128-row tile) and
// 16-element block `blk` (block index within the row) inside a run of 512-byte
// scale atoms: one atom per 64 elements of K, 4 atoms per 256-element chunk.
__device__ __forceinline__ uint32_t sf_atom_offset(uint32_t row, uint32_t blk) {
  const uint32_t chunk = blk >> 4, step = (blk >> 2) & 3u, q = blk & 3u;
  return ((chunk * 4u + step) * 512u) + (row & 31u) * 16u + ((row >> 5) & 3u) * 4u + q;
}

}  // namespace biloco
