// NVFP4 group encoder shared by the activation kernel and the weight codec.
//
// SVDQuant (paperlayer.ai summary of arXiv 2411.05007v4): per-group symmetric
// quantization with NVFP4 groups of 16 and FP8 (E4M3) scales (App. D), FP4
// qmax 6 (§3).  For a group v[0..15]:
//   amax = max |v|;  s = E4M3_rn_satfinite(amax / 6)  (IEEE fp32 division)
//   r = 1 / decode(s) (IEEE fp32 reciprocal), or 0 when s decodes to 0
//   q_i = E2M1_rn_satfinite(v_i * r)  (IEEE fp32 multiply), zero codes as +0
// Reciprocal-then-multiply keeps the per-element work to one multiply.  The
// division and the reciprocal are computed by exact shortcuts, both checked
// against the IEEE intrinsics over their whole domains by svdq_selftest_codec:
// - amax / 6: q0 = RN(amax * RN(1/6)), then one fused correction with the
//   exact remainder fma(-q0, 6, amax), the method of Brisebarre, Muller and
//   Raina, "Accelerating correctly rounded floating-point division when the
//   divisor is known in advance" (IEEE Trans. Computers 53(8), 2004); for every
//   fp32 mantissa it gives RN(amax / 6) (checked exhaustively), and below the
//   normal range the E4M3 scale is 0 either way.
// - 1 / decode(s): decode(s) is (1 + m/8) 2^(e-7), or m 2^-9 when e = 0, with a
//   3-bit m, and
//   RN(1 / (2^k x)) = 2^-k RN(1 / x) in the normal range, so a 16-entry table of
//   RN(1 / (1 + m/8)) and RN(1 / m) (filled with the IEEE reciprocal itself)
//   plus an exponent shift gives the IEEE reciprocal exactly.
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace dev {

struct Fp4Group {
  uint32_t lo, hi;  // codes of elements 0..7 and 8..15, element 0 in bits 0..3
  uint32_t scale;   // E4M3 byte
};

// RN(x / 6) for every finite fp32 x whose quotient is normal (Brisebarre,
// Muller and Raina 2004: multiply by the rounded reciprocal, then one fused
// correction with the exact remainder).
__device__ __forceinline__ float div6_rn(float x) {
  const float c = __uint_as_float(0x3E2AAAABu);  // RN(1/6)
  const float q0 = __fmul_rn(x, c);
  const float r = __fmaf_rn(-q0, 6.0f, x);
  return __fmaf_rn(r, c, q0);
}

// Entry i of the reciprocal table: RN(1 / (1 + i/8)) for i < 8, RN(1 / (i - 8)) for i > 8.
__device__ __forceinline__ float rcp_table_entry(int i) {
  return i < 8 ? __frcp_rn(1.0f + 0.125f * static_cast<float>(i)) : (i > 8 ? __frcp_rn(static_cast<float>(i - 8)) : 0.0f);
}

// RN(1 / decode(b)) for a positive finite E4M3 byte b, 0 for b = 0.
__device__ __forceinline__ float e4m3_rcp(uint32_t b, const float* tbl) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  const float t = tbl[e ? m : 8u + m];
  // normal: decode = (1 + m/8) 2^(e-7); subnormal: decode = m 2^-9
  const int shift = e ? 7 - static_cast<int>(e) : 9;
  const float r = __uint_as_float(static_cast<uint32_t>(static_cast<int>(__float_as_uint(t)) + shift * (1 << 23)));
  return b ? r : 0.0f;
}

__device__ __forceinline__ Fp4Group nvfp4_encode16(const float (&v)[16], const float* rcp_tbl) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  Fp4Group g;
  g.scale = f32_to_e4m3_rn_sat(div6_rn(amax));
  const float r = e4m3_rcp(g.scale, rcp_tbl);
  float t[16];
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float2 m = mul_f32x2(make_float2(v[i], v[i + 1]), make_float2(r, r));
    t[i] = m.x;
    t[i + 1] = m.y;
  }
  g.lo = e2m1_canonical_zero(f32x8_to_e2m1(t[0], t[1], t[2], t[3], t[4], t[5], t[6], t[7]));
  g.hi = e2m1_canonical_zero(f32x8_to_e2m1(t[8], t[9], t[10], t[11], t[12], t[13], t[14], t[15]));
  return g;
}

// Byte offset of scale (row, kb) in the block-scale atom layout: 128-row x
// 4-column atoms of 512 bytes, K-atoms fastest; kb_total = K / 16.
__host__ __device__ __forceinline__ size_t sf_atom_offset(int row, int kb, int kb_total) {
  const size_t atom = static_cast<size_t>(row >> 7) * static_cast<size_t>(kb_total >> 2) +
                      static_cast<size_t>(kb >> 2);
  return atom * 512 + static_cast<size_t>((row & 31) * 16 + ((row >> 5) & 3) * 4 + (kb & 3));
}

}  // namespace dev
}  // namespace svdq
