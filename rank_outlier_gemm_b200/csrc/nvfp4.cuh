// NVFP4 group encoder shared by the activation kernel and the weight codec.
//
// SVDQuant (paperlayer.ai summary of arXiv 2411.05007v4): per-group symmetric
// quantization with NVFP4 groups of 16 and FP8 (E4M3) scales (App. D), FP4
// qmax 6 (§3).  For a group v[0..15]:
//   amax = max |v|;  s = E4M3_rn_satfinite(amax / 6)  (IEEE fp32 division)
//   r = 1 / decode(s) (IEEE fp32 reciprocal), or 0 when s decodes to 0
//   q_i = E2M1_rn_satfinite(v_i * r)  (IEEE fp32 multiply), zero codes as +0
// Reciprocal-then-multiply keeps the per-element work to one multiply; the
// explicit __fdiv_rn/__frcp_rn/__fmul_rn intrinsics keep every step a single
// IEEE rounding (no contraction into FMAs).
#pragma once

#include "ptx.cuh"

namespace svdq {
namespace dev {

struct Fp4Group {
  uint32_t lo, hi;  // codes of elements 0..7 and 8..15, element 0 in bits 0..3
  uint32_t scale;   // E4M3 byte
};

__device__ __forceinline__ Fp4Group nvfp4_encode16(const float (&v)[16]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  Fp4Group g;
  g.scale = f32_to_e4m3_rn_sat(__fdiv_rn(amax, 6.0f));
  const float s = e4m3_to_f32(g.scale);
  const float r = s > 0.0f ? __frcp_rn(s) : 0.0f;
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
