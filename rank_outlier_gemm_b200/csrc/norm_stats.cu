// Per-token LayerNorm statistics for the fused norm + activation path.
//
// The configured DiT blocks feed their linear layers adaLN(z) = (1 + scale) *
// LayerNorm(z) + shift; the activation kernel applies that per element and
// needs mu and rstd of each token over its K channels first.  One warp per
// row and one read of it: each lane accumulates, in fp32, the sum and the sum
// of squares of d = z - z0, with z0 the row's first value (a shift that keeps
// the one-pass variance E[d^2] - E[d]^2 from cancelling when the mean is far
// from zero); a fixed shuffle tree combines the lanes; mu = z0 + E[d] and
// rstd = 1 / sqrt(var + eps) with IEEE square root and reciprocal.
#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int kRowsPerBlock = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(32 * kRowsPerBlock) row_stats_kernel(const uint16_t* __restrict__ Z, int M, int K,
                                                                    float eps, float2* __restrict__ stats) {
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  if (m >= M) return;
  const uint4* row = reinterpret_cast<const uint4*>(Z + static_cast<size_t>(m) * K);
  const int n8 = K / 8;  // 16-byte chunks of 8 values
  const float z0 = __uint_as_float(static_cast<uint32_t>(__ldg(Z + static_cast<size_t>(m) * K)) << 16);
  float s1 = 0.0f, s2 = 0.0f;
#pragma unroll 4
  for (int i = lane; i < n8; i += 32) {
    const uint4 w = __ldg(row + i);
    const float d[8] = {bf16_lo(w.x) - z0, bf16_hi(w.x) - z0, bf16_lo(w.y) - z0, bf16_hi(w.y) - z0,
                        bf16_lo(w.z) - z0, bf16_hi(w.z) - z0, bf16_lo(w.w) - z0, bf16_hi(w.w) - z0};
    s1 += ((d[0] + d[1]) + (d[2] + d[3])) + ((d[4] + d[5]) + (d[6] + d[7]));
    float q = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) q = __fmaf_rn(d[j], d[j], q);
    s2 += q;
  }
  const float inv_k = 1.0f / static_cast<float>(K);
  const float m1 = warp_sum(s1) * inv_k;
  const float var = fmaxf(warp_sum(s2) * inv_k - m1 * m1, 0.0f);
  const float mu = z0 + m1;
  if (lane == 0) stats[m] = make_float2(mu, __frcp_rn(__fsqrt_rn(__fadd_rn(var, eps))));
}

}  // namespace

svdq_status launch_row_stats(const void* Z, int M, int K, float eps, float* stats, cudaStream_t stream) {
  const int blocks = (M + kRowsPerBlock - 1) / kRowsPerBlock;
  row_stats_kernel<<<blocks, 32 * kRowsPerBlock, 0, stream>>>(static_cast<const uint16_t*>(Z), M, K, eps,
                                                             reinterpret_cast<float2*>(stats));
  SVDQ_CUDA_TRY(cudaGetLastError());
  return SVDQ_OK;
}

}  // namespace svdq
