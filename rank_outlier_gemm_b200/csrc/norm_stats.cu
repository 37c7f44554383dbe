// Per-token LayerNorm statistics for the fused norm + activation path.
//
// The configured DiT blocks feed their linear layers adaLN(z) = (1 + scale) *
// LayerNorm(z) + shift; the activation kernel applies that per element and
// needs mu and rstd of each token over its K channels first.  One warp per
// row: a pass for the mean and a second pass (mostly from L2) for the centred
// sum of squares, both accumulated in fp32 per lane and combined by a fixed
// shuffle tree; rstd = 1 / sqrt(var + eps) with IEEE square root and
// reciprocal.
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
  float s = 0.0f;
  for (int i = lane; i < n8; i += 32) {
    const uint4 w = __ldg(row + i);
    s += bf16_lo(w.x) + bf16_hi(w.x) + bf16_lo(w.y) + bf16_hi(w.y) + bf16_lo(w.z) + bf16_hi(w.z) +
         bf16_lo(w.w) + bf16_hi(w.w);
  }
  const float mu = __fdiv_rn(warp_sum(s), static_cast<float>(K));
  float q = 0.0f;
  for (int i = lane; i < n8; i += 32) {
    const uint4 w = __ldg(row + i);
    const float d[8] = {bf16_lo(w.x) - mu, bf16_hi(w.x) - mu, bf16_lo(w.y) - mu, bf16_hi(w.y) - mu,
                        bf16_lo(w.z) - mu, bf16_hi(w.z) - mu, bf16_lo(w.w) - mu, bf16_hi(w.w) - mu};
#pragma unroll
    for (int j = 0; j < 8; ++j) q = __fmaf_rn(d[j], d[j], q);
  }
  const float var = __fdiv_rn(warp_sum(q), static_cast<float>(K));
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
