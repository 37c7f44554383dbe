// Offline NVFP4 codec of the weight residual R / alpha_w (SVDQuant §4.2: the
// residual left after the low-rank split is quantized to 4 bits; App. D: NVFP4
// groups of 16 with E4M3 scales).  Uses the same group encoder as the
// activation kernel.  One thread encodes 64 consecutive values of one row
// (four groups); rows past the end produce zero scales for the padded atoms.
#include "nvfp4.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

using namespace dev;

__global__ void weight_codec_kernel(const float* __restrict__ src, int rows, int rows_pad, int K,
                                    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  __shared__ float rcp_tbl[16];
  if (threadIdx.x < 16) rcp_tbl[threadIdx.x] = rcp_table_entry(static_cast<int>(threadIdx.x));
  __syncthreads();
  const int q_total = K / 64;
  const long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long>(rows_pad) * q_total) return;
  const int row = static_cast<int>(idx / q_total);
  const int qb = static_cast<int>(idx % q_total);
  uint32_t w[8];
  uint32_t sc = 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float v[16];
    if (row < rows) {
      const float4* s4 = reinterpret_cast<const float4*>(src + static_cast<size_t>(row) * K + qb * 64 + g * 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 t = s4[j];
        v[4 * j] = t.x;
        v[4 * j + 1] = t.y;
        v[4 * j + 2] = t.z;
        v[4 * j + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = 0.0f;
    }
    const Fp4Group gq = nvfp4_encode16(v, rcp_tbl);
    w[2 * g] = gq.lo;
    w[2 * g + 1] = gq.hi;
    sc |= gq.scale << (8 * g);
  }
  if (row < rows) {
    uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<size_t>(row) * (K / 2) + qb * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  const size_t off = sf_atom_offset(row, qb * 4, K / 16);
  *reinterpret_cast<uint32_t*>(sf + off) = sc;
}

// Checks the encoder's exact shortcuts against the IEEE intrinsics: div6_rn for
// every fp32 mantissa at each exponent in [-100, 12] (block x = exponent), and
// e4m3_rcp for every positive finite E4M3 byte.  Counts mismatches.
__global__ void selftest_codec_kernel(unsigned int* mismatches) {
  __shared__ float rcp_tbl[16];
  if (threadIdx.x < 16) rcp_tbl[threadIdx.x] = rcp_table_entry(static_cast<int>(threadIdx.x));
  __syncthreads();
  const int ex = static_cast<int>(blockIdx.y) - 100;
  unsigned int bad = 0;
  for (uint32_t mant = blockIdx.x * blockDim.x + threadIdx.x; mant < (1u << 23); mant += gridDim.x * blockDim.x) {
    const float x = __uint_as_float((static_cast<uint32_t>(ex + 127) << 23) | mant);
    bad += __float_as_uint(div6_rn(x)) != __float_as_uint(__fdiv_rn(x, 6.0f));
  }
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 127) {
    const uint32_t b = threadIdx.x;  // 0..126 (0x7F is NaN)
    const float want = b ? __frcp_rn(e4m3_to_f32(b)) : 0.0f;
    bad += __float_as_uint(e4m3_rcp(b, rcp_tbl)) != __float_as_uint(want);
  }
  if (bad) atomicAdd(mismatches, bad);
}

}  // namespace

svdq_status selftest_codec(unsigned int* mismatches_out) {
  unsigned int* d = nullptr;
  SVDQ_CUDA_TRY(cudaMalloc(&d, sizeof(unsigned int)));
  cudaError_t e = cudaMemset(d, 0, sizeof(unsigned int));
  if (e == cudaSuccess) {
    selftest_codec_kernel<<<dim3(512, 113), 256>>>(d);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpy(mismatches_out, d, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  cudaFree(d);
  if (e != cudaSuccess) return cuda_fail(e, "codec self-test");
  return SVDQ_OK;
}

svdq_status launch_weight_codec(const float* d_src, int rows, int K, uint8_t* codes, uint8_t* sf,
                                cudaStream_t stream) {
  const int rows_pad = round_up(rows, 128);
  const long n = static_cast<long>(rows_pad) * (K / 64);
  const int threads = 256;
  const long blocks = (n + threads - 1) / threads;
  weight_codec_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(d_src, rows, rows_pad, K,
                                                                            codes, sf);
  SVDQ_CUDA_TRY(cudaGetLastError());
  return SVDQ_OK;
}

}  // namespace svdq
