// Offline choice of the smoothing strength alpha per layer.
//
// SVDQuant App. D: the smoothing factor lam_j = max|X_j|^alpha / max|W_j|^(1-alpha)
// is computed per channel from activation and weight maxima; the migration
// strength alpha is a per-layer knob (0.5 by default).  svdq_search_alpha
// prepares the layer for each candidate alpha with the library's own
// preparation, runs both runtime kernels on a calibration batch, and scores
// each candidate by the relative Frobenius error of its output against
// X W^T + b accumulated in fp32 from the same bf16 inputs.
#include <algorithm>
#include <cmath>
#include <vector>

#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int kRefTile = 32;

// Y_ref[m, n] = sum_k X[m, k] W[n, k] + b[n] in fp32 (bf16 inputs): a plain
// shared-memory tiled product, used once per search on a calibration batch.
__global__ void reference_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ W,
                                 const float* __restrict__ bias, int M, int N, int K, float* __restrict__ Y) {
  __shared__ float xs[kRefTile][kRefTile + 1];
  __shared__ float ws[kRefTile][kRefTile + 1];
  const int m = blockIdx.y * kRefTile + threadIdx.y;
  const int n = blockIdx.x * kRefTile + threadIdx.x;
  float acc = 0.0f;
  for (int k0 = 0; k0 < K; k0 += kRefTile) {
    const int mx = blockIdx.y * kRefTile + threadIdx.y, kx = k0 + threadIdx.x;
    xs[threadIdx.y][threadIdx.x] =
        (mx < M && kx < K) ? __uint_as_float(static_cast<uint32_t>(X[static_cast<size_t>(mx) * K + kx]) << 16) : 0.0f;
    const int nw = blockIdx.x * kRefTile + threadIdx.y;
    ws[threadIdx.y][threadIdx.x] =
        (nw < N && kx < K) ? __uint_as_float(static_cast<uint32_t>(W[static_cast<size_t>(nw) * K + kx]) << 16) : 0.0f;
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kRefTile; ++k) acc = fmaf(xs[threadIdx.y][k], ws[threadIdx.x][k], acc);
    __syncthreads();
  }
  if (m < M && n < N) Y[static_cast<size_t>(m) * N + n] = acc + (bias ? bias[n] : 0.0f);
}

// sums[0] += sum (Y - Y_ref)^2, sums[1] += sum Y_ref^2 over M*N elements (Y bf16).
__global__ void sq_err_kernel(const uint16_t* __restrict__ Y, const float* __restrict__ Yref, size_t n,
                              double* sums) {
  double e = 0.0, r = 0.0;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const double y = __uint_as_float(static_cast<uint32_t>(Y[i]) << 16), ref = Yref[i];
    e += (y - ref) * (y - ref);
    r += ref * ref;
  }
  for (int o = 16; o > 0; o >>= 1) {
    e += __shfl_xor_sync(0xffffffffu, e, o);
    r += __shfl_xor_sync(0xffffffffu, r, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&sums[0], e);
    atomicAdd(&sums[1], r);
  }
}

struct DevBuf {
  void* p = nullptr;
  ~DevBuf() {
    if (p) cudaFree(p);
  }
};

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" svdq_status svdq_search_alpha(const uint16_t* W_bf16, const uint16_t* X_bf16, int M,
                                         const uint16_t* bias_bf16, int N, int K, const float* alphas,
                                         int n_alpha, const svdq_prepare_opts* opts, void* stream,
                                         double* rel_err, int* best) {
  if (!W_bf16 || !X_bf16 || !alphas || !rel_err || !best)
    return fail(SVDQ_ERR_INVALID_ARG, "W, X, alphas, rel_err and best are required");
  if (M < 1 || n_alpha < 1) return fail(SVDQ_ERR_INVALID_ARG, "M=%d and n_alpha=%d must be >= 1", M, n_alpha);
  for (int i = 0; i < n_alpha; ++i)
    if (!(alphas[i] >= 0.0f && alphas[i] <= 1.0f))
      return fail(SVDQ_ERR_INVALID_ARG, "alphas[%d] must be in [0, 1]", i);
  svdq_prepare_opts o;
  svdq_prepare_opts_default(&o);
  if (opts) o = *opts;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // calibration maxima of the batch itself
  std::vector<float> absmax(K, 0.0f);
  for (int m = 0; m < M; ++m)
    for (int k = 0; k < K; ++k)
      absmax[k] = std::max(absmax[k], std::fabs(bf16_to_f32(X_bf16[static_cast<size_t>(m) * K + k])));
  std::vector<float> bias;
  if (bias_bf16) {
    bias.resize(N);
    for (int n = 0; n < N; ++n) bias[n] = bf16_to_f32(bias_bf16[n]);
  }

  DevBuf dX, dW, dB, dYref, dY, dSums;
  SVDQ_CUDA_TRY(cudaMalloc(&dX.p, static_cast<size_t>(M) * K * 2));
  SVDQ_CUDA_TRY(cudaMalloc(&dW.p, static_cast<size_t>(N) * K * 2));
  SVDQ_CUDA_TRY(cudaMalloc(&dYref.p, static_cast<size_t>(M) * N * 4));
  SVDQ_CUDA_TRY(cudaMalloc(&dY.p, static_cast<size_t>(M) * N * 2));
  SVDQ_CUDA_TRY(cudaMalloc(&dSums.p, 2 * sizeof(double)));
  if (bias_bf16) {
    SVDQ_CUDA_TRY(cudaMalloc(&dB.p, static_cast<size_t>(N) * 4));
    SVDQ_CUDA_TRY(cudaMemcpyAsync(dB.p, bias.data(), static_cast<size_t>(N) * 4, cudaMemcpyHostToDevice, s));
  }
  SVDQ_CUDA_TRY(cudaMemcpyAsync(dX.p, X_bf16, static_cast<size_t>(M) * K * 2, cudaMemcpyHostToDevice, s));
  SVDQ_CUDA_TRY(cudaMemcpyAsync(dW.p, W_bf16, static_cast<size_t>(N) * K * 2, cudaMemcpyHostToDevice, s));
  const dim3 grid((N + kRefTile - 1) / kRefTile, (M + kRefTile - 1) / kRefTile);
  reference_kernel<<<grid, dim3(kRefTile, kRefTile), 0, s>>>(
      static_cast<const uint16_t*>(dX.p), static_cast<const uint16_t*>(dW.p), static_cast<const float*>(dB.p), M,
      N, K, static_cast<float*>(dYref.p));
  SVDQ_CUDA_TRY(cudaGetLastError());

  int best_i = 0;
  for (int i = 0; i < n_alpha; ++i) {
    o.alpha = alphas[i];
    svdq_weights* w = nullptr;
    svdq_status st = svdq_prepare_weights(W_bf16, absmax.data(), bias_bf16, N, K, &o, stream, &w);
    if (st != SVDQ_OK) return st;
    DevBuf ws;
    const size_t wsb = svdq_forward_workspace_bytes(w, M);
    cudaError_t e = cudaMalloc(&ws.p, wsb);
    if (e != cudaSuccess) {
      svdq_weights_destroy(w);
      return cuda_fail(e, "cudaMalloc(workspace)");
    }
    st = svdq_forward(w, dX.p, M, dY.p, ws.p, wsb, stream);
    if (st == SVDQ_OK) {
      e = cudaMemsetAsync(dSums.p, 0, 2 * sizeof(double), s);
      if (e == cudaSuccess) {
        sq_err_kernel<<<148, 256, 0, s>>>(static_cast<const uint16_t*>(dY.p), static_cast<const float*>(dYref.p),
                                          static_cast<size_t>(M) * N, static_cast<double*>(dSums.p));
        e = cudaGetLastError();
      }
      double sums[2] = {0.0, 0.0};
      if (e == cudaSuccess) e = cudaMemcpyAsync(sums, dSums.p, sizeof(sums), cudaMemcpyDeviceToHost, s);
      if (e == cudaSuccess) e = cudaStreamSynchronize(s);
      if (e != cudaSuccess) st = cuda_fail(e, "alpha search scoring");
      rel_err[i] = sums[1] > 0.0 ? std::sqrt(sums[0] / sums[1]) : std::sqrt(sums[0]);
    }
    svdq_weights_destroy(w);
    if (st != SVDQ_OK) return st;
    if (rel_err[i] < rel_err[best_i]) best_i = i;
  }
  *best = best_i;
  return SVDQ_OK;
}
