// C ABI of the SVDQuant W4A4 layer: argument validation, the weights handle,
// tensor maps over device buffers, and the kernel launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "svdq_internal.h"

namespace {

thread_local char g_err[512] = "";
uint64_t g_wait_ns = 2000000000ull;
std::mutex g_mu;
int* g_err_words[64] = {};
int g_arch_ok[64] = {};  // 0 unknown, 1 sm_100, -1 other

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

namespace svdq {

svdq_status fail(svdq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

svdq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(e == cudaErrorMemoryAllocation ? SVDQ_ERR_OOM : SVDQ_ERR_CUDA, "%s: %s", what,
              cudaGetErrorString(e));
}

uint64_t wait_limit_ns() { return g_wait_ns; }

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_words[dev]) {
    int* p = nullptr;
    if (cudaMalloc(&p, sizeof(int)) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, sizeof(int)) != cudaSuccess) return nullptr;
    g_err_words[dev] = p;
  }
  return g_err_words[dev];
}

svdq_status check_device() {
  int dev = 0;
  SVDQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
  if (g_arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    SVDQ_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    SVDQ_CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (g_arch_ok[dev] != 1) return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "device %d is not sm_100", dev);
  return SVDQ_OK;
}

svdq_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t inner,
                         uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                         CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for [%llu x %llu] box [%u x %u]",
                static_cast<int>(r), static_cast<unsigned long long>(outer),
                static_cast<unsigned long long>(inner), box_outer, box_inner);
  return SVDQ_OK;
}

svdq_status make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, const uint64_t dims[3],
                         const uint64_t strides[2], const uint32_t box[3]) {
  auto fn = encode_fn();
  if (!fn) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  cuuint64_t st[2] = {strides[0], strides[1]};
  cuuint32_t bx[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for a 3-D map [%llu x %llu x %llu]",
                static_cast<int>(r), static_cast<unsigned long long>(dims[2]),
                static_cast<unsigned long long>(dims[1]), static_cast<unsigned long long>(dims[0]));
  return SVDQ_OK;
}

namespace {

void free_device(svdq_weights* w) {
  cudaFree(w->d_wq);
  cudaFree(w->d_wsf);
  cudaFree(w->d_inv_lam);
  cudaFree(w->d_L1t);
  cudaFree(w->d_L2t);
  cudaFree(w->d_bias);
  w->d_wq = w->d_wsf = nullptr;
  w->d_inv_lam = w->d_bias = nullptr;
  w->d_L1t = w->d_L2t = nullptr;
}

// (Re)builds the device low-rank factors L1'^T [r_pad, K] and L2^T/alpha_w
// [N, r_pad] from the host copies, and their tensor maps.
svdq_status upload_lowrank(svdq_weights* w, cudaStream_t stream) {
  const int K = w->K, N = w->N, r = w->rank;
  const int rp = round_up(r, 16);
  cudaFree(w->d_L1t);
  cudaFree(w->d_L2t);
  w->d_L1t = w->d_L2t = nullptr;
  w->r_pad = rp;
  if (rp == 0) return SVDQ_OK;
  std::vector<uint16_t> l1t(static_cast<size_t>(rp) * K, 0), l2t(static_cast<size_t>(N) * rp, 0);
  for (int k = 0; k < K; ++k)
    for (int i = 0; i < r; ++i) l1t[static_cast<size_t>(i) * K + k] = w->L1p[static_cast<size_t>(k) * r + i];
  const double inv_aw = 1.0 / static_cast<double>(w->alpha_w);
  for (int i = 0; i < r; ++i)
    for (int n = 0; n < N; ++n) {
      const float v = bf16_to_f32(w->L2[static_cast<size_t>(i) * N + n]);
      l2t[static_cast<size_t>(n) * rp + i] = f32_to_bf16_rne(static_cast<float>(v * inv_aw));  // exact
    }
  SVDQ_CUDA_TRY(cudaMalloc(&w->d_L1t, l1t.size() * 2));
  SVDQ_CUDA_TRY(cudaMalloc(&w->d_L2t, l2t.size() * 2));
  SVDQ_CUDA_TRY(cudaMemcpyAsync(w->d_L1t, l1t.data(), l1t.size() * 2, cudaMemcpyHostToDevice, stream));
  SVDQ_CUDA_TRY(cudaMemcpyAsync(w->d_L2t, l2t.data(), l2t.size() * 2, cudaMemcpyHostToDevice, stream));
  SVDQ_CUDA_TRY(cudaStreamSynchronize(stream));
  svdq_status st = make_tmap_2d(&w->map_l1, w->d_L1t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, rp,
                                static_cast<uint64_t>(K) * 2, 64, rp, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  st = make_tmap_2d(&w->map_l2_256, w->d_L2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rp, N,
                    static_cast<uint64_t>(rp) * 2, 32, 256, CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != SVDQ_OK) return st;
  return make_tmap_2d(&w->map_l2_128, w->d_L2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rp, N,
                      static_cast<uint64_t>(rp) * 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B);
}

svdq_status build_handle(int N, int K, int rank, const float* inv_lam, const uint16_t* L1p,
                         const uint16_t* L2, const float* R, const float* bias, int keep_residual, int format,
                         cudaStream_t stream, svdq_weights** out) {
  svdq_weights* w = new (std::nothrow) svdq_weights();
  if (!w) return fail(SVDQ_ERR_OOM, "host allocation failed");
  auto bail = [&](svdq_status s) {
    free_device(w);
    delete w;
    return s;
  };
  cudaGetDevice(&w->device);
  w->N = N;
  w->K = K;
  w->rank = rank;
  w->format = format;
  const size_t nk = static_cast<size_t>(N) * K;
  // INT4's bf16 scales span fp32's exponent range: no per-tensor factor
  w->alpha_w = format == SVDQ_FORMAT_INT4 ? 1.0f : weight_factor(R, nk);
  w->inv_lam.assign(inv_lam, inv_lam + K);
  if (rank > 0) {
    w->L1p.assign(L1p, L1p + static_cast<size_t>(K) * rank);
    w->L2.assign(L2, L2 + static_cast<size_t>(rank) * N);
  }
  w->bias.assign(N, 0.0f);
  if (bias) std::copy(bias, bias + N, w->bias.begin());
  std::vector<float> Rp(nk);
  for (size_t i = 0; i < nk; ++i) Rp[i] = static_cast<float>(static_cast<double>(R[i]) / w->alpha_w);
  if (keep_residual) w->residual = Rp;

  const int npad = format == SVDQ_FORMAT_INT4 ? round_up(N, 256) : round_up(N, 128);
  const size_t sf_bytes = format == SVDQ_FORMAT_INT4 ? static_cast<size_t>(K / 64) * npad * 2
                                                      : static_cast<size_t>(npad) * (K / 16);
  cudaError_t e;
  if ((e = cudaMalloc(&w->d_wq, nk / 2)) != cudaSuccess) return bail(cuda_fail(e, "cudaMalloc codes"));
  if ((e = cudaMalloc(&w->d_wsf, sf_bytes)) != cudaSuccess) return bail(cuda_fail(e, "cudaMalloc scales"));
  if ((e = cudaMalloc(&w->d_inv_lam, static_cast<size_t>(K) * 4)) != cudaSuccess)
    return bail(cuda_fail(e, "cudaMalloc inv_lam"));
  const size_t bias_n = static_cast<size_t>(round_up(N, 256));
  if ((e = cudaMalloc(&w->d_bias, bias_n * 4)) != cudaSuccess) return bail(cuda_fail(e, "cudaMalloc bias"));
  std::vector<float> bias_pad(bias_n, 0.0f);
  std::copy(w->bias.begin(), w->bias.end(), bias_pad.begin());
  float* d_R = nullptr;
  if ((e = cudaMalloc(&d_R, nk * 4)) != cudaSuccess) return bail(cuda_fail(e, "cudaMalloc residual"));
  svdq_status st = SVDQ_OK;
  std::vector<uint8_t> h_codes;
  std::vector<uint16_t> h_scales;
  if (format == SVDQ_FORMAT_INT4) {  // offline host codec; the device gets packed codes and scales
    h_codes.assign(nk / 2, 0);
    h_scales.assign(sf_bytes / 2, 0);
    int4_encode_rows(Rp.data(), N, K, npad, h_codes.data(), h_scales.data());
  }
  do {
    if (format == SVDQ_FORMAT_INT4) {
      if ((e = cudaMemcpyAsync(w->d_wq, h_codes.data(), nk / 2, cudaMemcpyHostToDevice, stream)) != cudaSuccess ||
          (e = cudaMemcpyAsync(w->d_wsf, h_scales.data(), sf_bytes, cudaMemcpyHostToDevice, stream)) !=
              cudaSuccess) {
        st = cuda_fail(e, "cudaMemcpyAsync INT4 codes");
        break;
      }
    }
    if ((e = cudaMemcpyAsync(d_R, Rp.data(), nk * 4, cudaMemcpyHostToDevice, stream)) != cudaSuccess ||
        (e = cudaMemcpyAsync(w->d_inv_lam, inv_lam, static_cast<size_t>(K) * 4, cudaMemcpyHostToDevice,
                             stream)) != cudaSuccess ||
        (e = cudaMemcpyAsync(w->d_bias, bias_pad.data(), bias_n * 4, cudaMemcpyHostToDevice, stream)) !=
            cudaSuccess) {
      st = cuda_fail(e, "cudaMemcpyAsync weights");
      break;
    }
    if (format != SVDQ_FORMAT_INT4) {
      st = launch_weight_codec(d_R, N, K, w->d_wq, w->d_wsf, stream);
      if (st != SVDQ_OK) break;
    }
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) st = cuda_fail(e, "weight codec");
  } while (0);
  cudaFree(d_R);
  if (st != SVDQ_OK) return bail(st);
  st = upload_lowrank(w, stream);
  if (st != SVDQ_OK) return bail(st);
  if (format == SVDQ_FORMAT_INT4) {  // one 64-wide group (32 bytes) of 256 rows per load
    st = make_tmap_2d(&w->map_wq_256, w->d_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, 32, 256,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != SVDQ_OK) return bail(st);
    *out = w;
    return SVDQ_OK;
  }
  st = make_tmap_2d(&w->map_wq_256, w->d_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, 128, 256,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  if (st == SVDQ_OK)
    st = make_tmap_2d(&w->map_wq_128, w->d_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (st == SVDQ_OK) {  // scale atoms [npad/128][K/64][512 bytes] as 32-bit words
    const uint64_t dims[3] = {128, static_cast<uint64_t>(K / 64), static_cast<uint64_t>(npad / 128)};
    const uint64_t strides[2] = {512, static_cast<uint64_t>(K / 64) * 512};
    const uint32_t box[3] = {128, 4, 2};
    st = make_tmap_3d(&w->map_wsf, w->d_wsf, CU_TENSOR_MAP_DATA_TYPE_UINT32, dims, strides, box);
  }
  if (st != SVDQ_OK) return bail(st);
  *out = w;
  return SVDQ_OK;
}

svdq_status check_shape(int N, int K) {
  if (N <= 0 || K <= 0) return fail(SVDQ_ERR_INVALID_ARG, "N and K must be positive (N=%d K=%d)", N, K);
  if (K % 64) return fail(SVDQ_ERR_INVALID_ARG, "K=%d must be a multiple of 64", K);
  if (N % 16) return fail(SVDQ_ERR_INVALID_ARG, "N=%d must be a multiple of 16", N);
  return SVDQ_OK;
}

svdq_status check_runtime(const svdq_weights* w, int M) {
  if (!w) return fail(SVDQ_ERR_INVALID_ARG, "null weights handle");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARG, "M=%d must be >= 1", M);
  int dev = -1;
  SVDQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != w->device)
    return fail(SVDQ_ERR_INVALID_ARG, "current device %d differs from the handle's device %d", dev, w->device);
  return check_device();
}

svdq_status check_dev_ptr(const void* p, const char* name) {
  if (!p) return fail(SVDQ_ERR_INVALID_ARG, "%s is null", name);
  if (!aligned16(p)) return fail(SVDQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return SVDQ_OK;
}

}  // namespace
}  // namespace svdq

using namespace svdq;

namespace {

// Copy streams and events of svdq_forward_host, one set per device, created on
// first use and kept for the life of the process.
struct HostPipe {
  static constexpr int kMaxChunks = 4;
  std::mutex mu;  // one call at a time enqueues on a device's pipe
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t loaded[kMaxChunks] = {}, computed[kMaxChunks] = {};
};
HostPipe g_host_pipe[64];
std::mutex g_host_pipe_mu;

svdq_status host_pipe(HostPipe** out) {
  int dev = 0;
  SVDQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_host_pipe_mu);
  HostPipe& hp = g_host_pipe[dev];
  if (!hp.ready) {
    SVDQ_CUDA_TRY(cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking));
    SVDQ_CUDA_TRY(cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking));
    SVDQ_CUDA_TRY(cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming));
    SVDQ_CUDA_TRY(cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming));
    for (int c = 0; c < HostPipe::kMaxChunks; ++c) {
      SVDQ_CUDA_TRY(cudaEventCreateWithFlags(&hp.loaded[c], cudaEventDisableTiming));
      SVDQ_CUDA_TRY(cudaEventCreateWithFlags(&hp.computed[c], cudaEventDisableTiming));
    }
    hp.ready = true;
  }
  *out = &hp;
  return SVDQ_OK;
}

}  // namespace

extern "C" {

void svdq_prepare_opts_default(svdq_prepare_opts* o) {
  if (!o) return;
  o->alpha = 0.5f;
  o->rank = 32;
  o->power_iters = 4;
  o->oversample = 16;
  o->seed = 0;
  o->keep_residual = 0;
  o->refine_iters = 1;
  o->format = SVDQ_FORMAT_NVFP4;
}

svdq_status svdq_prepare_weights(const uint16_t* W_bf16, const float* act_absmax, const uint16_t* bias_bf16,
                                 int N, int K, const svdq_prepare_opts* opts, void* stream,
                                 svdq_weights** out) {
  if (!out) return fail(SVDQ_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  if (!W_bf16 || !act_absmax) return fail(SVDQ_ERR_INVALID_ARG, "W_bf16 and act_absmax are required");
  SVDQ_TRY(check_shape(N, K));
  svdq_prepare_opts o;
  svdq_prepare_opts_default(&o);
  if (opts) o = *opts;
  if (o.rank < 0 || o.rank > 128 || o.rank > std::min(N, K))
    return fail(SVDQ_ERR_INVALID_ARG, "rank=%d must be in [0, min(128, N, K)]", o.rank);
  if (!(o.alpha >= 0.0f && o.alpha <= 1.0f)) return fail(SVDQ_ERR_INVALID_ARG, "alpha must be in [0, 1]");
  if (o.refine_iters < 1 || o.refine_iters > 64)
    return fail(SVDQ_ERR_INVALID_ARG, "refine_iters=%d must be in [1, 64]", o.refine_iters);
  if (o.format != SVDQ_FORMAT_NVFP4 && o.format != SVDQ_FORMAT_INT4)
    return fail(SVDQ_ERR_INVALID_ARG, "format=%d is neither NVFP4 (0) nor INT4 (1)", o.format);
  if (o.format == SVDQ_FORMAT_INT4 && o.refine_iters != 1)
    return fail(SVDQ_ERR_INVALID_ARG, "refinement (refine_iters > 1) is implemented for NVFP4 only");
  for (int k = 0; k < K; ++k)
    if (!std::isfinite(act_absmax[k]) || act_absmax[k] < 0)
      return fail(SVDQ_ERR_INVALID_ARG, "act_absmax[%d] is negative or not finite", k);
  SVDQ_TRY(check_device());
  HostSplit hs;
  SVDQ_TRY(host_prepare_split(W_bf16, act_absmax, N, K, o, &hs));
  std::vector<float> bias;
  if (bias_bf16) {
    bias.resize(N);
    for (int n = 0; n < N; ++n) bias[n] = bf16_to_f32(bias_bf16[n]);
  }
  SVDQ_TRY(build_handle(N, K, o.rank, hs.inv_lam.data(), hs.L1p.data(), hs.L2.data(), hs.R.data(),
                        bias_bf16 ? bias.data() : nullptr, o.keep_residual, o.format,
                        static_cast<cudaStream_t>(stream), out));
  (*out)->refine_err = hs.refine_err;
  return SVDQ_OK;
}

svdq_status svdq_weights_refine_errors(const svdq_weights* w, double* errors, int max_count, int* count) {
  if (!w || !count) return fail(SVDQ_ERR_INVALID_ARG, "null weights handle or count");
  if (max_count > 0 && !errors) return fail(SVDQ_ERR_INVALID_ARG, "errors is null");
  *count = static_cast<int>(w->refine_err.size());
  for (int i = 0; i < std::min(*count, max_count); ++i) errors[i] = w->refine_err[i];
  return SVDQ_OK;
}

svdq_status svdq_weights_from_factors(int N, int K, int rank, const float* inv_lam, const uint16_t* L1p_bf16,
                                      const uint16_t* L2_bf16, const float* R, const float* bias, void* stream,
                                      svdq_weights** out) {
  if (!out) return fail(SVDQ_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  SVDQ_TRY(check_shape(N, K));
  if (rank < 0 || rank > 128) return fail(SVDQ_ERR_INVALID_ARG, "rank=%d must be in [0, 128]", rank);
  if (!inv_lam || !R) return fail(SVDQ_ERR_INVALID_ARG, "inv_lam and R are required");
  if (rank > 0 && (!L1p_bf16 || !L2_bf16)) return fail(SVDQ_ERR_INVALID_ARG, "rank > 0 needs L1p and L2");
  const size_t nk = static_cast<size_t>(N) * K;
  for (size_t i = 0; i < nk; ++i)
    if (!std::isfinite(R[i])) return fail(SVDQ_ERR_INVALID_ARG, "R has a non-finite value");
  for (int k = 0; k < K; ++k)
    if (!std::isfinite(inv_lam[k])) return fail(SVDQ_ERR_INVALID_ARG, "inv_lam has a non-finite value");
  SVDQ_TRY(check_device());
  return build_handle(N, K, rank, inv_lam, L1p_bf16, L2_bf16, R, bias, 1, SVDQ_FORMAT_NVFP4,
                      static_cast<cudaStream_t>(stream), out);
}

svdq_status svdq_weights_from_factors_fmt(int N, int K, int rank, const float* inv_lam, const uint16_t* L1p_bf16,
                                          const uint16_t* L2_bf16, const float* R, const float* bias, int format,
                                          void* stream, svdq_weights** out) {
  if (format != SVDQ_FORMAT_NVFP4 && format != SVDQ_FORMAT_INT4)
    return fail(SVDQ_ERR_INVALID_ARG, "format=%d is neither NVFP4 (0) nor INT4 (1)", format);
  if (format == SVDQ_FORMAT_NVFP4)
    return svdq_weights_from_factors(N, K, rank, inv_lam, L1p_bf16, L2_bf16, R, bias, stream, out);
  if (!out) return fail(SVDQ_ERR_INVALID_ARG, "out is null");
  *out = nullptr;
  SVDQ_TRY(check_shape(N, K));
  if (rank < 0 || rank > 128) return fail(SVDQ_ERR_INVALID_ARG, "rank=%d must be in [0, 128]", rank);
  if (!inv_lam || !R) return fail(SVDQ_ERR_INVALID_ARG, "inv_lam and R are required");
  if (rank > 0 && (!L1p_bf16 || !L2_bf16)) return fail(SVDQ_ERR_INVALID_ARG, "rank > 0 needs L1p and L2");
  const size_t nk = static_cast<size_t>(N) * K;
  for (size_t i = 0; i < nk; ++i)
    if (!std::isfinite(R[i])) return fail(SVDQ_ERR_INVALID_ARG, "R has a non-finite value");
  SVDQ_TRY(check_device());
  return build_handle(N, K, rank, inv_lam, L1p_bf16, L2_bf16, R, bias, 1, format, static_cast<cudaStream_t>(stream),
                      out);
}

svdq_status svdq_weights_format(const svdq_weights* w, int* format) {
  if (!w || !format) return fail(SVDQ_ERR_INVALID_ARG, "null weights handle or format");
  *format = w->format;
  return SVDQ_OK;
}

size_t svdq_weights_sf_bytes(const svdq_weights* w) {
  if (!w) return 0;
  return w->format == SVDQ_FORMAT_INT4 ? static_cast<size_t>(w->K / 64) * round_up(w->N, 256) * 2
                                       : svdq_act_sf_bytes(w->N, w->K);
}

svdq_status svdq_attach_lora(svdq_weights* w, const uint16_t* A_bf16, const uint16_t* B_bf16, int r_l,
                             float scale, void* stream) {
  if (!w) return fail(SVDQ_ERR_INVALID_ARG, "null weights handle");
  if (!A_bf16 || !B_bf16) return fail(SVDQ_ERR_INVALID_ARG, "A and B are required");
  if (r_l <= 0 || w->rank + r_l > 128)
    return fail(SVDQ_ERR_INVALID_ARG, "r_l=%d: total rank must stay within 128", r_l);
  if (!std::isfinite(scale)) return fail(SVDQ_ERR_INVALID_ARG, "scale is not finite");
  SVDQ_TRY(check_device());
  const int K = w->K, N = w->N, r0 = w->rank, r1 = r0 + r_l;
  std::vector<uint16_t> L1p(static_cast<size_t>(K) * r1), L2(static_cast<size_t>(r1) * N);
  for (int k = 0; k < K; ++k) {
    for (int i = 0; i < r0; ++i) L1p[static_cast<size_t>(k) * r1 + i] = w->L1p[static_cast<size_t>(k) * r0 + i];
    for (int i = 0; i < r_l; ++i) L1p[static_cast<size_t>(k) * r1 + r0 + i] = A_bf16[static_cast<size_t>(k) * r_l + i];
  }
  std::copy(w->L2.begin(), w->L2.end(), L2.begin());
  for (int i = 0; i < r_l; ++i)
    for (int n = 0; n < N; ++n)
      L2[static_cast<size_t>(r0 + i) * N + n] =
          f32_to_bf16_rne(static_cast<float>(static_cast<double>(scale) * bf16_to_f32(B_bf16[static_cast<size_t>(i) * N + n])));
  w->L1p.swap(L1p);
  w->L2.swap(L2);
  w->rank = r1;
  return upload_lowrank(w, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_quantize_act_lowrank_down(const svdq_weights* w, const void* X_bf16, int M, void* xq,
                                           void* xsf, void* T, void* stream) {
  SVDQ_TRY(check_runtime(w, M));
  SVDQ_TRY(check_dev_ptr(X_bf16, "X"));
  SVDQ_TRY(check_dev_ptr(xq, "xq"));
  SVDQ_TRY(check_dev_ptr(xsf, "xsf"));
  if (w->r_pad > 0) SVDQ_TRY(check_dev_ptr(T, "T"));
  ActArgs a{M, w->K, w->r_pad, X_bf16, &w->map_l1, w->d_inv_lam, static_cast<uint8_t*>(xq),
            static_cast<uint8_t*>(xsf), static_cast<uint16_t*>(T), 0, 0};
  a.int4 = w->format == SVDQ_FORMAT_INT4;
  return launch_act_quant(a, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_act_row_stats(const void* Z_bf16, int M, int K, float eps, float* stats, void* stream) {
  if (M < 1 || K < 64 || K % 64)
    return fail(SVDQ_ERR_INVALID_ARG, "M=%d must be >= 1 and K=%d a positive multiple of 64", M, K);
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return fail(SVDQ_ERR_INVALID_ARG, "eps must be finite and >= 0");
  SVDQ_TRY(check_dev_ptr(Z_bf16, "Z"));
  SVDQ_TRY(check_dev_ptr(stats, "stats"));
  SVDQ_TRY(check_device());
  return launch_row_stats(Z_bf16, M, K, eps, stats, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_norm_quantize_act_lowrank_down(const svdq_weights* w, const void* Z_bf16, int M, const float* stats,
                                                const float* norm_a, const float* norm_c, void* xq, void* xsf,
                                                void* T, void* stream) {
  SVDQ_TRY(check_runtime(w, M));
  SVDQ_TRY(check_dev_ptr(Z_bf16, "Z"));
  SVDQ_TRY(check_dev_ptr(stats, "stats"));
  SVDQ_TRY(check_dev_ptr(norm_a, "norm_a"));
  SVDQ_TRY(check_dev_ptr(norm_c, "norm_c"));
  SVDQ_TRY(check_dev_ptr(xq, "xq"));
  SVDQ_TRY(check_dev_ptr(xsf, "xsf"));
  if (w->r_pad > 0) SVDQ_TRY(check_dev_ptr(T, "T"));
  ActArgs a{M, w->K, w->r_pad, Z_bf16, &w->map_l1, w->d_inv_lam, static_cast<uint8_t*>(xq),
            static_cast<uint8_t*>(xsf), static_cast<uint16_t*>(T), 0, 0};
  a.int4 = w->format == SVDQ_FORMAT_INT4;
  a.stats = stats;
  a.norm_a = norm_a;
  a.norm_c = norm_c;
  return launch_act_quant(a, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_debug_launch_stalled_act(const svdq_weights* w, const void* X_bf16, int M, void* xq, void* xsf,
                                          void* T, void* stream) {
  SVDQ_TRY(check_runtime(w, M));
  SVDQ_TRY(check_dev_ptr(X_bf16, "X"));
  SVDQ_TRY(check_dev_ptr(xq, "xq"));
  SVDQ_TRY(check_dev_ptr(xsf, "xsf"));
  if (w->r_pad > 0) SVDQ_TRY(check_dev_ptr(T, "T"));
  ActArgs a{M, w->K, w->r_pad, X_bf16, &w->map_l1, w->d_inv_lam, static_cast<uint8_t*>(xq),
            static_cast<uint8_t*>(xsf), static_cast<uint16_t*>(T), 1, 0};
  a.int4 = w->format == SVDQ_FORMAT_INT4;
  return launch_act_quant(a, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_selftest_codec(unsigned int* mismatches) {
  if (!mismatches) return fail(SVDQ_ERR_INVALID_ARG, "mismatches is null");
  SVDQ_TRY(check_device());
  return selftest_codec(mismatches);
}

namespace {
svdq_status launch_int4(const svdq_weights* w, const void* xq, const void* xsf, const void* T, int M, void* Y,
                        void* stream) {
  GemmInt4Args a{M, w->N, w->K, w->r_pad, xq, xsf, T, &w->map_wq_256, &w->map_l2_256,
                 reinterpret_cast<const uint16_t*>(w->d_wsf), w->d_bias, Y};
  return launch_gemm_int4(a, static_cast<cudaStream_t>(stream));
}
}  // namespace

svdq_status svdq_linear_w4a4(const svdq_weights* w, const void* xq, const void* xsf, const void* T, int M,
                             void* Y_bf16, void* stream) {
  SVDQ_TRY(check_runtime(w, M));
  SVDQ_TRY(check_dev_ptr(xq, "xq"));
  SVDQ_TRY(check_dev_ptr(xsf, "xsf"));
  SVDQ_TRY(check_dev_ptr(Y_bf16, "Y"));
  if (w->r_pad > 0) SVDQ_TRY(check_dev_ptr(T, "T"));
  if (w->format == SVDQ_FORMAT_INT4) return launch_int4(w, xq, xsf, T, M, Y_bf16, stream);
  GemmArgs a{M, w->N, w->K, w->r_pad, xq, xsf, T, &w->map_wq_256, &w->map_wq_128, &w->map_l2_256,
             &w->map_l2_128, w->d_wsf, w->d_bias, w->alpha_w, Y_bf16, 0};
  a.map_wsf = &w->map_wsf;
  return launch_gemm_w4a4(a, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_debug_forward_small_m(const svdq_weights* w, const void* X_bf16, int M, void* Y_bf16, int ksplit,
                                       void* stream) {
  if (ksplit < 0 || ksplit > 8) return fail(SVDQ_ERR_INVALID_ARG, "ksplit=%d must be in [0, 8]", ksplit);
  SVDQ_TRY(check_runtime(w, M));
  SVDQ_TRY(check_dev_ptr(X_bf16, "X"));
  SVDQ_TRY(check_dev_ptr(Y_bf16, "Y"));
  if (!small_m_supported(M, w->r_pad, w->format))
    return fail(SVDQ_ERR_INVALID_ARG, "the fused small-M layer takes NVFP4 handles, M <= 16 and rank <= 64");
  return launch_small_m_for(w, X_bf16, M, Y_bf16, ksplit, nullptr, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_debug_linear_w4a4_ksplit(const svdq_weights* w, const void* xq, const void* xsf, const void* T,
                                          int M, void* Y_bf16, int ksplit, void* stream) {
  if (ksplit < 1 || ksplit > 8) return fail(SVDQ_ERR_INVALID_ARG, "ksplit=%d must be in [1, 8]", ksplit);
  SVDQ_TRY(check_runtime(w, M));
  SVDQ_TRY(check_dev_ptr(xq, "xq"));
  SVDQ_TRY(check_dev_ptr(xsf, "xsf"));
  SVDQ_TRY(check_dev_ptr(Y_bf16, "Y"));
  if (w->r_pad > 0) SVDQ_TRY(check_dev_ptr(T, "T"));
  if (w->format == SVDQ_FORMAT_INT4) return launch_int4(w, xq, xsf, T, M, Y_bf16, stream);  // no split-K
  GemmArgs a{M, w->N, w->K, w->r_pad, xq, xsf, T, &w->map_wq_256, &w->map_wq_128, &w->map_l2_256,
             &w->map_l2_128, w->d_wsf, w->d_bias, w->alpha_w, Y_bf16, ksplit};
  a.map_wsf = &w->map_wsf;
  return launch_gemm_w4a4(a, static_cast<cudaStream_t>(stream));
}

size_t svdq_act_codes_bytes(int M, int K) {
  return M > 0 && K > 0 ? static_cast<size_t>(M) * K / 2 : 0;
}
size_t svdq_act_sf_bytes(int M, int K) {
  return M > 0 && K > 0 ? static_cast<size_t>(round_up(M, 128)) * (K / 16) : 0;
}
size_t svdq_lowrank_bytes(const svdq_weights* w, int M) {
  return w && M > 0 ? static_cast<size_t>(M) * 2 * w->r_pad * 2 : 0;
}
size_t svdq_forward_workspace_bytes(const svdq_weights* w, int M) {
  if (!w || M < 1) return 0;
  return up256(svdq_act_codes_bytes(M, w->K)) + up256(svdq_act_sf_bytes(M, w->K)) +
         up256(svdq_lowrank_bytes(w, M));
}
size_t svdq_forward_norm_workspace_bytes(const svdq_weights* w, int M) {
  if (!w || M < 1) return 0;
  return svdq_forward_workspace_bytes(w, M) + up256(static_cast<size_t>(M) * 8);
}
size_t svdq_forward_host_workspace_bytes(const svdq_weights* w, int M) {
  if (!w || M < 1) return 0;
  return svdq_forward_workspace_bytes(w, M) + up256(static_cast<size_t>(M) * w->K * 2) +
         up256(static_cast<size_t>(M) * w->N * 2);
}

svdq_status svdq_forward(const svdq_weights* w, const void* X_bf16, int M, void* Y_bf16, void* workspace,
                         size_t workspace_bytes, void* stream) {
  SVDQ_TRY(check_runtime(w, M));
  SVDQ_TRY(check_dev_ptr(workspace, "workspace"));
  if (workspace_bytes < svdq_forward_workspace_bytes(w, M))
    return fail(SVDQ_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", workspace_bytes,
                svdq_forward_workspace_bytes(w, M));
  if (small_m_preferred(M, w->N, w->K, w->r_pad, w->format)) {
    SVDQ_TRY(check_dev_ptr(X_bf16, "X"));
    SVDQ_TRY(check_dev_ptr(Y_bf16, "Y"));
    return launch_small_m_for(w, X_bf16, M, Y_bf16, 0, nullptr, static_cast<cudaStream_t>(stream));
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* xq = ws;
  uint8_t* xsf = xq + up256(svdq_act_codes_bytes(M, w->K));
  uint8_t* T = xsf + up256(svdq_act_sf_bytes(M, w->K));
  SVDQ_TRY(svdq_quantize_act_lowrank_down(w, X_bf16, M, xq, xsf, w->r_pad ? T : nullptr, stream));
  return svdq_linear_w4a4(w, xq, xsf, w->r_pad ? T : nullptr, M, Y_bf16, stream);
}

svdq_status svdq_forward_norm(const svdq_weights* w, const void* Z_bf16, int M, const float* norm_a,
                              const float* norm_c, float eps, void* Y_bf16, void* workspace, size_t workspace_bytes,
                              void* stream) {
  SVDQ_TRY(check_runtime(w, M));
  SVDQ_TRY(check_dev_ptr(workspace, "workspace"));
  if (workspace_bytes < svdq_forward_norm_workspace_bytes(w, M))
    return fail(SVDQ_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", workspace_bytes,
                svdq_forward_norm_workspace_bytes(w, M));
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* xq = ws;
  uint8_t* xsf = xq + up256(svdq_act_codes_bytes(M, w->K));
  uint8_t* T = xsf + up256(svdq_act_sf_bytes(M, w->K));
  float* stats = reinterpret_cast<float*>(ws + svdq_forward_workspace_bytes(w, M));
  SVDQ_TRY(svdq_act_row_stats(Z_bf16, M, w->K, eps, stats, stream));
  SVDQ_TRY(svdq_norm_quantize_act_lowrank_down(w, Z_bf16, M, stats, norm_a, norm_c, xq, xsf, w->r_pad ? T : nullptr,
                                               stream));
  return svdq_linear_w4a4(w, xq, xsf, w->r_pad ? T : nullptr, M, Y_bf16, stream);
}

svdq_status svdq_forward_host(const svdq_weights* w, const void* X_host, int M, void* Y_host, void* workspace,
                              size_t workspace_bytes, void* stream) {
  SVDQ_TRY(check_runtime(w, M));
  if (!X_host || !Y_host) return fail(SVDQ_ERR_INVALID_ARG, "X_host and Y_host are required");
  SVDQ_TRY(check_dev_ptr(workspace, "workspace"));
  if (workspace_bytes < svdq_forward_host_workspace_bytes(w, M))
    return fail(SVDQ_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", workspace_bytes,
                svdq_forward_host_workspace_bytes(w, M));
  const size_t fw = svdq_forward_workspace_bytes(w, M);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* xq = ws;
  uint8_t* xsf = xq + up256(svdq_act_codes_bytes(M, w->K));
  uint8_t* T = xsf + up256(svdq_act_sf_bytes(M, w->K));
  uint8_t* dX = ws + fw;
  uint8_t* dY = dX + up256(static_cast<size_t>(M) * w->K * 2);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t xrow = static_cast<size_t>(w->K) * 2, yrow = static_cast<size_t>(w->N) * 2;
  const uint8_t* Xh = static_cast<const uint8_t*>(X_host);
  uint8_t* Yh = static_cast<uint8_t*>(Y_host);

  // Rows are split into chunks (multiples of 128 rows) so that the upload of
  // chunk c+1 and the download of chunk c-1 run on their own streams while the
  // kernels of chunk c run on the caller's stream.  Every chunk owns disjoint
  // rows of the workspace, so only the per-chunk events order the three streams.
  const int nch = std::max(1, std::min(HostPipe::kMaxChunks, M / 512));
  const int rows = round_up((M + nch - 1) / nch, 128);
  HostPipe* hp = nullptr;
  SVDQ_TRY(host_pipe(&hp));
  std::lock_guard<std::mutex> lk(hp->mu);
  SVDQ_CUDA_TRY(cudaEventRecord(hp->start, s));
  SVDQ_CUDA_TRY(cudaStreamWaitEvent(hp->in, hp->start, 0));
  SVDQ_CUDA_TRY(cudaStreamWaitEvent(hp->out, hp->start, 0));
  for (int c = 0, m0 = 0; m0 < M; ++c, m0 += rows) {
    const int mc = std::min(rows, M - m0);
    SVDQ_CUDA_TRY(cudaMemcpyAsync(dX + m0 * xrow, Xh + m0 * xrow, mc * xrow, cudaMemcpyHostToDevice, hp->in));
    SVDQ_CUDA_TRY(cudaEventRecord(hp->loaded[c], hp->in));
    SVDQ_CUDA_TRY(cudaStreamWaitEvent(s, hp->loaded[c], 0));
    uint8_t* Tc = w->r_pad ? T + static_cast<size_t>(m0) * 4 * w->r_pad : nullptr;
    SVDQ_TRY(svdq_quantize_act_lowrank_down(w, dX + m0 * xrow, mc, xq + static_cast<size_t>(m0) * (w->K / 2),
                                            xsf + static_cast<size_t>(m0) * (w->K / 16), Tc, stream));
    SVDQ_TRY(svdq_linear_w4a4(w, xq + static_cast<size_t>(m0) * (w->K / 2),
                              xsf + static_cast<size_t>(m0) * (w->K / 16), Tc, mc, dY + m0 * yrow, stream));
    SVDQ_CUDA_TRY(cudaEventRecord(hp->computed[c], s));
    SVDQ_CUDA_TRY(cudaStreamWaitEvent(hp->out, hp->computed[c], 0));
    SVDQ_CUDA_TRY(cudaMemcpyAsync(Yh + m0 * yrow, dY + m0 * yrow, mc * yrow, cudaMemcpyDeviceToHost, hp->out));
  }
  SVDQ_CUDA_TRY(cudaEventRecord(hp->done, hp->out));
  SVDQ_CUDA_TRY(cudaStreamWaitEvent(s, hp->done, 0));
  return SVDQ_OK;
}

int svdq_weights_rank(const svdq_weights* w) { return w ? w->rank : -1; }

svdq_status svdq_weights_info(const svdq_weights* w, int* N, int* K, int* rank, int* r_pad, float* alpha_w) {
  if (!w) return fail(SVDQ_ERR_INVALID_ARG, "null weights handle");
  if (N) *N = w->N;
  if (K) *K = w->K;
  if (rank) *rank = w->rank;
  if (r_pad) *r_pad = w->r_pad;
  if (alpha_w) *alpha_w = w->alpha_w;
  return SVDQ_OK;
}

svdq_status svdq_weights_export(const svdq_weights* w, uint8_t* codes, uint8_t* sf, uint16_t* L1p_bf16,
                                uint16_t* L2_bf16, float* inv_lam, float* bias, float* residual) {
  if (!w) return fail(SVDQ_ERR_INVALID_ARG, "null weights handle");
  if (residual && w->residual.empty()) return fail(SVDQ_ERR_INVALID_ARG, "the handle kept no residual");
  SVDQ_CUDA_TRY(cudaDeviceSynchronize());
  if (codes) SVDQ_CUDA_TRY(cudaMemcpy(codes, w->d_wq, static_cast<size_t>(w->N) * w->K / 2, cudaMemcpyDeviceToHost));
  if (sf) SVDQ_CUDA_TRY(cudaMemcpy(sf, w->d_wsf, svdq_weights_sf_bytes(w), cudaMemcpyDeviceToHost));
  if (L1p_bf16) std::copy(w->L1p.begin(), w->L1p.end(), L1p_bf16);
  if (L2_bf16) std::copy(w->L2.begin(), w->L2.end(), L2_bf16);
  if (inv_lam) std::copy(w->inv_lam.begin(), w->inv_lam.end(), inv_lam);
  if (bias) std::copy(w->bias.begin(), w->bias.end(), bias);
  if (residual) std::copy(w->residual.begin(), w->residual.end(), residual);
  return SVDQ_OK;
}

svdq_status svdq_weights_destroy(svdq_weights* w) {
  if (!w) return SVDQ_OK;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != w->device) cudaSetDevice(w->device);
  free_device(w);
  if (cur != w->device) cudaSetDevice(cur);
  delete w;
  return SVDQ_OK;
}

void svdq_set_wait_limit_ns(uint64_t ns) { g_wait_ns = ns ? ns : 1; }

svdq_status svdq_check_device_errors(void* stream) {
  SVDQ_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int* word = device_error_word();
  if (!word) return fail(SVDQ_ERR_CUDA, "device error word unavailable");
  // the allocation-free path keeps its own static word; read and clear both
  int* words[2] = {word, noalloc_error_word_if_ready()};
  int first = 0;
  for (int* wp : words) {
    if (!wp) continue;
    int v = 0;
    SVDQ_CUDA_TRY(cudaMemcpy(&v, wp, sizeof(int), cudaMemcpyDeviceToHost));
    if (v != 0) {
      const int zero = 0;
      SVDQ_CUDA_TRY(cudaMemcpy(wp, &zero, sizeof(int), cudaMemcpyHostToDevice));
      if (!first) first = v;
    }
  }
  if (first) return fail(static_cast<svdq_status>(first), "device error word = %d", first);
  return SVDQ_OK;
}

const char* svdq_last_error(void) { return g_err; }

const char* svdq_version(void) { return "svdq-b200 0.1.0 (sm_100a)"; }

}  // extern "C"
