// svdq_forward_noalloc: both kernels of the layer with their intermediates
// (activation codes, scales and the low-rank T) in a fixed block of static
// device memory instead of a caller-provided workspace, for callers that must
// not allocate: code running inside a caching allocator's callbacks (a
// cudaMalloc there can re-enter the allocator or fail against its reserve), or
// a serving loop whose device memory is fully reserved up front.
//
// The block belongs to this file's device-code module.  CUDA loads a module on
// a device the first time one of its symbols is used there, so the block is
// committed (32 MiB) by the first svdq_forward_noalloc call on each device,
// which looks up its device address -- in host code the array's name is only a
// host-side stand-in -- and from then on stays until the process exits.  Every
// later call allocates nothing.
#include <mutex>

#include "svdq_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
static __device__ int g_noalloc_err;

struct DeviceScratch {
  uint8_t* base = nullptr;
  int* err = nullptr;
};
DeviceScratch g_scratch[64];
std::mutex g_scratch_mu;

inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Device addresses of the static block and error word for the current device.
svdq_status scratch_for_current_device(DeviceScratch* out) {
  int dev = -1;
  SVDQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return svdq::fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  DeviceScratch& d = g_scratch[dev];
  if (!d.base) {
    void* base = nullptr;
    void* err = nullptr;
    SVDQ_CUDA_TRY(cudaGetSymbolAddress(&base, g_noalloc_scratch));
    SVDQ_CUDA_TRY(cudaGetSymbolAddress(&err, g_noalloc_err));
    d.base = static_cast<uint8_t*>(base);
    d.err = static_cast<int*>(err);
  }
  *out = d;
  return SVDQ_OK;
}

}  // namespace

namespace svdq {

// The static error word of this path on the current device, or nullptr while
// no svdq_forward_noalloc call has set the path up there (the lookup is not
// made here, so reading errors never loads the block).
int* noalloc_error_word_if_ready() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  return g_scratch[dev].err;
}

}  // namespace svdq

using namespace svdq;

extern "C" svdq_status svdq_forward_noalloc(const svdq_weights* w, const void* X_bf16, int M, void* Y_bf16,
                                            void* stream) {
  if (!w) return fail(SVDQ_ERR_INVALID_ARG, "null weights handle");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARG, "M=%d must be >= 1", M);
  if (!X_bf16 || !Y_bf16) return fail(SVDQ_ERR_INVALID_ARG, "X and Y are required");
  if (!aligned16(X_bf16) || !aligned16(Y_bf16))
    return fail(SVDQ_ERR_INVALID_ARG, "X and Y must be 16-byte aligned");
  const size_t codes = up256(static_cast<size_t>(M) * w->K / 2);
  const size_t sf = up256(static_cast<size_t>(round_up(M, 128)) * (w->K / 16));
  const size_t t = up256(static_cast<size_t>(M) * 2 * w->r_pad * 2);
  const size_t need = codes + sf + t;
  if (need > kNoAllocScratchBytes)
    return fail(SVDQ_ERR_INVALID_ARG,
                "M=%d, K=%d, rank pad %d needs %zu bytes of intermediates; the allocation-free path holds %zu",
                M, w->K, w->r_pad, need, kNoAllocScratchBytes);
  int dev = -1;
  SVDQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != w->device)
    return fail(SVDQ_ERR_INVALID_ARG, "current device %d differs from the handle's device %d", dev, w->device);
  svdq_status st = check_device();
  if (st != SVDQ_OK) return st;
  DeviceScratch d;
  st = scratch_for_current_device(&d);
  if (st != SVDQ_OK) return st;
  // a few tokens: the one-kernel layer, which keeps no intermediates in memory
  if (small_m_preferred(M, w->N, w->K, w->r_pad, w->format))
    return launch_small_m_for(w, X_bf16, M, Y_bf16, 0, d.err, static_cast<cudaStream_t>(stream));

  uint8_t* xq = d.base;
  uint8_t* xsf = xq + codes;
  uint16_t* T = w->r_pad ? reinterpret_cast<uint16_t*>(xsf + sf) : nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ActArgs a{M, w->K, w->r_pad, X_bf16, &w->map_l1, w->d_inv_lam, xq, xsf, T, 0, 0};
  a.err = d.err;
  a.int4 = w->format == SVDQ_FORMAT_INT4;
  st = launch_act_quant(a, s);
  if (st != SVDQ_OK) return st;
  if (w->format == SVDQ_FORMAT_INT4) {
    GemmInt4Args g{M, w->N, w->K, w->r_pad, xq, xsf, T, &w->map_wq_256, &w->map_l2_256,
                   reinterpret_cast<const uint16_t*>(w->d_wsf), w->d_bias, Y_bf16};
    g.err = d.err;
    return launch_gemm_int4(g, s);
  }
  GemmArgs g{M, w->N, w->K, w->r_pad, xq, xsf, T, &w->map_wq_256, &w->map_wq_128, &w->map_l2_256,
             &w->map_l2_128, w->d_wsf, w->d_bias, w->alpha_w, Y_bf16, 0};
  g.map_wsf = &w->map_wsf;
  g.err = d.err;
  return launch_gemm_w4a4(g, s);
}
