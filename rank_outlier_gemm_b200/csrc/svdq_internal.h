// Internal declarations shared by the library's host code and kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "svdq.h"

namespace svdq {

// Records a failure message for svdq_last_error() and returns `s`.
svdq_status fail(svdq_status s, const char* fmt, ...);
// Maps a CUDA runtime error to SVDQ_ERR_CUDA with a message.
svdq_status cuda_fail(cudaError_t e, const char* what);

#define SVDQ_CUDA_TRY(expr)                                 \
  do {                                                      \
    cudaError_t _e = (expr);                                \
    if (_e != cudaSuccess) return ::svdq::cuda_fail(_e, #expr); \
  } while (0)

// Returns the status of `expr` from the enclosing function unless it is SVDQ_OK.
#define SVDQ_TRY(expr)                 \
  do {                                 \
    svdq_status _s = (expr);           \
    if (_s != SVDQ_OK) return _s;      \
  } while (0)

// Device error word of the current device (lazily allocated, zeroed).
int* device_error_word();
// The allocation-free path's static error word on the current device, or
// nullptr if that path has not run there yet.
int* noalloc_error_word_if_ready();
uint64_t wait_limit_ns();
// SVDQ_OK if the current device is sm_100, else SVDQ_ERR_UNSUPPORTED_DEVICE.
svdq_status check_device();

// 2-D tiled tensor map over a row-major [outer, inner] array.
svdq_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                         uint32_t box_outer, CUtensorMapSwizzle swizzle);
// 3-D tiled tensor map, no swizzle: dims[0] innermost, strides in bytes of dims 1 and 2.
svdq_status make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, const uint64_t dims[3],
                         const uint64_t strides[2], const uint32_t box[3]);

inline int round_up(int x, int m) { return (x + m - 1) / m * m; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------- kernels
struct ActArgs {
  int M, K, r_pad;
  const void* X;            // device bf16 [M, K]
  const CUtensorMap* map_l1;  // L1'^T [r_pad, K] bf16 (ignored when r_pad == 0)
  const float* inv_lam;     // device [K]
  uint8_t* xq;
  uint8_t* xsf;
  uint16_t* T;              // device [M, 2 r_pad] bf16 (hi/lo chunks)
  int stall;                // test hook: a wait that never completes
  int splits;               // K-splits per 128-row block (0 = automatic)
  int* err = nullptr;       // device error word (nullptr = the device's default word)
  int int4 = 0;             // INT4 variant: group-64 codes, bf16 scales [K/64][rows padded to 128]
  const void* stats = nullptr;   // norm front end: device (mu, rstd) per row; X is then the pre-norm Z
  const float* norm_a = nullptr;  // norm front end: device per-channel multiplier [K]
  const float* norm_c = nullptr;  // norm front end: device per-channel offset [K]
};
svdq_status launch_act_quant(const ActArgs& a, cudaStream_t stream);
// Per-row LayerNorm statistics (mu, rstd) of a device bf16 [M, K] array into device float [M][2].
svdq_status launch_row_stats(const void* Z, int M, int K, float eps, float* stats, cudaStream_t stream);

struct GemmArgs {
  int M, N, K, r_pad;
  const void* xq;           // device [M, K/2]
  const void* xsf;          // device act scales (atom layout)
  const void* T;            // device [M, 2 r_pad] bf16
  const CUtensorMap* map_wq_256;  // weight codes, box rows 256
  const CUtensorMap* map_wq_128;  // weight codes, box rows 128
  const CUtensorMap* map_l2_256;  // L2^T/alpha_w [N, r_pad] bf16, box rows 256
  const CUtensorMap* map_l2_128;
  const uint8_t* wsf;       // device weight scales (atom layout)
  const float* bias;        // device [N]
  float alpha_w;
  void* Y;                  // device bf16 [M, N]
  int ksplit;               // CTAs per output tile along K (0 = automatic, 1 = no split)
  int* err = nullptr;       // device error word (nullptr = the device's default word)
  // weight scale atoms as [128-row blocks][64-element K blocks][128 x u32], box 4 K blocks x 2 row
  // blocks (both halves of a 256-row tile in one copy); nullptr = the CTA-pair kernel is not used
  const CUtensorMap* map_wsf = nullptr;
};
svdq_status launch_gemm_w4a4(const GemmArgs& a, cudaStream_t stream);

// The fused single-kernel layer for M <= 16 tokens (NVFP4, rank <= 64).
struct SmallMArgs {
  int M, N, K, r_pad;
  const void* X;                   // device bf16 [M, K]
  const CUtensorMap* map_wq_128;   // weight codes, box rows 128
  const CUtensorMap* map_l1;       // L1'^T [r_pad, K] bf16, box 64 x r_pad
  const CUtensorMap* map_l2_128;   // L2^T/alpha_w [N, r_pad] bf16, box 32 x 128
  const uint8_t* wsf;              // weight scales (atom layout)
  const float* inv_lam;            // device [K]
  const float* bias;               // device [round_up(N, 256)]
  float alpha_w;
  void* Y;                         // device bf16 [M, N]
  int ksplit = 0;                  // CTAs per 128-row tile along K (0 = automatic)
  int* err = nullptr;
};
bool small_m_supported(int M, int r_pad, int format);
// small_m_supported and expected to beat the two-kernel path on this shape
bool small_m_preferred(int M, int N, int K, int r_pad, int format);
svdq_status launch_small_m(const SmallMArgs& a, cudaStream_t stream);
// launch_small_m for a weights handle (ksplit 0 = automatic; err nullptr = the device's word)
svdq_status launch_small_m_for(const svdq_weights* w, const void* X, int M, void* Y, int ksplit, int* err,
                               cudaStream_t stream);

struct GemmInt4Args {
  int M, N, K, r_pad;
  const void* xq;           // device [M, K/2] packed INT4
  const void* xsf;          // device bf16 [K/64][round_up(M, 128)]
  const void* T;            // device [M, 2 r_pad] bf16
  const CUtensorMap* map_wq;      // weight codes [N, K/2], box 32 bytes x 256 rows
  const CUtensorMap* map_l2_256;  // L2^T [N, r_pad] bf16, box rows 256
  const uint16_t* wsf;      // device bf16 [K/64][round_up(N, 256)]
  const float* bias;        // device [round_up(N, 256)]
  void* Y;                  // device bf16 [M, N]
  int* err = nullptr;
};
svdq_status launch_gemm_int4(const GemmInt4Args& a, cudaStream_t stream);

// INT4 codec of fp32 rows [rows, K] (host, offline): packed codes [rows, K/2]
// and bf16 scales group-major [K/64][rows_pad] (padded rows left untouched).
void int4_encode_rows(const float* R, int rows, int K, int rows_pad, uint8_t* codes, uint16_t* scales);

// Device self-test of the encoder's exact division and reciprocal shortcuts.
svdq_status selftest_codec(unsigned int* mismatches_out);

// NVFP4 codes + atom-layout scales of a device fp32 [rows, K] matrix.
svdq_status launch_weight_codec(const float* d_src, int rows, int K, uint8_t* codes, uint8_t* sf,
                                cudaStream_t stream);

// ------------------------------------------------------------- host math
struct HostSplit {
  std::vector<float> inv_lam;      // [K]
  std::vector<uint16_t> L1p;       // [K, r] bf16
  std::vector<uint16_t> L2;        // [r, N] bf16
  std::vector<float> R;            // [N, K]
  std::vector<double> refine_err;  // ||R - Q(R)||_F of each split tried (refinement)
};
// Smoothing + randomized SVD split + residual on the host (float64 math).
svdq_status host_prepare_split(const uint16_t* W_bf16, const float* act_absmax, int N, int K,
                               const svdq_prepare_opts& opts, HostSplit* out);
uint16_t f32_to_bf16_rne(float x);
float bf16_to_f32(uint16_t b);
float weight_factor(const float* R, size_t n);

}  // namespace svdq

// The opaque handle.
struct svdq_weights {
  int device = 0;
  int format = 0;     // SVDQ_FORMAT_NVFP4 or SVDQ_FORMAT_INT4
  int N = 0, K = 0;
  int rank = 0;       // SVD rank + LoRA ranks
  int r_pad = 0;      // rank rounded up to 16
  float alpha_w = 1.0f;
  uint8_t* d_wq = nullptr;       // [N, K/2]
  uint8_t* d_wsf = nullptr;      // NVFP4: [ceil(N/128)*128, K/16] atom layout;
                                 // INT4: bf16 [K/64][round_up(N, 256)]
  float* d_inv_lam = nullptr;    // [K]
  uint16_t* d_L1t = nullptr;     // [r_pad, K] bf16 = L1'^T
  uint16_t* d_L2t = nullptr;     // [N, r_pad] bf16 = L2^T / alpha_w
  float* d_bias = nullptr;       // [N]
  // host copies (export, LoRA growth)
  std::vector<float> inv_lam;
  std::vector<uint16_t> L1p;     // [K, rank]
  std::vector<uint16_t> L2;      // [rank, N]
  std::vector<float> bias;
  std::vector<float> residual;   // [N, K] R / alpha_w (only if kept)
  std::vector<double> refine_err;  // residual quantization error of each split tried by prepare
  // tensor maps over the weight-side buffers
  CUtensorMap map_l1{};
  CUtensorMap map_wq_256{}, map_wq_128{};
  CUtensorMap map_wsf{};  // NVFP4 scale atoms, 3-D (see GemmArgs::map_wsf)
  CUtensorMap map_l2_256{}, map_l2_128{};
};
