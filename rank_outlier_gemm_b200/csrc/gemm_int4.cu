// The INT4 variant's GEMM: group-64 INT4 codes with bf16 scales on both sides,
// the low-rank up-projection folded into the same accumulator.
//
// SVDQuant App. D: INT4 quantizes activations and weights per group of 64 with
// 16-bit scales.  sm_100 has no INT4 (or block-scaled integer) MMA, so the
// codes are expanded on chip: with bf16 scales every dequantized value q * s
// (|q| <= 7, 8-bit scale significand) has at most 11 significant bits and is
// exact in fp16 (for |q s| within fp16's range), so one fp16 tcgen05
// contraction of the dequantized tiles computes sum_g s_x s_w sum_k q_x q_w
// with only fp32 accumulation rounding.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles taken round-robin.
// Per tile: the low-rank slab (T hi/lo and L2^T, as in the NVFP4 GEMM), then
// one step per 64-wide K group.
//   warp 0      producer: per group, TMA of the packed codes (activations
//               [128 x 32 B], weights [256 x 32 B]) and 1-D bulk copies of the
//               group's bf16 scales into a 6-deep ring; per slab step, TMA of
//               T and L2^T into the slab buffer
//   warp 1      MMA issuer: kind::f16 (fp16 operands for a group, bf16 for the
//               slab), M128 N256 K16 x 4 per group from the two dequantized-tile
//               buffers, the slab from its own buffer
//   warps 2-13  dequantizers: packed codes x scale -> fp16 tiles in the 128-byte
//               swizzled K-major layout the MMA reads (one tile row of 64
//               values per thread and group), then an async-proxy fence
//   warps 14-17 epilogue: tcgen05.ld, y = acc + b, bf16 RNE, 32-byte stores
// TMEM holds two 256-column accumulators, so one tile's epilogue overlaps the
// next tile's main loop.  Each buffer has one writer and one reader that take
// every one of its uses in turn (the slab has a buffer of its own): a parity
// wait could not tell a phase from the one two uses earlier.  Launched as a programmatic dependent of the
// activation kernel; the producer waits for it before its first load.
#include <algorithm>
#include <cstddef>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

using namespace dev;

constexpr int kBN = 256;
constexpr int kThreads = 18 * 32;
constexpr int kDqWarps = 12;                       // one tile row (128 + 256) per thread
constexpr int kPStages = 6;                        // packed-code ring
constexpr int kPA = 128 * 32;                      // activation codes of one group (128 rows)
constexpr int kPB = kBN * 32;                      // weight codes of one group (256 rows)
constexpr int kPStage = 13 * 1024;                 // codes + 256 + 512 bytes of scales, padded
constexpr int kDA = 128 * 128;                     // dequantized activation tile: 128 rows x 64 fp16
constexpr int kDB = kBN * 128;                     // dequantized weight tile: 256 rows x 64 fp16
constexpr int kDBuf = kDA + kDB;
constexpr int kSlab = 128 * 128 + kBN * 64;          // T (128 x 64 bf16) and L2^T (256 x 32 bf16)
static_assert(kPA + kPB + 256 + 512 <= kPStage, "packed stage");

struct K2IParams {
  int M, N, K, r_pad;
  int groups;      // K / 64
  int slab;        // ceil(r_pad / 32)
  int mtiles, ntiles;
  int m_pad, n_pad;  // rows of the group-major scale arrays
  const uint16_t* xsf;  // [groups][m_pad] bf16
  const uint16_t* wsf;  // [groups][n_pad] bf16
  const float* bias;
  uint16_t* Y;
  int y32;
  int* err;
  uint64_t wait_ns;
};

struct K2IShared {
  alignas(16) float bias[4][kBN];
  uint64_t pfull[kPStages];
  uint64_t pempty[kPStages];
  uint64_t slab_full;    // a slab step landed in the slab buffer (TMA)
  uint64_t slab_empty;   // the MMAs reading it have completed
  uint64_t dfull[2];     // dequantizers filled buffer b
  uint64_t dempty[2];    // the MMAs reading buffer b have completed
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

__device__ __noinline__ bool wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) return false;
  }
  return true;
}

// Eight two's-complement INT4 codes (elements 2k in nibble k, 2k+1 in nibble
// k + 4) times scale s -> eight fp16 values in element order.  Offset-binary
// nibbles OR'ed into the fp16 pattern of 1024 give 1024 + (q + 8) exactly;
// subtracting 1032 gives q.  Mask k picks nibbles k and k + 4, i.e. elements
// 2k and 2k + 1, already in the low and high halves of a half2.
__device__ __forceinline__ uint4 int4x8_to_f16x8(uint32_t w, __half2 s2) {
  const uint32_t u = w ^ 0x88888888u;
  const uint32_t in[4] = {(u & 0x000F000Fu) | 0x64006400u, ((u >> 4) & 0x000F000Fu) | 0x64006400u,
                          ((u >> 8) & 0x000F000Fu) | 0x64006400u, ((u >> 12) & 0x000F000Fu) | 0x64006400u};
  const __half2 bias = __halves2half2(__ushort_as_half(0x6408u), __ushort_as_half(0x6408u));  // 1032
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&in[i]), bias);
    const __half2 v = __hmul2(q, s2);
    out[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// y = acc + b for 32 consecutive columns of one row, bf16 RNE.
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], const float* bias_s, const K2IParams& p,
                                            int m, int n) {
  if (m >= p.M || n >= p.N) return;
  uint32_t packed[16];
  const float4* b4 = reinterpret_cast<const float4*>(bias_s);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 bv = b4[i];
    packed[2 * i] = bf16x2_rn(__fadd_rn(__uint_as_float(r[4 * i]), bv.x), __fadd_rn(__uint_as_float(r[4 * i + 1]), bv.y));
    packed[2 * i + 1] =
        bf16x2_rn(__fadd_rn(__uint_as_float(r[4 * i + 2]), bv.z), __fadd_rn(__uint_as_float(r[4 * i + 3]), bv.w));
  }
  uint16_t* dst = p.Y + static_cast<size_t>(m) * p.N + n;
  if (p.y32) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
      if (n + 16 * i < p.N) st_global_v8(dst + 16 * i, &packed[8 * i]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (n + 8 * i < p.N)
        *reinterpret_cast<uint4*>(dst + 8 * i) =
            make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
  }
}

__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  // fp32 accumulator, fp16 A and B (format 0), both K-major
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__global__ void __launch_bounds__(kThreads, 1) gemm_int4_kernel(
    const __grid_constant__ CUtensorMap map_xq, const __grid_constant__ CUtensorMap map_wq,
    const __grid_constant__ CUtensorMap map_t, const __grid_constant__ CUtensorMap map_l2,
    const K2IParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* dq = smem;                                  // 2 dequantized-tile buffers
  uint8_t* sl = smem + 2 * kDBuf;                      // slab buffer
  uint8_t* pk = sl + kSlab;                            // packed ring
  K2IShared* sh = reinterpret_cast<K2IShared*>(pk + kPStages * kPStage);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int ntiles_total = p.mtiles * p.ntiles;
  // the next layer's activation kernel may launch now (it waits for this grid
  // before touching X or the activation buffers)
  grid_dep_launch_dependents();
  const int per_tile = p.slab + p.groups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&sh->pfull[s], 1);
      mbar_init(&sh->pempty[s], kDqWarps);
    }
    mbar_init(&sh->slab_full, 1);
    mbar_init(&sh->slab_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->dfull[b], kDqWarps);
      mbar_init(&sh->dempty[b], 1);
      mbar_init(&sh->acc_full[b], 1);
      mbar_init(&sh->acc_empty[b], 4);
    }
    mbar_init(&sh->done, 1);
    sh->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const WaitCtl wc{p.err, p.wait_ns, &sh->abort};
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&map_xq);
      tma_prefetch_desc(&map_wq);
      if (p.slab) {
        tma_prefetch_desc(&map_t);
        tma_prefetch_desc(&map_l2);
      }
      grid_dep_wait();  // the activation codes, scales and T come from the kernel ahead
      int pst = 0, sst = 0;  // packed stages and slab steps issued
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles_total; t += gridDim.x) {
        const int m0 = (t % p.mtiles) * 128;
        const int n0 = (t / p.mtiles) * kBN;
        for (int k = 0; k < per_tile; ++k) {
          if (k < p.slab) {
            if (!wait_bounded(&sh->slab_empty, (sst & 1) ^ 1, wc)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&sh->slab_full, kSlab);
            tma_load_2d(sl, &map_t, &sh->slab_full, 64 * k, m0);
            tma_load_2d(sl + 128 * 128, &map_l2, &sh->slab_full, 32 * k, n0);
            ++sst;
          } else {
            const int g = k - p.slab;
            const int s = pst % kPStages;
            if (!wait_bounded(&sh->pempty[s], ((pst / kPStages) & 1) ^ 1, wc)) {
              ok = false;
              break;
            }
            uint8_t* st = pk + s * kPStage;
            mbar_arrive_expect_tx(&sh->pfull[s], kPA + kPB + 256 + 512);
            tma_load_2d(st, &map_xq, &sh->pfull[s], 32 * g, m0);
            tma_load_2d(st + kPA, &map_wq, &sh->pfull[s], 32 * g, n0);
            bulk_load(st + kPA + kPB, p.xsf + static_cast<size_t>(g) * p.m_pad + m0, 256, &sh->pfull[s]);
            bulk_load(st + kPA + kPB + 256, p.wsf + static_cast<size_t>(g) * p.n_pad + n0, 512, &sh->pfull[s]);
            ++pst;
          }
        }
      }
      if (sh->abort) {  // let copies in flight land before the CTA exits
        for (int i = max(0, pst - kPStages); i < pst; ++i)
          wait_drain(&sh->pfull[i % kPStages], (i / kPStages) & 1, p.wait_ns);
        if (sst > 0) wait_drain(&sh->slab_full, (sst - 1) & 1, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_f16 = idesc_f16(128, kBN);
      const uint32_t id_bf16 = idesc_bf16(128, kBN);
      const uint32_t dq0 = smem_u32(dq), sl0 = smem_u32(sl);
      int gst = 0, sst = 0, j = 0;  // group steps, slab steps, tiles
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles_total; t += gridDim.x, ++j) {
        const int a = j & 1;
        if (!wait_bounded(&sh->acc_empty[a], ((j >> 1) & 1) ^ 1, wc)) break;
        tc_fence_after();
        const uint32_t acc = tmem + a * 256;
        uint32_t accum = 0;
        for (int k = 0; k < per_tile; ++k) {
          if (k < p.slab) {
            if (!wait_bounded(&sh->slab_full, sst & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t da = desc_kmajor_sw128(sl0), dl = desc_kmajor_sw64(sl0 + 128 * 128);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (32 * k + 16 * c >= p.r_pad) break;
              mma_bf16(acc, da + 4 * c, dl + 2 * c, id_bf16, accum);      // T_hi
              mma_bf16(acc, da + 4 * c + 2, dl + 2 * c, id_bf16, 1);      // T_lo
              accum = 1;
            }
            mma_commit(&sh->slab_empty);
            ++sst;
          } else {
            const int b = gst & 1;
            if (!wait_bounded(&sh->dfull[b], (gst >> 1) & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t base = dq0 + b * kDBuf;
            mma_bf16_x4(acc, desc_kmajor_sw128(base), desc_kmajor_sw128(base + kDA), id_f16, accum);
            accum = 1;
            mma_commit(&sh->dempty[b]);
            ++gst;
          }
        }
        if (ok) mma_commit(&sh->acc_full[a]);
      }
      mma_commit(&sh->done);
    }
  } else if (warp < 2 + kDqWarps) {
    // --------------------------------------------------------- dequantizers
    // thread -> one row: activation rows 0..127, then weight rows 0..255
    const int tid = static_cast<int>(threadIdx.x) - 64;  // 0..383
    const bool is_a = tid < 128;
    const int row = is_a ? tid : tid - 128;
    const int code_off = (is_a ? 0 : kPA) + row * 32;
    const int out_off = (is_a ? 0 : kDA) + (row >> 3) * 1024 + (row & 7) * 128;
    int pst = 0;  // group steps (packed stages = uses of the dequantized-tile buffers)
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles_total; t += gridDim.x) {
      for (int g = 0; g < p.groups; ++g) {
        const int s = pst % kPStages;
        const int b = pst & 1;
        if (!wait_warp(&sh->pfull[s], (pst / kPStages) & 1, wc)) {
          ok = false;
          break;
        }
        if (!wait_warp(&sh->dempty[b], ((pst >> 1) & 1) ^ 1, wc)) {
          ok = false;
          break;
        }
        const uint8_t* st = pk + s * kPStage;
        const uint16_t* scales = reinterpret_cast<const uint16_t*>(st + kPA + kPB);  // 128 then 256
        const uint4 c0 = *reinterpret_cast<const uint4*>(st + code_off);
        const uint4 c1 = *reinterpret_cast<const uint4*>(st + code_off + 16);
        const __half sh16 = __float2half_rn(__uint_as_float(static_cast<uint32_t>(scales[tid]) << 16));
        const __half2 s2 = __halves2half2(sh16, sh16);
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};  // 8 codes each
        uint8_t* orow = dq + b * kDBuf + out_off;
#pragma unroll
        for (int c = 0; c < 8; ++c)  // 128-byte swizzle: chunk c of row r at chunk c ^ (r % 8)
          *reinterpret_cast<uint4*>(orow + ((c ^ (row & 7)) << 4)) = int4x8_to_f16x8(cw[c], s2);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sh->pempty[s]);
          mbar_arrive(&sh->dfull[b]);
        }
        ++pst;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int row = q * 32 + lane;
    int j = 0;
    for (int t = blockIdx.x; t < ntiles_total; t += gridDim.x, ++j) {
      const int a = j & 1;
      const int m = (t % p.mtiles) * 128 + row;
      const int n0 = (t / p.mtiles) * kBN;
      float* bias_s = sh->bias[warp - (2 + kDqWarps)];
      {
        const float4* src = reinterpret_cast<const float4*>(p.bias + n0) + 2 * lane;
        float4* dstb = reinterpret_cast<float4*>(bias_s) + 2 * lane;
        dstb[0] = __ldg(src);
        dstb[1] = __ldg(src + 1);
      }
      __syncwarp();
      if (!wait_warp(&sh->acc_full[a], (j >> 1) & 1, wc)) break;
      tc_fence_after();
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t rr[32];
        tmem_ld_x32(tmem + a * 256 + lane_off + 32 * c, rr);
        tmem_ld_wait();
        store_chunk(rr, bias_s + 32 * c, p, m, n0 + 32 * c);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->acc_empty[a]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) wait_drain(&sh->done, 0, p.wait_ns);  // every MMA has retired
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int num_sms_int4() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

svdq_status launch_gemm_int4(const GemmInt4Args& a, cudaStream_t stream) {
  K2IParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.r_pad = a.r_pad;
  p.groups = a.K / 64;
  p.slab = (a.r_pad + 31) / 32;
  p.mtiles = (a.M + 127) / 128;
  p.ntiles = (a.N + kBN - 1) / kBN;
  p.m_pad = round_up(a.M, 128);
  p.n_pad = round_up(a.N, kBN);
  p.xsf = static_cast<const uint16_t*>(a.xsf);
  p.wsf = a.wsf;
  p.bias = a.bias;
  p.Y = static_cast<uint16_t*>(a.Y);
  p.y32 = (reinterpret_cast<uintptr_t>(a.Y) & 31u) == 0;
  p.err = a.err ? a.err : device_error_word();
  p.wait_ns = wait_limit_ns();
  if (!p.err) return fail(SVDQ_ERR_CUDA, "device error word unavailable");

  CUtensorMap map_xq;
  svdq_status st = make_tmap_2d(&map_xq, a.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.K / 2, a.M, a.K / 2, 32, 128,
                                CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != SVDQ_OK) return st;
  CUtensorMap map_t = map_xq;
  if (a.r_pad > 0) {
    st = make_tmap_2d(&map_t, a.T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2 * a.r_pad, a.M,
                      static_cast<uint64_t>(4 * a.r_pad), 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != SVDQ_OK) return st;
  }
  const CUtensorMap& map_l2 = a.r_pad > 0 ? *a.map_l2_256 : map_xq;

  const size_t smem = 1024 + 2 * static_cast<size_t>(kDBuf) + kSlab + static_cast<size_t>(kPStages) * kPStage +
                      sizeof(K2IShared);
  static bool attr_set[64] = {};
  int cur_dev = 0;
  SVDQ_CUDA_TRY(cudaGetDevice(&cur_dev));
  if (cur_dev < 0 || cur_dev >= 64 || !attr_set[cur_dev]) {
    SVDQ_CUDA_TRY(cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
    if (cur_dev >= 0 && cur_dev < 64) attr_set[cur_dev] = true;
  }
  const int tiles = p.mtiles * p.ntiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::min(tiles, num_sms_int4()), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  SVDQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_int4_kernel, map_xq, *a.map_wq, map_t, map_l2, p));
  return SVDQ_OK;
}

}  // namespace svdq
