// Kernel 2: block-scaled NVFP4 GEMM with the low-rank up-projection folded into
// the same tensor-memory accumulator.
//
// SVDQuant §4.3 (Nunchaku, Fig. 6): the up-projection is fused into the 4-bit
// computation kernel so the output tile is produced once.  Per 128 x BN tile:
//   warp 0     producer: TMA loads of activation codes [128 x 256 FP4] and
//              weight codes [BN x 256 FP4] (128-byte swizzled rows) plus 1-D
//              bulk copies of the matching 512-byte scale atoms; then the
//              low-rank slab: T (hi/lo bf16, 128-byte rows) and L2^T/alpha_w
//              (64-byte rows)
//   warp 1     MMA issuer: tcgen05.cp of the scale atoms into TMEM (two
//              alternating buffers), tcgen05.mma kind::mxf4nvf4 block16
//              (M=128, N=BN, K=64) per 64-element K block, then tcgen05.mma
//              kind::f16 (K=16) for T_hi L2 and T_lo L2 into the same accumulator
//   warps 2-5  epilogue: tcgen05.ld of the fp32 accumulator, y = alpha_w*acc + b,
//              bf16 round-to-nearest-even, 16-byte stores
#include <algorithm>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

using namespace dev;

constexpr int kThreads = 192;
constexpr int kATile = 128 * 128;  // 128 rows x 128 bytes (256 FP4 along K)

struct K2Params {
  int M, N, K, r_pad;
  int kt;          // ceil(K / 256)
  int kb_total;    // K / 64 (scale-atom columns of four 16-groups)
  int nblk_total;  // ceil(N / 128)
  int slab;        // ceil(r_pad / 32)
  const uint8_t* xsf;
  const uint8_t* wsf;
  const float* bias;
  float alpha_w;
  uint16_t* Y;
  int* err;
  uint64_t wait_ns;
};

template <int BN>
struct Layout {
  static constexpr int kB = BN * 128;
  static constexpr int kSfa = 2048;
  static constexpr int kSfb = (BN / 128) * 2048;
  static constexpr int kStage = kATile + kB + kSfa + kSfb;
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kSfCols = 16 + 4 * (BN / 32);  // TMEM columns of one scale buffer
  static constexpr uint32_t kTmemCols = BN + 2 * kSfCols <= 256 ? 256 : 512;
};

struct K2Shared {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full;
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

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_w4a4_kernel(
    const __grid_constant__ CUtensorMap map_xq, const __grid_constant__ CUtensorMap map_wq,
    const __grid_constant__ CUtensorMap map_t, const __grid_constant__ CUtensorMap map_l2,
    const K2Params p) {
  using L = Layout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  K2Shared* sh = reinterpret_cast<K2Shared*>(smem + L::kStages * L::kStage);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int m0 = blockIdx.x * 128;
  const int n0 = blockIdx.y * BN;
  const int total = p.kt + p.slab;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->acc_full, 1);
    sh->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const WaitCtl wc{p.err, p.wait_ns, &sh->abort};
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&map_xq);
      tma_prefetch_desc(&map_wq);
      if (p.slab) {
        tma_prefetch_desc(&map_t);
        tma_prefetch_desc(&map_l2);
      }
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % L::kStages;
        const uint32_t ph = (it / L::kStages) & 1;
        if (!wait_bounded(&sh->empty[s], ph ^ 1, wc)) break;
        uint8_t* st = smem + s * L::kStage;
        if (it < p.kt) {
          const int nkb = min(4, p.kb_total - 4 * it);
          int nb_valid = 0;
          for (int nb = 0; nb < BN / 128; ++nb) nb_valid += (n0 / 128 + nb < p.nblk_total);
          const uint32_t bytes = kATile + L::kB + 512u * nkb * (1 + nb_valid);
          mbar_arrive_expect_tx(&sh->full[s], bytes);
          tma_load_2d(st, &map_xq, &sh->full[s], it * 128, m0);
          tma_load_2d(st + kATile, &map_wq, &sh->full[s], it * 128, n0);
          bulk_load(st + kATile + L::kB,
                    p.xsf + (static_cast<size_t>(m0 / 128) * p.kb_total + 4 * it) * 512, 512u * nkb,
                    &sh->full[s]);
          for (int nb = 0; nb < BN / 128; ++nb) {
            const int nblk = n0 / 128 + nb;
            if (nblk < p.nblk_total)
              bulk_load(st + kATile + L::kB + L::kSfa + nb * 2048,
                        p.wsf + (static_cast<size_t>(nblk) * p.kb_total + 4 * it) * 512, 512u * nkb,
                        &sh->full[s]);
          }
        } else {
          const int j = it - p.kt;
          mbar_arrive_expect_tx(&sh->full[s], kATile + BN * 64);
          tma_load_2d(st, &map_t, &sh->full[s], 64 * j, m0);
          tma_load_2d(st + kATile, &map_l2, &sh->full[s], 32 * j, n0);
        }
        issued = it + 1;
      }
      if (sh->abort) {
        for (int i = max(0, issued - L::kStages); i < issued; ++i)
          wait_drain(&sh->full[i % L::kStages], (i / L::kStages) & 1, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_fp4 = idesc_nvfp4(128, BN);
      const uint32_t id_bf16 = idesc_bf16(128, BN);
      for (int it = 0; it < total; ++it) {
        const int s = it % L::kStages;
        const uint32_t ph = (it / L::kStages) & 1;
        if (!wait_bounded(&sh->full[s], ph, wc)) break;
        tc_fence_after();
        const uint32_t a_s = smem_u32(smem + s * L::kStage);
        const uint32_t b_s = a_s + kATile;
        if (it < p.kt) {
          const int nkb = min(4, p.kb_total - 4 * it);
          const uint32_t sfa_t = tmem + BN + (it & 1) * L::kSfCols;
          const uint32_t sfb_t = sfa_t + 16;
          const uint32_t sfa_s = b_s + L::kB;
          const uint32_t sfb_s = sfa_s + L::kSfa;
          for (int kb = 0; kb < nkb; ++kb) {
            tmem_cp_sf_atom(sfa_t + 4 * kb, desc_sf_atom(sfa_s + 512 * kb));
#pragma unroll
            for (int nb = 0; nb < BN / 128; ++nb)
              tmem_cp_sf_atom(sfb_t + kb * (BN / 32) + 4 * nb,
                              desc_sf_atom(sfb_s + nb * 2048 + 512 * kb));
          }
          for (int kb = 0; kb < nkb; ++kb)
            mma_nvfp4(tmem, desc_kmajor_sw128(a_s + 32 * kb), desc_kmajor_sw128(b_s + 32 * kb),
                      id_fp4, sfa_t + 4 * kb, sfb_t + kb * (BN / 32), (it | kb) != 0);
        } else {
          const int j = it - p.kt;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (32 * j + 16 * c >= p.r_pad) break;
            const uint64_t bdesc = desc_kmajor_sw64(b_s + 32 * c);
            mma_bf16(tmem, desc_kmajor_sw128(a_s + 64 * c), bdesc, id_bf16, 1);       // T_hi
            mma_bf16(tmem, desc_kmajor_sw128(a_s + 64 * c + 32), bdesc, id_bf16, 1);  // T_lo
          }
        }
        mma_commit(&sh->empty[s]);
      }
      mma_commit(&sh->acc_full);
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int m = m0 + row;
    if (wait_bounded(&sh->acc_full, 0, wc)) {
      tc_fence_after();
      for (int j = 0; j < BN / 32; ++j) {
        uint32_t r[32];
        tmem_ld_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + 32 * j, r);
        tmem_ld_wait();
        const int n = n0 + 32 * j;
        if (m < p.M && n < p.N) {
          uint32_t packed[16];
          const float4* b4 = reinterpret_cast<const float4*>(p.bias + n);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 b = __ldg(b4 + i);
            const float y0 = __fadd_rn(__fmul_rn(__uint_as_float(r[4 * i + 0]), p.alpha_w), b.x);
            const float y1 = __fadd_rn(__fmul_rn(__uint_as_float(r[4 * i + 1]), p.alpha_w), b.y);
            const float y2 = __fadd_rn(__fmul_rn(__uint_as_float(r[4 * i + 2]), p.alpha_w), b.z);
            const float y3 = __fadd_rn(__fmul_rn(__uint_as_float(r[4 * i + 3]), p.alpha_w), b.w);
            packed[2 * i] = __bfloat16_as_ushort(__float2bfloat16_rn(y0)) |
                            (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(y1))) << 16);
            packed[2 * i + 1] = __bfloat16_as_ushort(__float2bfloat16_rn(y2)) |
                                (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(y3))) << 16);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(m) * p.N + n);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (n + 8 * i < p.N)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) wait_drain(&sh->acc_full, 0, p.wait_ns);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Layout<BN>::kTmemCols);
  }
}

template <int BN>
svdq_status launch_bn(const GemmArgs& a, const CUtensorMap& map_xq, const CUtensorMap& map_wq,
                      const CUtensorMap& map_t, const CUtensorMap& map_l2, const K2Params& p,
                      cudaStream_t stream) {
  using L = Layout<BN>;
  const size_t smem = 1024 + static_cast<size_t>(L::kStages) * L::kStage + sizeof(K2Shared);
  static bool attr_set = false;
  if (!attr_set) {
    SVDQ_CUDA_TRY(cudaFuncSetAttribute(gemm_w4a4_kernel<BN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
    attr_set = true;
  }
  dim3 grid((a.M + 127) / 128, (a.N + BN - 1) / BN, 1);
  gemm_w4a4_kernel<BN><<<grid, kThreads, smem, stream>>>(map_xq, map_wq, map_t, map_l2, p);
  SVDQ_CUDA_TRY(cudaGetLastError());
  return SVDQ_OK;
}

}  // namespace

svdq_status launch_gemm_w4a4(const GemmArgs& a, cudaStream_t stream) {
  K2Params p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.r_pad = a.r_pad;
  p.kt = (a.K + 255) / 256;
  p.kb_total = a.K / 64;
  p.nblk_total = (a.N + 127) / 128;
  p.slab = (a.r_pad + 31) / 32;
  p.xsf = static_cast<const uint8_t*>(a.xsf);
  p.wsf = a.wsf;
  p.bias = a.bias;
  p.alpha_w = a.alpha_w;
  p.Y = static_cast<uint16_t*>(a.Y);
  p.err = device_error_word();
  p.wait_ns = wait_limit_ns();
  if (!p.err) return fail(SVDQ_ERR_CUDA, "device error word unavailable");

  int bn = a.force_bn;
  if (bn != 128 && bn != 256) {
    const long tiles256 = static_cast<long>((a.M + 127) / 128) * ((a.N + 255) / 256);
    bn = (a.N % 256 == 0 && tiles256 >= 148) ? 256 : 128;
  }
  CUtensorMap map_xq;
  svdq_status st = make_tmap_2d(&map_xq, a.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.K / 2, a.M, a.K / 2,
                                128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  CUtensorMap map_t = map_xq;
  if (a.r_pad > 0) {
    st = make_tmap_2d(&map_t, a.T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2 * a.r_pad, a.M,
                      static_cast<uint64_t>(4 * a.r_pad), 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != SVDQ_OK) return st;
  }
  if (bn == 256)
    return launch_bn<256>(a, map_xq, *a.map_wq_256, map_t, a.r_pad ? *a.map_l2_256 : map_xq, p, stream);
  return launch_bn<128>(a, map_xq, *a.map_wq_128, map_t, a.r_pad ? *a.map_l2_128 : map_xq, p, stream);
}

}  // namespace svdq
