// Kernel 1: activation quantization with the low-rank down-projection fused in.
//
// SVDQuant §4.3 (Nunchaku, Fig. 6): the down-projection shares the activation
// read with the quantization kernel.  One CTA owns 128 rows of X and a slice of
// K; S CTAs of a thread-block cluster split K and reduce their partial
// T = X L1' through distributed shared memory.
//
// Per 64-column K tile (one TMA box, 128-byte swizzled rows):
//   warp 0     producer: TMA of the X tile [128 x 64] bf16 and the L1'^T tile
//              [r_pad x 64], bulk copy of the 64 smoothing multipliers
//   warp 1     tcgen05.mma kind::f16 (M=128, N=r_pad, K=16 x 4) into TMEM from
//              the same shared-memory X tile the quantizers read
//   warps 2-9  quantizers: a thread takes two adjacent 16-groups of one row:
//              smoothing multiply, amax, E4M3 scale, E2M1 codes; 16 code bytes
//              and, with its neighbour lane, one 4-byte scale word per row
// After the K loop the quantizer warps move T from TMEM to shared memory, the
// cluster syncs, each CTA sums its share of rows over all S partials (fixed
// order) and writes T as a bf16 hi/lo pair.
//
// The INT4 instantiation (SVDQuant App. D: groups of 64, 16-bit scales; §3:
// qmax 7) quantizes each row's 64-column tile as one group: the lane pair
// holding its two halves combines their maxima, s = bf16(fp32(amax / 7)),
// q = clamp(rint(fp32(v * fp32(1 / s))), -7, 7), two's-complement nibbles (per
// 8 elements one word, even elements in nibbles 0-3, odd ones in 4-7),
// and the bf16 scale goes to a group-major [K/64][rows padded to 128] array.
//
// The norm instantiation reads the pre-norm activations Z instead of X and
// first applies the adaLN front end of the configured DiT blocks per element,
// x = bf16(((z - mu) * rstd) * a_j + c_j) with the row's mu and rstd from the
// row-statistics kernel (zero for padding rows).  Each quantizer thread writes
// its normalized values back into the stage's tile, so the down-projection MMA
// (which waits for that) and the quantizer both see X; the rest is unchanged.
#include <cooperative_groups.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "nvfp4.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

using namespace dev;

constexpr int kStages = 4;
constexpr int kQuantWarps = 8;
constexpr int kThreads = (2 + kQuantWarps) * 32;
constexpr int kXTile = 128 * 128;  // 128 rows x 64 bf16
constexpr int kInvTile = 64 * 4;   // 64 fp32 smoothing multipliers

struct K1Params {
  int M, K, r_pad, kt_total, splits;
  const float* inv_lam;
  uint8_t* xq;
  uint8_t* xsf;
  uint16_t* T;
  int* err;
  uint64_t wait_ns;
  int stall;
  int m_pad;           // INT4: rows of the group-major scale array
  const float2* stats;  // norm: (mu, rstd) per row
  const float* norm_a;  // norm: per-channel multiplier [K]
  const float* norm_c;  // norm: per-channel offset [K]
  uint32_t l1_tile;    // r_pad * 128 bytes
  uint32_t tmem_cols;
};

struct K1Shared {
  float rcp_tbl[16];  // reciprocals of the E4M3 mantissa patterns (see nvfp4.cuh)
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t normed[kStages];  // norm: the quantizer warps wrote X into the stage
  uint64_t tfull;
  uint64_t never;
  uint32_t tmem_base;
  int abort;
};

// Waits for a phase with a time limit only (used when draining after an abort).
__device__ __noinline__ bool wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ void bar_sync_quant() {
  asm volatile("bar.sync 1, %0;" ::"n"(kQuantWarps * 32) : "memory");
}

// INT4: the eight codes of v[0..7] times r as one word, even elements in
// nibbles 0-3 and odd ones in nibbles 4-7.
__device__ __forceinline__ uint32_t int4x8(const float* v, float r) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = min(7, max(-7, __float2int_rn(__fmul_rn(v[i], r))));
    w |= (static_cast<uint32_t>(q) & 0xFu) << (4 * ((i & 1) ? 4 + (i >> 1) : (i >> 1)));
  }
  return w;
}

template <bool kInt4, bool kNorm>
__global__ void __launch_bounds__(kThreads, 2) act_quant_lowrank_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_l1,
    const K1Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem;
  uint8_t* l1s = xs + kStages * kXTile;
  constexpr int kAux = kInvTile * (kNorm ? 3 : 1);  // inv_lam (then a and c) of a tile
  uint8_t* invs = l1s + kStages * p.l1_tile;
  K1Shared* sh = reinterpret_cast<K1Shared*>(invs + kStages * kAux);
  float* red = reinterpret_cast<float*>(smem);  // reuses the stage buffers after the K loop
  const int red_stride = p.r_pad + 4;

  const uint32_t warp = warp_id(), lane = lane_id();
  const int mb = blockIdx.x;
  const int m0 = mb * 128;
  const int split = static_cast<int>(blockIdx.y);
  const int base = p.kt_total / p.splits, rem = p.kt_total % p.splits;
  const int nt = base + (split < rem ? 1 : 0);
  const int t0 = split * base + min(split, rem);
  const bool lowrank = p.r_pad > 0;
  // the GEMM behind this kernel may start its set-up and weight loads now; it
  // waits for this grid to finish before reading what this kernel writes
  grid_dep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], kQuantWarps + (lowrank ? 1 : 0));
      mbar_init(&sh->normed[s], kQuantWarps);
    }
    mbar_init(&sh->tfull, 1);
    mbar_init(&sh->never, 1);
    sh->abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 16) sh->rcp_tbl[threadIdx.x] = rcp_table_entry(static_cast<int>(threadIdx.x));
  if (warp == 1 && lowrank) {
    tmem_alloc(&sh->tmem_base, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const WaitCtl wc{p.err, p.wait_ns, &sh->abort};
  const uint32_t tmem = lowrank ? sh->tmem_base : 0u;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&map_x);
      if (lowrank) tma_prefetch_desc(&map_l1);
      const uint32_t bytes = kXTile + (lowrank ? p.l1_tile : 0u) + kAux;
      // A stage's loads come in two halves: the layer's own constants (L1'
      // tile, smoothing multipliers), which no kernel of the forward pass
      // writes, and X (with the norm front end's a and c), which the kernel
      // ahead may produce.  The first stages' constants go out before the
      // wait for that kernel (a programmatic launch lets this kernel start
      // while the one ahead finishes).
      auto consts = [&](int i, int s) {
        mbar_arrive_expect_tx(&sh->full[s], bytes);
        const int k0 = (t0 + i) * 64;
        if (lowrank) tma_load_2d(l1s + s * p.l1_tile, &map_l1, &sh->full[s], k0, 0);
        bulk_load(invs + s * kAux, p.inv_lam + k0, kInvTile, &sh->full[s]);
      };
      auto acts = [&](int i, int s) {
        const int k0 = (t0 + i) * 64;
        tma_load_2d(xs + s * kXTile, &map_x, &sh->full[s], k0, m0);
        if (kNorm) {
          bulk_load(invs + s * kAux + kInvTile, p.norm_a + k0, kInvTile, &sh->full[s]);
          bulk_load(invs + s * kAux + 2 * kInvTile, p.norm_c + k0, kInvTile, &sh->full[s]);
        }
      };
      const int npre = min(kStages, nt);
      for (int i = 0; i < npre; ++i) consts(i, i);
      grid_dep_wait();  // X comes from the kernel ahead, which may still read xq, xsf and T
      for (int i = 0; i < npre; ++i) acts(i, i);
      int issued = npre;
      for (int i = npre; i < nt; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!wait_bounded(&sh->empty[s], ph ^ 1, wc)) break;
        consts(i, s);
        acts(i, s);
        issued = i + 1;
      }
      if (sh->abort) {  // let copies in flight land before the buffers are reused
        for (int i = max(0, issued - kStages); i < issued; ++i)
          wait_drain(&sh->full[i % kStages], (i / kStages) & 1, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    if (lowrank && lane == 0) {
      const uint32_t idesc = idesc_bf16(128, p.r_pad);
      for (int i = 0; i < nt; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!wait_bounded(kNorm ? &sh->normed[s] : &sh->full[s], ph, wc)) break;  // X in the tile
        tc_fence_after();
        mma_bf16_x4(tmem, desc_kmajor_sw128(smem_u32(xs + s * kXTile)),
                    desc_kmajor_sw128(smem_u32(l1s + s * p.l1_tile)), idesc, i != 0);
        mma_commit(&sh->empty[s]);
      }
      mma_commit(&sh->tfull);
    }
  } else {
    // ------------------------------------------------------------ quantizers
    const int wq = static_cast<int>(warp) - 2;           // 0..7
    const int row = 16 * wq + static_cast<int>(lane >> 1);
    const int h = lane & 1;                              // columns [32h, 32h + 32) of the tile
    const int m = m0 + row;
    float mu = 0.0f, rstd = 0.0f;
    if (kNorm) grid_dep_wait();  // the statistics come from the kernel ahead
    if (kNorm && m < p.M) {
      const float2 st = p.stats[m];
      mu = st.x;
      rstd = st.y;
    }
    if (p.stall) wait_warp(&sh->never, 0, wc);
    for (int i = 0; i < nt; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      if (!wait_warp(&sh->full[s], ph, wc)) break;
      if (m0 + 16 * wq >= p.M) {
        // every row of this warp is padding (the TMA filled it with zeros): no
        // codes to write, and the scales of padding rows are 0 by definition
        __syncwarp();
        if (lane == 0) {
          if (kNorm) mbar_arrive(&sh->normed[s]);
          mbar_arrive(&sh->empty[s]);
        }
        const int kt = t0 + i;
        if (h == 0) {
          if constexpr (kInt4)
            reinterpret_cast<uint16_t*>(p.xsf)[static_cast<size_t>(kt) * p.m_pad + m] = 0;
          else
            *reinterpret_cast<uint32_t*>(p.xsf + (static_cast<size_t>(mb) * p.kt_total + kt) * 512 +
                                         (row & 31) * 16 + (row >> 5) * 4) = 0u;
        }
        continue;
      }
      uint8_t* xrow = xs + s * kXTile + row * 128;
      const float4* inv4 = reinterpret_cast<const float4*>(invs + s * kAux) + 8 * h;
      if constexpr (kNorm) {
        // z -> x = bf16(((z - mu) * rstd) * a + c) in place (zero on padding rows)
        const float* na = reinterpret_cast<const float*>(invs + s * kAux + kInvTile) + 32 * h;
        const float* nc = reinterpret_cast<const float*>(invs + s * kAux + 2 * kInvTile) + 32 * h;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4* cp = reinterpret_cast<uint4*>(xrow + (((4 * h + c) ^ (row & 7)) << 4));
          const uint4 z = *cp;
          const uint32_t zw[4] = {z.x, z.y, z.z, z.w};
          uint32_t xw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 8 * c + 2 * e;
            const float z0 = __uint_as_float(zw[e] << 16), z1 = __uint_as_float(zw[e] & 0xFFFF0000u);
            const float x0 = __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(z0, mu), rstd), na[j]), nc[j]);
            const float x1 = __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(z1, mu), rstd), na[j + 1]), nc[j + 1]);
            const __nv_bfloat162 xb = __floats2bfloat162_rn(x0, x1);
            xw[e] = m < p.M ? *reinterpret_cast<const uint32_t*>(&xb) : 0u;
          }
          *cp = make_uint4(xw[0], xw[1], xw[2], xw[3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the MMA reads X through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->normed[s]);
      }
      const int kt = t0 + i;
      const int k0 = kt * 64;
      float v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8).
        const uint4 w = *reinterpret_cast<const uint4*>(xrow + (((4 * h + c) ^ (row & 7)) << 4));
        const float4 i0 = inv4[2 * c], i1 = inv4[2 * c + 1];
        const float2 a0 = mul_f32x2(make_float2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u)), make_float2(i0.x, i0.y));
        const float2 a1 = mul_f32x2(make_float2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u)), make_float2(i0.z, i0.w));
        const float2 a2 = mul_f32x2(make_float2(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xFFFF0000u)), make_float2(i1.x, i1.y));
        const float2 a3 = mul_f32x2(make_float2(__uint_as_float(w.w << 16), __uint_as_float(w.w & 0xFFFF0000u)), make_float2(i1.z, i1.w));
        v[8 * c + 0] = a0.x; v[8 * c + 1] = a0.y; v[8 * c + 2] = a1.x; v[8 * c + 3] = a1.y;
        v[8 * c + 4] = a2.x; v[8 * c + 5] = a2.y; v[8 * c + 6] = a3.x; v[8 * c + 7] = a3.y;
      }
      if constexpr (kInt4) {
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));  // the other half of the group
        const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
        const float sv = __bfloat162float(sb);
        const float r = sv > 0.0f ? __frcp_rn(sv) : 0.0f;
        const uint4 codes = make_uint4(int4x8(v, r), int4x8(v + 8, r), int4x8(v + 16, r), int4x8(v + 24, r));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->empty[s]);  // this warp is done reading the stage
        if (m < p.M)
          *reinterpret_cast<uint4*>(p.xq + static_cast<size_t>(m) * (p.K / 2) + k0 / 2 + 16 * h) = codes;
        if (h == 0)
          reinterpret_cast<uint16_t*>(p.xsf)[static_cast<size_t>(kt) * p.m_pad + m] = __bfloat16_as_ushort(sb);
      } else {
        float g0[16], g1[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          g0[j] = v[j];
          g1[j] = v[16 + j];
        }
        const Fp4Group q0 = nvfp4_encode16(g0, sh->rcp_tbl);
        const Fp4Group q1 = nvfp4_encode16(g1, sh->rcp_tbl);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->empty[s]);  // this warp is done reading the stage
        if (m < p.M) {
          uint4* dst = reinterpret_cast<uint4*>(p.xq + static_cast<size_t>(m) * (p.K / 2) + k0 / 2 + 16 * h);
          *dst = make_uint4(q0.lo, q0.hi, q1.lo, q1.hi);
        }
        const uint32_t mine = q0.scale | (q1.scale << 8);
        const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
        if (h == 0) {
          const size_t atom = static_cast<size_t>(mb) * p.kt_total + kt;
          *reinterpret_cast<uint32_t*>(p.xsf + atom * 512 + (row & 31) * 16 + (row >> 5) * 4) =
              mine | (other << 16);
        }
      }
    }
    if (lowrank) {
      bar_sync_quant();  // every quantizer is done with the stage buffers
      if (wait_warp(&sh->tfull, 0, wc)) {
        tc_fence_after();
        const int q = warp & 3;           // TMEM lane quarter this warp may access
        const int half = wq >> 2;         // the two warps of a quarter split the 16-column chunks
        const int trow = q * 32 + static_cast<int>(lane);
        float* dst = red + trow * red_stride;
        for (int c = 16 * half; c < p.r_pad; c += 32) {
          uint32_t r[16];
          tmem_ld_x16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(dst + c + j) =
                make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                            __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
        }
      }
    }
  }

  // ---- cluster-wide reduction of the partial T over the K splits
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  tc_fence_before();
  cluster.sync();
  if (lowrank && !sh->abort) {
    const int rows_per = (128 + p.splits - 1) / p.splits;
    const int r_lo = split * rows_per;
    const int r_hi = min(128, r_lo + rows_per);
    const int c4n = p.r_pad / 4;
    const float* peers[8];
#pragma unroll
    for (int qr = 0; qr < 8; ++qr) peers[qr] = cluster.map_shared_rank(red, qr < p.splits ? qr : 0);
    for (int it = threadIdx.x; it < (r_hi - r_lo) * c4n; it += kThreads) {
      const int rr = r_lo + it / c4n;
      const int c = (it % c4n) * 4;
      const int m = m0 + rr;
      if (m >= p.M) continue;
      const int off = rr * red_stride + c;
      float4 v[8];
#pragma unroll
      for (int qr = 0; qr < 8; ++qr)
        if (qr < p.splits) v[qr] = *reinterpret_cast<const float4*>(peers[qr] + off);
      float4 acc = v[0];
#pragma unroll
      for (int qr = 1; qr < 8; ++qr)
        if (qr < p.splits) {
          acc.x += v[qr].x;
          acc.y += v[qr].y;
          acc.z += v[qr].z;
          acc.w += v[qr].w;
        }
      const float a[4] = {acc.x, acc.y, acc.z, acc.w};
      uint16_t hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat16 hb = __float2bfloat16_rn(a[j]);
        hi[j] = __bfloat16_as_ushort(hb);
        lo[j] = __bfloat16_as_ushort(__float2bfloat16_rn(a[j] - __bfloat162float(hb)));
      }
      uint16_t* trow = p.T + static_cast<size_t>(m) * (2 * p.r_pad) + 32 * (c / 16) + (c % 16);
      *reinterpret_cast<uint2*>(trow) =
          make_uint2(hi[0] | (uint32_t(hi[1]) << 16), hi[2] | (uint32_t(hi[3]) << 16));
      *reinterpret_cast<uint2*>(trow + 16) =
          make_uint2(lo[0] | (uint32_t(lo[1]) << 16), lo[2] | (uint32_t(lo[3]) << 16));
    }
  }
  cluster.sync();  // peers are done reading this CTA's partial

  if (warp == 1 && lowrank) {
    if (lane == 0) wait_drain(&sh->tfull, 0, p.wait_ns);  // every MMA has retired
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

// The kernel instantiation for a format and front end.
using K1Kernel = void (*)(const CUtensorMap, const CUtensorMap, const K1Params);
K1Kernel k1_kernel(bool int4, bool norm) {
  if (norm) return int4 ? act_quant_lowrank_kernel<true, true> : act_quant_lowrank_kernel<false, true>;
  return int4 ? act_quant_lowrank_kernel<true, false> : act_quant_lowrank_kernel<false, false>;
}

// Clusters of this kernel that fit on the device at once for a K-split of S
// (cluster = S CTAs); cached per (S, shared memory size).
int max_active_clusters(int S, size_t smem, bool int4, bool norm) {
  static std::mutex mu;
  static std::map<std::pair<int, size_t>, int> cache;
  std::lock_guard<std::mutex> lk(mu);
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_pair(S + 64 * dev + (int4 ? 4096 : 0) + (norm ? 8192 : 0), smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, S, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = S;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  const cudaError_t qe = cudaOccupancyMaxActiveClusters(&n, k1_kernel(int4, norm), &cfg);
  if (qe != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 1;
  }
  cache[key] = n;
  return n;
}

// K-split for `mblocks` row blocks of `kt_total` 64-column tiles.  The T
// reduction needs the S CTAs of a row block in one cluster, and clusters are
// placed one CTA per SM within a GPC, so splitting more only pays while the
// clusters still fit: the cost is (waves of clusters) x (tiles per CTA), ties
// going to the larger split (more CTAs in flight).  At least 4 tiles per CTA.
int auto_splits(int mblocks, int kt_total, size_t smem, bool int4, bool norm) {
  const int s_max = std::max(1, std::min(8, kt_total / 4));
  int best = 1;
  long best_cost = -1;
  for (int S = 1; S <= s_max; ++S) {
    const int fit = max_active_clusters(S, smem, int4, norm);
    const long waves = (mblocks + fit - 1) / fit;
    const long cost = waves * ((kt_total + S - 1) / S);
    if (best_cost < 0 || cost <= best_cost) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

}  // namespace

svdq_status launch_act_quant(const ActArgs& a, cudaStream_t stream) {
  const int mblocks = (a.M + 127) / 128;
  const int kt_total = a.K / 64;
  const uint32_t l1_tile = static_cast<uint32_t>(a.r_pad) * 128u;
  const bool norm = a.stats != nullptr;
  const size_t smem = 1024 + kStages * (kXTile + l1_tile + kInvTile * (norm ? 3 : 1)) + sizeof(K1Shared);
  static bool attr_set[64] = {};  // per device: the attribute is set on the current one
  int cur_dev = 0;
  SVDQ_CUDA_TRY(cudaGetDevice(&cur_dev));
  if (cur_dev < 0 || cur_dev >= 64 || !attr_set[cur_dev]) {
    for (int v = 0; v < 4; ++v)
      SVDQ_CUDA_TRY(cudaFuncSetAttribute(k1_kernel(v & 1, v & 2), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024));
    if (cur_dev >= 0 && cur_dev < 64) attr_set[cur_dev] = true;
  }
  const int splits = a.splits > 0 ? std::min(std::min(a.splits, 8), kt_total)
                                   : auto_splits(mblocks, kt_total, smem, a.int4 != 0, norm);

  CUtensorMap map_x;
  svdq_status st = make_tmap_2d(&map_x, a.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.K, a.M,
                                static_cast<uint64_t>(a.K) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  CUtensorMap map_l1 = a.r_pad > 0 ? *a.map_l1 : map_x;

  K1Params p;
  p.M = a.M;
  p.K = a.K;
  p.r_pad = a.r_pad;
  p.kt_total = kt_total;
  p.splits = splits;
  p.inv_lam = a.inv_lam;
  p.xq = a.xq;
  p.xsf = a.xsf;
  p.T = a.T;
  p.err = a.err ? a.err : device_error_word();
  p.wait_ns = wait_limit_ns();
  p.stall = a.stall;
  p.m_pad = mblocks * 128;
  p.stats = static_cast<const float2*>(a.stats);
  p.norm_a = a.norm_a;
  p.norm_c = a.norm_c;
  p.l1_tile = l1_tile;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(a.r_pad)) cols <<= 1;
  p.tmem_cols = cols;
  if (!p.err) return fail(SVDQ_ERR_CUDA, "device error word unavailable");

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(mblocks, splits, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // a programmatic dependent of the kernel ahead: set-up and constant loads
  // overlap its tail; everything it may produce or still read waits for it
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = splits;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  SVDQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, k1_kernel(a.int4 != 0, norm), map_x, map_l1, p));
  return SVDQ_OK;
}

}  // namespace svdq
