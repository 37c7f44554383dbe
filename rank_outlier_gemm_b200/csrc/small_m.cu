// The whole layer in one kernel for a few tokens (M <= 16): activation
// quantization, the low-rank down-projection, the block-scaled FP4 GEMM and
// the up-projection.
//
// SVDQuant §4.3 (Nunchaku, Fig. 6) fuses the down-projection into the
// quantization kernel and the up-projection into the 4-bit GEMM.  With one to
// sixteen tokens the layer streams the weights (N x K/2 code bytes) once and
// everything else is small, so a second kernel and the round trip of the
// activation codes through global memory would cost more than the work; here
// the GEMM's own CTAs quantize the activations they need.
//
// Orientation: the output tile is Y^T, 128 weight rows (MMA M = 128) by 16
// tokens (MMA N = 16), so the weights are the A operand and the tensor work
// scales with the tokens actually present.  One CTA owns 128 output features
// and a contiguous range of 256-wide K tiles; S CTAs of a cluster split K and
// sum their fp32 partials through distributed shared memory in split order.
//
// Per K tile (one stage):
//   warp 0      producer: TMA of the weight codes [128 x 128 B] and bulk copy
//               of their scale atoms, TMA of the X slices [16 tokens x 64] and
//               of the L1'^T slices [r_pad x 64] (one per 64 columns), bulk
//               copy of the 256 smoothing multipliers
//   warps 2-9   quantizers: one 16-group of one token per thread (smoothing
//               multiply, E4M3 scale, E2M1 codes), codes into the K-major B
//               tile of the FP4 MMA, scales into one 512-byte atom per K block
//   warp 1      MMA issuer: tcgen05.cp of the weight and activation scale
//               atoms into tensor memory, four kind::mxf4nvf4 block16 MMAs
//               (M 128, N 16, K 64) into the accumulator, and the
//               down-projection T^T += L1'^T X^T as kind::f16 MMAs (M 64, N 16)
// After the K loop, warps 2-5 read T from tensor memory, split it into the
// bf16 pair T = T_hi + T_lo in shared memory, and the MMA issuer adds
// L2^T (T_hi + T_lo)^T into the same accumulator (each split applies L2 to
// its own partial T: the branch is linear in K).  The epilogue computes
// y = alpha_w * acc + b in bf16 and stores Y (M x N), after the cluster sum
// when K is split.
#include <algorithm>
#include <mutex>

#include "nvfp4.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

using namespace dev;

constexpr int kThreads = 320;
constexpr int kStages = 3;
constexpr int kNTok = 16;                       // MMA N: tokens, padded
constexpr int kWTile = 128 * 128;               // weight codes, 128 rows x 128 bytes (256 FP4)
constexpr int kWSf = 2048;                      // four 512-byte scale atoms
constexpr int kXSlice = kNTok * 128;            // 16 tokens x 64 bf16
constexpr int kL1Slice = 64 * 128;              // up to 64 ranks x 64 bf16 (rows >= r_pad stay zero)
constexpr int kInv = 256 * 4;                   // 256 fp32 smoothing multipliers
constexpr int kACodes = kNTok * 128;            // activation codes, 16 tokens x 128 bytes
constexpr int kASf = 4 * 512;                   // activation scale atoms, one per 64-wide K block
constexpr int kStageUsed = kWTile + kWSf + 4 * kXSlice + 4 * kL1Slice + kInv + kACodes + kASf;
constexpr int kStage = (kStageUsed + 1023) / 1024 * 1024;
constexpr int kL2Tile = 128 * 64;               // L2^T, 128 rows x 32 ranks (64-byte swizzle)
constexpr int kTTile = kNTok * 128;             // T_hi/T_lo of 32 ranks for 16 tokens (128-byte swizzle)
constexpr int kMaxSplit = 8;
constexpr int kPartStride = kNTok + 4;          // fp32 per partial row
// tensor memory columns
constexpr uint32_t kColY = 0;                   // Y^T accumulator, 16 columns
constexpr uint32_t kColT = 16;                  // T^T accumulator (M = 64 layout), 16 columns
constexpr uint32_t kColSfa = 32;                // 16 columns per stage (4 per 64-wide K block)
constexpr uint32_t kColSfb = 32 + 16 * kStages; // 16 columns per stage (4 per 64-wide K block)
constexpr uint32_t kTmemCols = 128;
static_assert(kColSfb + 16 * kStages <= kTmemCols, "tensor memory plan");
static_assert(kStage % 1024 == 0, "stage buffers keep 1024-byte alignment");

// offsets inside a stage
constexpr int kOffWSf = kWTile;
constexpr int kOffX = kOffWSf + kWSf;
constexpr int kOffL1 = kOffX + 4 * kXSlice;
constexpr int kOffInv = kOffL1 + 4 * kL1Slice;
constexpr int kOffACodes = kOffInv + kInv;
constexpr int kOffASf = kOffACodes + kACodes;
static_assert(kOffX % 1024 == 0 && kOffL1 % 1024 == 0 && kOffACodes % 1024 == 0, "swizzled tiles aligned");

struct SmParams {
  int M, N, K, r_pad;
  int kt;          // ceil(K / 256)
  int kb_total;    // K / 64
  int ksplit;      // CTAs per 128-row tile along K
  const uint8_t* wsf;
  const float* inv_lam;
  const float* bias;  // padded to a multiple of 256
  float alpha_w;
  uint16_t* Y;
  int* err;
  uint64_t wait_ns;
};

struct SmShared {
  alignas(1024) uint8_t l2[2][kL2Tile];         // L2^T / alpha_w for the tile's rows, ranks 0-31, 32-63
  alignas(1024) uint8_t t[2][kTTile];           // T_hi | T_lo pairs for ranks 0-31, 32-63
  float rcp_tbl[16];
  uint64_t full[kStages];
  uint64_t qdone[kStages];
  uint64_t empty[kStages];
  uint64_t l2full;
  uint64_t tdone;
  uint64_t tready;
  uint64_t accdone;
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

__global__ void __launch_bounds__(kThreads, 1) small_m_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_wq,
    const __grid_constant__ CUtensorMap map_l1, const __grid_constant__ CUtensorMap map_l2, const SmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmShared* sh = reinterpret_cast<SmShared*>(smem + kStages * kStage);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int S = p.ksplit;
  const int split = static_cast<int>(blockIdx.x) % S;
  const int tile = static_cast<int>(blockIdx.x) / S;
  const int n0 = tile * 128;
  const int kt_base = p.kt / S, kt_rem = p.kt % S;
  const int kt_lo = split * kt_base + min(split, kt_rem);
  const int nk = kt_base + (split < kt_rem ? 1 : 0);
  const bool lowrank = p.r_pad > 0;
  const int ntt = (p.r_pad + 31) / 32;  // 32-rank groups of T and L2
  grid_dep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->qdone[s], 8);
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->l2full, 1);
    mbar_init(&sh->tdone, 1);
    mbar_init(&sh->tready, 4);
    mbar_init(&sh->accdone, 1);
    mbar_init(&sh->done, 1);
    sh->abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 16) sh->rcp_tbl[threadIdx.x] = rcp_table_entry(static_cast<int>(threadIdx.x));
  // The L1' slices hold r_pad <= 64 ranks of 64 rows: the rows r_pad..63,
  // which the TMA never writes, must read as zero for the M = 64
  // down-projection MMA.  The activation scale atoms are zero outside the 16
  // token rows.  (The T tiles need no clearing: the ranks of every 32-rank
  // group in use are all written, as zero past r_pad.)
  {
    const int zrow = lowrank ? p.r_pad : 64;
    const int zwords = (64 - zrow) * 128 / 4;  // per slice
    for (int i = threadIdx.x; i < kStages * 4 * zwords; i += kThreads) {
      const int sl = i / zwords;  // stage * 4 + slice
      reinterpret_cast<uint32_t*>(smem + (sl >> 2) * kStage + kOffL1 + (sl & 3) * kL1Slice + zrow * 128)[i % zwords] = 0u;
    }
    for (int i = threadIdx.x; i < kStages * kASf / 4; i += kThreads)
      reinterpret_cast<uint32_t*>(smem + (i / (kASf / 4)) * kStage + kOffASf)[i % (kASf / 4)] = 0u;
  }
  fence_proxy_async_smem();  // the zeros are seen by the async proxy (TMA, MMA)
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, kTmemCols);
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
      tma_prefetch_desc(&map_x);
      tma_prefetch_desc(&map_wq);
      if (lowrank) {
        tma_prefetch_desc(&map_l1);
        tma_prefetch_desc(&map_l2);
        mbar_arrive_expect_tx(&sh->l2full, static_cast<uint32_t>(ntt * kL2Tile));
        for (int g = 0; g < ntt; ++g) tma_load_2d(sh->l2[g], &map_l2, &sh->l2full, 32 * g, n0);
      }
      // A stage's loads: the weight side (codes, scales, L1', multipliers),
      // which no kernel of the forward pass writes, then the activations.  The
      // first stages' weight sides go out before the wait for the kernel ahead.
      auto weight_side = [&](int i, int s) {
        const int kk = kt_lo + i;
        const int nkb = min(4, p.kb_total - 4 * kk);
        uint8_t* st = smem + s * kStage;
        const uint32_t bytes = kWTile + 512u * nkb + static_cast<uint32_t>(nkb) * kXSlice +
                               (lowrank ? static_cast<uint32_t>(nkb * p.r_pad * 128) : 0u) + 256u * nkb;
        mbar_arrive_expect_tx(&sh->full[s], bytes);
        tma_load_2d(st, &map_wq, &sh->full[s], kk * 128, n0);
        bulk_load(st + kOffWSf, p.wsf + (static_cast<size_t>(n0 / 128) * p.kb_total + 4 * kk) * 512, 512u * nkb,
                  &sh->full[s]);
        if (lowrank)
          for (int sl = 0; sl < nkb; ++sl)
            tma_load_2d(st + kOffL1 + sl * kL1Slice, &map_l1, &sh->full[s], kk * 256 + 64 * sl, 0);
        bulk_load(st + kOffInv, p.inv_lam + kk * 256, 256u * nkb, &sh->full[s]);
      };
      auto act_side = [&](int i, int s) {
        const int kk = kt_lo + i;
        const int nkb = min(4, p.kb_total - 4 * kk);
        uint8_t* st = smem + s * kStage;
        for (int sl = 0; sl < nkb; ++sl)
          tma_load_2d(st + kOffX + sl * kXSlice, &map_x, &sh->full[s], kk * 256 + 64 * sl, 0);
      };
      const int npre = min(kStages, nk);
      for (int i = 0; i < npre; ++i) weight_side(i, i);
      grid_dep_wait();  // X comes from the kernel ahead, and Y may still be read by it
      for (int i = 0; i < npre; ++i) act_side(i, i);
      int issued = npre;
      for (int i = npre; i < nk; ++i) {
        const int s = i % kStages;
        if (!wait_bounded(&sh->empty[s], ((i / kStages) & 1) ^ 1, wc)) break;
        weight_side(i, s);
        act_side(i, s);
        issued = i + 1;
      }
      if (sh->abort) {  // let copies in flight land before the buffers are reused
        for (int i = max(0, issued - kStages); i < issued; ++i)
          wait_drain(&sh->full[i % kStages], (i / kStages) & 1, p.wait_ns);
        if (lowrank) wait_drain(&sh->l2full, 0, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_fp4 = idesc_nvfp4(128, kNTok);
      const uint32_t id_t = idesc_bf16(64, kNTok);
      const uint32_t id_slab = idesc_bf16(128, kNTok);
      bool ok = true;
      for (int i = 0; ok && i < nk; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!wait_bounded(&sh->full[s], ph, wc) || !wait_bounded(&sh->qdone[s], ph, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int nkb = min(4, p.kb_total - 4 * (kt_lo + i));
        const uint32_t st = smem_u32(smem + s * kStage);
        const uint32_t sfa = tmem + kColSfa + 16u * s, sfb = tmem + kColSfb + 16u * s;
        // scale-factor columns stay 4-aligned: each K block's weight and
        // activation scales take a 4-column group of their own
        for (int kb = 0; kb < nkb; ++kb) {
          tmem_cp_sf_atom(sfa + 4u * kb, desc_sf_atom(st + kOffWSf + 512 * kb));
          tmem_cp_sf_atom(sfb + 4u * kb, desc_sf_atom(st + kOffASf + 512 * kb));
        }
        const uint64_t wd = desc_kmajor_sw128(st), ad = desc_kmajor_sw128(st + kOffACodes);
        for (int kb = 0; kb < nkb; ++kb)
          mma_nvfp4(tmem + kColY, wd + 2 * kb, ad + 2 * kb, id_fp4, sfa + 4u * kb, sfb + 4u * kb, (i | kb) != 0);
        if (lowrank)
          for (int sl = 0; sl < nkb; ++sl)
            mma_bf16_x4(tmem + kColT, desc_kmajor_sw128(st + kOffL1 + sl * kL1Slice),
                        desc_kmajor_sw128(st + kOffX + sl * kXSlice), id_t, (i | sl) != 0);
        mma_commit(&sh->empty[s]);
      }
      if (ok) mma_commit(&sh->tdone);
      if (ok && lowrank) {
        // up-projection: Y^T += L2^T (T_hi + T_lo)^T, 16 ranks per MMA
        if (wait_bounded(&sh->l2full, 0, wc) && wait_bounded(&sh->tready, 0, wc)) {
          tc_fence_after();
          for (int c = 0; c < p.r_pad / 16; ++c) {
            const uint64_t a = desc_kmajor_sw64(smem_u32(sh->l2[c >> 1])) + 2 * (c & 1);
            const uint64_t b = desc_kmajor_sw128(smem_u32(sh->t[c >> 1])) + 4 * (c & 1);
            mma_bf16(tmem + kColY, a, b, id_slab, 1);      // T_hi
            mma_bf16(tmem + kColY, a, b + 2, id_slab, 1);  // T_lo
          }
        } else {
          ok = false;
        }
      }
      if (ok) mma_commit(&sh->accdone);
      mma_commit(&sh->done);
    }
  } else {
    // ------------------------------------------------------------ quantizers
    const int tq = static_cast<int>(threadIdx.x) - 64;  // 0..255
    const int tok = tq >> 4;                            // token row of the tile
    const int g = tq & 15;                              // 16-group of the 256-wide K tile
    bool ok = true;
    for (int i = 0; i < nk; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      // a stage is refilled only after the MMAs of its previous use completed,
      // so once its data landed the code and scale buffers are free as well
      if (!wait_warp(&sh->full[s], ph, wc)) {
        ok = false;
        break;
      }
      uint8_t* st = smem + s * kStage;
      const int nkb = min(4, p.kb_total - 4 * (kt_lo + i));
      uint2 codes = make_uint2(0u, 0u);
      uint32_t scale = 0u;
      if ((g >> 2) < nkb) {
        const uint8_t* xrow = st + kOffX + (g >> 2) * kXSlice + tok * 128;
        const float4* inv4 = reinterpret_cast<const float4*>(st + kOffInv) + 4 * g;
        float v[16];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(xrow + (((2 * (g & 3) + c) ^ (tok & 7)) << 4));
          const float4 i0 = inv4[2 * c], i1 = inv4[2 * c + 1];
          const float2 a0 = mul_f32x2(make_float2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u)), make_float2(i0.x, i0.y));
          const float2 a1 = mul_f32x2(make_float2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u)), make_float2(i0.z, i0.w));
          const float2 a2 = mul_f32x2(make_float2(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xFFFF0000u)), make_float2(i1.x, i1.y));
          const float2 a3 = mul_f32x2(make_float2(__uint_as_float(w.w << 16), __uint_as_float(w.w & 0xFFFF0000u)), make_float2(i1.z, i1.w));
          v[8 * c + 0] = a0.x; v[8 * c + 1] = a0.y; v[8 * c + 2] = a1.x; v[8 * c + 3] = a1.y;
          v[8 * c + 4] = a2.x; v[8 * c + 5] = a2.y; v[8 * c + 6] = a3.x; v[8 * c + 7] = a3.y;
        }
        const Fp4Group q = nvfp4_encode16(v, sh->rcp_tbl);
        codes = make_uint2(q.lo, q.hi);
        scale = q.scale;
      }
      // codes: row tok of the K-major B tile, bytes [8g, 8g + 8) (128-byte swizzle);
      // scale: in the atom of K block g/4, byte (g % 4) of row tok's first word,
      // i.e. TMEM lane tok of the block's first column (N = 16 <= 32 rows)
      *reinterpret_cast<uint2*>(st + kOffACodes + tok * 128 + ((((g >> 1) ^ (tok & 7)) << 4) | ((g & 1) << 3))) = codes;
      st[kOffASf + (g >> 2) * 512 + tok * 16 + (g & 3)] = static_cast<uint8_t>(scale);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->qdone[s]);
    }
    if (warp < 6 && lowrank && ok) {
      // T from tensor memory (M = 64 layout: ranks 16q..16q+15 in the first
      // 16 lanes of quarter q) into the bf16 pair tiles
      const int q = warp & 3;
      if (wait_warp(&sh->tdone, 0, wc)) {
        tc_fence_after();
        uint32_t r[16];
        tmem_ld_x16(tmem + kColT + (static_cast<uint32_t>(q * 32) << 16), r);
        tmem_ld_wait();
        const int rank = 16 * q + static_cast<int>(lane);
        if (lane < 16 && rank < 32 * ntt) {
          uint8_t* tt = sh->t[rank >> 5];
          const int rr = rank & 31;
          const int hb = (rr >> 4) * 64 + (rr & 15) * 2;  // byte of T_hi in the logical 128-byte row
#pragma unroll
          for (int j = 0; j < kNTok; ++j) {
            const float x = __uint_as_float(r[j]);
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
            uint8_t* row = tt + j * 128;
            *reinterpret_cast<__nv_bfloat16*>(row + ((((hb >> 4)) ^ (j & 7)) << 4) + (hb & 15)) = hi;
            *reinterpret_cast<__nv_bfloat16*>(row + ((((hb + 32) >> 4) ^ (j & 7)) << 4) + ((hb + 32) & 15)) = lo;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->tready);
      }
    }
  }

  // ---- epilogue: warps 2-5 read the accumulator (lane = output feature)
  float* part = reinterpret_cast<float*>(smem);  // split partials, in the stage buffers
  const bool epi = warp >= 2 && warp < 6;
  const int q = warp & 3;
  const int nrow = q * 32 + static_cast<int>(lane);
  float acc[kNTok];
  bool have = false;
  if (epi) {
    const bool ok = lowrank ? wait_warp(&sh->accdone, 0, wc) : wait_warp(&sh->tdone, 0, wc);
    if (ok) {
      tc_fence_after();
      uint32_t r[16];
      tmem_ld_x16(tmem + kColY + (static_cast<uint32_t>(q * 32) << 16), r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < kNTok; ++j) acc[j] = __uint_as_float(r[j]);
      have = true;
    }
    have = __all_sync(0xffffffffu, have);
  }
  // every stage buffer is free once all MMAs are done (accdone / tdone seen)
  tc_fence_before();
  __syncthreads();
  if (S == 1) {
    if (epi && have) {
      const int n = n0 + nrow;
      if (n < p.N) {
        const float b = p.bias[n];
#pragma unroll
        for (int j = 0; j < kNTok; ++j)
          if (j < p.M)
            reinterpret_cast<__nv_bfloat16*>(p.Y)[static_cast<size_t>(j) * p.N + n] =
                __float2bfloat16_rn(__fmaf_rn(acc[j], p.alpha_w, b));
      }
    }
  } else {
    if (epi && have) {
      float4* prow = reinterpret_cast<float4*>(part + nrow * kPartStride);
#pragma unroll
      for (int j = 0; j < kNTok; j += 4) prow[j / 4] = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
    }
    cluster_sync_all();  // every split's partial is in its CTA's shared memory
    if (!sh->abort) {
      const int per = (128 + S - 1) / S;
      const int r_lo = split * per, r_hi = min(128, r_lo + per);
      const uint32_t base = smem_u32(part);
      for (int it = threadIdx.x; it < (r_hi - r_lo) * p.M; it += kThreads) {
        const int j = it / (r_hi - r_lo);          // token
        const int nr = r_lo + it % (r_hi - r_lo);  // tile row, fastest over threads
        const int n = n0 + nr;
        if (n >= p.N) continue;
        const uint32_t off = static_cast<uint32_t>(nr * kPartStride + j) * 4u;
        float sum = 0.0f;
        for (int qq = 0; qq < S; ++qq) {
          float v;
          asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(mapa_shared(base + off, qq)) : "memory");
          sum = qq ? __fadd_rn(sum, v) : v;
        }
        reinterpret_cast<__nv_bfloat16*>(p.Y)[static_cast<size_t>(j) * p.N + n] =
            __float2bfloat16_rn(__fmaf_rn(sum, p.alpha_w, p.bias[n]));
      }
    }
    cluster_sync_relaxed();  // the peers have read this CTA's partial
  }
  if (warp == 1) {
    if (lane == 0) wait_drain(&sh->done, 0, p.wait_ns);  // every MMA and copy has retired
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

int num_sms_sm() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

size_t small_m_smem() { return 1024 + static_cast<size_t>(kStages) * kStage + sizeof(SmShared); }

// Clusters of S CTAs that fit on the device at once (cached per device and S).
int max_active_clusters_sm(int S) {
  static int cache[64][kMaxSplit + 1] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cache[dev][S]) return cache[dev][S];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = small_m_smem();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, small_m_kernel, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = -1;
  }
  if (dev >= 0 && dev < 64) cache[dev][S] = n;
  return n;
}

}  // namespace

bool small_m_supported(int M, int r_pad, int format) {
  return format == SVDQ_FORMAT_NVFP4 && M >= 1 && M <= kNTok && r_pad <= 64;
}

// The one-kernel layer pays per K tile for the activation work that the
// two-kernel path does once (every CTA quantizes its K range and computes its
// share of T: 16 down-projection MMAs and 8 scale copies per K tile, each
// tcgen05 operation costing ~100 cycles of issue on the MMA thread), plus
// ~2.5k cycles of set-up and ~3.5k of split reduction.  Measured on B200 with
// rank 32 + LoRA 16 (CUDA-graph replay): M = 1 / 16, N = 3072: 12.1 / 14.2 us
// against 12.5 / 13.4 us for the two kernels; N = 12288: 23.6 / 23.9 against
// 15.2 / 16.0.  So svdq_forward keeps the two-kernel path everywhere; the
// kernel stays available (svdq_debug_forward_small_m) as the fused design's
// measured alternative.
bool small_m_preferred(int M, int N, int K, int r_pad, int format) {
  (void)N;
  (void)K;
  (void)small_m_supported(M, r_pad, format);
  return false;
}

svdq_status launch_small_m(const SmallMArgs& a, cudaStream_t stream) {
  if (!small_m_supported(a.M, a.r_pad, SVDQ_FORMAT_NVFP4))
    return fail(SVDQ_ERR_INVALID_ARG, "the fused small-M kernel takes M <= %d and rank <= 64", kNTok);
  SmParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.r_pad = a.r_pad;
  p.kt = (a.K + 255) / 256;
  p.kb_total = a.K / 64;
  p.wsf = a.wsf;
  p.inv_lam = a.inv_lam;
  p.bias = a.bias;
  p.alpha_w = a.alpha_w;
  p.Y = static_cast<uint16_t*>(a.Y);
  p.err = a.err ? a.err : device_error_word();
  p.wait_ns = wait_limit_ns();
  if (!p.err) return fail(SVDQ_ERR_CUDA, "device error word unavailable");

  CUtensorMap map_x;
  SVDQ_TRY(make_tmap_2d(&map_x, a.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.K, a.M, static_cast<uint64_t>(a.K) * 2, 64,
                        kNTok, CU_TENSOR_MAP_SWIZZLE_128B));
  const CUtensorMap& map_l1 = a.r_pad > 0 ? *a.map_l1 : map_x;
  const CUtensorMap& map_l2 = a.r_pad > 0 ? *a.map_l2_128 : map_x;

  const size_t smem = small_m_smem();
  static bool attr_set[64] = {};
  int cur_dev = 0;
  SVDQ_CUDA_TRY(cudaGetDevice(&cur_dev));
  if (cur_dev < 0 || cur_dev >= 64 || !attr_set[cur_dev]) {
    SVDQ_CUDA_TRY(cudaFuncSetAttribute(small_m_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
    if (cur_dev >= 0 && cur_dev < 64) attr_set[cur_dev] = true;
  }
  // one wave: tiles x S CTAs on the SMs, S splits of K in a cluster
  const int tiles = (a.N + 127) / 128;
  int S = std::max(1, std::min(std::min(kMaxSplit, p.kt), num_sms_sm() / std::max(1, tiles)));
  if (a.ksplit > 0) S = std::min(std::min(a.ksplit, kMaxSplit), p.kt);
  while (S > 1 && max_active_clusters_sm(S) < tiles) --S;
  p.ksplit = S;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * S, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  SVDQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, small_m_kernel, map_x, *a.map_wq_128, map_l1, map_l2, p));
  return SVDQ_OK;
}

svdq_status launch_small_m_for(const svdq_weights* w, const void* X, int M, void* Y, int ksplit, int* err,
                               cudaStream_t stream) {
  SmallMArgs a{M, w->N, w->K, w->r_pad, X, &w->map_wq_128, &w->map_l1, &w->map_l2_128, w->d_wsf, w->d_inv_lam,
               w->d_bias, w->alpha_w, Y};
  a.ksplit = ksplit;
  a.err = err;
  return launch_small_m(a, stream);
}

}  // namespace svdq
