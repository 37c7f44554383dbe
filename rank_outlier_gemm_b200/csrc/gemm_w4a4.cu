// Kernel 2: block-scaled NVFP4 GEMM with the low-rank up-projection folded into
// the same tensor-memory accumulator.
//
// SVDQuant §4.3 (Nunchaku, Fig. 6): the up-projection is fused into the 4-bit
// computation kernel so the output tile is produced once.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles taken round-robin.
//   warp 0     producer: per tile, first the low-rank slab -- T (hi/lo bf16)
//              and L2^T/alpha_w (64-byte swizzle) -- then per 256-wide K tile,
//              TMA loads of activation codes [128 x 128 B] and weight codes
//              [256 x 128 B] (128-byte swizzle) plus 1-D bulk copies of the
//              512-byte scale atoms
//   warp 1     MMA issuer: kind::f16 (K16) T_hi L2 and T_lo L2, then
//              tcgen05.mma kind::mxf4nvf4 block16 (M128 N256 K64) per 64-element
//              K block, all into the same accumulator.  For a K tile it waits
//              only for the scale writers, which have seen its data land
//   warps 2-5  scale writers: read the scale atoms of a K tile from shared
//              memory and write them into TMEM with tcgen05.st, replicated into
//              each 32-lane quarter (the layout the block-scaled MMA reads)
//   warps 6-9  epilogue: tcgen05.ld, y = alpha_w*acc + b, bf16 RNE; 32 x 32
//              chunks staged in shared memory and written by TMA stores while
//              a long main loop follows, stored from registers otherwise
// TMEM (512 columns) holds two 256-column accumulators.  Tile j accumulates in
// acc[j%2] and keeps its scale slots (2 x 48 columns, one K tile each) in the first 96 columns
// of acc[(j+1)%2], which the epilogue of tile j-1 releases first; so the
// epilogue of one tile runs under the main loop of the next, and the slab MMAs,
// which need no scales, keep the tensor pipe busy during that hand-over.
//
// Few output tiles (small M): split-K.  A cluster of S CTAs shares one tile,
// each CTA accumulating a contiguous range of K tiles (the last split also
// takes the low-rank slab); the partial accumulators go to shared memory and,
// after a cluster barrier, each CTA sums a slice of the tile's rows over the S
// partials through distributed shared memory in split order (0, 1, ..., S-1),
// so the result does not depend on timing.
//
// The kernel is launched as a programmatic dependent of the kernel ahead of
// it in the stream (the activation kernel): its set-up and the weight-side
// loads of the first stages run before that kernel has finished, and the
// producer waits for it only before loading activation codes, scales and T.
#include <algorithm>
#include <cstddef>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

using namespace dev;

constexpr int kBN = 256;
constexpr int kThreads = 320;
constexpr int kMaxStages = 4;
constexpr int kATile = 128 * 128;               // 128 rows x 128 bytes (256 FP4 along K)
constexpr int kBTile = kBN * 128;               // 256 rows x 128 bytes
constexpr int kSfa = 2048;                      // four 512-byte atoms
constexpr int kSfb = 2 * 2048;                  // two 128-row blocks x four atoms
constexpr int kStage = kATile + kBTile + kSfa + kSfb;
constexpr int kSfCols = 16 + 32;                // TMEM columns of one scale slot (one K tile)
constexpr int kSfSlots = 2;                     // 2 x 48 = 96 columns
constexpr int kMaxSplit = 8;                    // portable cluster size
constexpr int kPartStride = kBN + 4;            // fp32 words per partial row (bank spread)
static_assert(128 * kPartStride * 4 <= 3 * kStage, "partials fit in the stage buffers");

struct K2Params {
  int M, N, K, r_pad;
  int kt;          // ceil(K / 256)
  int kb_total;    // K / 64
  int nblk_total;  // ceil(N / 128)
  int slab;        // ceil(r_pad / 32)
  int mtiles, ntiles;
  int ksplit;      // CTAs (one cluster) per output tile along K; 1 = persistent
  const uint8_t* xsf;
  const uint8_t* wsf;
  const float* bias;
  float alpha_w;
  uint16_t* Y;
  int y32;         // Y is 32-byte aligned: one 32-byte store per 16 columns (direct stores)
  int tma_y;       // tiles long enough to hide a staged epilogue use TMA stores of Y
  int* err;
  uint64_t wait_ns;
};

// Two configurations: 4 operand stages and one Y staging buffer per epilogue
// warp (long K: the main loop hides the epilogue), or 3 stages and a ring of
// 4 Y buffers per warp (short K: the epilogue is the longer of the two, and
// its TMA stores then overlap instead of waiting for each other).
template <int kStages, int kYBufs>
struct K2Shared {
  // per epilogue warp, kYBufs 32 x 32 bf16 chunks of Y in the 64-byte-swizzled
  // layout of the Y tensor map
  alignas(1024) uint8_t ystage[4][kYBufs][2048];
  float bias[kBN];  // the current tile's bias columns (fp32)
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t sf_full[kSfSlots];
  uint64_t sf_empty[kSfSlots];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t sfreg_free[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  int epi_stop;  // the epilogue warps leave their tile loop together
};

__device__ __noinline__ bool wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) return false;
  }
  return true;
}

// Two floats to a bf16x2 word (round to nearest even), the first in the low half.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// y = alpha_w * acc + b for 32 consecutive columns of one row, bf16 RNE, packed
// in pairs.  alpha_w is a power of two, so alpha_w * acc is exact (outside the
// subnormal range) and one fused multiply-add rounds exactly like the product
// followed by the sum.
__device__ __forceinline__ void epi_pack(const uint32_t (&r)[32], const K2Params& p, const float* bias_s,
                                         uint32_t (&packed)[16]) {
  const float4* b4 = reinterpret_cast<const float4*>(bias_s);  // this chunk's 32 bias columns (shared)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 bv = b4[i];
    const float y0 = __fmaf_rn(__uint_as_float(r[4 * i + 0]), p.alpha_w, bv.x);
    const float y1 = __fmaf_rn(__uint_as_float(r[4 * i + 1]), p.alpha_w, bv.y);
    const float y2 = __fmaf_rn(__uint_as_float(r[4 * i + 2]), p.alpha_w, bv.z);
    const float y3 = __fmaf_rn(__uint_as_float(r[4 * i + 3]), p.alpha_w, bv.w);
    packed[2 * i] = bf16x2_rn(y0, y1);
    packed[2 * i + 1] = bf16x2_rn(y2, y3);
  }
}

// One 32 x 32 chunk of the warp's rows (row `lane`, 32 columns per lane) to Y
// through the warp's staging buffer and one TMA store: four conflict-free
// 16-byte shared stores per lane instead of 32 scattered row segments per
// global store instruction, which keeps the epilogue's traffic off the load /
// store pipe the main loop's shared-memory accesses share.  The store clips rows
// >= M; its issue waits for the previous chunk's store to read the buffer, so a
// chunk takes longer than a direct store: used while the next tile's main loop
// is long enough to hide it.
template <int kYBufs>
__device__ __forceinline__ void store_chunk_tma(const uint32_t (&r)[32], const K2Params& p, const CUtensorMap* map_y,
                                                uint8_t (*ys)[2048], int& ybuf, const float* bias_s, uint32_t lane,
                                                int m_warp, int n) {
  if (m_warp >= p.M || n >= p.N) return;
  uint32_t packed[16];
  epi_pack(r, p, bias_s, packed);
  // the ring's buffers are used by the warp's stores in turn: the store that
  // last used this one is kYBufs groups back, so at most kYBufs - 1 may still read
  uint8_t* stage = ys[ybuf];
  ybuf = ybuf + 1 == kYBufs ? 0 : ybuf + 1;
  if (lane == 0) bulk_wait_read<kYBufs - 1>();
  __syncwarp();
  // 64-byte rows, 64-byte swizzle: row r's 16-byte piece i sits at piece i ^ ((r >> 1) & 3)
  uint4* row = reinterpret_cast<uint4*>(stage + lane * 64);
  const uint32_t sw = (lane >> 1) & 3u;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    row[i ^ sw] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map_y, stage, n, m_warp);
    bulk_commit_group();
  }
}

// The same chunk stored straight from registers: each lane writes its row's 64
// bytes as whole 32-byte sectors when Y allows it (else 16-byte halves).
__device__ __forceinline__ void store_chunk_direct(const uint32_t (&r)[32], const K2Params& p, const float* bias_s,
                                                   int m, int n) {
  if (m >= p.M || n >= p.N) return;
  uint32_t packed[16];
  epi_pack(r, p, bias_s, packed);
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

// One warp's share of a tile's epilogue (its 32 rows, 256 columns): chunks 0-2
// first, whose accumulator columns then take the next tile's scale slots, then
// chunks 3-7, each chunk's TMEM load in flight while the one before is stored.
template <bool kTma, int kYBufs>
__device__ __forceinline__ void epilogue_tile(const K2Params& p, const CUtensorMap* map_y, uint32_t acc,
                                              uint64_t* sfreg_free, uint64_t* sfreg_free2, uint8_t (*ys)[2048],
                                              int& ybuf, const float* bias_s, uint32_t lane, int m_warp, int n0) {
  auto put = [&](const uint32_t(&rr)[32], int c) {
    if constexpr (kTma)
      store_chunk_tma<kYBufs>(rr, p, map_y, ys, ybuf, bias_s + 32 * c, lane, m_warp, n0 + 32 * c);
    else
      store_chunk_direct(rr, p, bias_s + 32 * c, m_warp + static_cast<int>(lane), n0 + 32 * c);
  };
  uint32_t r[3][32];
#pragma unroll
  for (int c = 0; c < 3; ++c) tmem_ld_x32(acc + 32 * c, r[c]);
  tmem_ld_wait();
  // columns 0..95 read: the next tile's scale slots may go there
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(sfreg_free);
  uint32_t nx[32];
  tmem_ld_x32(acc + 96, nx);
#pragma unroll
  for (int c = 0; c < 3; ++c) put(r[c], c);
#pragma unroll
  for (int c = 3; c < kBN / 32; ++c) {
    tmem_ld_wait_regs(nx);
    if (sfreg_free2 && c == 4) {
      // columns 96..159 read: a third scale slot (columns 96..143) may go there
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sfreg_free2);
    }
    uint32_t cur[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) cur[i] = nx[i];
    if (c + 1 < kBN / 32) tmem_ld_x32(acc + 32 * (c + 1), nx);
    put(cur, c);
  }
}

// Split-K: this CTA's share of the tile's rows, summed over the S partials in
// split order, then y = alpha_w * acc + b in bf16 RNE.
__device__ __forceinline__ void split_reduce(const K2Params& p, const float* part, int split, int t) {
  const int m0 = (t % p.mtiles) * 128, n0 = (t / p.mtiles) * kBN;
  const int rows = min(128, p.M - m0);
  const int per = (rows + p.ksplit - 1) / p.ksplit;
  const int r_lo = split * per, r_hi = min(rows, r_lo + per);
  const uint32_t base = smem_u32(part);
  for (int i = threadIdx.x; i < (r_hi - r_lo) * (kBN / 4); i += kThreads) {
    const int r = r_lo + i / (kBN / 4), c = 4 * (i % (kBN / 4));
    const int n = n0 + c;
    if (n >= p.N) continue;
    const uint32_t off = static_cast<uint32_t>(r * kPartStride + c) * 4u;
    float4 v[kMaxSplit];
#pragma unroll
    for (int q = 0; q < kMaxSplit; ++q)
      if (q < p.ksplit) v[q] = ld_dsmem_f4(mapa_shared(base + off, q));
    float4 acc = v[0];
#pragma unroll
    for (int q = 1; q < kMaxSplit; ++q)
      if (q < p.ksplit) {
        acc.x = __fadd_rn(acc.x, v[q].x);
        acc.y = __fadd_rn(acc.y, v[q].y);
        acc.z = __fadd_rn(acc.z, v[q].z);
        acc.w = __fadd_rn(acc.w, v[q].w);
      }
    const float4 b = *reinterpret_cast<const float4*>(p.bias + n);
    const uint32_t lo = bf16x2_rn(__fmaf_rn(acc.x, p.alpha_w, b.x), __fmaf_rn(acc.y, p.alpha_w, b.y));
    const uint32_t hi = bf16x2_rn(__fmaf_rn(acc.z, p.alpha_w, b.z), __fmaf_rn(acc.w, p.alpha_w, b.w));
    *reinterpret_cast<uint2*>(p.Y + static_cast<size_t>(m0 + r) * p.N + n) = make_uint2(lo, hi);
  }
}

// Named barrier of the four epilogue warps (ids 0 and 1 are __syncthreads and unused).
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

template <int kStages, int kYBufs>
__global__ void __launch_bounds__(kThreads, 1) gemm_w4a4_kernel(
    const __grid_constant__ CUtensorMap map_xq, const __grid_constant__ CUtensorMap map_wq,
    const __grid_constant__ CUtensorMap map_t, const __grid_constant__ CUtensorMap map_l2,
    const __grid_constant__ CUtensorMap map_y,
    const K2Params p) {
  using Shared = K2Shared<kStages, kYBufs>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared* sh = reinterpret_cast<Shared*>(smem + kStages * kStage);
  static_assert(offsetof(Shared, ystage) == 0, "Y staging buffers keep the 1024-byte alignment the swizzle needs");
  static_assert((kStages * kStage) % 1024 == 0, "stage buffers keep 1024-byte alignment");

  const uint32_t warp = warp_id(), lane = lane_id();
  const int ntiles_total = p.mtiles * p.ntiles;
  // split-K: CTA blockIdx.x is rank (blockIdx.x % S) of the cluster that owns
  // tile blockIdx.x / S; it takes a contiguous range of the K tiles, and the
  // last split the slab as well (its range is never the longer one)
  const int S = p.ksplit;
  const int split = static_cast<int>(blockIdx.x) % S;
  const int tile0 = static_cast<int>(blockIdx.x) / S, tile_step = static_cast<int>(gridDim.x) / S;
  const int kt_base = p.kt / S, kt_rem = p.kt % S;
  const int kt_lo = split * kt_base + min(split, kt_rem);
  const int nslab = split == S - 1 ? p.slab : 0;
  const int per_tile = nslab + kt_base + (split < kt_rem ? 1 : 0);
  float* part = reinterpret_cast<float*>(smem);  // split-K partials, after the tile's MMAs
  // the next layer's activation kernel may launch now and take SMs as this
  // grid's CTAs retire; it waits for this grid before touching X, xq, xsf or T
  grid_dep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1 + 4);  // MMA commit + the four scale writers
    }
    for (int b = 0; b < kSfSlots; ++b) {
      mbar_init(&sh->sf_full[b], 4);
      mbar_init(&sh->sf_empty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->acc_full[b], 1);
      mbar_init(&sh->acc_empty[b], 4);
      mbar_init(&sh->sfreg_free[b], 4);
    }
    mbar_init(&sh->done, 1);
    sh->abort = 0;
    sh->epi_stop = 0;
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
      // A stage's loads come in two halves: the weight side (codes, scales,
      // L2), which no kernel of the forward pass writes, and the activation
      // side (codes, scales, T) from the kernel ahead.  The first stages'
      // weight halves go out before the wait for that kernel.
      int m0 = (tile0 % p.mtiles) * 128, n0 = (tile0 / p.mtiles) * kBN;
      int nb_valid = min(2, p.nblk_total - n0 / 128);
      const int npre = tile0 < ntiles_total ? min(kStages, per_tile) : 0;
      for (int k = 0; k < npre; ++k) {
        uint8_t* st = smem + k * kStage;
        if (k >= nslab) {
          const int kk = kt_lo + k - nslab;
          const int nkb = min(4, p.kb_total - 4 * kk);
          mbar_arrive_expect_tx(&sh->full[k], kATile + kBTile + 512u * nkb * (1 + nb_valid));
          tma_load_2d(st + kATile, &map_wq, &sh->full[k], kk * 128, n0);
          for (int nb = 0; nb < nb_valid; ++nb)
            bulk_load(st + kATile + kBTile + kSfa + nb * 2048,
                      p.wsf + (static_cast<size_t>(n0 / 128 + nb) * p.kb_total + 4 * kk) * 512, 512u * nkb,
                      &sh->full[k]);
        } else {
          mbar_arrive_expect_tx(&sh->full[k], kATile + kBN * 64);
          tma_load_2d(st + kATile, &map_l2, &sh->full[k], 32 * k, n0);
        }
      }
      grid_dep_wait();
      int it = 0;
      bool ok = true;
      for (int t = tile0; ok && t < ntiles_total; t += tile_step) {
        m0 = (t % p.mtiles) * 128;
        n0 = (t / p.mtiles) * kBN;
        nb_valid = min(2, p.nblk_total - n0 / 128);
        for (int k = 0; k < per_tile; ++k, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          const bool pre = it < npre;  // weight half already issued
          if (!pre && !wait_bounded(&sh->empty[s], ph ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStage;
          if (k >= nslab) {
            const int kk = kt_lo + k - nslab;
            const int nkb = min(4, p.kb_total - 4 * kk);
            if (!pre) mbar_arrive_expect_tx(&sh->full[s], kATile + kBTile + 512u * nkb * (1 + nb_valid));
            tma_load_2d(st, &map_xq, &sh->full[s], kk * 128, m0);
            if (!pre) tma_load_2d(st + kATile, &map_wq, &sh->full[s], kk * 128, n0);
            bulk_load(st + kATile + kBTile,
                      p.xsf + (static_cast<size_t>(m0 / 128) * p.kb_total + 4 * kk) * 512, 512u * nkb,
                      &sh->full[s]);
            if (!pre)
              for (int nb = 0; nb < nb_valid; ++nb)
                bulk_load(st + kATile + kBTile + kSfa + nb * 2048,
                          p.wsf + (static_cast<size_t>(n0 / 128 + nb) * p.kb_total + 4 * kk) * 512,
                          512u * nkb, &sh->full[s]);
          } else {
            if (!pre) mbar_arrive_expect_tx(&sh->full[s], kATile + kBN * 64);
            tma_load_2d(st, &map_t, &sh->full[s], 64 * k, m0);
            if (!pre) tma_load_2d(st + kATile, &map_l2, &sh->full[s], 32 * k, n0);
          }
        }
      }
      if (sh->abort) {  // let copies in flight land before the CTA exits
        for (int i = max(0, it - kStages); i < it; ++i)
          wait_drain(&sh->full[i % kStages], (i / kStages) & 1, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_fp4 = idesc_nvfp4(128, kBN);
      const uint32_t id_bf16 = idesc_bf16(128, kBN);
      // descriptors of stage 0; stage s starts kStage bytes further (the start
      // address field counts 16-byte units)
      const uint32_t stage0 = smem_u32(smem);
      const uint64_t da0 = desc_kmajor_sw128(stage0);
      const uint64_t db0 = desc_kmajor_sw128(stage0 + kATile);
      const uint64_t dl0 = desc_kmajor_sw64(stage0 + kATile);
      int it = 0, sfi = 0, j = 0;
      bool ok = true;
      for (int t = tile0; ok && t < ntiles_total; t += tile_step, ++j) {
        const int a = j & 1;
        if (!wait_bounded(&sh->acc_empty[a], ((j >> 1) & 1) ^ 1, wc)) break;
        tc_fence_after();
        const uint32_t acc = tmem + a * 256;
        const uint32_t sf_region = tmem + (a ^ 1) * 256;
        uint32_t accum = 0;  // the tile's first MMA overwrites the accumulator
        for (int k = 0; k < per_tile; ++k, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          const uint64_t soff = static_cast<uint64_t>(s * (kStage >> 4));
          if (k >= nslab) {
            const int nkb = min(4, p.kb_total - 4 * (kt_lo + k - nslab));
            const int b = sfi & (kSfSlots - 1);
            // the writers waited for this stage's data before publishing its scales
            if (!wait_bounded(&sh->sf_full[b], (sfi / kSfSlots) & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sfa = sf_region + b * kSfCols;
            const uint32_t sfb = sfa + 16;
            const uint64_t adesc = da0 + soff, bdesc = db0 + soff;
            if (nkb == 4) {
              mma_nvfp4_x4(acc, adesc, bdesc, id_fp4, sfa, sfb, accum);
            } else {  // K tail: fewer than four 64-element blocks
              for (int kb = 0; kb < nkb; ++kb)
                mma_nvfp4(acc, adesc + 2 * kb, bdesc + 2 * kb, id_fp4, sfa + 4 * kb, sfb + 8 * kb, kb ? 1u : accum);
            }
            accum = 1;
            mma_commit(&sh->sf_empty[b]);
            mma_commit(&sh->empty[s]);
            ++sfi;
          } else {
            if (!wait_bounded(&sh->full[s], ph, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (32 * k + 16 * c >= p.r_pad) break;
              const uint64_t ldesc = dl0 + soff + 2 * c;
              mma_bf16(acc, da0 + soff + 4 * c, ldesc, id_bf16, accum);      // T_hi
              mma_bf16(acc, da0 + soff + 4 * c + 2, ldesc, id_bf16, 1);      // T_lo
              accum = 1;
            }
            mma_commit(&sh->empty[s]);
          }
        }
        if (ok) mma_commit(&sh->acc_full[a]);
      }
      mma_commit(&sh->done);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------ scale writers
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    int it = 0, sfi = 0, j = 0;
    bool ok = true;
    for (int t = tile0; ok && t < ntiles_total; t += tile_step, ++j) {
      const int a = j & 1;
      const uint32_t sf_region = tmem + (a ^ 1) * 256 + lane_off;
      for (int k = 0; k < per_tile; ++k, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (k >= nslab) {
          if (!wait_warp(&sh->full[s], ph, wc)) {
            ok = false;
            break;
          }
          const uint8_t* sfa_s = smem + s * kStage + kATile + kBTile;
          const uint8_t* sfb_s = sfa_s + kSfa;
          // read the K tile's scale atoms first, then release the stage and
          // wait for the TMEM slot: only the tcgen05.st is on the MMA's path
          uint32_t ra[16], rb[32];
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint4 v = *reinterpret_cast<const uint4*>(sfa_s + kb * 512 + lane * 16);
            ra[4 * kb] = v.x;
            ra[4 * kb + 1] = v.y;
            ra[4 * kb + 2] = v.z;
            ra[4 * kb + 3] = v.w;
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
              const uint4 u = *reinterpret_cast<const uint4*>(sfb_s + nb * 2048 + kb * 512 + lane * 16);
              rb[8 * kb + 4 * nb] = u.x;
              rb[8 * kb + 4 * nb + 1] = u.y;
              rb[8 * kb + 4 * nb + 2] = u.z;
              rb[8 * kb + 4 * nb + 3] = u.w;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->empty[s]);
          if (k == nslab) {
            // the scale slots live in acc[a^1]: before the tile's first store into
            // them, wait until the previous tile's epilogue has read its first 96 columns
            if (!wait_warp(&sh->sfreg_free[a ^ 1], ((j - 1) >> 1) & 1, wc)) {
              ok = false;
              break;
            }
          }
          const int b = sfi & (kSfSlots - 1);
          if (!wait_warp(&sh->sf_empty[b], ((sfi / kSfSlots) & 1) ^ 1, wc)) {
            ok = false;
            break;
          }
          const uint32_t dst = sf_region + b * kSfCols;
          tmem_st_x16(dst, ra);
          tmem_st_x32(dst + 16, rb);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->sf_full[b]);
          ++sfi;
        } else {
          if (!wait_warp(&sh->full[s], ph, wc)) {
            ok = false;
            break;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->empty[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int row = q * 32 + lane;
    uint8_t(*ys)[2048] = sh->ystage[warp - 6];
    const int et = static_cast<int>(threadIdx.x) - 6 * 32;  // 0..127 over the epilogue warps
    int ybuf = 0;  // next buffer of the warp's Y staging ring
    int j = 0;
    for (int t = tile0; t < ntiles_total; t += tile_step, ++j) {
      const int a = j & 1;
      const int m_warp = (t % p.mtiles) * 128 + q * 32;
      const int m = m_warp + static_cast<int>(lane);
      const int n0 = (t / p.mtiles) * kBN;
      // staged TMA stores while another tile's main loop follows (or always,
      // with a ring of buffers); the CTA's last tile stores directly
      const bool tma = p.tma_y && (kYBufs > 1 || t + tile_step < ntiles_total);
      // this tile's bias columns (the bias is padded to a multiple of 256),
      // loaded before the wait so that the load latency hides under the MMAs
      const float2 bpre = __ldg(reinterpret_cast<const float2*>(p.bias + n0) + et);
      if (!wait_warp(&sh->acc_full[a], (j >> 1) & 1, wc) && lane == 0) sh->epi_stop = 1;
      epi_bar();  // every epilogue warp is done with the previous tile's bias
      const bool stop = sh->epi_stop != 0;  // the same for all four warps (written before the barrier)
      if (!stop) reinterpret_cast<float2*>(sh->bias)[et] = bpre;
      epi_bar();
      if (stop) break;
      tc_fence_after();
      if (S > 1) {
        // split-K (one tile per CTA): this split's partial rows into the
        // stage buffers, which the tile's completed MMAs no longer read
        float* prow = part + row * kPartStride;
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t rr[32];
          tmem_ld_x32(tmem + a * 256 + lane_off + 32 * c, rr);
          tmem_ld_wait();
          if (m < p.M) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<float4*>(prow + 32 * c + 4 * i) =
                  make_float4(__uint_as_float(rr[4 * i]), __uint_as_float(rr[4 * i + 1]),
                              __uint_as_float(rr[4 * i + 2]), __uint_as_float(rr[4 * i + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sh->sfreg_free[a]);
          mbar_arrive(&sh->acc_empty[a]);
        }
        continue;
      }
      if (tma)
        epilogue_tile<true, kYBufs>(p, &map_y, tmem + a * 256 + lane_off, &sh->sfreg_free[a], nullptr, ys, ybuf,
                                    sh->bias, lane, m_warp, n0);
      else
        epilogue_tile<false, kYBufs>(p, &map_y, tmem + a * 256 + lane_off, &sh->sfreg_free[a], nullptr, ys, ybuf,
                                     sh->bias, lane, m_warp, n0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->acc_empty[a]);
    }
    if (lane == 0) bulk_wait_all();  // Y written, the staging buffer no longer read
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (S > 1) {
    cluster_sync_all();  // every split's partial is in its CTA's shared memory
    if (!sh->abort && tile0 < ntiles_total) split_reduce(p, part, split, tile0);
    cluster_sync_relaxed();  // the peers have read this CTA's partial
  }
  if (warp == 1) {
    if (lane == 0) wait_drain(&sh->done, 0, p.wait_ns);  // every MMA has retired
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ CTA pair
// Many output tiles: a cluster of two CTAs takes 256 x 256 tiles, each MMA an
// M = 256 pair operation issued by rank 0.  Each CTA stages its own 128 rows
// of the activation codes and 128 of the 256 weight rows, so a K tile brings
// 38 KB into each SM instead of 54 KB and five stages fit where four did; each
// CTA's TMEM holds its 128 accumulator rows and the scale atoms of its rows and
// of all 256 weight rows (the layout the pair MMA reads in both CTAs).
// Every load completes on a barrier of its own CTA, so each CTA can account
// for its copies in flight; what the leader's MMA issuer needs of the peer
// (its operands landed, its scale slots filled, its accumulator rows drained)
// reaches it as arrivals on the leader's barriers, and the leader's commits
// arrive on the same barrier in both CTAs.  Three scale slots: the MMAs of a
// K tile wait only for the slot filled after the K tile three back retired.
constexpr int kPBTile = 128 * 128;                             // this CTA's 128 weight rows x 128 bytes
constexpr int kPStage = kATile + kPBTile + kSfa + kSfb;        // 38 KB
constexpr int kPSlots = 3;                                     // 3 x 48 = 144 columns of the idle accumulator
static_assert(kPStage % 1024 == 0, "stage buffers keep 1024-byte alignment");

template <int kStages, int kYBufs>
struct K2PairShared {
  alignas(1024) uint8_t ystage[4][kYBufs][2048];
  float bias[kBN];
  uint64_t full[kStages];       // this CTA's bytes of the stage (operands, scales, T, L2)
  uint64_t empty[kStages];      // the leader's MMA commit
  uint64_t peer_full[kStages];  // leader: the peer's bytes of the stage have landed
  uint64_t sf_full[kPSlots];    // leader: the pair's eight scale-writer warps
  uint64_t sf_empty[kPSlots];   // the leader's MMA commit
  uint64_t acc_full[2];         // the leader's MMA commit
  uint64_t acc_empty[2];        // leader: the pair's eight epilogue warps
  uint64_t sfreg_free[2];       // this CTA's epilogue warps have read columns 0..95
  uint64_t sfreg_free2[2];      // ... and columns 96..159
  uint64_t done;                // leader: every MMA has retired
  uint32_t tmem_base;
  int abort;
  int epi_stop;
};

// p.mtiles counts 256-row pair tiles here.
constexpr int kPThreads = 352;  // the 320 of the single-CTA kernel plus a weight-side producer warp
template <int kStages, int kYBufs>
__global__ void __launch_bounds__(kPThreads, 1) gemm_w4a4_pair_kernel(
    const __grid_constant__ CUtensorMap map_xq, const __grid_constant__ CUtensorMap map_wq,
    const __grid_constant__ CUtensorMap map_t, const __grid_constant__ CUtensorMap map_l2,
    const __grid_constant__ CUtensorMap map_y, const __grid_constant__ CUtensorMap map_wsf, const K2Params p) {
  using Shared = K2PairShared<kStages, kYBufs>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared* sh = reinterpret_cast<Shared*>(smem + kStages * kPStage);
  static_assert(offsetof(Shared, ystage) == 0, "Y staging buffers keep the 1024-byte alignment the swizzle needs");

  const uint32_t warp = warp_id(), lane = lane_id();
  const int rank = static_cast<int>(cluster_ctarank());  // 0 = leader
  const bool leader = rank == 0;
  const int ntiles_total = p.mtiles * p.ntiles;
  const int pair0 = static_cast<int>(blockIdx.x) >> 1, npairs = static_cast<int>(gridDim.x) >> 1;
  const int per_tile = p.slab + p.kt;
  grid_dep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
      mbar_init(&sh->peer_full[s], 1);
    }
    for (int b = 0; b < kPSlots; ++b) {
      mbar_init(&sh->sf_full[b], 8);
      mbar_init(&sh->sf_empty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->acc_full[b], 1);
      mbar_init(&sh->acc_empty[b], 8);
      mbar_init(&sh->sfreg_free[b], 4);
      mbar_init(&sh->sfreg_free2[b], 4);
    }
    mbar_init(&sh->done, 1);
    sh->abort = 0;
    sh->epi_stop = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&sh->tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const WaitCtl wc{p.err, p.wait_ns, &sh->abort};
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------ producers
    // Warp 10 issues the weight half of every stage (codes and both 128-row
    // blocks of scale atoms in one 3-D copy, or L2), which no kernel of the
    // forward pass writes, and arms the stage's barrier for all its bytes; warp
    // 0 issues the activation half (codes and scales, or T) once the kernel
    // ahead has finished.  A thread issuing a copy waits for the copy engine to
    // take it (~130 cycles each): one thread for all of a stage's copies was
    // the bound on the K-tile rate.
    if (lane == 0) {
      const bool wside = warp == 10;
      if (wside) {
        tma_prefetch_desc(&map_wq);
        tma_prefetch_desc(&map_wsf);
        if (p.slab) tma_prefetch_desc(&map_l2);
      } else {
        tma_prefetch_desc(&map_xq);
        if (p.slab) tma_prefetch_desc(&map_t);
        grid_dep_wait();
      }
      int it = 0;
      bool ok = true;
      for (int t = pair0; ok && t < ntiles_total; t += npairs) {
        const int m0 = (t % p.mtiles) * 256 + 128 * rank;
        const int n0 = (t / p.mtiles) * kBN;
        const int sfa_valid = m0 < p.M ? 1 : 0;
        for (int k = 0; k < per_tile; ++k, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!wait_bounded(&sh->empty[s], ph ^ 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kPStage;
          if (k >= p.slab) {
            const int kk = k - p.slab;
            const int nkb = min(4, p.kb_total - 4 * kk);
            if (wside) {
              // a tiled copy counts its whole box, the parts outside the array included
              mbar_arrive_expect_tx(&sh->full[s], kATile + kPBTile + kSfb + 512u * nkb * sfa_valid);
              tma_load_2d(st + kATile, &map_wq, &sh->full[s], kk * 128, n0 + 128 * rank);
              tma_load_3d(st + kATile + kPBTile + kSfa, &map_wsf, &sh->full[s], 0, 4 * kk, n0 / 128);
            } else {
              tma_load_2d(st, &map_xq, &sh->full[s], kk * 128, m0);
              if (sfa_valid)
                bulk_load(st + kATile + kPBTile, p.xsf + (static_cast<size_t>(m0 / 128) * p.kb_total + 4 * kk) * 512,
                          512u * nkb, &sh->full[s]);
            }
          } else {
            if (wside) {
              mbar_arrive_expect_tx(&sh->full[s], kATile + 128 * 64);
              tma_load_2d(st + kATile, &map_l2, &sh->full[s], 32 * k, n0 + 128 * rank);
            } else {
              tma_load_2d(st, &map_t, &sh->full[s], 64 * k, m0);
            }
          }
        }
      }
      if (sh->abort) {  // this CTA's copies in flight land before it exits
        for (int i = max(0, it - kStages); i < it; ++i)
          wait_drain(&sh->full[i % kStages], (i / kStages) & 1, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      const uint32_t id_fp4 = idesc_nvfp4(256, kBN);
      const uint32_t id_bf16 = idesc_bf16(256, kBN);
      const uint32_t stage0 = smem_u32(smem);
      const uint64_t da0 = desc_kmajor_sw128(stage0);
      const uint64_t db0 = desc_kmajor_sw128(stage0 + kATile);
      const uint64_t dl0 = desc_kmajor_sw64(stage0 + kATile);
      int it = 0, j = 0;
      int b = 0;
      uint32_t bph = 0;  // scale slot and the parity of its current fill
      bool ok = true;
      for (int t = pair0; ok && t < ntiles_total; t += npairs, ++j) {
        const int a = j & 1;
        if (!wait_bounded(&sh->acc_empty[a], ((j >> 1) & 1) ^ 1, wc)) break;
        tc_fence_after();
        const uint32_t acc = tmem + a * 256;
        const uint32_t sf_region = tmem + (a ^ 1) * 256;
        uint32_t accum = 0;
        for (int k = 0; k < per_tile; ++k, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          const uint64_t soff = static_cast<uint64_t>(s * (kPStage >> 4));
          if (k >= p.slab) {
            const int nkb = min(4, p.kb_total - 4 * (k - p.slab));
            // both CTAs' writers saw their CTA's bytes of the stage land first
            if (!wait_bounded(&sh->sf_full[b], bph, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sfa = sf_region + b * kSfCols;
            const uint32_t sfb = sfa + 16;
            const uint64_t adesc = da0 + soff, bdesc = db0 + soff;
            if (nkb == 4) {
              mma_nvfp4_pair_x4(acc, adesc, bdesc, id_fp4, sfa, sfb, accum);
            } else {
              for (int kb = 0; kb < nkb; ++kb)
                mma_nvfp4_pair(acc, adesc + 2 * kb, bdesc + 2 * kb, id_fp4, sfa + 4 * kb, sfb + 8 * kb,
                               kb ? 1u : accum);
            }
            accum = 1;
            mma_commit_both(&sh->sf_empty[b]);
            mma_commit_both(&sh->empty[s]);
            if (++b == kPSlots) {
              b = 0;
              bph ^= 1;
            }
          } else {
            if (!wait_bounded(&sh->full[s], ph, wc) || !wait_bounded(&sh->peer_full[s], ph, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (32 * k + 16 * c >= p.r_pad) break;
              const uint64_t ldesc = dl0 + soff + 2 * c;
              mma_bf16_pair(acc, da0 + soff + 4 * c, ldesc, id_bf16, accum);  // T_hi
              mma_bf16_pair(acc, da0 + soff + 4 * c + 2, ldesc, id_bf16, 1);  // T_lo
              accum = 1;
            }
            mma_commit_both(&sh->empty[s]);
          }
        }
        if (ok) mma_commit_both(&sh->acc_full[a]);
      }
      mma_commit_pair_local(&sh->done);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------ scale writers
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t sf_full_l = mapa_shared(smem_u32(&sh->sf_full[0]), 0);
    const uint32_t peer_full_l = mapa_shared(smem_u32(&sh->peer_full[0]), 0);
    int it = 0, j = 0;
    int b = 0;
    uint32_t bph = 0;
    bool ok = true;
    for (int t = pair0; ok && t < ntiles_total; t += npairs, ++j) {
      const int a = j & 1;
      const uint32_t sf_region = tmem + (a ^ 1) * 256 + lane_off;
      bool third_free = false;  // the previous tile's epilogue has read columns 96..159
      for (int k = 0; k < per_tile; ++k, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!wait_warp(&sh->full[s], ph, wc)) {
          ok = false;
          break;
        }
        // the peer tells the leader's MMA issuer that its bytes of the stage are in
        if (!leader && warp == 2 && lane == 0) mbar_arrive_cluster(peer_full_l + 8u * s);
        if (k < p.slab) continue;
        const uint8_t* sfa_s = smem + s * kPStage + kATile + kPBTile;
        const uint8_t* sfb_s = sfa_s + kSfa;
        uint32_t ra[16], rb[32];
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          const uint4 v = *reinterpret_cast<const uint4*>(sfa_s + kb * 512 + lane * 16);
          ra[4 * kb] = v.x;
          ra[4 * kb + 1] = v.y;
          ra[4 * kb + 2] = v.z;
          ra[4 * kb + 3] = v.w;
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            const uint4 u = *reinterpret_cast<const uint4*>(sfb_s + nb * 2048 + kb * 512 + lane * 16);
            rb[8 * kb + 4 * nb] = u.x;
            rb[8 * kb + 4 * nb + 1] = u.y;
            rb[8 * kb + 4 * nb + 2] = u.z;
            rb[8 * kb + 4 * nb + 3] = u.w;
          }
        }
        // the scale slots live in acc[a^1]: before the tile's first store into
        // a slot, wait until the previous tile's epilogue of this CTA has read it
        if (k == p.slab && !wait_warp(&sh->sfreg_free[a ^ 1], ((j - 1) >> 1) & 1, wc)) {
          ok = false;
          break;
        }
        if (b == 2 && !third_free) {
          if (!wait_warp(&sh->sfreg_free2[a ^ 1], ((j - 1) >> 1) & 1, wc)) {
            ok = false;
            break;
          }
          third_free = true;
        }
        if (!wait_warp(&sh->sf_empty[b], bph ^ 1, wc)) {
          ok = false;
          break;
        }
        const uint32_t dst = sf_region + b * kSfCols;
        tmem_st_x16(dst, ra);
        tmem_st_x32(dst + 16, rb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(sf_full_l + 8u * b);
        if (++b == kPSlots) {
          b = 0;
          bph ^= 1;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t acc_empty_l = mapa_shared(smem_u32(&sh->acc_empty[0]), 0);
    uint8_t(*ys)[2048] = sh->ystage[warp - 6];
    const int et = static_cast<int>(threadIdx.x) - 6 * 32;
    int ybuf = 0;
    int j = 0;
    for (int t = pair0; t < ntiles_total; t += npairs, ++j) {
      const int a = j & 1;
      const int m_warp = (t % p.mtiles) * 256 + 128 * rank + q * 32;
      const int n0 = (t / p.mtiles) * kBN;
      const bool tma = p.tma_y && (kYBufs > 1 || t + npairs < ntiles_total);
      const float2 bpre = __ldg(reinterpret_cast<const float2*>(p.bias + n0) + et);
      if (!wait_warp(&sh->acc_full[a], (j >> 1) & 1, wc) && lane == 0) sh->epi_stop = 1;
      epi_bar();
      const bool stop = sh->epi_stop != 0;
      if (!stop) reinterpret_cast<float2*>(sh->bias)[et] = bpre;
      epi_bar();
      if (stop) break;
      tc_fence_after();
      if (tma)
        epilogue_tile<true, kYBufs>(p, &map_y, tmem + a * 256 + lane_off, &sh->sfreg_free[a], &sh->sfreg_free2[a], ys, ybuf,
                                    sh->bias, lane, m_warp, n0);
      else
        epilogue_tile<false, kYBufs>(p, &map_y, tmem + a * 256 + lane_off, &sh->sfreg_free[a], &sh->sfreg_free2[a], ys, ybuf,
                                     sh->bias, lane, m_warp, n0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_l + 8u * a);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1 && leader && lane == 0) wait_drain(&sh->done, 0, p.wait_ns);  // every MMA has retired
  __syncthreads();
  cluster_sync_all();  // no cross-CTA arrival or MMA access is still in flight
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

using K2Kernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                         const CUtensorMap, const K2Params);
using K2PairKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                             const CUtensorMap, const CUtensorMap, const K2Params);

// The two instantiations: long K (4 stages, one Y buffer per epilogue warp)
// and short K (3 stages, a ring of 4 Y buffers per warp).
struct K2Config {
  K2Kernel fn;        // single-CTA kernel (nullptr for the pair kernel)
  K2PairKernel pfn;   // CTA-pair kernel
  size_t smem;
  int id;
  const void* entry() const { return fn ? reinterpret_cast<const void*>(fn) : reinterpret_cast<const void*>(pfn); }
};
K2Config k2_config(bool short_k) {
  if (short_k)
    return {gemm_w4a4_kernel<3, 4>, nullptr, 1024 + 3 * static_cast<size_t>(kStage) + sizeof(K2Shared<3, 4>), 1};
  return {gemm_w4a4_kernel<4, 1>, nullptr, 1024 + 4 * static_cast<size_t>(kStage) + sizeof(K2Shared<4, 1>), 0};
}
// The CTA-pair kernel: five stages and a ring of four Y buffers per epilogue warp.
constexpr int kPairStages = 5, kPairYBufs = 4;
constexpr int kPairMinKTiles = 16;  // K > 3840
K2Config k2_pair_config() {
  return {nullptr, gemm_w4a4_pair_kernel<kPairStages, kPairYBufs>,
          1024 + kPairStages * static_cast<size_t>(kPStage) + sizeof(K2PairShared<kPairStages, kPairYBufs>), 2};
}
static_assert(1024 + kPairStages * kPStage + sizeof(K2PairShared<kPairStages, kPairYBufs>) <= 232448,
              "the pair kernel's shared memory fits one CTA per SM");

// Clusters of S CTAs of this kernel that fit on the device at once (cached
// per device, configuration and S).
int max_active_clusters(const K2Config& kc, int S) {
  static int cache[64][3][kMaxSplit + 1] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cache[dev][kc.id][S]) return cache[dev][kc.id][S];
  const size_t smem = kc.smem;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, 1, 1);
  cfg.blockDim = dim3(kc.id == 2 ? kPThreads : kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kc.entry(), &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = -1;  // cached as "does not fit"
  }
  if (dev >= 0 && dev < 64) cache[dev][kc.id][S] = n;
  return n;
}

// Split-K factor for `tiles` output tiles of `kt` K tiles plus `slab` low-rank
// stages.  Splitting pays when the tiles leave most SMs idle: the time of a
// tile is its longest split (the last split also runs the slab, one stage's
// worth of MMAs each) plus about two K tiles for the reduction; every tile's
// cluster must be resident at once.  Ties go to the smaller split.
int choose_ksplit(const K2Config& kc, int tiles, int kt, int slab) {
  if (2 * tiles > num_sms()) return 1;
  int best = 1;
  long best_cost = kt + slab;
  for (int S = 2; S <= std::min(kMaxSplit, kt); ++S) {
    if (max_active_clusters(kc, S) < tiles) continue;
    const int base = kt / S, rem = kt % S;
    const long cost = std::max(base + (rem ? 1 : 0), base + slab) + 2;
    if (cost < best_cost) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
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
  p.mtiles = (a.M + 127) / 128;
  p.ntiles = (a.N + kBN - 1) / kBN;
  p.ksplit = 1;
  p.xsf = static_cast<const uint8_t*>(a.xsf);
  p.wsf = a.wsf;
  p.bias = a.bias;
  p.alpha_w = a.alpha_w;
  p.Y = static_cast<uint16_t*>(a.Y);
  // N % 16 == 0, so every 16-column piece starts 32 bytes after the last
  p.y32 = (reinterpret_cast<uintptr_t>(a.Y) & 31u) == 0;
  // A tile of at least 8 K steps (K >= 1792) hides the staged epilogue of the
  // one before; shorter tiles are epilogue-bound and take the configuration
  // with fewer stages and a ring of Y buffers, whose TMA stores overlap.
  const bool short_k = p.kt + p.slab < 8;
  const K2Config kc = k2_config(short_k);
  p.tma_y = 1;
  p.err = a.err ? a.err : device_error_word();
  p.wait_ns = wait_limit_ns();
  if (!p.err) return fail(SVDQ_ERR_CUDA, "device error word unavailable");

  CUtensorMap map_xq;
  svdq_status st = make_tmap_2d(&map_xq, a.xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.K / 2, a.M, a.K / 2, 128,
                                128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != SVDQ_OK) return st;
  CUtensorMap map_t = map_xq;
  if (a.r_pad > 0) {
    st = make_tmap_2d(&map_t, a.T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2 * a.r_pad, a.M,
                      static_cast<uint64_t>(4 * a.r_pad), 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != SVDQ_OK) return st;
  }
  const CUtensorMap& map_l2 = a.r_pad > 0 ? *a.map_l2_256 : map_xq;
  // Y in 32 x 32 boxes (64-byte rows, 64-byte swizzle) for the epilogue's stores
  CUtensorMap map_y;
  st = make_tmap_2d(&map_y, a.Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.N, a.M, static_cast<uint64_t>(a.N) * 2, 32, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != SVDQ_OK) return st;

  const size_t smem = kc.smem;
  static bool attr_set[64] = {};  // per device: the attributes are set on the current one
  int cur_dev = 0;
  SVDQ_CUDA_TRY(cudaGetDevice(&cur_dev));
  if (cur_dev < 0 || cur_dev >= 64 || !attr_set[cur_dev]) {
    for (int v = 0; v < 3; ++v) {
      const K2Config c = v == 2 ? k2_pair_config() : k2_config(v == 1);
      SVDQ_CUDA_TRY(
          cudaFuncSetAttribute(c.entry(), cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(c.smem)));
    }
    if (cur_dev >= 0 && cur_dev < 64) attr_set[cur_dev] = true;
  }
  const int tiles = p.mtiles * p.ntiles;
  if (a.ksplit > 0) {
    p.ksplit = std::min(std::min(a.ksplit, kMaxSplit), p.kt);
    if (p.ksplit > 1 && max_active_clusters(kc, p.ksplit) < tiles) p.ksplit = 1;
  } else {
    p.ksplit = choose_ksplit(kc, tiles, p.kt, p.slab);
  }

  // Many tiles, long K and no split requested: the CTA-pair kernel over
  // 256 x 256 tiles, one pair per resident cluster of two.  Measured against
  // the single-CTA kernel (GEMM alone, CUDA-graph replay, us): ahead from 16 K
  // tiles (FLUX 12288 -> 3072 75.4 vs 79.2, SDXL 10240 -> 1280 23.5 vs 25.2,
  // PixArt 4608 -> 1152 21.7 vs 22.0), level within noise at 5-12 K tiles
  // (and behind in the full step, where its clusters of two start later behind
  // the activation kernel), behind below 4 (SDXL 640-wide: 33.5 vs 31.6).
  if (a.ksplit == 0 && p.ksplit == 1 && p.kt >= kPairMinKTiles && a.map_wq_128 && a.map_wsf &&
      (a.r_pad == 0 || a.map_l2_128)) {
    const K2Config pc = k2_pair_config();
    const int pairs_fit = max_active_clusters(pc, 2);
    if (pairs_fit >= 1) {
      K2Params pp = p;
      pp.mtiles = (a.M + 255) / 256;
      const int ptiles = pp.mtiles * pp.ntiles;
      const CUtensorMap& map_l2_p = a.r_pad > 0 ? *a.map_l2_128 : map_xq;
      cudaLaunchConfig_t pcfg = {};
      pcfg.gridDim = dim3(2 * std::min(ptiles, pairs_fit), 1, 1);
      pcfg.blockDim = dim3(kPThreads, 1, 1);
      pcfg.dynamicSmemBytes = pc.smem;
      pcfg.stream = stream;
      cudaLaunchAttribute pattr[2];
      pattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      pattr[0].val.programmaticStreamSerializationAllowed = 1;
      pattr[1].id = cudaLaunchAttributeClusterDimension;
      pattr[1].val.clusterDim.x = 2;
      pattr[1].val.clusterDim.y = 1;
      pattr[1].val.clusterDim.z = 1;
      pcfg.attrs = pattr;
      pcfg.numAttrs = 2;
      SVDQ_CUDA_TRY(cudaLaunchKernelEx(&pcfg, pc.pfn, map_xq, *a.map_wq_128, map_t, map_l2_p, map_y, *a.map_wsf, pp));
      return SVDQ_OK;
    }
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ksplit > 1 ? tiles * p.ksplit : std::min(tiles, num_sms()), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.ksplit;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.ksplit > 1 ? 2 : 1;
  SVDQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, kc.fn, map_xq, *a.map_wq_256, map_t, map_l2, map_y, p));
  return SVDQ_OK;
}

}  // namespace svdq
