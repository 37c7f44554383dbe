/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 + low-rank linear layer.
 *
 * The layer (SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit
 * Diffusion Models; paperlayer.ai summary of arXiv 2411.05007v4, §4.2 and §4.3):
 *
 *   Y = Q4(X diag(lam)^-1) Q4(R)^T * alpha_w  +  (X diag(lam)^-1 L1) L2  +  b
 *
 * X is M x K (tokens x in-features), W is N x K (out x in, the PyTorch
 * Linear.weight layout), b is N.  A 16-bit rank-r branch L1 (K x r), L2 (r x N)
 * from the SVD of the smoothed weight W_hat = W diag(lam) takes the outliers,
 * and the residual R = W_hat - (L1 L2)^T is quantized to NVFP4: E2M1 codes
 * with one E4M3 scale per 16 consecutive elements along K (App. D).  The
 * runtime is two kernels (§4.3, Fig. 6): the activation kernel quantizes X and
 * computes the down-projection from the same read of X; the GEMM kernel folds
 * the up-projection into its 4-bit accumulator.
 *
 * Conventions for every call:
 *  - Element types: bf16 values are passed as their uint16 bit patterns;
 *    fp32 as float.  All matrices are row-major with the last index
 *    contiguous.
 *  - "host" pointers are ordinary CPU memory (pinned memory makes the copies
 *    of svdq_forward_host asynchronous); "device" pointers are global memory of
 *    the current CUDA device and must be 16-byte aligned.
 *  - Ownership: the caller owns every buffer it passes and keeps device
 *    buffers alive until the work queued on the stream has finished.  The
 *    library owns the svdq_weights handle and the device memory inside it;
 *    svdq_weights_destroy frees both.
 *  - CUDA graphs: the runtime calls (both kernels and svdq_forward) can be
 *    captured into a graph once the same call has run eagerly on the device,
 *    since a first call sets up per-device state (error word, kernel
 *    attributes, occupancy queries).
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *    default stream).  Runtime calls only enqueue work; they do not
 *    synchronize.  Weight preparation and LoRA attachment synchronize.
 *  - Errors: every call validates its arguments on the host before touching
 *    the GPU and returns a status; svdq_last_error() gives a message for the
 *    last failure on the calling thread.  Device-side failures (a wait that ran
 *    past its time limit) are recorded in a device error word that
 *    svdq_check_device_errors() reads.
 *  - Shape limits: K % 64 == 0; N % 16 == 0; 1 <= M; rank + LoRA ranks <= 128.
 *    The device must be sm_100 (B200).
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct svdq_weights svdq_weights; /* opaque, library-owned */

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* a null pointer, bad shape or misaligned pointer */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 2, /* the current device is not sm_100 */
  SVDQ_ERR_CUDA = 3,               /* a CUDA runtime/driver call failed */
  SVDQ_ERR_OOM = 4,                /* device or host allocation failed */
  SVDQ_ERR_TIMEOUT = 5,            /* a kernel wait passed its time limit */
  SVDQ_ERR_DEVICE_CHECK = 6        /* a kernel's own bounds/launch check failed */
} svdq_status;

/* 4-bit format of the residual and the activations. */
typedef enum {
  SVDQ_FORMAT_NVFP4 = 0, /* E2M1 codes, E4M3 scale per 16 (App. D, Blackwell); the default */
  SVDQ_FORMAT_INT4 = 1   /* signed INT4 codes (qmax 7, §3), bf16 scale per 64 (App. D "16-bit scales") */
} svdq_format;

/* Options of the offline weight transform. */
typedef struct {
  float alpha;        /* smoothing migration strength (App. D); default 0.5 */
  int rank;           /* low-rank branch rank r (§4.2: 16 or 32); default 32 */
  int power_iters;    /* subspace iterations of the randomized SVD; default 4 */
  int oversample;     /* extra columns of the random subspace; default 16 */
  uint64_t seed;      /* seed of the random starting subspace; default 0 */
  int keep_residual;  /* nonzero: keep a host copy of R/alpha_w for export */
  int refine_iters;   /* splits tried (§4.2 refinement, see svdq_prepare_weights); default 1 */
  int format;         /* svdq_format; default SVDQ_FORMAT_NVFP4 */
} svdq_prepare_opts;

/* Fills *opts with the defaults above. */
void svdq_prepare_opts_default(svdq_prepare_opts* opts);

/*
 * Offline weight transform (§4.2 and App. D): smoothing factors
 * lam_j = act_absmax_j^alpha / max_n |W_nj|^(1-alpha) (lam_j = 1 when either
 * maximum is 0), W_hat = W diag(1/fp32(1/lam)), a top-r SVD of W_hat by
 * randomized subspace iteration on the host, 16-bit factors
 * L1' = bf16(diag(inv_lam) L1) and L2 = bf16(V_r^T), the residual
 * R = W_hat - (diag(1/inv_lam) L1' L2)^T, the power-of-two factor
 * alpha_w = 2^ceil(log2(max|R| / 2688)), and the NVFP4 codes of R/alpha_w
 * (computed on the device).
 * With opts->refine_iters = t > 1 the split is refined (§4.2: the
 * decomposition can be refined over several iterations; the update is a
 * reading): with Q(R) = alpha_w times the NVFP4 round trip of R/alpha_w,
 * L_{i+1} = SVD_r(W_hat - Q(W_hat - L_i)) for i < t, and the split whose
 * residual quantization error ||R - Q(R)||_F is smallest is kept
 * (svdq_weights_refine_errors reports the errors).
 * With opts->format = SVDQ_FORMAT_INT4 the residual is coded in INT4 instead
 * (groups of 64 along K, s = bf16(fp32(amax / 7)),
 * q = clamp(rint(fp32(r_i * fp32(1/s))), -7, 7), round half to even, on the
 * host; alpha_w = 1); refinement is NVFP4-only (refine_iters must be 1).
 *   W_bf16      host, N x K bf16 (out x in)
 *   act_absmax  host, K floats: per-input-channel max |x| over calibration data
 *   bias_bf16   host, N bf16, or NULL for no bias
 *   opts        NULL for the defaults
 *   out         receives the new handle (NULL on failure)
 * Synchronizes `stream`.
 */
svdq_status svdq_prepare_weights(const uint16_t* W_bf16, const float* act_absmax,
                                 const uint16_t* bias_bf16, int N, int K,
                                 const svdq_prepare_opts* opts, void* stream,
                                 svdq_weights** out);

/*
 * Per-layer choice of the smoothing strength (App. D: alpha sets how much of
 * the activation range migrates into the weights; 0.5 by default).  For each
 * of the n_alpha candidates in `alphas` (each in [0, 1]) the layer is prepared
 * as svdq_prepare_weights does with opts->alpha = alphas[i] and the per-channel
 * maxima of the calibration batch, both kernels run on the batch, and
 * rel_err[i] = ||Y_i - (X W^T + b)||_F / ||X W^T + b||_F with the reference
 * accumulated in fp32 on the device.  *best is the index of the smallest
 * error.  Synchronous; allocates and frees its own device buffers.
 *   W_bf16     host, N x K bf16
 *   X_bf16     host, M x K bf16 calibration activations
 *   bias_bf16  host, N bf16, or NULL
 *   opts       NULL for the defaults (its alpha is ignored)
 *   rel_err    host, n_alpha doubles (out);  best  host int (out)
 */
svdq_status svdq_search_alpha(const uint16_t* W_bf16, const uint16_t* X_bf16, int M, const uint16_t* bias_bf16,
                              int N, int K, const float* alphas, int n_alpha, const svdq_prepare_opts* opts,
                              void* stream, double* rel_err, int* best);

/*
 * The residual quantization error ||R - Q(R)||_F (Frobenius, float64, in the
 * smoothed-weight space) of each split svdq_prepare_weights tried, in order:
 * one value without refinement, refine_iters values with it (the kept split
 * has the smallest); 0 values for handles made by svdq_weights_from_factors.
 * Writes min(count, max_count) values to `errors` (host) and the count to *count.
 */
svdq_status svdq_weights_refine_errors(const svdq_weights* w, double* errors, int max_count, int* count);

/*
 * Builds a handle from a given split (the second half of
 * svdq_prepare_weights): alpha_w is chosen from R as above and R/alpha_w is
 * quantized on the device.  This lets a caller supply factors computed
 * elsewhere (for instance an exact SVD).
 *   inv_lam   host, K floats (the runtime activation multipliers 1/lam)
 *   L1p_bf16  host, K x rank bf16 (L1' = diag(inv_lam) L1), or NULL if rank == 0
 *   L2_bf16   host, rank x N bf16, or NULL if rank == 0
 *   R         host, N x K floats: the residual (not yet divided by alpha_w)
 *   bias      host, N floats, or NULL
 * Synchronizes `stream`.
 */
svdq_status svdq_weights_from_factors(int N, int K, int rank, const float* inv_lam,
                                      const uint16_t* L1p_bf16, const uint16_t* L2_bf16,
                                      const float* R, const float* bias, void* stream,
                                      svdq_weights** out);

/* svdq_weights_from_factors with the residual's format chosen (svdq_format;
 * SVDQ_FORMAT_INT4 codes R as svdq_prepare_weights describes). */
svdq_status svdq_weights_from_factors_fmt(int N, int K, int rank, const float* inv_lam,
                                          const uint16_t* L1p_bf16, const uint16_t* L2_bf16,
                                          const float* R, const float* bias, int format, void* stream,
                                          svdq_weights** out);

/* The handle's svdq_format. */
svdq_status svdq_weights_format(const svdq_weights* w, int* format);

/*
 * LoRA without re-quantization (§2; §5.2 and Fig. 9: the low-rank branch
 * absorbs the LoRA by growing its rank).  Appends A as new columns of L1'
 * (A acts on the unsmoothed X, so it is not scaled by inv_lam) and
 * bf16(scale * B) as new rows of L2.  The 4-bit codes, scales and alpha_w are
 * not touched.
 *   A_bf16  host, K x r_l bf16 (LoRA down)
 *   B_bf16  host, r_l x N bf16 (LoRA up)
 * Synchronizes `stream`.
 */
svdq_status svdq_attach_lora(svdq_weights* w, const uint16_t* A_bf16, const uint16_t* B_bf16,
                             int r_l, float scale, void* stream);

/*
 * Kernel 1, activation side (§4.3: the down-projection is fused into the
 * quantization kernel so X is read once).  For each row m and group of 16
 * along K: x_hat = fp32(x * inv_lam_j); amax = max|x_hat|;
 * s = E4M3_rne_satfinite(fp32(amax/6)); codes = E2M1_rne_satfinite(
 * fp32(x_hat * fp32(1/s))) (all +0 when s decodes to 0; a code that rounds to
 * magnitude 0 is stored as +0).  In the same pass T = X L1' (fp32 on the
 * tensor cores) is written as an unevaluated bf16 pair T = T_hi + T_lo.
 *   X_bf16  device, M x K bf16
 *   xq      device, M x K/2 bytes: two codes per byte, element 2i in the low nibble
 *   xsf     device, svdq_act_sf_bytes(M, K) bytes: E4M3 scales in the Blackwell
 *           block-scale layout (128-row x 4-column atoms of 512 bytes, K-atoms
 *           fastest; inside an atom row m, column j is byte
 *           (m%32)*16 + (m/32)*4 + j; padded rows get scale 0)
 *   T       device, svdq_lowrank_bytes(w, M) bytes: M rows of 2*r_pad bf16 where,
 *           for each 16-wide chunk c of the rank, columns [32c, 32c+16) hold T_hi
 *           and [32c+16, 32c+32) hold T_lo.  May be NULL when the rank is 0.
 */
svdq_status svdq_quantize_act_lowrank_down(const svdq_weights* w, const void* X_bf16, int M,
                                           void* xq, void* xsf, void* T, void* stream);

/*
 * For an INT4 handle the same call writes INT4 codes (two's-complement
 * nibbles; per 8 elements one little-endian 32-bit word holding elements
 * 0, 2, 4, 6 in nibbles 0-3 and 1, 3, 5, 7 in nibbles 4-7) into xq and bf16 scales,
 * group-major [K/64][round_up(M, 128)] with zeros for the padding rows, into
 * xsf; the buffer sizes above cover both formats.
 */

/*
 * Kernel 2, the 4-bit GEMM with the up-projection folded in (§4.3):
 * Y = bf16_rne(alpha_w * (sum_k deq(xq) deq(wq) + (T_hi + T_lo) (L2 / alpha_w)) + b),
 * accumulated in fp32 in tensor memory.
 *   xq, xsf, T  as written by svdq_quantize_act_lowrank_down for the same M
 *   Y_bf16      device, M x N bf16
 * When the 128 x 256 output tiles would leave most SMs idle (small M), K is
 * split over a cluster of up to 8 CTAs per tile and the fp32 partials are
 * summed in a fixed order through distributed shared memory; the result is
 * then deterministic but its rounding differs from the unsplit sum within
 * fp32 accumulation error.  With many tiles and K > 3840 the tiles are
 * 256 x 256 over clusters of two CTAs (one M = 256 MMA per K block, issued
 * by one CTA of the pair); every output element is the same sum in the same
 * order, so Y is bitwise the one-CTA result.  The launch is a programmatic
 * dependent of the kernel ahead of it in the stream: it reads xq, xsf and T
 * only once that kernel has completed.
 * For an INT4 handle the codes and scales are expanded on chip into fp16 tiles
 * (q * s with a bf16 s is exact in fp16 while |q s| stays in fp16's range)
 * and contracted by fp16 tensor-core MMAs:
 * Y = bf16_rne(sum_g s_x s_w sum_k q_x q_w + (T_hi + T_lo) L2 + b); no split-K.
 */
svdq_status svdq_linear_w4a4(const svdq_weights* w, const void* xq, const void* xsf,
                             const void* T, int M, void* Y_bf16, void* stream);

/*
 * The activation kernel fused with the adaLN front end of a DiT block
 * (SVDQuant §4.3 fuses the down-projection into the quantization kernel; this
 * extends the fusion to the norm ahead of the layer): per token
 * x_j = bf16(fp32(fp32(fp32(z_j - mu) * rstd) * a_j) + c_j), then exactly what
 * svdq_quantize_act_lowrank_down does with X = x.  The pre-norm activations are
 * read in place of X (the layer never stores X).
 *   Z_bf16   device, M x K bf16 pre-norm activations
 *   stats    device, M x 2 floats (mu, rstd) from svdq_act_row_stats
 *   norm_a   device, K floats (1 + scale);  norm_c  device, K floats (shift)
 *   xq, xsf, T as for svdq_quantize_act_lowrank_down
 */
svdq_status svdq_norm_quantize_act_lowrank_down(const svdq_weights* w, const void* Z_bf16, int M,
                                                const float* stats, const float* norm_a,
                                                const float* norm_c, void* xq, void* xsf, void* T,
                                                void* stream);

/*
 * LayerNorm statistics per token: mu = mean_j z_j and
 * rstd = 1 / sqrt(mean_j (z_j - mu)^2 + eps), in one read of the row: fp32 sums
 * of d = z - z0 and d^2 (z0 = the row's first value, so the one-pass variance
 * E[d^2] - E[d]^2 does not cancel for a mean far from zero), IEEE square root
 * and reciprocal.
 *   Z_bf16  device, M x K bf16;  stats  device, M x 2 floats (out)
 * SVDQ_ERR_INVALID_ARG for bad sizes, eps < 0 or misaligned pointers.
 */
svdq_status svdq_act_row_stats(const void* Z_bf16, int M, int K, float eps, float* stats, void* stream);

/*
 * The layer with the norm in front: row statistics, the fused activation
 * kernel and the GEMM.  `workspace` is device memory of at least
 * svdq_forward_norm_workspace_bytes(w, M) bytes.
 */
svdq_status svdq_forward_norm(const svdq_weights* w, const void* Z_bf16, int M, const float* norm_a,
                              const float* norm_c, float eps, void* Y_bf16, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Both kernels back to back.  `workspace` is device memory of at least
 * svdq_forward_workspace_bytes(w, M) bytes holding xq, xsf and T.
 */
svdq_status svdq_forward(const svdq_weights* w, const void* X_bf16, int M, void* Y_bf16,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * svdq_forward with host input and output: copies X (host, M x K bf16) into
 * the workspace, runs both kernels and copies Y (M x N bf16) back into Y_host.
 * `workspace` is device memory of at least svdq_forward_host_workspace_bytes(w, M)
 * bytes.  For M >= 1024 the rows are processed in up to four chunks of a
 * multiple of 128 rows: uploads and downloads run on two copy streams the
 * library keeps per device, the kernels on `stream`, so the copies of one
 * chunk overlap the kernels of its neighbours (X_host and Y_host should be
 * pinned for the copies to be asynchronous).  Nothing synchronizes: the work
 * is ordered after what `stream` already holds, and `stream` is ordered after
 * all of it.  Calls for one device are enqueued one at a time.
 */
svdq_status svdq_forward_host(const svdq_weights* w, const void* X_host, int M, void* Y_host,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * svdq_forward without a workspace, for callers that cannot call cudaMalloc:
 * code running inside a caching allocator's callbacks (an allocation there
 * re-enters the allocator or fails against its reserve), or a serving loop
 * whose device memory is fully reserved up front.  (The paper has no
 * counterpart; this is a deployment convenience of this library.)
 *
 * The intermediates (activation codes, scales, T) live in one static block of
 * device memory of 32 MiB per device; layers whose intermediates exceed it
 * (M*K/2 + ceil(M/128)*128*K/16 + 4*M*r_pad bytes, each rounded up to 256)
 * are rejected with SVDQ_ERR_INVALID_ARG before any GPU work.  The block is
 * part of the library's device code: the FIRST call on a device, with that
 * device current, looks up its device address, which makes CUDA load that
 * code and commit the 32 MiB on the device (kept until the process exits).
 * Make that first call before reserving the rest of the device's memory and
 * before any stream capture.  Later calls allocate nothing: no cudaMalloc,
 * cudaFree or allocating library routine.
 *
 * All calls on a device share the one block and leave their intermediates in
 * it; calls whose kernels overlap on the GPU (other streams, other threads)
 * race on it and must be serialized by the caller.  Nothing in the block needs
 * to start at zero.  A device-side wait that runs out is recorded in a static
 * error word of this path, which svdq_check_device_errors reads and clears
 * together with the library's other word; the outputs of that call are then
 * unspecified.
 *   X_bf16  device, M x K bf16          Y_bf16  device, M x N bf16
 */
svdq_status svdq_forward_noalloc(const svdq_weights* w, const void* X_bf16, int M, void* Y_bf16,
                                 void* stream);

/* Sizes in bytes. */
size_t svdq_act_codes_bytes(int M, int K);                 /* M * K / 2 */
size_t svdq_act_sf_bytes(int M, int K);                    /* ceil(M/128)*128 * K/16 */
size_t svdq_lowrank_bytes(const svdq_weights* w, int M);   /* M * 2 * r_pad * 2 */
size_t svdq_forward_workspace_bytes(const svdq_weights* w, int M);
size_t svdq_forward_host_workspace_bytes(const svdq_weights* w, int M);
size_t svdq_forward_norm_workspace_bytes(const svdq_weights* w, int M);
size_t svdq_weights_sf_bytes(const svdq_weights* w);       /* the handle's weight scales */

/* Rank of the handle's 16-bit branch (§4.2, rank r of L1 and L2, plus the
 * ranks of the LoRAs attached by svdq_attach_lora, §5.2); -1 for NULL. */
int svdq_weights_rank(const svdq_weights* w);

/* Shape of a handle: rank counts the SVD rank plus attached LoRA ranks, r_pad
 * is that rounded up to a multiple of 16 (the width of T's hi and lo parts). */
svdq_status svdq_weights_info(const svdq_weights* w, int* N, int* K, int* rank, int* r_pad,
                              float* alpha_w);

/*
 * Copies the handle's contents to host memory (tests and inspection).  Any
 * output may be NULL to skip it.
 *   codes     N x K/2 bytes
 *   sf        svdq_weights_sf_bytes(w) bytes: NVFP4 atom layout, or INT4 bf16
 *             scales group-major [K/64][round_up(N, 256)]
 *   L1p_bf16  K x rank bf16        L2_bf16 rank x N bf16 (not divided by alpha_w)
 *   inv_lam   K floats             bias    N floats
 *   residual  N x K floats R/alpha_w; only if the handle kept it, else
 *             SVDQ_ERR_INVALID_ARG
 * Synchronizes the device.
 */
svdq_status svdq_weights_export(const svdq_weights* w, uint8_t* codes, uint8_t* sf,
                                uint16_t* L1p_bf16, uint16_t* L2_bf16, float* inv_lam,
                                float* bias, float* residual);

/* Frees the handle and its device memory (NULL is allowed). */
svdq_status svdq_weights_destroy(svdq_weights* w);

/*
 * Time limit, in nanoseconds, of every wait inside the kernels (default
 * 2e9).  When a wait passes it the kernel records SVDQ_ERR_TIMEOUT in the
 * device error word, skips its remaining work and exits cleanly.
 */
void svdq_set_wait_limit_ns(uint64_t ns);

/*
 * Synchronizes `stream`, then reads and clears the current device's error
 * words (the library's, and the allocation-free path's once that path has run
 * on the device): SVDQ_OK, SVDQ_ERR_TIMEOUT or SVDQ_ERR_DEVICE_CHECK.
 */
svdq_status svdq_check_device_errors(void* stream);

/*
 * Test hook for the bounded waits: launches the activation kernel with a
 * wait that nothing completes (its pipeline barrier expects one more arrival
 * than it gets), so that the wait runs out after svdq_set_wait_limit_ns and
 * the kernel exits with SVDQ_ERR_TIMEOUT in the device error word.  Buffers
 * as for svdq_quantize_act_lowrank_down.
 */
svdq_status svdq_debug_launch_stalled_act(const svdq_weights* w, const void* X_bf16, int M,
                                          void* xq, void* xsf, void* T, void* stream);

/*
 * Test hook: svdq_linear_w4a4 with the split-K factor fixed to `ksplit` CTAs
 * per output tile (1 = no split, one CTA per 128 x 256 tile and never the
 * CTA pair) instead of the automatic choice.  The split
 * is clamped to the number of 256-wide K tiles; a split whose clusters would
 * not all be resident at once falls back to 1.  INT4 handles have no split-K:
 * for them the call is svdq_linear_w4a4.  SVDQ_ERR_INVALID_ARG unless
 * 1 <= ksplit <= 8; otherwise as svdq_linear_w4a4.
 */
svdq_status svdq_debug_linear_w4a4_ksplit(const svdq_weights* w, const void* xq, const void* xsf,
                                          const void* T, int M, void* Y_bf16, int ksplit, void* stream);

/*
 * The layer as one kernel for a few tokens (NVFP4 handle, 1 <= M <= 16,
 * rank + LoRA ranks <= 64), kept beside the two-kernel path as a measured
 * alternative (on B200 it is no faster, so svdq_forward does not use it), with
 * its split of K
 * over a cluster fixed to `ksplit` CTAs per 128 output features (0 = the
 * automatic choice; a split whose clusters would not all be resident at once
 * is lowered).  Each CTA quantizes the activations of its K range itself (the
 * same NVFP4 codec as svdq_quantize_act_lowrank_down), computes its share of
 * T = X L1' and applies L2 to it, and the splits' fp32 partials of Y are
 * summed in split order.  SVDQ_ERR_INVALID_ARG for other shapes or ksplit
 * outside [0, 8].
 *   X_bf16  device, M x K bf16          Y_bf16  device, M x N bf16
 */
svdq_status svdq_debug_forward_small_m(const svdq_weights* w, const void* X_bf16, int M, void* Y_bf16,
                                       int ksplit, void* stream);

/*
 * Device self-test of the NVFP4 group encoder's exact shortcuts (both kernels
 * use them; SVDQuant App. D fixes the codec as IEEE fp32 division by qmax = 6
 * and reciprocal of the decoded E4M3 scale).  Compares, on the current device,
 * the fused division by 6 with IEEE division for every fp32 mantissa at
 * exponents -100..12, and the table reciprocal with the IEEE reciprocal for
 * every positive finite E4M3 byte.  Synchronous; writes the number of
 * mismatches (0 when the shortcuts are exact) to *mismatches.
 * SVDQ_ERR_INVALID_ARG for a null pointer, SVDQ_ERR_UNSUPPORTED_DEVICE off sm_100.
 */
svdq_status svdq_selftest_codec(unsigned int* mismatches);

/* Message for the last failed call on this thread ("" if none). */
const char* svdq_last_error(void);

/* Library version string. */
const char* svdq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
