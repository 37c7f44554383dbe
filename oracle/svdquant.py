"""SVDQuant W4A4 linear layer, step by step, in float64 on the CPU.

TEST INFRASTRUCTURE ONLY: part of the CPU oracle (see ``oracle/__init__.py``).

Source: SVDQuant (paperlayer.ai summary of arXiv 2411.05007v4).  The layer is

    Y = Q4(X diag(lam)^-1) Q4(R)^T * alpha_w  +  (X diag(lam)^-1 L1) L2  +  b

Steps and where they come from:
  1. Smoothing (§4.2; App. D "the smoothing factor is computed per channel
     using activation and weight maxima", following SmoothQuant):
     lam_j = max_m |X_mj|^alpha / max_n |W_nj|^(1-alpha), alpha = 0.5.
     Reading: lam_j = 1 when either maximum is 0.  lam is kept as fp32 and the
     runtime multiplies activations by inv_lam = fp32(1/lam) (correctly
     rounded); the smoothed weight is W_hat = W diag(1/inv_lam), so that
     X_hat W_hat^T equals X W^T for the inv_lam actually used.
  2. Low-rank split (§4.2: a 16-bit low-rank branch of rank 16 or 32 from the
     SVD of the smoothed weight, keeping the dominant singular values; App. D:
     rank 32 for 4-bit).  With W_hat^T = U S V^T (K x N), L1 = U_r S_r (K x r)
     and L2 = V_r^T (r x N).  Reading: S goes to L1.
     Stored 16-bit factors: L1' = bf16(diag(inv_lam) L1) (the smoothing
     divide folded in, so the branch runs on the raw X) and L2b = bf16(L2).
     Reading: the residual absorbs the rounding of the stored factors in the
     form they are used, R = W_hat - (diag(1/inv_lam) L1' L2b)^T (N x K),
     computed in float64 and stored as fp32.
  3. Per-tensor weight factor (not in the pages; a reading):
     alpha_w = 2^ceil(log2(max|R| / (6 * 448))) (1 when R = 0), R' = R/alpha_w
     (exact).  It keeps the weight block scales out of the E4M3 subnormals;
     a power of two adds no rounding.
  4. NVFP4 codec (see ``codec.py``) on R' rows and on X_hat = fp32(x * inv_lam).
  4b. Optional refinement (§4.2: the decomposition "can be refined over several
     iterations"; the pages give no formula).  Reading: with Q(R) the weight
     quantization as the runtime sees it (alpha_w times the dequantized codes of
     R/alpha_w, App. A.2's Q(R) = s_R Q_R), iterate
     L_{t+1} = SVD_r(W_hat - Q(W_hat - L_t)) starting from the plain split, and
     keep the split whose residual quantization error ||R - Q(R)||_F is
     smallest (R computed from the stored 16-bit factors as in step 2).
  5. Output in float64 with no intermediate rounding:
     Y = alpha_w deq(Qx) deq(Qw)^T + (X L1') L2b + b.
  6. LoRA (§2 and §5.2 Fig. 9: off-the-shelf LoRAs are absorbed into the
     low-rank branch "by slightly increasing its rank", without re-quantizing
     R): L1' <- [L1' | A], L2b <- [L2b ; scale B].  Reading: the LoRA acts on
     the unsmoothed X, so A enters unscaled.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

from .codec import dequantize_groups, quantize_groups
from .formats import round_bf16

FP4_QMAX = 6.0
E4M3_MAX = 448.0


def smoothing_factors(act_absmax, W, alpha: float = 0.5):
    """(lam fp32 [K], inv_lam fp32 [K]) from activation and weight channel maxima."""
    ax = np.asarray(act_absmax, dtype=np.float64)
    wx = np.abs(np.asarray(W, dtype=np.float64)).max(axis=0)
    ok = (ax > 0) & (wx > 0)
    lam = np.ones_like(ax)
    lam[ok] = ax[ok] ** alpha / wx[ok] ** (1.0 - alpha)
    lam32 = lam.astype(np.float32)
    inv32 = (1.0 / lam32.astype(np.float64)).astype(np.float32)
    return lam32, inv32


def smooth_weight(W, inv_lam) -> np.ndarray:
    """W_hat = W diag(1/inv_lam) in float64 (N x K)."""
    return np.asarray(W, np.float64) / np.asarray(inv_lam, np.float64)[None, :]


def svd_split(W_hat, r: int):
    """Top-r factors of W_hat^T: L1 = U_r S_r (K x r), L2 = V_r^T (r x N), and
    the full singular values."""
    W_hat = np.asarray(W_hat, np.float64)
    N, K = W_hat.shape
    u, s, vt = np.linalg.svd(W_hat, full_matrices=False)   # W_hat = u diag(s) vt
    L1 = vt[:r].T * s[:r][None, :]                          # K x r
    L2 = u[:, :r].T.copy()                                  # r x N
    return L1, L2, s


def weight_factor(R) -> float:
    """alpha_w = 2^ceil(log2(max|R| / (6*448))), or 1 for R == 0."""
    m = float(np.abs(np.asarray(R, np.float64)).max(initial=0.0))
    if m == 0.0:
        return 1.0
    frac, e = np.frexp(m / (FP4_QMAX * E4M3_MAX))            # m' = frac * 2^e, frac in [0.5, 1)
    ceil_log2 = int(e) - 1 if frac == 0.5 else int(e)
    return float(np.ldexp(1.0, ceil_log2))


@dataclasses.dataclass
class Prepared:
    """Everything the oracle's runtime step needs for one layer."""

    N: int
    K: int
    rank: int
    lam: np.ndarray          # fp32 [K]
    inv_lam: np.ndarray      # fp32 [K]
    L1p: np.ndarray          # float64 values of bf16 L1' [K, r_tot]
    L2b: np.ndarray          # float64 values of bf16 L2  [r_tot, N]
    R: np.ndarray            # fp32 residual [N, K]
    alpha_w: float
    Rp: np.ndarray           # fp32 R / alpha_w [N, K]
    w_codes: np.ndarray      # uint8 [N, K] one code per element
    w_scales: np.ndarray     # uint8 [N, K/16]
    bias: np.ndarray         # float64 [N]
    sigma: Optional[np.ndarray] = None       # singular values of W_hat
    refine_errors: Optional[list] = None     # ||R - Q(R)||_F of each split tried (step 4b)
    lora_B_exact: Optional[np.ndarray] = None  # float64 scale*B rows appended to L2b
    lora_rank: int = 0


def prepare_from_factors(W_hat, inv_lam, L1p, L2b, bias, lam=None, sigma=None) -> Prepared:
    """Residual, weight factor and weight codes from given 16-bit factors."""
    W_hat = np.asarray(W_hat, np.float64)
    N, K = W_hat.shape
    inv64 = np.asarray(inv_lam, np.float32).astype(np.float64)
    L1p = np.asarray(L1p, np.float64).reshape(K, -1)
    L2b = np.asarray(L2b, np.float64).reshape(-1, N)
    low = (L1p / inv64[:, None]) @ L2b                    # K x N, in W_hat space
    R = (W_hat - low.T).astype(np.float32)
    aw = weight_factor(R)
    Rp = (R.astype(np.float64) / aw).astype(np.float32)  # exact: power of two
    codes, scales = quantize_groups(Rp)
    b = np.zeros(N) if bias is None else np.asarray(bias, np.float64)
    lam = (1.0 / inv64).astype(np.float32) if lam is None else lam
    return Prepared(N, K, L1p.shape[1], np.asarray(lam, np.float32), np.asarray(inv_lam, np.float32),
                    L1p, L2b, R, aw, Rp, codes, scales, b, sigma)


def fake_quantize_weights(R) -> np.ndarray:
    """Q(R) = alpha_w * dequantized NVFP4 codes of R / alpha_w, float64 (step 4b)."""
    R = np.asarray(R, np.float32)
    aw = weight_factor(R)
    codes, scales = quantize_groups((R.astype(np.float64) / aw).astype(np.float32))
    return dequantize_groups(codes, scales) * aw


def prepare(W, act_absmax, bias, rank: int, alpha: float = 0.5, iters: int = 1) -> Prepared:
    """Smoothing, SVD split, residual quantization (steps 1-4 for the weights);
    ``iters`` > 1 refines the split (step 4b) and keeps the best of ``iters``."""
    lam, inv_lam = smoothing_factors(act_absmax, W, alpha)
    W_hat = smooth_weight(W, inv_lam)
    inv64 = inv_lam.astype(np.float64)[:, None]
    A = W_hat
    best, errors = None, []
    for _ in range(max(1, iters)):
        L1, L2, s = svd_split(A, rank)
        prep = prepare_from_factors(W_hat, inv_lam, round_bf16(L1 * inv64), round_bf16(L2), bias, lam=lam,
                                    sigma=s if best is None else best.sigma)
        Q = fake_quantize_weights(prep.R)
        errors.append(float(np.linalg.norm(prep.R.astype(np.float64) - Q)))
        if best is None or errors[-1] < min(errors[:-1]):
            best = prep
        A = W_hat - Q
    best.refine_errors = errors
    return best


def search_alpha(W, X, bias, rank: int, alphas, iters: int = 1):
    """Per-layer smoothing strength (App. D: alpha is the migration strength of
    the smoothing; choosing it per layer this way is a reading): for each candidate, prepare
    with the calibration batch's per-channel maxima and score the layer output
    by ||Y - (X W^T + b)||_F / ||X W^T + b||_F in float64.  Returns (errors,
    index of the smallest)."""
    X = np.asarray(X, np.float32)
    exact = X.astype(np.float64) @ np.asarray(W, np.float64).T
    if bias is not None:
        exact = exact + np.asarray(bias, np.float64)[None, :]
    absmax = np.abs(X).max(axis=0)
    errs = []
    for a in alphas:
        prep = prepare(W, absmax, bias, rank, alpha=float(a), iters=iters)
        errs.append(float(np.linalg.norm(linear(prep, X) - exact) / np.linalg.norm(exact)))
    return errs, int(np.argmin(errs))


def smooth_activations(X, inv_lam) -> np.ndarray:
    """X_hat = fp32(x * inv_lam) elementwise (one fp32 rounding)."""
    return (np.asarray(X, np.float32) * np.asarray(inv_lam, np.float32)[None, :]).astype(np.float32)


def quantize_activations(X, inv_lam):
    """(codes [M, K], scales [M, K/16]) of the smoothed activations."""
    return quantize_groups(smooth_activations(X, inv_lam))


def lowrank_down(X, prep: Prepared) -> np.ndarray:
    """T = X L1' in float64 (M x r_tot)."""
    return np.asarray(X, np.float64) @ prep.L1p


def linear(prep: Prepared, X, rows=None, cols=None) -> np.ndarray:
    """Y in float64 for all rows of X, or for the listed row indices and/or
    output columns (the same arithmetic restricted to those outputs)."""
    X = np.asarray(X, np.float32)
    if rows is not None:
        X = X[np.asarray(rows)]
    c = slice(None) if cols is None else np.asarray(cols)
    xc, xs = quantize_activations(X, prep.inv_lam)
    main = dequantize_groups(xc, xs) @ dequantize_groups(prep.w_codes[c], prep.w_scales[c]).T
    L2 = prep.L2b if prep.lora_B_exact is None else prep.lora_B_exact
    return prep.alpha_w * main + lowrank_down(X, prep) @ L2[:, c] + prep.bias[None, c]


def attach_lora(prep: Prepared, A, B, scale: float = 1.0) -> Prepared:
    """Concatenate a LoRA (A: K x r_l on raw X, B: r_l x N) onto the branch.

    The stored 16-bit up-factor gets bf16(scale * B); the exact reference keeps
    scale * B in float64.  Codes, scales and alpha_w are untouched."""
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    L1p = np.concatenate([prep.L1p, A], axis=1)
    L2b = np.concatenate([prep.L2b, round_bf16(scale * B)], axis=0)
    exact = np.concatenate([prep.L2b if prep.lora_B_exact is None else prep.lora_B_exact,
                            scale * B], axis=0)
    return dataclasses.replace(prep, L1p=L1p, L2b=L2b, rank=L1p.shape[1], lora_B_exact=exact,
                               lora_rank=prep.lora_rank + A.shape[1])


def prop41_bound(X, W, QX, QW) -> float:
    """Right side of Prop. 4.1 (App. A.1): ||X|| ||W-Q(W)|| + ||X-Q(X)|| (||W|| + ||W-Q(W)||)."""
    f = np.linalg.norm
    dW = f(W - QW)
    return f(X) * dW + f(X - QX) * (f(W) + dW)
