"""INT4 variant of the layer: group-64 integer codec with 16-bit scales.

TEST INFRASTRUCTURE ONLY: part of the CPU oracle (see ``oracle/__init__.py``).

Source: SVDQuant (paperlayer.ai summary of arXiv 2411.05007v4).  App. D
(Implementation details): the 4-bit setting quantizes activations and weights
per group, symmetric, with group size 64 and 16-bit scales for INT4; §3
(Quantization Preliminary): signed k-bit integers have qmax = 2^(k-1) - 1 = 7,
and dequantization multiplies the low-bit tensor by its scaling factor.

For each group of 64 consecutive values v along K:

  amax = max |v|                                   (fp32, exact)
  s    = bf16_rne(fp32(amax / 7))
  if s == 0: every code is 0
  else: r = fp32(1 / s);  q = clamp(round_half_even(fp32(v * r)), -7, 7)
  dequantized value: q * s

Readings of steps the pages leave open: the 16-bit scale format is bfloat16;
the scale is rounded from the IEEE fp32 quotient; codes come from
reciprocal-then-multiply like the NVFP4 codec; the clamp is symmetric (+-qmax)
and never binds, since rounding s to bf16 moves v/s by at most 2^-9 relative;
the layer has no per-tensor weight factor (bf16 scales span fp32's exponent
range).  Everything else -- smoothing, the low-rank split, the residual, LoRA
-- is the NVFP4 layer's (``svdquant.py``).

Storage (not fixed by the pages; chosen so that the GEMM unpacks pairs of
consecutive elements without byte permutes): codes are two's-complement
nibbles; each run of 8 elements is a little-endian 32-bit word whose nibbles
0-3 hold the even elements (0, 2, 4, 6) and nibbles 4-7 the odd ones
(1, 3, 5, 7).  Scales are bf16 bit patterns, stored group-major ([K/64, rows]).
"""

from __future__ import annotations

import dataclasses

import numpy as np

from . import svdquant as S
from .formats import bf16_bits_to_f64, round_bf16

GROUP = 64
QMAX = 7


def quantize_groups(v) -> tuple:
    """Quantize float32 rows [R, K] (K % 64 == 0) group-wise along K.

    Returns (codes int8 [R, K] in -7..7, scales float64 [R, K/64] holding the
    bf16 scale values)."""
    v = np.asarray(v, dtype=np.float32)
    R, K = v.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 64")
    if not np.all(np.isfinite(v)):
        raise ValueError("non-finite input to the codec")
    g = v.reshape(R, K // GROUP, GROUP)
    amax = np.abs(g).max(axis=-1)                                     # exact
    s = round_bf16((amax / np.float32(QMAX)).astype(np.float32))      # fp32 div, then RNE to bf16
    s32 = s.astype(np.float32)                                        # exact (bf16 fits fp32)
    nz = s32 > 0
    r = np.where(nz, np.float32(1.0) / np.where(nz, s32, np.float32(1.0)), np.float32(0.0)).astype(np.float32)
    t = (g * r[..., None]).astype(np.float32)                         # fp32 multiply
    q = np.clip(np.rint(t), -QMAX, QMAX).astype(np.int8)              # rint: half to even
    return q.reshape(R, K), s


def dequantize_groups(codes, scales) -> np.ndarray:
    """q * s in float64, [R, K]."""
    codes = np.asarray(codes, np.int64)
    R, K = codes.shape
    s = np.asarray(scales, np.float64)
    return (codes.reshape(R, K // GROUP, GROUP) * s[..., None]).reshape(R, K)


def pack_codes(codes) -> np.ndarray:
    """uint8 [R, K/2]: per 8 elements a little-endian word with the even
    elements in nibbles 0-3 and the odd ones in nibbles 4-7."""
    c = np.asarray(codes, np.int64) & 0xF
    R, K = c.shape
    c = c.reshape(R, K // 8, 8)
    word = np.zeros((R, K // 8), np.uint64)
    for k in range(4):
        word |= (c[..., 2 * k].astype(np.uint64) << np.uint64(4 * k)) | \
                (c[..., 2 * k + 1].astype(np.uint64) << np.uint64(16 + 4 * k))
    return word.astype("<u4").view(np.uint8).reshape(R, K // 2)


def unpack_codes(packed) -> np.ndarray:
    """Inverse of pack_codes: int8 [R, K]."""
    p = np.ascontiguousarray(np.asarray(packed, np.uint8))
    R = p.shape[0]
    word = p.view("<u4").astype(np.int64)
    out = np.empty((R, word.shape[1], 8), np.int64)
    for k in range(4):
        out[..., 2 * k] = (word >> (4 * k)) & 0xF
        out[..., 2 * k + 1] = (word >> (16 + 4 * k)) & 0xF
    out = out.reshape(R, -1)
    return np.where(out >= 8, out - 16, out).astype(np.int8)


def scales_to_bits(scales) -> np.ndarray:
    """bf16 bit patterns of bf16-valued scales (exact)."""
    return np.asarray(scales, np.float32).view(np.uint32).__rshift__(16).astype(np.uint16)


def scales_from_bits(bits) -> np.ndarray:
    return bf16_bits_to_f64(np.asarray(bits, np.uint16))


@dataclasses.dataclass
class PreparedInt4:
    """The INT4 layer's weights: the NVFP4 layer's split with an INT4 residual."""

    base: S.Prepared         # smoothing, factors, residual R (its NVFP4 fields unused here)
    w_codes: np.ndarray      # int8 [N, K] in -7..7
    w_scales: np.ndarray     # float64 bf16 values [N, K/64]

    def __getattr__(self, name):          # N, K, rank, inv_lam, L1p, L2b, R, bias, ...
        if name == "base":
            raise AttributeError(name)
        return getattr(self.base, name)


def prepare(W, act_absmax, bias, rank: int, alpha: float = 0.5) -> PreparedInt4:
    """Smoothing and low-rank split as in the NVFP4 layer, then the INT4 codec
    on the residual R."""
    base = S.prepare(W, act_absmax, bias, rank, alpha=alpha)
    return from_base(base)


def from_base(base: S.Prepared) -> PreparedInt4:
    codes, scales = quantize_groups(base.R)
    return PreparedInt4(base, codes, scales)


def attach_lora(prep: PreparedInt4, A, B, scale: float = 1.0) -> PreparedInt4:
    return dataclasses.replace(prep, base=S.attach_lora(prep.base, A, B, scale))


def quantize_activations(X, inv_lam):
    """(codes, scales) of the smoothed activations X_hat = fp32(x * inv_lam)."""
    return quantize_groups(S.smooth_activations(X, inv_lam))


def linear(prep: PreparedInt4, X, rows=None, cols=None) -> np.ndarray:
    """Y = deq(Qx) deq(Qw)^T + (X L1') L2 + b in float64."""
    X = np.asarray(X, np.float32)
    if rows is not None:
        X = X[np.asarray(rows)]
    c = slice(None) if cols is None else np.asarray(cols)
    xc, xs = quantize_activations(X, prep.inv_lam)
    main = dequantize_groups(xc, xs) @ dequantize_groups(prep.w_codes[c], prep.w_scales[c]).T
    b = prep.base
    L2 = b.L2b if b.lora_B_exact is None else b.lora_B_exact
    return main + S.lowrank_down(X, b) @ L2[:, c] + b.bias[None, c]
