"""LayerNorm in front of the layer, as the fused activation kernel applies it.

TEST INFRASTRUCTURE ONLY: part of the CPU oracle (see ``oracle/__init__.py``).

SVDQuant (paperlayer.ai summary of arXiv 2411.05007v4), §4.3: the down-projection
shares the activation read with the quantization kernel; the fused path here
carries that one step further, into the norm ahead of the layer.  In the DiT blocks of
the configured models the linear layers read LayerNorm(z) modulated per channel
(adaLN: (1 + scale) * LN(z) + shift), so the fused input is

  x_j = bf16( fp32( fp32( fp32(z_j - mu) * rstd ) * a_j ) + c_j )

per token, with mu = mean_j z_j, rstd = 1 / sqrt(mean_j (z_j - mu)^2 + eps) over
the K channels, a = 1 + scale and c = shift.  Readings: the per-element steps are
the IEEE fp32 operations written above (no fused multiply-add), and the result
is rounded to bf16, the activation format of the unfused pipeline (a norm
kernel writing bf16 X followed by the activation kernel), so the fused layer
equals that pipeline.  The statistics themselves are a reduction whose rounding
depends on the summation order: ``row_stats`` gives them in float64, and
``normalize`` takes mu and rstd as inputs so that a caller can reproduce the
codes of a kernel from the kernel's own statistics.
"""

from __future__ import annotations

import numpy as np

from .formats import round_bf16


def row_stats(Z, eps: float):
    """(mu, rstd) per row in float64."""
    Z = np.asarray(Z, np.float64)
    mu = Z.mean(axis=1)
    var = ((Z - mu[:, None]) ** 2).mean(axis=1)
    return mu, 1.0 / np.sqrt(var + eps)


def normalize(Z, mu, rstd, a, c) -> np.ndarray:
    """x = bf16(((z - mu) * rstd) * a + c) with fp32 steps, float32 values [M, K]."""
    Z = np.asarray(Z, np.float32)
    mu = np.asarray(mu, np.float32)[:, None]
    rstd = np.asarray(rstd, np.float32)[:, None]
    d = (Z - mu).astype(np.float32)
    n = (d * rstd).astype(np.float32)
    x = ((n * np.asarray(a, np.float32)[None, :]).astype(np.float32) + np.asarray(c, np.float32)[None, :])
    return round_bf16(x.astype(np.float32)).astype(np.float32)
