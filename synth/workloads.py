"""Seeded synthetic layer inputs with the shapes and value structure of the
SVDQuant evaluation models (FLUX.1, PixArt-Sigma, SDXL; SVDQuant paper,
App. B "Benchmark models").

No model weights or prompts are used: every tensor is drawn from a seeded
PCG64 generator, rounded to bf16 (the 16-bit format of the model weights and
activations) with PyTorch's own cast, and returned both as raw bf16 bit
patterns (uint16) and as the float32 values those bits encode.

Recipe, per layer (X is tokens x in-features, W is out x in):
  * X ~ N(0, 1); a random set of input channels ("outlier channels") is
    multiplied by a large factor.
  * W ~ N(0, 0.02); only the tiny layer also has outlier input columns.
  * bias ~ N(0, 0.01).
  * LoRA factors A (K x r_l) and B (r_l x N) ~ N(0, 0.01), scale 1.
  * act_absmax is the per-input-channel max |x| over the layer's own X, the
    calibration statistic the smoothing step consumes.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (PyTorch's cast) and return the bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Float32 values encoded by bf16 bit patterns (bf16 is the top half of fp32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class LayerCase:
    """One linear layer of a workload: Y[M,N] = X[M,K] W[N,K]^T + b."""

    config: str
    name: str
    M: int
    K: int
    N: int
    rank: int
    x_outlier_count: int
    x_outlier_scale: float
    w_outlier_count: int = 0
    w_outlier_scale: float = 1.0
    lora_rank: int = 0
    seed: int = 0
    alpha: float = 0.5

    @property
    def flops(self) -> int:
        """Dense 4-bit GEMM flops 2*M*N*K."""
        return 2 * self.M * self.N * self.K

    @property
    def label(self) -> str:
        return f"{self.config}/{self.name}"


@dataclasses.dataclass
class LayerInputs:
    case: LayerCase
    X_bits: np.ndarray        # uint16 [M, K]
    X: np.ndarray             # float32 [M, K]
    W_bits: np.ndarray        # uint16 [N, K]
    W: np.ndarray             # float32 [N, K]
    bias_bits: np.ndarray     # uint16 [N]
    bias: np.ndarray          # float32 [N]
    act_absmax: np.ndarray    # float32 [K]
    lora_A_bits: Optional[np.ndarray] = None  # uint16 [K, r_l]
    lora_A: Optional[np.ndarray] = None
    lora_B_bits: Optional[np.ndarray] = None  # uint16 [r_l, N]
    lora_B: Optional[np.ndarray] = None
    lora_scale: float = 1.0


def _outliers(frac: float, K: int) -> int:
    return int(round(frac * K))


def _build_configs() -> Dict[str, List[LayerCase]]:
    cfg: Dict[str, List[LayerCase]] = {}
    cfg["tiny"] = [LayerCase("tiny", "layer", 64, 256, 256, 16, 4, 40.0, 4, 20.0, seed=0)]

    pix = [("attn_qkv_out", 1152, 1152), ("mlp_up", 1152, 4608), ("mlp_down", 4608, 1152)]
    cfg["pixart"] = [
        LayerCase("pixart", n, 4096, k, nn, 32, _outliers(0.01, k), 30.0, seed=1100 + j)
        for j, (n, k, nn) in enumerate(pix)
    ]

    flux = [("attn_out", 3072, 3072), ("qkv", 3072, 9216), ("mlp_up", 3072, 12288),
            ("mlp_down", 12288, 3072)]
    cfg["flux"] = [
        LayerCase("flux", n, 4608, k, nn, 32, _outliers(0.005, k), 50.0, seed=1200 + j)
        for j, (n, k, nn) in enumerate(flux)
    ]

    sdxl = [("r64_attn", 8192, 640, 640), ("r64_ff_up", 8192, 640, 5120),
            ("r64_ff_down", 8192, 5120, 640), ("r32_attn", 2048, 1280, 1280),
            ("r32_ff_up", 2048, 1280, 10240), ("r32_ff_down", 2048, 10240, 1280)]
    cfg["sdxl"] = [
        LayerCase("sdxl", n, m, k, nn, 32, _outliers(0.01, k), 30.0, seed=1300 + j)
        for j, (n, m, k, nn) in enumerate(sdxl)
    ]

    small = []
    j = 0
    for m in (1, 16, 256):
        for nn in (3072, 12288):
            small.append(LayerCase("small_m_lora", f"M{m}_N{nn}", m, 3072, nn, 32,
                                   _outliers(0.005, 3072), 50.0, lora_rank=16, seed=1400 + j))
            j += 1
    cfg["small_m_lora"] = small
    return cfg


CONFIGS: Dict[str, List[LayerCase]] = _build_configs()


def config_cases(name: str) -> List[LayerCase]:
    return list(CONFIGS[name])


def make_layer_inputs(case: LayerCase, M: Optional[int] = None) -> LayerInputs:
    """Draw one layer's inputs.  ``M`` overrides the token count (the weights,
    outlier channels and the first rows of X do not depend on it)."""
    rng = np.random.Generator(np.random.PCG64(case.seed))
    K, N = case.K, case.N
    M_full = case.M
    M = M_full if M is None else M
    # Draw the weight side first so that it does not depend on M.
    W = rng.normal(0.0, 0.02, size=(N, K)).astype(np.float32)
    if case.w_outlier_count:
        cols = rng.choice(K, size=case.w_outlier_count, replace=False)
        W[:, cols] *= np.float32(case.w_outlier_scale)
    bias = rng.normal(0.0, 0.01, size=(N,)).astype(np.float32)
    xcols = rng.choice(K, size=case.x_outlier_count, replace=False) if case.x_outlier_count else []
    lA = lB = None
    if case.lora_rank:
        lA = rng.normal(0.0, 0.01, size=(K, case.lora_rank)).astype(np.float32)
        lB = rng.normal(0.0, 0.01, size=(case.lora_rank, N)).astype(np.float32)
    # Activations come from their own stream so that changing M keeps W fixed.
    xr = np.random.Generator(np.random.PCG64(case.seed + 7919))
    X = xr.normal(0.0, 1.0, size=(M, K)).astype(np.float32)
    if len(xcols):
        X[:, xcols] *= np.float32(case.x_outlier_scale)

    Xb, Wb, bb = f32_to_bf16_bits(X), f32_to_bf16_bits(W), f32_to_bf16_bits(bias)
    Xf = bf16_bits_to_f32(Xb)
    out = LayerInputs(case, Xb, Xf, Wb, bf16_bits_to_f32(Wb), bb, bf16_bits_to_f32(bb),
                      np.abs(Xf).max(axis=0).astype(np.float32))
    if lA is not None:
        Ab, Bb = f32_to_bf16_bits(lA), f32_to_bf16_bits(lB)
        out.lora_A_bits, out.lora_A = Ab, bf16_bits_to_f32(Ab)
        out.lora_B_bits, out.lora_B = Bb, bf16_bits_to_f32(Bb)
    return out


def make_lora_factors(K: int, N: int, r_l: int, seed: int):
    """A LoRA of rank ``r_l`` for a K -> N layer: A (K x r_l) and B (r_l x N)
    drawn N(0, 0.01) like the configured small-M LoRA, rounded to bf16.
    Returns (A_bits, A, B_bits, B)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    A = rng.normal(0.0, 0.01, size=(K, r_l)).astype(np.float32)
    B = rng.normal(0.0, 0.01, size=(r_l, N)).astype(np.float32)
    Ab, Bb = f32_to_bf16_bits(A), f32_to_bf16_bits(B)
    return Ab, bf16_bits_to_f32(Ab), Bb, bf16_bits_to_f32(Bb)


# Magnitudes a 4-bit E2M1 element can take (used only to build inputs that lie
# on the FP4 grid already).
_FP4_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


def make_fp4_grid_inputs(M: int, K: int, N: int, seed: int,
                         x_exp=(-1, 1), w_exp=(-3, -1)):
    """X [M,K] and W [N,K] whose every 16-element group along K is a set of
    FP4 grid values times a power-of-two group scale, with one element of each
    group at +-6 x scale, so that the group's 4-bit encoding is exact.

    Exponent ranges are small so that every partial sum of X W^T is exact in
    fp32.  Returns (X_bits, X, W_bits, W) with bf16 bit patterns."""
    rng = np.random.Generator(np.random.PCG64(seed))

    def draw(rows, exps):
        g = rng.choice(_FP4_GRID, size=(rows, K // 16, 16))
        g *= rng.choice(np.array([-1.0, 1.0], np.float32), size=g.shape)
        pos = rng.integers(0, 16, size=(rows, K // 16))
        sgn = rng.choice(np.array([-6.0, 6.0], np.float32), size=(rows, K // 16))
        np.put_along_axis(g, pos[..., None], sgn[..., None], axis=-1)
        e = rng.integers(exps[0], exps[1] + 1, size=(rows, K // 16, 1))
        v = (g * np.ldexp(np.float32(1.0), e).astype(np.float32)).reshape(rows, K)
        bits = f32_to_bf16_bits(v)
        return bits, bf16_bits_to_f32(bits)

    Xb, X = draw(M, x_exp)
    Wb, W = draw(N, w_exp)
    return Xb, X, Wb, W


def make_int4_grid_inputs(M: int, K: int, N: int, seed: int,
                          x_exp=(-2, 2), w_exp=(-9, -6), s_steps: int = 16):
    """X [M,K] and W [N,K] whose every 64-element group along K is a set of
    integers in -7..7 times a group scale s = 2^e (1 + j/s_steps), j <
    s_steps (a power of two <= 16), with one element of each group at +-7 s,
    so that amax / 7 = s exactly, s is a bf16 value and the group's INT4
    encoding is exact.  Every value (at most 3 + 5 significant bits) is a bf16
    value.  s_steps = 1 gives power-of-two scales.  Returns (X_bits, X, W_bits, W)."""
    rng = np.random.Generator(np.random.PCG64(seed))

    def draw(rows, exps):
        q = rng.integers(-7, 8, size=(rows, K // 64, 64)).astype(np.float32)
        pos = rng.integers(0, 64, size=(rows, K // 64))
        sgn = rng.choice(np.array([-7.0, 7.0], np.float32), size=(rows, K // 64))
        np.put_along_axis(q, pos[..., None], sgn[..., None], axis=-1)
        e = rng.integers(exps[0], exps[1] + 1, size=(rows, K // 64, 1))
        j = rng.integers(0, s_steps, size=(rows, K // 64, 1))
        s = (np.ldexp(np.float32(1.0), e) * (1.0 + j / float(s_steps))).astype(np.float32)
        v = (q * s).reshape(rows, K).astype(np.float32)
        bits = f32_to_bf16_bits(v)
        return bits, bf16_bits_to_f32(bits)

    Xb, X = draw(M, x_exp)
    Wb, W = draw(N, w_exp)
    return Xb, X, Wb, W
