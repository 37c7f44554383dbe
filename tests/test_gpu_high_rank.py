"""GPU parity at branch widths above the default rank 32, through the C ABI.

SVDQuant App. E.5 (Fig. 18) trades rank 16 to 64 against latency, and §5.2
(Fig. 9) grows the branch by the rank of each attached LoRA; the library takes
rank + LoRA ranks up to 128.  A wider branch changes both kernels: the
activation kernel's down-projection MMA width, its tensor-memory columns and
its L1' tiles, the T buffer (2 r_pad columns of hi/lo pairs) and the number of
low-rank steps the GEMM folds into its accumulator.  Each case is compared with
the oracle: activation codes and scales bit-exact, T within the fp32
accumulation bound, Y within the layer tolerance.

r_pad covered: 64 (rank 64), 80 (rank 48 + LoRA 32), 112 (rank 96 + LoRA 16)
and 128 (rank 64 + LoRA 64), on the FLUX.1 attn_out (K = 3072) and mlp_down
(K = 12288) shapes and the mlp_up shape the benchmark's rank sweep times."""

import functools

import numpy as np
import pytest

from oracle import formats as OF
from oracle import int4 as OI
from oracle import svdquant as OS
from synth import config_cases, f32_to_bf16_bits, make_layer_inputs, make_lora_factors
from tests import gpu_common as G

pytestmark = pytest.mark.gpu

MAX_RANK = 128


@functools.lru_cache(maxsize=None)
def _svd(name: str):
    """The oracle's exact SVD of a FLUX layer's smoothed weight, kept to rank
    128 so that every rank below reuses the same decomposition (prepare() at
    rank r takes exactly the first r singular pairs).  The smoothing maxima
    come from the full-size activations, as for the benchmark's layer."""
    case = [c for c in config_cases("flux") if c.name == name][0]
    t = make_layer_inputs(case)
    lam, inv_lam = OS.smoothing_factors(t.act_absmax, t.W)
    W_hat = OS.smooth_weight(t.W, inv_lam)
    L1, L2, s = OS.svd_split(W_hat, MAX_RANK)
    return lam, inv_lam, W_hat, L1, L2, s


@functools.lru_cache(maxsize=None)
def _split(name: str, M: int):
    """Inputs of a FLUX layer at M tokens (weights and leading rows do not
    depend on M) and the shared decomposition."""
    case = [c for c in config_cases("flux") if c.name == name][0]
    t = make_layer_inputs(case, M=M)
    return (case, t) + _svd(name)


def _prep(name: str, M: int, rank: int) -> OS.Prepared:
    case, t, lam, inv_lam, W_hat, L1, L2, s = _split(name, M)
    inv64 = inv_lam.astype(np.float64)[:, None]
    return OS.prepare_from_factors(W_hat, inv_lam, OF.round_bf16(L1[:, :rank] * inv64),
                                   OF.round_bf16(L2[:rank]), t.bias, lam=lam, sigma=s)


def _handle(prep: OS.Prepared, fmt: str = "nvfp4"):
    L1p = f32_to_bf16_bits(prep.L1p.astype(np.float32))
    L2 = f32_to_bf16_bits(prep.L2b.astype(np.float32))
    return G.lib().svdq_weights_from_factors(prep.N, prep.K, prep.rank, prep.inv_lam, L1p, L2, prep.R,
                                             prep.bias.astype(np.float32), fmt=fmt)


def _with_lora(w, prep: OS.Prepared, r_l: int, seed: int):
    if r_l == 0:
        return prep
    Ab, A, Bb, B = make_lora_factors(prep.K, prep.N, r_l, seed)
    G.lib().svdq_attach_lora(w, Ab, Bb, 1.0)
    return OS.attach_lora(prep, A, B, 1.0)


def test_prepare_at_rank_equals_the_truncated_split():
    """The shared decomposition is the oracle's own prepare() at that rank."""
    case = [c for c in config_cases("flux") if c.name == "attn_out"][0]
    t = make_layer_inputs(case)
    a = _prep("attn_out", 64, 16)
    b = OS.prepare(t.W, t.act_absmax, t.bias, 16)
    np.testing.assert_array_equal(a.L1p, b.L1p)
    np.testing.assert_array_equal(a.L2b, b.L2b)
    np.testing.assert_array_equal(a.R, b.R)


@pytest.mark.parametrize("name", ["attn_out", "mlp_down", "mlp_up"])
@pytest.mark.parametrize("rank,r_l", [(64, 0), (48, 32), (96, 16), (64, 64)])
def test_wide_branch_layer(name, rank, r_l):
    M = 300                                   # three row blocks, the last ragged
    if name == "mlp_up" and r_l not in (0, 16):
        pytest.skip("mlp_up is covered at the rank the benchmark times and one LoRA width")
    case, t, *_ = _split(name, M)
    prep = _prep(name, M, rank)
    w = _handle(prep)
    ref = _with_lora(w, prep, r_l, seed=9000 + rank + r_l)
    info = w.info
    assert G.lib().svdq_weights_rank(w) == rank + r_l
    assert info["r_pad"] == (rank + r_l + 15) // 16 * 16
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    assert T.shape == (M, 2 * info["r_pad"])
    G.check_codes(xq, xsf, t.X, prep.inv_lam)
    G.check_T(T, t.X, ref)
    G.check_Y(Y, OS.linear(ref, t.X))


@pytest.mark.parametrize("name", ["attn_out", "mlp_down"])
def test_widest_branch_full_size(name):
    """r_pad = 128 (rank 64 + LoRA 64) at the full M = 4608 the benchmark runs:
    the activation kernel's larger tiles change its K-split, the GEMM runs four
    low-rank steps per tile.  Codes and scales of every row bit-exact, T and Y
    within bounds on rows from the start, middle and end."""
    case, t, *_ = _split(name, 4608)
    prep = _prep(name, 4608, 64)
    w = _handle(prep)
    ref = _with_lora(w, prep, 64, seed=9128)
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    M = Y.shape[0]
    rows = np.r_[0:48, M // 2 - 24:M // 2 + 24, M - 48:M]
    G.check_codes(xq, xsf, t.X, prep.inv_lam)
    G.check_T(T, t.X, ref, rows=rows)
    G.check_Y(Y[rows], OS.linear(ref, t.X, rows=rows))


@pytest.mark.parametrize("split", [2, 5, 8])
def test_wide_branch_split_k(split):
    """The split-K GEMM (small M) with the widest branch: the last split takes
    all four low-rank steps."""
    case, t, *_ = _split("attn_out", 16)
    prep = _prep("attn_out", 16, 64)
    w = _handle(prep)
    ref = _with_lora(w, prep, 64, seed=9129)
    _, xq, xsf, T = G.run_act(w, t.X_bits)
    import torch
    Y = torch.empty((16, case.N), dtype=torch.bfloat16, device="cuda")
    G.lib().svdq_debug_linear_w4a4_ksplit(w, xq, xsf, T, 16, Y, split)
    assert G.lib().svdq_check_device_errors() == 0
    G.check_Y(Y.float().cpu().numpy().astype(np.float64), OS.linear(ref, t.X))


def test_int4_widest_branch():
    """The INT4 variant (App. D) with r_pad = 128: its own GEMM runs the four
    low-rank steps from its slab buffer."""
    case, t, *_ = _split("attn_out", 300)
    base = _prep("attn_out", 300, 64)
    prep = OI.from_base(base)
    w = _handle(base, fmt="int4")
    Ab, A, Bb, B = make_lora_factors(case.K, case.N, 64, 9130)
    G.lib().svdq_attach_lora(w, Ab, Bb, 1.0)
    ref = OI.attach_lora(prep, A, B, 1.0)
    Y, _ = G.run_layer(w, t.X_bits)
    G.check_Y(Y, OI.linear(ref, t.X))
