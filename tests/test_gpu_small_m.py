"""GPU parity of the one-kernel layer for a few tokens (M <= 16, NVFP4 handle,
rank + LoRA ranks <= 64; reached through svdq_debug_forward_small_m, while
svdq_forward keeps the faster two-kernel path), through the C ABI.

That kernel quantizes the activations inside the GEMM's CTAs, computes each
CTA's share of the down-projection T = X L1' on the tensor cores, applies L2
to it and sums the K splits' fp32 partials in split order (SVDQuant §4.3: the
branch is linear in K).  Checked against the oracle: the exact product on
inputs already on the FP4 grid (rank 0, ragged K and N, every split), the
small-M + LoRA layers of the benchmark (M = 1, 5, 16; K = 3072; N = 3072 and
12288; rank 32 + LoRA 16) within the layer tolerance, run-to-run bitwise
repeatability, agreement with the two-kernel path, and the fallback to the
two-kernel path above its limits (M = 17, rank 64 + LoRA 16)."""

import functools

import numpy as np
import pytest
import torch

from oracle import formats as OF
from oracle import svdquant as OS
from synth import config_cases, make_fp4_grid_inputs, make_layer_inputs, make_lora_factors
from tests import gpu_common as G

pytestmark = pytest.mark.gpu


def _rank0_prep(W, inv_lam, bias=None):
    K = W.shape[1]
    return OS.prepare_from_factors(OS.smooth_weight(W, inv_lam), inv_lam, np.zeros((K, 0)),
                                   np.zeros((0, W.shape[0])), bias)


def _forward(w, X_bits, ksplit=None):
    L = G.lib()
    M = X_bits.shape[0]
    X = G.to_dev_bf16(X_bits)
    Y = torch.full((M, w.info["N"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    if ksplit is None:
        ws = torch.empty(L.svdq_forward_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
        L.svdq_forward(w, X, Y, ws)
    else:
        L.svdq_debug_forward_small_m(w, X, Y, ksplit)
    assert L.svdq_check_device_errors() == 0
    return Y.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M,K,N", [(1, 256, 128), (7, 640, 400), (16, 3072, 384), (16, 1280, 256)])
@pytest.mark.parametrize("ksplit", [1, 2, 3, 8])
def test_exact_product_on_fp4_grid(M, K, N, ksplit):
    """Rank 0, unit smoothing, inputs on the FP4 grid: every partial sum is
    exact in fp32, so Y equals bf16(X W^T) exactly -- for a ragged last K tile
    (K = 640), output features past the last full 128-row tile (N = 400, 384),
    and splits clamped to the number of K tiles."""
    Xb, X, Wb, W = make_fp4_grid_inputs(M, K, N, seed=11 * M + K + N + ksplit)
    w = G.weights_from_oracle(_rank0_prep(W, np.ones(K, np.float32)))
    exact = OF.round_bf16(X.astype(np.float64) @ W.astype(np.float64).T)
    np.testing.assert_array_equal(_forward(w, Xb, ksplit), exact)


@functools.lru_cache(maxsize=None)
def _small_case(name: str, M: int):
    case = [c for c in config_cases("small_m_lora") if c.name == name][0]
    t = make_layer_inputs(case, M=M)
    prep = OS.prepare(t.W, t.act_absmax, t.bias, case.rank)
    return case, t, prep


def _lora_handle(case, t, prep):
    w = G.weights_from_oracle(prep)
    G.lib().svdq_attach_lora(w, t.lora_A_bits, t.lora_B_bits, t.lora_scale)
    return w, OS.attach_lora(prep, t.lora_A, t.lora_B, t.lora_scale)


@pytest.mark.parametrize("name", ["M16_N3072", "M16_N12288"])
@pytest.mark.parametrize("M", [1, 5, 16])
def test_small_m_lora_layer(name, M):
    case, t, prep = _small_case(name, M)
    w, ref = _lora_handle(case, t, prep)
    assert w.info["r_pad"] == 48
    Y = _forward(w, t.X_bits, 0)                                  # the one-kernel layer
    G.check_Y(Y, OS.linear(ref, t.X))
    np.testing.assert_array_equal(_forward(w, t.X_bits, 0), Y)    # repeatable bit for bit
    G.check_Y(_forward(w, t.X_bits), OS.linear(ref, t.X))        # svdq_forward's choice of path
    # the two-kernel path computes the same layer (fp32 sums in another order)
    Y2, _ = G.run_layer(w, t.X_bits)
    assert np.max(np.abs(Y - Y2) / np.maximum(1.0, np.abs(Y2))) <= 2e-2
    assert np.mean(Y == Y2) >= 0.9


@pytest.mark.parametrize("ksplit", [1, 2, 4, 6, 8])
def test_small_m_every_split(ksplit):
    case, t, prep = _small_case("M16_N3072", 16)
    w, ref = _lora_handle(case, t, prep)
    Y = _forward(w, t.X_bits, ksplit)
    G.check_Y(Y, OS.linear(ref, t.X))


def test_rank0_and_rank64_handles():
    """No low-rank branch at all, and the widest branch the kernel takes
    (rank 64: r_pad 64, two 32-rank groups of T and L2)."""
    case, t, _ = _small_case("M16_N3072", 16)
    K, N = case.K, case.N
    lam, inv = OS.smoothing_factors(t.act_absmax, t.W)
    p0 = _rank0_prep(t.W, inv, t.bias)
    G.check_Y(_forward(G.weights_from_oracle(p0), t.X_bits), OS.linear(p0, t.X))
    p64 = OS.prepare(t.W, t.act_absmax, t.bias, 64)
    w64 = G.weights_from_oracle(p64)
    assert w64.info["r_pad"] == 64
    G.check_Y(_forward(w64, t.X_bits), OS.linear(p64, t.X))


def test_fallback_above_the_limits():
    """M = 17 and rank 64 + LoRA 16 (r_pad 80) are outside the one-kernel
    layer, which svdq_debug_forward_small_m refuses; svdq_forward matches the
    oracle there."""
    L = G.lib()
    case, t, prep = _small_case("M16_N3072", 17)
    w, ref = _lora_handle(case, t, prep)
    G.check_Y(_forward(w, t.X_bits), OS.linear(ref, t.X))
    X = G.to_dev_bf16(t.X_bits)
    Y = torch.empty((17, case.N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.SvdqError):
        L.svdq_debug_forward_small_m(w, X, Y)
    case16, t16, _ = _small_case("M16_N3072", 16)
    p64 = OS.prepare(t16.W, t16.act_absmax, t16.bias, 64)
    w80 = G.weights_from_oracle(p64)
    Ab, A, Bb, B = make_lora_factors(case16.K, case16.N, 16, 9500)
    L.svdq_attach_lora(w80, Ab, Bb, 1.0)
    ref80 = OS.attach_lora(p64, A, B, 1.0)
    assert w80.info["r_pad"] == 80
    G.check_Y(_forward(w80, t16.X_bits), OS.linear(ref80, t16.X))


@pytest.mark.parametrize("name", ["M16_N3072", "M16_N12288"])
def test_noalloc_matches_forward_at_small_m(name):
    """The allocation-free entry point takes the same path as svdq_forward."""
    L = G.lib()
    case, t, prep = _small_case(name, 16)
    w, _ = _lora_handle(case, t, prep)
    X = G.to_dev_bf16(t.X_bits)
    Y = torch.empty((16, case.N), dtype=torch.bfloat16, device="cuda")
    L.svdq_forward_noalloc(w, X, Y)
    assert L.svdq_check_device_errors() == 0
    np.testing.assert_array_equal(Y.float().cpu().numpy().astype(np.float64), _forward(w, t.X_bits))
