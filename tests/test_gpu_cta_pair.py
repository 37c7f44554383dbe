"""The CTA-pair GEMM (256 x 256 tiles, one M = 256 pair MMA per K block) that
svdq_linear_w4a4 runs when a layer has many output tiles and at least 16 K
tiles.  The shapes below take that path: more than 74 single-CTA tiles (no
split-K) and K > 3840.  They include a last pair tile whose second CTA lies
wholly past M (M = 1300: rows 1280-1299 are the only valid ones), a weight tile
cut by N (N = 2000), N = 3088 (a last tile of 16 columns) and a LoRA-grown rank.

Exactness on FP4-grid inputs pins the path to the product itself; the
comparison with the single-CTA kernel (svdq_debug_linear_w4a4_ksplit with one
CTA per tile) checks that both kernels sum the same terms in the same order."""

import dataclasses

import numpy as np
import pytest
import torch

from oracle import formats as OF
from oracle import svdquant as OS
from synth import config_cases, make_fp4_grid_inputs, make_layer_inputs, make_lora_factors
from tests import gpu_common as G

pytestmark = pytest.mark.gpu


def _rank0_prep(W, inv_lam):
    K = W.shape[1]
    W_hat = OS.smooth_weight(W, inv_lam)
    return OS.prepare_from_factors(W_hat, inv_lam, np.zeros((K, 0)), np.zeros((0, W.shape[0])), None)


@pytest.mark.parametrize("M,K,N", [(1300, 4096, 2000), (1000, 4096, 3088), (2148, 4096, 1152)])
def test_pair_exact_on_fp4_grid(M, K, N):
    """On FP4-grid inputs every partial product and sum is exact in fp32, so Y
    is bf16(X W^T) exactly, in every row and column of ragged pair tiles."""
    Xb, X, Wb, W = make_fp4_grid_inputs(M, K, N, seed=7 * M + K + N)
    w = G.weights_from_oracle(_rank0_prep(W, np.ones(K, np.float32)))
    Y, _ = G.run_layer(w, Xb)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_array_equal(Y, OF.round_bf16(exact))


def _single_cta(w, xq, xsf, T, M):
    L = G.lib()
    Y = torch.full((M, w.info["N"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.svdq_debug_linear_w4a4_ksplit(w, xq, xsf, T, M, Y, 1)
    assert L.svdq_check_device_errors() == 0
    return Y


@pytest.mark.parametrize("M,K,N,rank,lora", [(1300, 4096, 2000, 32, 0), (1500, 6144, 2304, 64, 16),
                                             (4608, 12288, 3072, 32, 0)])
def test_pair_equals_single_cta_bitwise(M, K, N, rank, lora):
    """Library-prepared layers with the low-rank slab (rank 32, rank 64 grown
    by a rank-16 LoRA to 80, and the FLUX mlp_down shape): the pair kernel's Y
    equals the single-CTA kernel's bit for bit, and every element is written."""
    L = G.lib()
    c = dataclasses.replace(config_cases("flux")[0], M=M, K=K, N=N, rank=rank, lora_rank=0)
    t = make_layer_inputs(c)
    w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=rank)
    if lora:
        A_bits, _, B_bits, _ = make_lora_factors(K, N, lora, seed=M + lora)
        L.svdq_attach_lora(w, A_bits, B_bits, 1.0)
    _, xq, xsf, T = G.run_act(w, t.X_bits)
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.svdq_linear_w4a4(w, xq, xsf, T, M, Y)
    assert L.svdq_check_device_errors() == 0
    assert not torch.isnan(Y.float()).any()
    assert torch.equal(Y, _single_cta(w, xq, xsf, T, M))
