"""GPU parity of the norm-fused activation path (LayerNorm + adaLN modulation
in front of the layer) against the CPU oracle, through the C ABI."""

import numpy as np
import pytest
import torch

from oracle import int4 as OI
from oracle import norm as ON
from oracle import svdquant as OS
from synth import f32_to_bf16_bits
from tests import gpu_common as G
from tests.test_gpu_int4 import _check_act as check_int4_act
from tests.test_gpu_int4 import _weights as int4_weights

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _inputs(M, K, seed):
    rng = np.random.default_rng(seed)
    Z = (rng.standard_normal((M, K)) * rng.uniform(0.5, 4, (M, 1)) + rng.uniform(-3, 3, (M, 1))).astype(np.float32)
    Z[:, rng.choice(K, 4, replace=False)] *= 20
    Zb = f32_to_bf16_bits(Z)
    Zf = (Zb.astype(np.uint32) << 16).view(np.float32)
    a = (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    c = (0.1 * rng.standard_normal(K)).astype(np.float32)
    return Zb, Zf, a, c


def _dev_f32(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def _stats(Zb):
    L = G.lib()
    Z = G.to_dev_bf16(Zb)
    st = torch.empty((Zb.shape[0], 2), dtype=torch.float32, device="cuda")
    L.svdq_act_row_stats(Z, EPS, st)
    torch.cuda.synchronize()
    return Z, st


def _prep(X, K, N, seed, fmt):
    rng = np.random.default_rng(seed + 1)
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    bias = rng.normal(0, 0.01, N).astype(np.float32)
    prep = OS.prepare(W, np.abs(X).max(axis=0), bias, 32)
    if fmt == "int4":
        prep = OI.from_base(prep)
        return prep, int4_weights(prep)
    return prep, G.weights_from_oracle(prep)


@pytest.mark.parametrize("M,K", [(1, 64), (300, 3072), (129, 1152)])
def test_row_stats_against_float64(M, K):
    Zb, Zf, _, _ = _inputs(M, K, M + K)
    _, st = _stats(Zb)
    got = st.cpu().numpy().astype(np.float64)
    mu, rstd = ON.row_stats(Zf, EPS)
    sd = 1.0 / rstd
    # fp32 one-pass sums over up to K / 32 values per lane: a few ulps of fp32 per step
    assert np.all(np.abs(got[:, 0] - mu) <= 1e-5 * (np.abs(mu) + sd))
    assert np.all(np.abs(got[:, 1] / rstd - 1.0) <= 1e-4)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
@pytest.mark.parametrize("M,K,N", [(300, 3072, 256), (1, 1152, 128), (200, 640, 384)])
def test_norm_fused_activation_bitexact_given_kernel_stats(fmt, M, K, N):
    """With the kernel's own (mu, rstd), the codes and scales equal the oracle's
    for X = bf16(((z - mu) rstd) a + c), T follows X L1', and Y is within the
    layer tolerance of the oracle."""
    L = G.lib()
    Zb, Zf, a, c = _inputs(M, K, 7 * M + K)
    Z, st = _stats(Zb)
    s = st.cpu().numpy()
    X = ON.normalize(Zf, s[:, 0], s[:, 1], a, c)
    prep, w = _prep(X, K, N, M + K, fmt)
    xq, xsf, T = L.act_buffers(w, M)
    L.svdq_norm_quantize_act_lowrank_down(w, Z, st, _dev_f32(a), _dev_f32(c), xq, xsf, T)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    L.svdq_linear_w4a4(w, xq, xsf, T, M, Y)
    assert L.svdq_check_device_errors() == 0
    if fmt == "int4":
        check_int4_act(xq, xsf, X, prep.inv_lam)
        G.check_T(T, X, prep.base)
        G.check_Y(Y.float().cpu().numpy().astype(np.float64), OI.linear(prep, X))
    else:
        G.check_codes(xq, xsf, X, prep.inv_lam)
        G.check_T(T, X, prep)
        G.check_Y(Y.float().cpu().numpy().astype(np.float64), OS.linear(prep, X))


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_forward_norm_equals_the_unfused_pipeline(fmt):
    """svdq_forward_norm (statistics, fused activation kernel, GEMM) gives the
    output, bit for bit, of svdq_forward on the bf16 X that a separate norm
    with the same statistics would have written."""
    L = G.lib()
    M, K, N = 1000, 3072, 512
    Zb, Zf, a, c = _inputs(M, K, 11)
    Z, st = _stats(Zb)
    s = st.cpu().numpy()
    X = ON.normalize(Zf, s[:, 0], s[:, 1], a, c)
    _, w = _prep(X, K, N, 11, fmt)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.svdq_forward_norm_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward_norm(w, Z, _dev_f32(a), _dev_f32(c), EPS, Y, ws)
    Xd = G.to_dev_bf16(f32_to_bf16_bits(X))
    Y2 = torch.empty_like(Y)
    ws2 = torch.empty(L.svdq_forward_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward(w, Xd, Y2, ws2)
    assert L.svdq_check_device_errors() == 0
    assert torch.equal(Y, Y2)
