"""GPU parity of the INT4 variant (group 64, bf16 scales) against the CPU
oracle, through the C ABI: activation and weight codes and scales bit-exact,
the output exact on INT4-grid inputs and within the layer tolerance elsewhere."""

import functools

import numpy as np
import pytest
import torch

from oracle import formats as OF
from oracle import int4 as OI
from oracle import svdquant as OS
from synth import config_cases, f32_to_bf16_bits, make_int4_grid_inputs, make_layer_inputs
from tests import gpu_common as G

pytestmark = pytest.mark.gpu


def _weights(prep: OI.PreparedInt4):
    """Library INT4 handle holding exactly the oracle's split (before any LoRA)."""
    b = prep.base
    r = b.rank - b.lora_rank
    L1p = f32_to_bf16_bits(b.L1p[:, :r].astype(np.float32)) if r else None
    L2 = f32_to_bf16_bits(b.L2b[:r].astype(np.float32)) if r else None
    return G.lib().svdq_weights_from_factors(b.N, b.K, r, b.inv_lam, L1p, L2, b.R, b.bias.astype(np.float32),
                                             fmt="int4")


def _rank0(W, inv_lam, bias=None):
    K = W.shape[1]
    base = OS.prepare_from_factors(OS.smooth_weight(W, inv_lam), inv_lam, np.zeros((K, 0)),
                                   np.zeros((0, W.shape[0])), bias)
    return OI.from_base(base)


def _check_act(xq, xsf, X, inv_lam):
    M, K = X.shape
    codes, scales = OI.quantize_activations(X, inv_lam)
    np.testing.assert_array_equal(xq.cpu().numpy().reshape(-1)[: M * K // 2].reshape(M, K // 2),
                                  OI.pack_codes(codes))
    mpad = (M + 127) // 128 * 128
    s16 = xsf.cpu().numpy()[: (K // 64) * mpad * 2].view(np.uint16).reshape(K // 64, mpad)
    np.testing.assert_array_equal(s16[:, :M].T, OI.scales_to_bits(scales))
    assert not s16[:, M:].any()          # padding rows of the last 128-row block carry zero scales


@functools.lru_cache(maxsize=None)
def _case(label: str, M: int):
    cfg, name = label.split("/")
    case = [c for c in config_cases(cfg) if c.name == name][0]
    t = make_layer_inputs(case, M=M)
    return case, t, OI.prepare(t.W, t.act_absmax, t.bias, case.rank)


@pytest.mark.parametrize("M,K", [(64, 256), (1, 64), (200, 640), (333, 3072), (130, 1152)])
def test_int4_activation_codes_bitexact(M, K):
    rng = np.random.default_rng(M * 5 + K)
    X = rng.normal(0, 1, (M, K)).astype(np.float32)
    X[:, rng.choice(K, 3, replace=False)] *= 50
    X[0, :64] = 0.0                       # an all-zero group
    X[-1, :64] = 1e-30                    # a scale in the bf16 subnormal range
    X[min(1, M - 1), :64] *= 1e4          # large values
    Xb = f32_to_bf16_bits(X)
    Xf = OF.bf16_bits_to_f64(Xb).astype(np.float32)
    inv_lam = np.exp2(rng.uniform(-3, 3, K)).astype(np.float32)
    W = rng.normal(0, 0.02, (64, K)).astype(np.float32)
    w = _weights(_rank0(W, inv_lam))
    _, xq, xsf, T = G.run_act(w, Xb)
    assert T is None
    _check_act(xq, xsf, Xf, inv_lam)


def test_int4_weight_codes_bitexact():
    case, t, prep = _case("pixart/attn_qkv_out", 128)
    w = _weights(prep)
    ex = G.lib().svdq_weights_export(w)
    assert ex["format"] == "int4" and ex["alpha_w"] == 1.0
    np.testing.assert_array_equal(ex["codes"], OI.pack_codes(prep.w_codes))
    npad = (prep.N + 255) // 256 * 256
    s16 = ex["sf"].view(np.uint16).reshape(prep.K // 64, npad)
    np.testing.assert_array_equal(s16[:, : prep.N].T, OI.scales_to_bits(prep.w_scales))


@pytest.mark.parametrize("M,K,N", [(128, 256, 256), (64, 256, 48), (300, 640, 400), (77, 1280, 512)])
def test_int4_exact_on_grid(M, K, N):
    """Power-of-two group scales: every dequantized product and every partial
    sum is exact in fp32, so Y = bf16(X W^T) exactly."""
    Xb, X, Wb, W = make_int4_grid_inputs(M, K, N, seed=M + K + N, x_exp=(-1, 1), w_exp=(-7, -5), s_steps=1)
    prep = _rank0(W, np.ones(K, np.float32))
    w = _weights(prep)
    Y, (xq, xsf, _) = G.run_layer(w, Xb)
    _check_act(xq, xsf, X, np.ones(K, np.float32))
    np.testing.assert_array_equal(Y, OF.round_bf16(X.astype(np.float64) @ W.astype(np.float64).T))


INT4_LAYERS = ["tiny/layer", "pixart/attn_qkv_out", "flux/attn_out", "sdxl/r64_attn"]


@pytest.mark.parametrize("label", INT4_LAYERS)
def test_int4_layer_matches_oracle(label):
    """Configured layers at full K, N with up to 300 tokens (ragged row blocks)."""
    cfg, name = label.split("/")
    full_m = [c for c in config_cases(cfg) if c.name == name][0].M
    case, t, prep = _case(label, min(300, full_m))
    w = _weights(prep)
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    _check_act(xq, xsf, t.X, prep.inv_lam)
    G.check_T(T, t.X, prep.base)
    G.check_Y(Y, OI.linear(prep, t.X))


@pytest.mark.parametrize("M", [1, 16, 200])
def test_int4_small_m_with_lora(M):
    case, t, prep = _case("small_m_lora/M16_N3072", M)
    w = _weights(prep)
    G.lib().svdq_attach_lora(w, t.lora_A_bits, t.lora_B_bits, t.lora_scale)
    ref = OI.attach_lora(prep, t.lora_A, t.lora_B, t.lora_scale)
    Y, _ = G.run_layer(w, t.X_bits)
    G.check_Y(Y, OI.linear(ref, t.X))


def test_int4_forward_entry_points_agree():
    L = G.lib()
    case, t, prep = _case("pixart/mlp_up", 300)
    w = _weights(prep)
    Y2, _ = G.run_layer(w, t.X_bits)
    M = t.X_bits.shape[0]
    X = G.to_dev_bf16(t.X_bits)
    Y = torch.empty((M, w.info["N"]), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.svdq_forward_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward(w, X, Y, ws)
    assert L.svdq_check_device_errors() == 0
    np.testing.assert_array_equal(Y.float().cpu().numpy(), Y2)
    Y.zero_()
    L.svdq_forward_noalloc(w, X, Y)
    assert L.svdq_check_device_errors() == 0
    np.testing.assert_array_equal(Y.float().cpu().numpy(), Y2)
    Xh = torch.from_numpy(t.X_bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((M, w.info["N"]), dtype=torch.bfloat16).pin_memory()
    wsh = torch.empty(L.svdq_forward_host_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward_host(w, Xh, Yh, wsh)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Yh.float().numpy(), Y2)


def test_int4_library_prepare():
    """svdq_prepare_weights(format=INT4): the handle reports INT4 with alpha_w = 1,
    its codes are the oracle codec of the library's own residual, and the layer
    follows X W^T + b about as closely as the NVFP4 layer does."""
    L = G.lib()
    case, t, _ = _case("pixart/attn_qkv_out", 256)
    w4 = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=32, fmt="int4", keep_residual=True)
    info = w4.info
    assert info["format"] == "int4" and info["alpha_w"] == 1.0
    ex = L.svdq_weights_export(w4, residual=True)
    codes, scales = OI.quantize_groups(ex["residual"])
    np.testing.assert_array_equal(ex["codes"], OI.pack_codes(codes))
    Y4, _ = G.run_layer(w4, t.X_bits)
    wf = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=32)
    Yf, _ = G.run_layer(wf, t.X_bits)
    exact = t.X.astype(np.float64) @ t.W.astype(np.float64).T + t.bias
    e4 = np.linalg.norm(Y4 - exact) / np.linalg.norm(exact)
    ef = np.linalg.norm(Yf - exact) / np.linalg.norm(exact)
    assert e4 < 0.1 and ef < 0.1, (e4, ef)
    with pytest.raises(Exception):
        L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=32, fmt="int4", refine_iters=2)


def test_int4_full_size_layer_repeatable():
    """FLUX attn_out at full size (36 x 12 tiles, several per CTA, so every
    buffer of the GEMM's rings turns over many times): rows from the start,
    middle and end within the layer tolerance of the oracle, and two launches
    bitwise equal."""
    L = G.lib()
    case, t, prep = _case("flux/attn_out", 4608)
    w = _weights(prep)
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    rows = np.r_[0:40, 2300:2340, case.M - 40:case.M]
    G.check_Y(Y[rows], OI.linear(prep, t.X, rows=rows))
    Y2 = torch.empty((case.M, case.N), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        L.svdq_linear_w4a4(w, xq, xsf, T, case.M, Y2)
    assert L.svdq_check_device_errors() == 0
    np.testing.assert_array_equal(Y2.float().cpu().numpy(), Y)


def test_int4_cuda_graph_capture_and_replay():
    """The INT4 forward pass (activation kernel, then the GEMM as its
    programmatic dependent) captured into a CUDA graph replays to the eager
    output and follows a rewrite of the captured input."""
    L = G.lib()
    case, t, prep = _case("pixart/mlp_up", 300)
    w = _weights(prep)
    M, N = t.X_bits.shape[0], w.info["N"]
    X = G.to_dev_bf16(t.X_bits)
    X2 = G.to_dev_bf16(t.X_bits[::-1].copy())
    ws = torch.empty(L.svdq_forward_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    eager = []
    for src in (X, X2):
        L.svdq_forward(w, src, Y, ws)
        eager.append(Y.clone())
    torch.cuda.synchronize()
    Xg = X.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        L.svdq_forward(w, Xg, Y, ws)
    Y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, eager[0])
    Xg.copy_(X2)
    g.replay()
    torch.cuda.synchronize()
    assert L.svdq_check_device_errors() == 0
    assert torch.equal(Y, eager[1])
    del g


def test_int4_alpha_search_runs_on_the_int4_layer():
    """svdq_search_alpha with the INT4 format scores every candidate through the
    INT4 kernels; its errors are finite, the pick is the smallest, and the
    α = 0.5 score matches preparing at 0.5 and measuring the output directly."""
    L = G.lib()
    case, t, _ = _case("tiny/layer", 64)
    alphas = (0.3, 0.5, 0.7)
    errs, best = L.svdq_search_alpha(t.W_bits, t.X_bits, t.bias_bits, alphas=alphas, rank=case.rank, fmt="int4")
    assert len(errs) == 3 and all(np.isfinite(errs)) and best == int(np.argmin(errs))
    w = L.svdq_prepare_weights(t.W_bits, np.abs(t.X).max(axis=0), t.bias_bits, rank=case.rank, alpha=0.5,
                               fmt="int4")
    Y, _ = G.run_layer(w, t.X_bits)
    exact = t.X.astype(np.float64) @ t.W.astype(np.float64).T + t.bias
    # the library scores against an fp32 reference; the float64 one differs in the last bits
    assert abs(errs[1] - np.linalg.norm(Y - exact) / np.linalg.norm(exact)) < 1e-4
