"""GPU parity of the two kernels against the CPU oracle, through the C ABI.

Codes and scales must match bit for bit; Y must be within the layer
tolerance (relative Frobenius 2e-3, per element 1e-2 * max(1, |ref|)); on
inputs that already lie on the FP4 grid Y must equal bf16(X W^T) exactly."""

import functools

import numpy as np
import pytest
import torch

from oracle import codec as OC
from oracle import formats as OF
from oracle import svdquant as OS
from synth import config_cases, f32_to_bf16_bits, make_fp4_grid_inputs, make_layer_inputs
from tests import gpu_common as G

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def _case_prep(label: str, M: int):
    cfg, name = label.split("/")
    case = [c for c in config_cases(cfg) if c.name == name][0]
    t = make_layer_inputs(case, M=M)
    prep = OS.prepare(t.W, t.act_absmax, t.bias, case.rank)
    return t, prep


def _rank0_prep(W, inv_lam, bias=None):
    K = W.shape[1]
    W_hat = OS.smooth_weight(W, inv_lam)
    return OS.prepare_from_factors(W_hat, inv_lam, np.zeros((K, 0)), np.zeros((0, W.shape[0])), bias)


@pytest.mark.parametrize("M,K", [(64, 256), (1, 64), (200, 640), (333, 3072), (128, 1152)])
def test_activation_codes_bitexact(M, K):
    rng = np.random.default_rng(M * 7 + K)
    X = rng.normal(0, 1, (M, K)).astype(np.float32)
    X[:, rng.choice(K, 3, replace=False)] *= 50
    X[0, :32] = 0.0                       # an all-zero group
    X[-1, 16:32] = 1e-7                   # scale rounds to zero
    X[-1, 32:48] = -1e-3                  # E4M3 subnormal scale, negatives
    X[min(1, M - 1), 48:64] = 3e4         # large values
    Xb = f32_to_bf16_bits(X)
    Xf = OF.bf16_bits_to_f64(Xb).astype(np.float32)
    inv_lam = np.exp2(rng.uniform(-3, 3, K)).astype(np.float32)
    W = rng.normal(0, 0.02, (64, K)).astype(np.float32)
    w = G.weights_from_oracle(_rank0_prep(W, inv_lam))
    _, xq, xsf, T = G.run_act(w, Xb)
    assert T is None
    G.check_codes(xq, xsf, Xf, inv_lam)


@pytest.mark.parametrize("M,K", [(4600, 1152), (8000, 640)])
def test_large_M_layer(M, K):
    """Large M (ragged last row block at M = 4600; K = 640 is a ragged number of
    256-wide GEMM K tiles): codes and scales bit-exact, T within the fp32
    accumulation bound, and the whole layer within the output tolerance on
    rows from the start, middle and end."""
    rng = np.random.default_rng(M + K)
    X = rng.normal(0, 1, (M, K)).astype(np.float32)
    X[:, rng.choice(K, 5, replace=False)] *= 30
    X[7, :64] = 0.0
    Xb = f32_to_bf16_bits(X)
    Xf = OF.bf16_bits_to_f64(Xb).astype(np.float32)
    W = rng.normal(0, 0.02, (64, K)).astype(np.float32)
    bias = rng.normal(0, 0.01, 64).astype(np.float32)
    prep = OS.prepare(W, np.abs(Xf).max(axis=0), bias, 32)
    w = G.weights_from_oracle(prep)
    Y, (xq, xsf, T) = G.run_layer(w, Xb)
    G.check_codes(xq, xsf, Xf, prep.inv_lam)
    G.check_T(T, Xf, prep)
    rows = np.r_[0:40, M // 2 : M // 2 + 40, M - 40 : M]
    G.check_Y(Y[rows], OS.linear(prep, Xf, rows=rows))


def test_weight_codes_and_factor_bitexact():
    t, prep = _case_prep("pixart/attn_qkv_out", 128)
    w = G.weights_from_oracle(prep)
    ex = G.lib().svdq_weights_export(w, residual=True)
    assert ex["alpha_w"] == prep.alpha_w
    np.testing.assert_array_equal(ex["residual"], prep.Rp)
    np.testing.assert_array_equal(ex["codes"], OC.pack_codes(prep.w_codes))
    np.testing.assert_array_equal(ex["sf"], OC.scales_to_atoms(prep.w_scales))


@pytest.mark.parametrize("M,K,N", [(128, 256, 256), (64, 256, 48), (300, 640, 400), (77, 1280, 512)])
def test_exact_product_on_fp4_grid(M, K, N):
    Xb, X, Wb, W = make_fp4_grid_inputs(M, K, N, seed=M + K + N)
    w = G.weights_from_oracle(_rank0_prep(W, np.ones(K, np.float32)))
    Y, (xq, xsf, _) = G.run_layer(w, Xb)
    G.check_codes(xq, xsf, X, np.ones(K, np.float32))
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_array_equal(Y, OF.round_bf16(exact))


def _run_split(w, X_bits: np.ndarray, ksplit: int) -> np.ndarray:
    L = G.lib()
    _, xq, xsf, T = G.run_act(w, X_bits)
    M = X_bits.shape[0]
    Y = torch.empty((M, w.info["N"]), dtype=torch.bfloat16, device="cuda")
    L.svdq_debug_linear_w4a4_ksplit(w, xq, xsf, T, M, Y, ksplit)
    assert L.svdq_check_device_errors() == 0
    return Y.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M,K,N", [(16, 3072, 512), (1, 1280, 256), (200, 640, 256), (130, 2304, 768)])
@pytest.mark.parametrize("ksplit", [2, 3, 5, 8])
def test_split_k_exact_on_fp4_grid(M, K, N, ksplit):
    """Split-K (S CTAs of a cluster per output tile, partials summed through
    distributed shared memory): on FP4-grid inputs every partial sum is exact
    in fp32, so Y equals bf16(X W^T) exactly for every split -- with ragged row
    tiles (M = 200, 130), a ragged K tail (K = 640) and splits clamped to the
    number of K tiles (K = 640, 1280 with S = 5, 8)."""
    Xb, X, Wb, W = make_fp4_grid_inputs(M, K, N, seed=3 * M + K + N + ksplit)
    w = G.weights_from_oracle(_rank0_prep(W, np.ones(K, np.float32)))
    exact = OF.round_bf16(X.astype(np.float64) @ W.astype(np.float64).T)
    np.testing.assert_array_equal(_run_split(w, Xb, ksplit), exact)


@pytest.mark.parametrize("M", [1, 16, 129])
def test_split_k_layer_matches_oracle(M):
    """The small-M + LoRA layer (rank 32 + 16, K = 3072) under every split:
    within the layer tolerance of the oracle, reproducible bit for bit from
    run to run, and within fp32 accumulation differences of the unsplit sum."""
    t, prep = _case_prep("small_m_lora/M16_N3072", M)
    w = G.weights_from_oracle(prep)
    G.lib().svdq_attach_lora(w, t.lora_A_bits, t.lora_B_bits, t.lora_scale)
    ref = OS.linear(OS.attach_lora(prep, t.lora_A, t.lora_B, t.lora_scale), t.X)
    Y1 = _run_split(w, t.X_bits, 1)
    G.check_Y(Y1, ref)
    for S in (2, 3, 6, 8):
        Ys = _run_split(w, t.X_bits, S)
        G.check_Y(Ys, ref)
        np.testing.assert_array_equal(_run_split(w, t.X_bits, S), Ys)
        assert np.max(np.abs(Ys - Y1) / np.maximum(1.0, np.abs(Y1))) <= 2e-2
        assert np.mean(Ys == Y1) >= 0.9


def test_tiny_layer():
    t, prep = _case_prep("tiny/layer", 64)
    w = G.weights_from_oracle(prep)
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    G.check_codes(xq, xsf, t.X, prep.inv_lam)
    G.check_T(T, t.X, prep)
    G.check_Y(Y, OS.linear(prep, t.X))


def test_rank0_plain_w4a4_layer():
    t, _ = _case_prep("tiny/layer", 64)
    K = t.case.K
    prep = OS.prepare_from_factors(t.W, np.ones(K, np.float32), np.zeros((K, 0)), np.zeros((0, t.case.N)),
                                   t.bias)
    w = G.weights_from_oracle(prep)
    Y, _ = G.run_layer(w, t.X_bits)
    G.check_Y(Y, OS.linear(prep, t.X))


ALL_LAYERS = [c.label for cfg in ["pixart", "flux", "sdxl", "small_m_lora"] for c in config_cases(cfg)]


@pytest.mark.parametrize("label", ALL_LAYERS)
def test_config_layer_reduced_M(label):
    """Every configured layer at full K, N with 300 tokens (3 row tiles, ragged)."""
    cfg, name = label.split("/")
    case = [c for c in config_cases(cfg) if c.name == name][0]
    M = min(case.M, 300)
    t, prep = _case_prep(label, M)
    w = G.weights_from_oracle(prep)
    ref_prep = prep
    if case.lora_rank:
        G.lib().svdq_attach_lora(w, t.lora_A_bits, t.lora_B_bits, t.lora_scale)
        ref_prep = OS.attach_lora(prep, t.lora_A, t.lora_B, t.lora_scale)
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    G.check_codes(xq, xsf, t.X, prep.inv_lam)
    G.check_T(T, t.X, ref_prep)
    G.check_Y(Y, OS.linear(ref_prep, t.X))


def test_lora_attach_keeps_codes():
    t, prep = _case_prep("small_m_lora/M16_N3072", 16)
    w = G.weights_from_oracle(prep)
    before = G.lib().svdq_weights_export(w)
    G.lib().svdq_attach_lora(w, t.lora_A_bits, t.lora_B_bits, 0.5)
    after = G.lib().svdq_weights_export(w)
    for k in ("codes", "sf", "inv_lam", "bias"):
        np.testing.assert_array_equal(before[k], after[k])
    assert after["rank"] == before["rank"] + 16 and after["alpha_w"] == before["alpha_w"]
    np.testing.assert_array_equal(after["L1p"][:, 32:], t.lora_A_bits)
    ref = OS.attach_lora(prep, t.lora_A, t.lora_B, 0.5)
    Y, _ = G.run_layer(w, t.X_bits)
    G.check_Y(Y, OS.linear(ref, t.X))


def test_forward_entry_points_agree():
    L = G.lib()
    t, prep = _case_prep("pixart/mlp_up", 300)
    w = G.weights_from_oracle(prep)
    Y2, _ = G.run_layer(w, t.X_bits)
    M = t.X_bits.shape[0]
    X = G.to_dev_bf16(t.X_bits)
    Y = torch.empty((M, w.info["N"]), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.svdq_forward_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward(w, X, Y, ws)
    assert L.svdq_check_device_errors() == 0
    np.testing.assert_array_equal(Y.float().cpu().numpy(), Y2)
    Xh = torch.from_numpy(t.X_bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((M, w.info["N"]), dtype=torch.bfloat16).pin_memory()
    wsh = torch.empty(L.svdq_forward_host_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward_host(w, Xh, Yh, wsh)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Yh.float().numpy(), Y2)


def test_forward_host_chunked_pipeline():
    """A host-buffer call large enough to be split into row chunks (two chunks,
    the second ragged) agrees with the device-buffer call and the oracle."""
    L = G.lib()
    t, prep = _case_prep("pixart/mlp_up", 1100)
    w = G.weights_from_oracle(prep)
    M = t.X_bits.shape[0]
    X = G.to_dev_bf16(t.X_bits)
    Y = torch.empty((M, w.info["N"]), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.svdq_forward_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward(w, X, Y, ws)
    Xh = torch.from_numpy(t.X_bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    Yh = torch.full((M, w.info["N"]), float("nan"), dtype=torch.bfloat16).pin_memory()
    wsh = torch.empty(L.svdq_forward_host_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward_host(w, Xh, Yh, wsh)
    torch.cuda.synchronize()
    assert L.svdq_check_device_errors() == 0
    # a chunk of 460 rows may take the split-K GEMM, the whole batch does not:
    # the two agree to fp32 accumulation order, and both with the oracle
    Yc, Yw = Yh.float().numpy().astype(np.float64), Y.float().cpu().numpy().astype(np.float64)
    assert np.mean(Yc == Yw) >= 0.9
    rows = np.r_[0:40, 600:640, M - 40:M]
    ref = OS.linear(prep, t.X, rows=rows)
    G.check_Y(Yc[rows], ref)
    G.check_Y(Yw[rows], ref)


@pytest.mark.parametrize("label,M", [("small_m_lora/M16_N3072", 16), ("pixart/mlp_up", 300)])
def test_cuda_graph_capture_and_replay(label, M):
    """The forward pass captured into a CUDA graph (the split-K GEMM at M = 16,
    the persistent one at M = 300; both launched as programmatic dependents of
    the activation kernel) replays to the eager output, and follows a rewrite
    of the captured input buffer."""
    L = G.lib()
    t, prep = _case_prep(label, M)
    w = G.weights_from_oracle(prep)
    X = G.to_dev_bf16(t.X_bits)
    X2 = G.to_dev_bf16(t.X_bits[::-1].copy())
    N = w.info["N"]
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
    G.check_Y(Y.float().cpu().numpy().astype(np.float64)[:8], OS.linear(prep, t.X[::-1][:8]))
    del g


def test_codec_shortcuts_match_ieee():
    """The encoder's fused division by 6 and its table reciprocal of the E4M3
    scale equal IEEE fp32 division / reciprocal over their whole domains
    (checked on the device against the IEEE intrinsics)."""
    assert G.lib().svdq_selftest_codec() == 0


def test_output_only_16_byte_aligned():
    """Y that is 16- but not 32-byte aligned takes the 16-byte store path; the
    values are the same as with an aligned Y (and rows/columns stay in place)."""
    L = G.lib()
    t, prep = _case_prep("pixart/mlp_up", 300)
    w = G.weights_from_oracle(prep)
    Y_ref, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    M, N = t.X_bits.shape[0], w.info["N"]
    buf = torch.full((M * N + 16,), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert buf.data_ptr() % 32 == 0
    Y = buf[8:8 + M * N].view(M, N)  # 16 bytes past a 32-byte boundary
    L.svdq_linear_w4a4(w, xq, xsf, T, M, Y)
    assert L.svdq_check_device_errors() == 0
    np.testing.assert_array_equal(Y.float().cpu().numpy(), Y_ref)
    assert torch.isnan(buf[:8].float()).all() and torch.isnan(buf[8 + M * N:].float()).all()


def test_staged_store_clips_a_ragged_row_block():
    """The GEMM epilogue's staged TMA stores (tiles of >= 8 K steps that are not
    their CTA's last) on a row block that ends inside a warp's 32-row box:
    M = 3900, so the last block holds rows 3840-3899 and its second warp's box
    is 28 rows of Y and 4 past it; K = 2048 at rank 0 (8 K steps); 31 x 8 = 248
    tiles, so CTAs 0-99 take two and the ragged block's tiles 30, 61 and 92 go
    through the staged path.  Y matches the oracle on rows around the ragged
    block, every element of Y is written, and guard rows after Y keep their NaNs."""
    L = G.lib()
    M, K, N = 3900, 2048, 2048
    rng = np.random.default_rng(3900)
    X = rng.normal(0, 1, (M, K)).astype(np.float32)
    X[:, rng.choice(K, 10, replace=False)] *= 30
    Xb = f32_to_bf16_bits(X)
    Xf = OF.bf16_bits_to_f64(Xb).astype(np.float32)
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    bias = rng.normal(0, 0.01, N).astype(np.float32)
    _, inv_lam = OS.smoothing_factors(np.abs(Xf).max(axis=0), W)
    prep = _rank0_prep(W, inv_lam, bias)
    w = G.weights_from_oracle(prep)
    _, xq, xsf, T = G.run_act(w, Xb)
    guard = 64
    buf = torch.full(((M + guard) * N,), float("nan"), dtype=torch.bfloat16, device="cuda")
    Y = buf[:M * N].view(M, N)
    L.svdq_linear_w4a4(w, xq, xsf, T, M, Y)
    assert L.svdq_check_device_errors() == 0
    assert torch.isnan(buf[M * N:].float()).all()
    Yh = Y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(Yh))
    rows = np.r_[0:16, 3830:3900]
    G.check_Y(Yh[rows], OS.linear(prep, Xf, rows=rows))


def test_library_prepare_invariants():
    """The library's own host SVD split: inv_lam as the oracle's, L1 L2 + R
    reconstructs W_hat, and the split is near the Eckart-Young optimum."""
    L = G.lib()
    t, prep = _case_prep("tiny/layer", 64)
    w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=16, keep_residual=True)
    ex = L.svdq_weights_export(w, residual=True)
    np.testing.assert_allclose(ex["inv_lam"], prep.inv_lam, rtol=1.2e-7, atol=0)
    W_hat = OS.smooth_weight(t.W, ex["inv_lam"])
    L1p = OF.bf16_bits_to_f64(ex["L1p"])
    L2 = OF.bf16_bits_to_f64(ex["L2"])
    low = ((L1p / ex["inv_lam"].astype(np.float64)[:, None]) @ L2).T
    recon = low + ex["residual"].astype(np.float64) * ex["alpha_w"]
    assert np.linalg.norm(recon - W_hat) / np.linalg.norm(W_hat) < 1e-6
    opt = np.sum(prep.sigma[16:] ** 2)
    assert np.linalg.norm(W_hat - low) ** 2 <= 1.02 * opt + 1e-3 * np.sum(prep.sigma ** 2)
    np.testing.assert_allclose(np.linalg.svd(low, compute_uv=False)[:16], prep.sigma[:16], rtol=2e-2)
    # its layer output is as accurate as the oracle's own split
    Y, _ = G.run_layer(w, t.X_bits)
    exact = t.X.astype(np.float64) @ t.W.astype(np.float64).T + t.bias
    e_lib = np.linalg.norm(Y - exact) / np.linalg.norm(exact)
    e_orc = np.linalg.norm(OS.linear(prep, t.X) - exact) / np.linalg.norm(exact)
    assert e_lib < 1.5 * e_orc + 1e-3


@pytest.mark.parametrize("name", ["attn_out", "qkv", "mlp_up", "mlp_down"])
def test_bench_configuration_full_size_sampled(name):
    """The FLUX.1 double-block layers exactly as the benchmark times them: full
    M = 4608, weights prepared by the library's own host SVD at rank 32, both
    kernels.  The oracle evaluates the library's exported split on 96 rows x
    256 columns spread over the output: the weight codes and scales of those
    columns and the activation codes and scales of those rows are bit-exact,
    and Y there is within the layer tolerance."""
    L = G.lib()
    case = [c for c in config_cases("flux") if c.name == name][0]
    t = make_layer_inputs(case)
    w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=case.rank, keep_residual=True)
    ex = L.svdq_weights_export(w, residual=True)
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    M, N = Y.shape
    rows = np.r_[0:32, M // 2:M // 2 + 32, M - 32:M]
    cols = np.r_[0:64, N // 2 - 64:N // 2 + 64, N - 64:N]
    inv = ex["inv_lam"]
    Rp = ex["residual"][cols]
    codes, scales = OC.quantize_groups(Rp)
    np.testing.assert_array_equal(ex["codes"][cols], OC.pack_codes(codes))
    np.testing.assert_array_equal(OC.atoms_to_scales(ex["sf"], N, case.K // 16)[cols], scales)
    prep = OS.Prepared(len(cols), case.K, ex["rank"], (1.0 / inv.astype(np.float64)).astype(np.float32), inv,
                       OF.bf16_bits_to_f64(ex["L1p"]), OF.bf16_bits_to_f64(ex["L2"])[:, cols],
                       (Rp.astype(np.float64) * ex["alpha_w"]).astype(np.float32), ex["alpha_w"], Rp, codes, scales,
                       ex["bias"][cols].astype(np.float64))
    G.check_codes(xq, xsf, t.X, inv, rows=rows)
    G.check_T(T, t.X, prep, rows=rows)
    G.check_Y(Y[np.ix_(rows, cols)], OS.linear(prep, t.X, rows=rows))


def test_library_refinement_matches_oracle():
    """Refined split (SVDQuant §4.2; the update rule is a reading of its iterations):
    the library's residual quantization errors follow the oracle's (exact SVD)
    closely, the kept split is the one with the smallest error (recomputed by
    the oracle from the exported residual), refinement lowers the error on the
    outlier layer, and the refined layer meets the output tolerance."""
    L = G.lib()
    t, _ = _case_prep("tiny/layer", 64)
    orc = OS.prepare(t.W, t.act_absmax, t.bias, 16, iters=4)
    w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=16, keep_residual=True,
                               refine_iters=4)
    errs = L.svdq_weights_refine_errors(w)
    assert len(errs) == 4
    np.testing.assert_allclose(errs, orc.refine_errors, rtol=2e-2)
    assert min(errs) < 0.95 * errs[0]
    ex = L.svdq_weights_export(w, residual=True)
    R = (ex["residual"].astype(np.float64) * ex["alpha_w"]).astype(np.float32)
    kept = np.linalg.norm(R.astype(np.float64) - OS.fake_quantize_weights(R))
    assert kept == pytest.approx(min(errs), rel=1e-9)
    plain = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=16)
    assert len(L.svdq_weights_refine_errors(plain)) == 1
    prep = OS.prepare_from_factors(OS.smooth_weight(t.W, ex["inv_lam"]), ex["inv_lam"],
                                   OF.bf16_bits_to_f64(ex["L1p"]), OF.bf16_bits_to_f64(ex["L2"]), t.bias)
    Y, _ = G.run_layer(w, t.X_bits)
    G.check_Y(Y, OS.linear(prep, t.X))


def test_library_alpha_search_matches_oracle():
    """NEXT-3 alpha search (App. D migration strength) run through the library's
    preparation and kernels: the per-candidate output errors follow the
    oracle's float64 ones, and the chosen alpha's error is the oracle's minimum
    up to the spread of near-ties."""
    L = G.lib()
    t, _ = _case_prep("tiny/layer", 64)
    alphas = [0.0, 0.25, 0.5, 0.75, 0.9]
    errs, best = L.svdq_search_alpha(t.W_bits, t.X_bits, t.bias_bits, alphas, rank=16)
    ref, ref_best = OS.search_alpha(t.W, t.X, t.bias, 16, alphas)
    np.testing.assert_allclose(errs, ref, rtol=3e-2)
    assert best == int(np.argmin(errs))
    assert errs[best] <= 1.02 * min(ref)
    assert errs[2] < errs[0]


def test_bounded_wait_reports_timeout():
    L = G.lib()
    t, prep = _case_prep("tiny/layer", 64)
    w = G.weights_from_oracle(prep)
    X = G.to_dev_bf16(t.X_bits)
    xq, xsf, T = L.act_buffers(w, 64)
    L.svdq_set_wait_limit_ns(2_000_000)
    try:
        L.svdq_debug_launch_stalled_act(w, X, xq, xsf, T)
        assert L.svdq_check_device_errors() == 5          # SVDQ_ERR_TIMEOUT
    finally:
        L.svdq_set_wait_limit_ns(2_000_000_000)
    # the context is still usable and the error word was cleared
    Y, _ = G.run_layer(w, t.X_bits)
    G.check_Y(Y, OS.linear(prep, t.X))


def test_full_size_layer_repeatable():
    """FLUX attn_out at full size (36 x 12 tiles over 148 persistent CTAs, so
    each CTA hands its accumulators and scale slots over between tiles): rows
    from the start, middle and end within the layer tolerance of the oracle,
    codes and scales of those rows bit-exact, and repeated launches bitwise
    equal."""
    L = G.lib()
    t, prep = _case_prep("flux/attn_out", 4608)
    w = G.weights_from_oracle(prep)
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    M, N = Y.shape
    rows = np.r_[0:40, 2300:2340, M - 40:M]
    G.check_codes(xq, xsf, t.X, prep.inv_lam, rows=rows)
    G.check_Y(Y[rows], OS.linear(prep, t.X, rows=rows))
    Y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        L.svdq_linear_w4a4(w, xq, xsf, T, M, Y2)
    assert L.svdq_check_device_errors() == 0
    np.testing.assert_array_equal(Y2.float().cpu().numpy(), Y)
