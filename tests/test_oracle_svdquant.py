"""Pins for the oracle's SVDQuant steps: closed forms, invariants and special
cases (SVDQuant, paperlayer.ai summary of arXiv 2411.05007v4)."""

import json
import os

import ml_dtypes
import numpy as np
import pytest

from oracle import codec as C
from oracle import formats as F
from oracle import svdquant as S
from synth import config_cases, make_fp4_grid_inputs, make_layer_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny():
    return make_layer_inputs(config_cases("tiny")[0])


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_paper_constants_fixture():
    with open(os.path.join(GOLDEN, "paper_constants.json")) as f:
        g = json.load(f)
    assert C.QMAX == g["fp4_e2m1_qmax"]["value"] == F.e2m1_decode(7)
    assert C.GROUP == g["nvfp4_group_size"]["value"]
    assert np.nanmax(F.e4m3_decode(np.arange(256))) == g["e4m3_max_finite"]["value"]
    assert g["default_rank_4bit"]["value"] in g["typical_ranks"]["value"]
    # signed k-bit integer qmax 2^(k-1)-1 (SVDQuant §3): 7 for INT4
    assert 2 ** (4 - 1) - 1 == g["int4_qmax"]["value"]


def test_smoothing_hand_example():
    act = np.array([4.0, 0.0, 9.0, 1.0], np.float32)
    W = np.array([[1.0, -2.0, 0.0, 4.0], [0.5, 1.0, 0.0, -1.0]], np.float32)
    lam, inv = S.smoothing_factors(act, W, 0.5)
    np.testing.assert_array_equal(lam, [2.0, 1.0, 1.0, 0.5])
    np.testing.assert_array_equal(inv, [0.5, 1.0, 1.0, 2.0])
    lam, _ = S.smoothing_factors(np.array([8.0], np.float32), np.array([[2.0]], np.float32), 0.25)
    assert lam[0] == np.float32(8 ** 0.25 / 2 ** 0.75)


def test_inverse_smoothing_is_the_reciprocal_of_the_stored_lambda():
    """inv_lam is fp32(1 / lam) of the fp32 lam the layer keeps.  Activation
    maximum 1, weight maximum 3: lam = 1/sqrt(3) rounds to fp32 0.57735026
    (0x3F13CD3A, 1.0e-8 low), whose reciprocal sqrt(3) (1 + 1.8e-8) rounds to
    1.7320509 (0x3FDDB3D8), one ulp above fp32(sqrt(3)) (0x3FDDB3D7), which
    the reciprocal of the unrounded lam would give."""
    lam, inv = S.smoothing_factors(np.array([1.0], np.float32), np.array([[3.0]], np.float32))
    assert lam.view(np.uint32)[0] == 0x3F13CD3A
    assert inv.view(np.uint32)[0] == 0x3FDDB3D8


def test_smoothing_preserves_product():
    t = _tiny()
    lam, inv = S.smoothing_factors(t.act_absmax, t.W)
    Xh = t.X.astype(np.float64) * inv.astype(np.float64)
    Wh = S.smooth_weight(t.W, inv)
    ref = t.X.astype(np.float64) @ t.W.astype(np.float64).T
    assert _rel(Xh @ Wh.T, ref) < 1e-12
    # smoothing shrinks the activation outliers
    assert np.abs(Xh).max() < np.abs(t.X).max()


def test_svd_split_known_spectrum():
    rng = np.random.default_rng(20)
    N, K, r = 40, 24, 5
    q1, _ = np.linalg.qr(rng.normal(size=(N, K)))
    q2, _ = np.linalg.qr(rng.normal(size=(K, K)))
    sig = np.linspace(10, 1, K)
    W_hat = q1 @ np.diag(sig) @ q2.T
    L1, L2, s = S.svd_split(W_hat, r)
    np.testing.assert_allclose(s, sig, rtol=1e-12)
    np.testing.assert_allclose((L1 @ L2).T, q1[:, :r] @ np.diag(sig[:r]) @ q2[:, :r].T, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(L1, axis=0), sig[:r], rtol=1e-12)   # S sits in L1
    np.testing.assert_allclose(L2 @ L2.T, np.eye(r), atol=1e-12)                   # L2 orthonormal rows


def test_eckart_young_and_reconstruction():
    t = _tiny()
    lam, inv = S.smoothing_factors(t.act_absmax, t.W)
    Wh = S.smooth_weight(t.W, inv)
    L1, L2, s = S.svd_split(Wh, 16)
    err2 = np.linalg.norm(Wh - (L1 @ L2).T) ** 2
    np.testing.assert_allclose(err2, np.sum(s[16:] ** 2), rtol=1e-9)
    prep = S.prepare(t.W, t.act_absmax, t.bias, 16)
    low = (prep.L1p / prep.inv_lam.astype(np.float64)[:, None]) @ prep.L2b
    recon = low.T + prep.R.astype(np.float64)
    assert _rel(recon, Wh) < 1e-6           # no quantization: L1 L2 + R = W_hat
    # the residual is much smaller than the smoothed weight (outliers absorbed)
    assert np.abs(prep.R).max() < 0.5 * np.abs(Wh).max()


def test_rank_zero_residual_is_smoothed_weight():
    t = _tiny()
    prep = S.prepare(t.W, t.act_absmax, t.bias, 0)
    _, inv = S.smoothing_factors(t.act_absmax, t.W)
    np.testing.assert_array_equal(prep.R, S.smooth_weight(t.W, inv).astype(np.float32))


def test_weight_factor_closed_forms():
    assert S.weight_factor(np.array([2688.0])) == 1.0
    assert S.weight_factor(np.array([2689.0])) == 2.0
    assert S.weight_factor(np.array([-1344.0])) == 0.5
    assert S.weight_factor(np.zeros(3)) == 1.0
    for m in [0.02, 0.3, 7.5, 1e-5, 123.0]:
        a = S.weight_factor(np.array([m]))
        assert np.log2(a) == int(np.log2(a))
        assert m / a <= 2688 < 2 * m / a


def _brute_w4a4(X, W, b):
    """Plain W4A4 (r = 0, lam = 1) with per-element loops and library casts."""
    def q(row):
        out = np.zeros(row.size)
        for g0 in range(0, row.size, 16):
            v = row[g0:g0 + 16]
            s = float((np.float32(np.abs(v).max()) / np.float32(6)).astype(ml_dtypes.float8_e4m3fn))
            if s == 0:
                continue
            r = np.float32(1) / np.float32(s)
            for i in range(16):
                out[g0 + i] = float((np.float32(v[i]) * r).astype(ml_dtypes.float4_e2m1fn)) * s
        return out
    aw = S.weight_factor(W)
    Qx = np.array([q(x) for x in X])
    Qw = np.array([q((w.astype(np.float64) / aw).astype(np.float32)) for w in W])
    Y = np.zeros((X.shape[0], W.shape[0]))
    for m in range(X.shape[0]):
        for n in range(W.shape[0]):
            Y[m, n] = aw * sum(Qx[m, k] * Qw[n, k] for k in range(X.shape[1])) + b[n]
    return Y


def test_rank0_unit_lambda_is_plain_w4a4():
    rng = np.random.default_rng(21)
    X = rng.normal(0, 1, (3, 64)).astype(np.float32)
    W = rng.normal(0, 0.02, (5, 64)).astype(np.float32)
    b = rng.normal(0, 0.01, 5).astype(np.float32)
    K = X.shape[1]
    prep = S.prepare_from_factors(W, np.ones(K, np.float32), np.zeros((K, 0)), np.zeros((0, 5)), b)
    np.testing.assert_array_equal(prep.R, W)
    np.testing.assert_allclose(S.linear(prep, X), _brute_w4a4(X, W, b), rtol=0, atol=1e-12)


def test_exact_product_on_fp4_grid():
    Xb, X, Wb, W = make_fp4_grid_inputs(32, 256, 48, seed=22)
    K = 256
    prep = S.prepare_from_factors(W, np.ones(K, np.float32), np.zeros((K, 0)), np.zeros((0, 48)), None)
    xc, xs = S.quantize_activations(X, prep.inv_lam)
    np.testing.assert_array_equal(C.dequantize_groups(xc, xs), X)
    np.testing.assert_array_equal(prep.alpha_w * C.dequantize_groups(prep.w_codes, prep.w_scales), W)
    np.testing.assert_array_equal(S.linear(prep, X), X.astype(np.float64) @ W.astype(np.float64).T)


@pytest.mark.parametrize("cfg", ["tiny", "pixart", "flux", "sdxl", "small_m_lora"])
def test_prop41_bound_holds(cfg):
    case = config_cases(cfg)[0]
    t = make_layer_inputs(case, M=min(case.M, 64))
    K = case.K
    W = t.W[:256].astype(np.float32)
    prep = S.prepare(W, t.act_absmax, None, case.rank)
    Xh = S.smooth_activations(t.X, prep.inv_lam).astype(np.float64)
    QX = C.dequantize_groups(*S.quantize_activations(t.X, prep.inv_lam))
    Rp = prep.Rp.astype(np.float64)
    QW = C.dequantize_groups(prep.w_codes, prep.w_scales)
    err = np.linalg.norm(Xh @ Rp.T - QX @ QW.T)
    assert 0 < err <= S.prop41_bound(Xh, Rp, QX, QW)
    assert K % 64 == 0


def test_prop41_bound_worked_example():
    """Prop. 4.1's right side on 1 x 2 matrices with round norms: ||X|| = 5,
    ||X - Q(X)|| = 4, ||W|| = 2, ||W - Q(W)|| = 1, so the bound is
    5 * 1 + 4 * (2 + 1) = 17; the product error |X W^T - Q(X) Q(W)^T| = 8 sits
    under it."""
    X, QX = np.array([[3.0, 4.0]]), np.array([[3.0, 0.0]])
    W, QW = np.array([[0.0, 2.0]]), np.array([[0.0, 1.0]])
    assert S.prop41_bound(X, W, QX, QW) == 17.0
    assert abs((X @ W.T - QX @ QW.T)[0, 0]) == 8.0


def test_method_beats_smoothing_beats_naive():
    t = _tiny()
    K = t.case.K
    ref = t.X.astype(np.float64) @ t.W.astype(np.float64).T + t.bias
    naive = S.prepare_from_factors(t.W, np.ones(K, np.float32), np.zeros((K, 0)),
                                   np.zeros((0, t.case.N)), t.bias)
    smooth = S.prepare(t.W, t.act_absmax, t.bias, 0)
    svdq = S.prepare(t.W, t.act_absmax, t.bias, 16)
    e_naive, e_smooth, e_svdq = (_rel(S.linear(p, t.X), ref) for p in (naive, smooth, svdq))
    assert e_svdq < e_smooth < e_naive


def test_lora_concat_equals_separate_sum_and_keeps_codes():
    t = make_layer_inputs(config_cases("small_m_lora")[2], M=8)
    W = t.W[:128]
    prep = S.prepare(W, t.act_absmax, t.bias[:128], 32)
    A, B = t.lora_A, t.lora_B[:, :128]
    both = S.attach_lora(prep, A, B, scale=0.75)
    np.testing.assert_array_equal(both.w_codes, prep.w_codes)
    np.testing.assert_array_equal(both.w_scales, prep.w_scales)
    assert both.alpha_w == prep.alpha_w and both.rank == 48
    sep = S.linear(prep, t.X) + 0.75 * (t.X.astype(np.float64) @ A) @ B
    assert _rel(S.linear(both, t.X), sep) < 1e-12


def _tiny_case():
    case = config_cases("tiny")[0]
    return case, make_layer_inputs(case)


def test_refinement_keeps_the_best_split_and_one_iteration_is_plain():
    """Step 4b (SVDQuant §4.2, refinement over several iterations): iters = 1 is
    the plain split; with more iterations the kept split is the one with the
    smallest residual quantization error, its first error is the plain split's,
    and the kept split still reconstructs W_hat exactly before quantization."""
    case, t = _tiny_case()
    plain = S.prepare(t.W, t.act_absmax, t.bias, case.rank)
    assert len(plain.refine_errors) == 1
    ref = S.prepare(t.W, t.act_absmax, t.bias, case.rank, iters=4)
    errs = ref.refine_errors
    assert len(errs) == 4
    assert errs[0] == pytest.approx(plain.refine_errors[0], rel=0, abs=0)
    q = S.fake_quantize_weights(ref.R)
    assert np.linalg.norm(ref.R.astype(np.float64) - q) == pytest.approx(min(errs), rel=1e-12)
    # the outlier layer gains from refinement (the qualitative claim of §4.2)
    assert min(errs) < 0.95 * errs[0]
    W_hat = S.smooth_weight(t.W, ref.inv_lam)
    low = (ref.L1p / ref.inv_lam.astype(np.float64)[:, None]) @ ref.L2b
    np.testing.assert_allclose(low.T + ref.R.astype(np.float64), W_hat, rtol=0, atol=1e-6)


def test_refinement_keeps_the_best_when_a_later_split_is_worse():
    """The iteration is not monotone: on this heavy-tailed weight (Gaussian
    cubed, rank 6, 8 iterations) the seventh split has the smallest residual
    quantization error and the eighth is worse, so keeping the best split and
    keeping the last one differ."""
    W = (np.random.default_rng(8).normal(0, 1, (32, 64)) ** 3).astype(np.float32)
    prep = S.prepare(W, np.ones(64, np.float32), None, 6, iters=8)
    errs = prep.refine_errors
    best = int(np.argmin(errs))
    assert best < len(errs) - 1 and errs[-1] > errs[best]
    kept = np.linalg.norm(prep.R.astype(np.float64) - S.fake_quantize_weights(prep.R))
    assert kept == pytest.approx(errs[best], rel=1e-12)


def test_refinement_of_an_exactly_low_rank_weight_stays_put():
    """A smoothed weight of rank r is split exactly by the SVD: every iterate's
    residual is only the 16-bit rounding of the factors, so all errors are tiny
    compared with quantizing the weight itself."""
    rng = np.random.default_rng(3)
    N, K, r = 96, 128, 8
    W = (rng.normal(0, 1, (N, r)) @ rng.normal(0, 0.05, (r, K))).astype(np.float32)
    absmax = np.ones(K, np.float32)
    prep = S.prepare(W, absmax, None, r, iters=3)
    W_hat = S.smooth_weight(W, prep.inv_lam)
    full = np.linalg.norm(W_hat - S.fake_quantize_weights(W_hat.astype(np.float32)))
    assert max(prep.refine_errors) < 1e-2 * full


def test_fake_quantize_weights_is_the_codec_round_trip():
    """Q(R) = alpha_w * dequantize(quantize(R / alpha_w)) (App. A.2: Q(R) = s_R Q_R);
    on a residual already on the FP4 grid times a power of two it is exact."""
    _, _, _, W = make_fp4_grid_inputs(16, 64, 32, seed=5)
    R = (W * np.float32(2.0 ** -9)).astype(np.float32)
    np.testing.assert_array_equal(S.fake_quantize_weights(R), R.astype(np.float64))


def test_alpha_search_scores_each_candidate_and_picks_the_smallest():
    """NEXT-3 (App. D migration strength): each candidate's error is the plain
    prepare-then-linear error at that alpha, the pick is the smallest, and on
    the outlier layer migrating some activation range into the weights beats
    none (alpha = 0 leaves the x40 outlier channels in the activations)."""
    case, t = _tiny_case()
    X = t.X[:32]
    alphas = [0.0, 0.5, 0.8]
    errs, best = S.search_alpha(t.W, X, t.bias, case.rank, alphas)
    exact = X.astype(np.float64) @ t.W.astype(np.float64).T + t.bias
    p5 = S.prepare(t.W, np.abs(X).max(axis=0), t.bias, case.rank, alpha=0.5)
    e5 = np.linalg.norm(S.linear(p5, X) - exact) / np.linalg.norm(exact)
    assert errs[1] == pytest.approx(e5, rel=1e-12)
    assert best == int(np.argmin(errs))
    assert errs[1] < 0.5 * errs[0]
