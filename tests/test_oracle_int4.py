"""Pins of the oracle's INT4 variant (group 64, bf16 scales, qmax 7) against
hand-worked groups, closed forms, brute force and exact products."""

import json
import os

import numpy as np
import pytest

from oracle import int4 as OI
from oracle import svdquant as OS
from synth import make_int4_grid_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paper_constants.json")


def _group(vals):
    g = np.zeros((1, 64), np.float32)
    g[0, : len(vals)] = vals
    return g


def test_constants_match_the_pages():
    c = json.load(open(GOLDEN))
    assert OI.QMAX == c["int4_qmax"]["value"] == 2 ** (4 - 1) - 1
    assert OI.GROUP == c["int4_group_size"]["value"]


def test_worked_group_with_unit_scale():
    """amax = 7 gives s = 1, so the codes are the values rounded half to even."""
    q, s = OI.quantize_groups(_group([7.0, -3.5, 0.5, 2.5, 1.5, -0.5, -6.5, 3.25, -7.0, 0.75]))
    assert s.shape == (1, 1) and s[0, 0] == 1.0
    np.testing.assert_array_equal(q[0, :10], [7, -4, 0, 2, 2, 0, -6, 3, -7, 1])
    assert not q[0, 10:].any()


def test_worked_group_with_scale_two():
    q, s = OI.quantize_groups(_group([14.0, 3.0, -5.0, 1.0, -13.0]))
    assert s[0, 0] == 2.0
    np.testing.assert_array_equal(q[0, :5], [7, 2, -2, 0, -6])   # 1.5 -> 2, -2.5 -> -2, 0.5 -> 0, -6.5 -> -6


@pytest.mark.parametrize("amax,scale", [(7 * (1 + 2.0 ** -9), 1.0),          # below half an ulp
                                        (7 * (1 + 2.0 ** -8), 1.0),          # tie to even (down)
                                        (7 * (1 + 3 * 2.0 ** -8), 1.015625),  # tie to even (up)
                                        (7 * 3.0, 3.0)])
def test_scale_is_the_bf16_rounding_of_amax_over_7(amax, scale):
    q, s = OI.quantize_groups(_group([amax, -amax / 2]))
    assert s[0, 0] == scale
    assert q[0, 0] == 7                     # the maximum always takes the extreme code


def test_zero_group():
    q, s = OI.quantize_groups(np.zeros((2, 128), np.float32))
    assert not q.any() and not s.any()


def test_roundtrip_error_within_half_a_step():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal((64, 512)) * np.exp2(rng.integers(-20, 20, (64, 1)))).astype(np.float32)
    q, s = OI.quantize_groups(v)
    assert np.abs(q).max() <= 7
    err = np.abs(v.astype(np.float64) - OI.dequantize_groups(q, s))
    step = np.repeat(s, 64, axis=1)
    assert np.all(err <= 0.5001 * step)
    # each group's largest magnitude is coded +-7
    g = np.abs(v).reshape(64, 8, 64)
    qa = np.take_along_axis(np.abs(q.reshape(64, 8, 64)), g.argmax(-1)[..., None], -1)
    assert np.all(qa == 7)


def test_brute_force_codes_are_nearest():
    """Each code is the integer in -7..7 nearest to v * fp32(1/s) (ties even)."""
    rng = np.random.default_rng(5)
    v = rng.uniform(-3, 3, (8, 128)).astype(np.float32)
    q, s = OI.quantize_groups(v)
    for r in range(8):
        for k in range(128):
            sv = np.float32(s[r, k // 64])
            t = np.float32(v[r, k] * (np.float32(1.0) / sv))
            cand = np.arange(-7, 8)
            d = np.abs(cand - np.float64(t))
            best = cand[d == d.min()]
            assert q[r, k] == (best[0] if len(best) == 1 else best[best % 2 == 0][0])


def test_pack_unpack():
    rng = np.random.default_rng(7)
    q = rng.integers(-7, 8, (5, 128)).astype(np.int8)
    p = OI.pack_codes(q)
    assert p.shape == (5, 64) and p.dtype == np.uint8
    np.testing.assert_array_equal(OI.unpack_codes(p), q)
    # nibbles (two's complement) 1, F, 9, 7, 0, 2, 3, D; evens 1 9 0 3 -> 0x3091, odds F 7 2 D -> 0xD27F
    np.testing.assert_array_equal(OI.pack_codes(np.array([[1, -1, -7, 7, 0, 2, 3, -3]], np.int8)),
                                  [[0x91, 0x30, 0x7F, 0xD2]])


def test_scale_bits_roundtrip():
    s = np.array([[1.0, 0.5, 3.0, 1.015625, 2.0 ** -100]])
    np.testing.assert_array_equal(OI.scales_from_bits(OI.scales_to_bits(s)), s)


def _rank0(W):
    K = W.shape[1]
    ones = np.ones(K, np.float32)
    base = OS.prepare_from_factors(OS.smooth_weight(W, ones), ones, np.zeros((K, 0)), np.zeros((0, W.shape[0])), None)
    return OI.from_base(base)


@pytest.mark.parametrize("M,K,N", [(8, 128, 16), (5, 1024, 24)])
def test_layer_exact_on_int4_grid(M, K, N):
    """Inputs on the INT4 grid quantize exactly, so the rank-0 layer equals X W^T."""
    _, X, _, W = make_int4_grid_inputs(M, K, N, seed=M + K)
    prep = _rank0(W)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_array_equal(OI.linear(prep, X), exact)
    np.testing.assert_array_equal(OI.dequantize_groups(prep.w_codes, prep.w_scales), W.astype(np.float64))


def test_layer_low_rank_and_bias_terms():
    """The INT4 layer adds the same low-rank branch and bias as the NVFP4 one;
    with an exactly rank-r weight the residual is ~0 and Y ~ X W^T + b."""
    rng = np.random.default_rng(11)
    K, N, r = 128, 32, 8
    W = (rng.standard_normal((N, r)) @ rng.standard_normal((r, K)) * 0.05).astype(np.float32)
    X = rng.standard_normal((6, K)).astype(np.float32)
    b = rng.standard_normal(N).astype(np.float32) * 0.1
    prep = OI.prepare(W, np.abs(X).max(0), b, r)
    ref = X.astype(np.float64) @ W.astype(np.float64).T + b
    y = OI.linear(prep, X)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 2e-2
    # the INT4 main term alone is the codec applied to R and X_hat
    xc, xs = OI.quantize_activations(X, prep.inv_lam)
    main = OI.dequantize_groups(xc, xs) @ OI.dequantize_groups(prep.w_codes, prep.w_scales).T
    np.testing.assert_allclose(y - main, OS.lowrank_down(X, prep.base) @ prep.L2b + b, rtol=0, atol=1e-12)


def test_lora_on_the_int4_layer():
    """A LoRA attached to the INT4 layer (SVDQuant §2, §5.2: absorbed into the
    low-rank branch without re-quantizing R) adds scale (X A) B to the output
    and leaves the residual's codes and scales as they were."""
    rng = np.random.default_rng(17)
    K, N, r, rl = 128, 32, 8, 4
    W = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    X = rng.standard_normal((6, K)).astype(np.float32)
    A = (rng.standard_normal((K, rl)) * 0.1).astype(np.float32)
    B = (rng.standard_normal((rl, N)) * 0.1).astype(np.float32)
    prep = OI.prepare(W, np.abs(X).max(0), None, r)
    withl = OI.attach_lora(prep, A, B, scale=0.5)
    np.testing.assert_array_equal(withl.w_codes, prep.w_codes)
    np.testing.assert_array_equal(withl.w_scales, prep.w_scales)
    assert withl.rank == r + rl
    added = 0.5 * (X.astype(np.float64) @ A.astype(np.float64)) @ B.astype(np.float64)
    np.testing.assert_allclose(OI.linear(withl, X) - OI.linear(prep, X), added, rtol=0, atol=1e-12)


def test_prop41_bound_holds_for_int4():
    rng = np.random.default_rng(13)
    X = rng.standard_normal((16, 256)).astype(np.float32)
    W = (rng.standard_normal((24, 256)) * 0.1).astype(np.float32)
    QX = OI.dequantize_groups(*OI.quantize_groups(X))
    QW = OI.dequantize_groups(*OI.quantize_groups(W))
    lhs = np.linalg.norm(X.astype(np.float64) @ W.T.astype(np.float64) - QX @ QW.T)
    assert lhs <= OS.prop41_bound(X.astype(np.float64), W.astype(np.float64), QX, QW)
