"""Pins of the oracle's LayerNorm front end (fused activation path)."""

import numpy as np

from oracle import norm as ON
from oracle.formats import round_bf16


def test_row_stats_closed_forms():
    Z = np.array([[1.0, 3.0, 5.0, 7.0], [2.0, 2.0, 2.0, 2.0], [-1.0, 1.0, -1.0, 1.0]])
    mu, rstd = ON.row_stats(Z, eps=1e-6)
    np.testing.assert_allclose(mu, [4.0, 2.0, 0.0])
    np.testing.assert_allclose(rstd, [1 / np.sqrt(5.0 + 1e-6), 1 / np.sqrt(1e-6), 1 / np.sqrt(1.0 + 1e-6)])


def test_normalize_worked_row():
    """mu = 4, rstd = 0.5: (z - 4) * 0.5 * a + c, all exact, then bf16."""
    Z = np.array([[1.0, 3.0, 5.0, 7.0]], np.float32)
    x = ON.normalize(Z, [4.0], [0.5], a=[1.0, 2.0, -1.0, 0.5], c=[0.0, 1.0, 0.25, -3.0])
    np.testing.assert_array_equal(x, [[-1.5, 0.0, -0.25, -2.25]])


def test_normalize_rounds_to_bf16_once():
    """A value that needs more than 8 significant bits is rounded (ties to even)."""
    Z = np.array([[1.0 + 2.0 ** -8, 0.0]], np.float32)     # halfway between two bf16 values at 1
    x = ON.normalize(Z, [0.0], [1.0], a=[1.0, 1.0], c=[0.0, 0.0])
    assert x[0, 0] == 1.0                                   # tie to even
    Z = np.array([[1.0 + 3 * 2.0 ** -8, 0.0]], np.float32)
    assert ON.normalize(Z, [0.0], [1.0], [1.0, 1.0], [0.0, 0.0])[0, 0] == 1.0 + 2.0 ** -6


def test_normalized_rows_have_zero_mean_unit_variance():
    rng = np.random.default_rng(2)
    Z = (rng.standard_normal((8, 512)) * 3 + 5).astype(np.float32)
    mu, rstd = ON.row_stats(Z, 1e-6)
    x = ON.normalize(Z, mu, rstd, np.ones(512), np.zeros(512)).astype(np.float64)
    np.testing.assert_allclose(x.mean(axis=1), 0.0, atol=2e-3)
    np.testing.assert_allclose(x.var(axis=1), 1.0, rtol=5e-3)
    np.testing.assert_array_equal(x, round_bf16(x))       # bf16 values


def test_normalize_rounds_each_step_in_fp32():
    """Each of the four steps rounds to fp32 before the last rounding to bf16.
    Worked element (fp32 bit patterns): z = 0x4067A449 (3.6194022),
    mu = 0xBF156111 (-0.58351237), rstd = 0x3F8D8666, a = 0x3F84A6F0,
    c = 0x3C4837D2.  The fp32 steps give z - mu = 4.2029147 (the exact
    difference 4.2029145 rounds up), times rstd 4.6470118, times a 4.815905,
    plus c 4.8281255: above the midpoint 4.828125 of the bf16 values 4.8125
    and 4.84375, so x = 4.84375.  Kept in float64 until the product with a,
    the same element gives 4.8159046 + c = 4.828125, the midpoint itself,
    which ties to the even 4.8125."""
    bits = np.array([0x4067A449, 0xBF156111, 0x3F8D8666, 0x3F84A6F0, 0x3C4837D2], np.uint32)
    z, mu, rstd, a, c = bits.view(np.float32)
    x = ON.normalize(np.array([[z]]), np.array([mu]), np.array([rstd]), np.array([a]), np.array([c]))
    assert x[0, 0] == np.float32(4.84375)
