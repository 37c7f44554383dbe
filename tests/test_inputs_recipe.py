"""The synthetic inputs follow their stated recipe: shapes of the configured
layers, round(frac * K) outlier channels scaled by the config's factor, bf16
values, determinism, and a weight side (and leading rows of X) that does not
depend on the token count M."""

import numpy as np
import pytest

from synth import config_cases, make_layer_inputs
from synth.workloads import bf16_bits_to_f32

SHAPES = {
    "tiny": [(64, 256, 256)],
    "pixart": [(4096, 1152, 1152), (4096, 1152, 4608), (4096, 4608, 1152)],
    "flux": [(4608, 3072, 3072), (4608, 3072, 9216), (4608, 3072, 12288), (4608, 12288, 3072)],
    "sdxl": [(8192, 640, 640), (8192, 640, 5120), (8192, 5120, 640), (2048, 1280, 1280), (2048, 1280, 10240),
             (2048, 10240, 1280)],
    "small_m_lora": [(m, 3072, n) for m in (1, 16, 256) for n in (3072, 12288)],
}
# outlier channels: 1 % of K (PixArt, SDXL), 0.5 % (FLUX, small M), rounded; tiny has 4
OUTLIERS = {"tiny": lambda K: 4, "pixart": lambda K: round(0.01 * K), "sdxl": lambda K: round(0.01 * K),
            "flux": lambda K: round(0.005 * K), "small_m_lora": lambda K: round(0.005 * K)}
FACTOR = {"tiny": 40.0, "pixart": 30.0, "sdxl": 30.0, "flux": 50.0, "small_m_lora": 50.0}


def test_configured_shapes_and_ranks():
    for name, shapes in SHAPES.items():
        cases = config_cases(name)
        assert [(c.M, c.K, c.N) for c in cases] == shapes
        for c in cases:
            assert c.rank == (16 if name == "tiny" else 32)
            assert c.lora_rank == (16 if name == "small_m_lora" else 0)
            assert c.K % 64 == 0 and c.N % 16 == 0
    assert [round(0.005 * 3072), round(0.005 * 12288), round(0.01 * 1152)] == [15, 61, 12]


@pytest.mark.parametrize("name", list(SHAPES))
def test_outlier_channels_follow_the_recipe(name):
    c = config_cases(name)[0]
    t = make_layer_inputs(c, M=256)                       # outlier channels do not depend on M
    assert c.x_outlier_count == OUTLIERS[name](c.K) and c.x_outlier_scale == FACTOR[name]
    # N(0, 1) columns stay below ~5.5 over 256 rows; scaled ones reach ~factor * 2
    colmax = np.abs(t.X).max(axis=0)
    big = np.flatnonzero(colmax > 8.0)
    assert len(big) == c.x_outlier_count
    np.testing.assert_array_equal(t.act_absmax, colmax)
    if name == "tiny":
        wmax = np.abs(t.W).max(axis=0)
        assert np.sum(wmax > 0.2) == c.w_outlier_count == 4


def test_values_are_bf16_and_draws_repeat():
    c = config_cases("tiny")[0]
    a, b = make_layer_inputs(c), make_layer_inputs(c)
    for f in ["X_bits", "W_bits", "bias_bits"]:
        np.testing.assert_array_equal(getattr(a, f), getattr(b, f))
    np.testing.assert_array_equal(a.X, bf16_bits_to_f32(a.X_bits))
    np.testing.assert_array_equal(a.W, bf16_bits_to_f32(a.W_bits))
    assert abs(float(a.W.std()) - 0.02 * np.sqrt(1 + 4 * (20 ** 2 - 1) / 256)) < 0.01


def test_weights_and_leading_rows_do_not_depend_on_m():
    c = config_cases("small_m_lora")[4]                 # M = 256, N = 3072
    full, small = make_layer_inputs(c), make_layer_inputs(c, M=16)
    np.testing.assert_array_equal(full.W_bits, small.W_bits)
    np.testing.assert_array_equal(full.lora_A_bits, small.lora_A_bits)
    np.testing.assert_array_equal(full.lora_B_bits, small.lora_B_bits)
    np.testing.assert_array_equal(full.X_bits[:16], small.X_bits)
    assert full.lora_A.shape == (3072, 16) and full.lora_B.shape == (16, 3072)
