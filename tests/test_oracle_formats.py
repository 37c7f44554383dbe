"""Pins for the oracle's number formats against library casts and brute force.

E2M1 (qmax 6, SVDQuant §3) and E4M3 scales (NVFP4, SVDQuant App. D) are pinned
against ml_dtypes / torch casts, which implement the same formats
independently, and against exhaustive nearest-value search."""

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats as F


def _ml_e2m1_value(codes):
    return np.asarray(codes, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def _ml_e2m1_cast(x):
    return np.asarray(x, np.float32).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)


def _ml_e4m3_cast(x):
    return np.asarray(x, np.float32).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)


def test_e2m1_decode_all_codes_match_ml_dtypes():
    codes = np.arange(16)
    np.testing.assert_array_equal(F.e2m1_decode(codes), _ml_e2m1_value(codes))
    assert F.e2m1_decode(7) == 6.0  # qmax = 6 for FP4 (SVDQuant §3)


def test_e4m3_decode_all_bytes_match_torch_and_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_decode(codes)
    t = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(t))
    ok = ~np.isnan(ours)
    np.testing.assert_array_equal(ours[ok], t[ok])
    np.testing.assert_array_equal(ours[ok], ml[ok])
    assert np.nanmax(ours) == 448.0
    assert F.e4m3_decode(1) == 2.0 ** -9


def _midpoints(vals):
    v = np.unique(np.abs(vals[np.isfinite(vals)]))
    return (v[:-1] + v[1:]) / 2


def test_e4m3_encode_matches_ml_dtypes_rne():
    rng = np.random.default_rng(1)
    mags = np.exp2(rng.uniform(-12, np.log2(448), 200000))
    x = np.concatenate([mags, -mags, _midpoints(F.e4m3_decode(np.arange(128))),
                        np.nextafter(_midpoints(F.e4m3_decode(np.arange(128))), 0),
                        [0.0, 448.0, 450.0, 463.9]]).astype(np.float32)
    ours = F.e4m3_decode(F.e4m3_encode(x))
    np.testing.assert_array_equal(ours, _ml_e4m3_cast(x))


def test_e4m3_encode_saturates():
    x = np.array([464.0, 480.0, 1e6, -1e6], np.float32)
    np.testing.assert_array_equal(F.e4m3_decode(F.e4m3_encode(x)), [448, 448, 448, -448])


def test_e2m1_encode_matches_ml_dtypes_rne():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.uniform(-7, 7, 200000), _midpoints(F.e2m1_decode(np.arange(8))),
                        -_midpoints(F.e2m1_decode(np.arange(8))), [8.0, -9.0, 1e-30]])
    x = x.astype(np.float32)
    ours = F.e2m1_decode(F.e2m1_encode(x))
    ref = _ml_e2m1_cast(x)
    np.testing.assert_array_equal(np.abs(ours), np.abs(ref))
    # sign kept for non-zero results; rounded-to-zero values are +0 (code 0)
    nz = ref != 0
    np.testing.assert_array_equal(np.sign(ours[nz]), np.sign(ref[nz]))
    assert np.all(F.e2m1_encode(x[~nz]) == 0)


def test_e2m1_ties_to_even_table():
    # Midpoints of the E2M1 grid and the even neighbour each must round to.
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for t, want in ties.items():
        assert F.e2m1_decode(F.e2m1_encode(np.float32(t))) == want
        assert F.e2m1_decode(F.e2m1_encode(np.float32(-t))) == -want


def test_e2m1_brute_force_nearest():
    rng = np.random.default_rng(3)
    x = rng.uniform(-6.5, 6.5, 1_000_000).astype(np.float32).astype(np.float64)
    grid = F.e2m1_decode(np.arange(16))
    dist = np.abs(x[:, None] - grid[None, :])
    best = dist.min(axis=1)
    got = F.e2m1_decode(F.e2m1_encode(x))
    sat = np.abs(x) > 6
    np.testing.assert_array_equal(np.abs(x - got)[~sat], best[~sat])
    np.testing.assert_array_equal(got[sat], np.sign(x[sat]) * 6)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.normal(0, 1, 100000), rng.normal(0, 1e-3, 1000) * 1e-30,
                        np.exp2(rng.uniform(-120, 120, 10000))]).astype(np.float32)
    # exact ties: a bf16 value plus half an ulp
    base = torch.from_numpy(rng.normal(0, 1, 1000).astype(np.float32)).to(torch.bfloat16)
    tie = (base.view(torch.int16).numpy().astype(np.int64) & 0xFFFF).astype(np.uint32) << 16
    tie = (tie | 0x8000).view(np.float32)
    x = np.concatenate([x, tie])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(F.f32_to_bf16_bits(x), ref)
