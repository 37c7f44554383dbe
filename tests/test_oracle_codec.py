"""Pins for the oracle's NVFP4 group codec and block-scale layout.

Group size 16, E4M3 scales (SVDQuant App. D), qmax 6 (SVDQuant §3).  The
group codec is checked against a loop-by-loop restatement that takes its
roundings from ml_dtypes casts, against brute-force nearest-code search, and
against closed-form special cases."""

import ml_dtypes
import numpy as np

from oracle import codec as C
from oracle import formats as F


def _groups(rng, n):
    g = rng.normal(0, 1, (n, 16)).astype(np.float32)
    g[: n // 8] *= np.float32(1e-3)                       # tiny scales (E4M3 subnormals)
    g[n // 8: n // 4] *= np.float32(300.0)               # large
    g[n // 4: n // 4 + 4] = 0.0                           # all-zero groups
    g[n // 4 + 4: n // 4 + 8] *= np.float32(1e-6)         # scale rounds to 0
    return g


def _brute_group(v):
    """One group, loop by loop, roundings from ml_dtypes casts."""
    amax = max(abs(float(x)) for x in v)
    q = np.float32(amax) / np.float32(6.0)
    s = float(np.float32(q).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)) if q <= 448 else 448.0
    if s == 0.0:
        return [0.0] * 16, 0.0
    r = np.float32(1.0) / np.float32(s)
    out = []
    for x in v:
        vp = np.float32(x) * r
        out.append(float(np.float32(vp).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)))
    return out, s


def test_group_codec_matches_loop_restatement():
    rng = np.random.default_rng(10)
    g = _groups(rng, 2000)
    codes, scales = C.quantize_groups(g.reshape(125, 256))
    deq = C.dequantize_groups(codes, scales).reshape(-1, 16)
    sv = F.e4m3_decode(scales).reshape(-1)
    for i in range(g.shape[0]):
        vals, s = _brute_group(g[i])
        assert sv[i] == s
        np.testing.assert_array_equal(deq[i], np.array(vals) * s)


def test_codes_are_nearest_grid_points():
    rng = np.random.default_rng(11)
    g = _groups(rng, 4096).reshape(256, 256)
    codes, scales = C.quantize_groups(g)
    s = F.e4m3_decode(scales)
    grid = F.e2m1_decode(np.arange(16))
    for i in range(0, 256, 17):
        for b in range(16):
            if s[i, b] == 0:
                assert np.all(codes[i, 16 * b:16 * b + 16] == 0)
                continue
            r = np.float32(1.0) / np.float32(s[i, b])
            vp = (g[i, 16 * b:16 * b + 16] * r).astype(np.float64)
            got = F.e2m1_decode(codes[i, 16 * b:16 * b + 16])
            best = np.abs(np.clip(vp, -6, 6)[:, None] - grid[None, :]).min(axis=1)
            np.testing.assert_array_equal(np.abs(np.clip(vp, -6, 6) - got), best)


def test_scale_is_rne_of_amax_over_qmax():
    rng = np.random.default_rng(12)
    g = _groups(rng, 4096)
    _, scales = C.quantize_groups(g.reshape(256, 256))
    amax = np.abs(g).max(axis=1)
    q = (amax / np.float32(6)).astype(np.float32)
    ref = q.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(F.e4m3_decode(scales.reshape(-1)), ref)


def test_scale_on_e4m3_midpoints():
    """The scale is E4M3_RNE of the correctly rounded quotient amax / 6, worked
    at the places where a slip shows.  amax = 6.375: the quotient 1.0625 is
    exact and halfway between the E4M3 values 1.0 and 1.125; the tie goes to the
    even mantissa, 1.0 (byte 0x38), so a scale nudged upward first would give
    1.125.  amax = 7.1249995 (0x40E3FFFF, one ulp below 7.125): the exact
    quotient is 1.1875 - 7.9e-8, which rounds to the fp32 value one ulp (1.2e-7)
    below the 1.125 / 1.25 midpoint 1.1875, so the scale is 1.125 (0x39);
    multiplying by fp32(1/6) = 1/6 + 5.0e-9 instead lands on 1.1875 itself and
    the tie would give 1.25."""
    g = np.zeros((2, 16), np.float32)
    g[0, 3] = 6.375
    g[1, 0] = np.array([0x40E3FFFF], np.uint32).view(np.float32)[0]
    _, scales = C.quantize_groups(g)
    np.testing.assert_array_equal(scales[:, 0], [0x38, 0x39])


def test_codes_multiply_by_the_reciprocal_of_the_scale():
    """Reading of the codec step: v' = fp32(v * fp32(1/s)).  A worked group where
    it differs from dividing by s: amax = 10.5 gives s = 10.5 / 6 = 1.75 (exact,
    E4M3 byte 0x3E) and fp32(1/1.75) = 4/7 + 2.6e-8.  For v = 3.0624998
    (0x4043FFFF, one ulp below 3.0625 = 1.75 * 1.75) the product is
    1.75 - 5.8e-8, within half an ulp (6.0e-8) of 1.75, so v' = 1.75 exactly,
    the E2M1 midpoint of 1.5 and 2.0, and the tie gives 2.0 (code 4); v / s
    would be 1.75 - 1.4e-7, which rounds below the midpoint to 1.5 (code 3).
    10.5 itself becomes 10.5 * fp32(1/1.75) = 6.0000005, saturated to 6 (code 7)."""
    g = np.zeros((1, 16), np.float32)
    g[0, 0] = 10.5
    g[0, 1] = np.array([0x4043FFFF], np.uint32).view(np.float32)[0]
    g[0, 2] = -g[0, 1]
    codes, scales = C.quantize_groups(g)
    assert scales[0, 0] == 0x3E
    np.testing.assert_array_equal(codes[0, :3], [0x7, 0x4, 0xC])
    assert np.all(codes[0, 3:] == 0)


def test_special_groups():
    v = np.zeros((1, 32), np.float32)
    v[0, 16:] = np.float32(1e-6)                   # amax/6 below half the smallest subnormal
    codes, scales = C.quantize_groups(v)
    assert np.all(codes == 0) and np.all(scales == 0)
    # A group holding exactly the grid times 2: scale 2, codes reproduce it exactly.
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0.5, -1, -1.5, -2, -3, -4, -6, 0], np.float32)
    codes, scales = C.quantize_groups((2 * grid)[None, :])
    assert F.e4m3_decode(scales[0, 0]) == 2.0
    np.testing.assert_array_equal(C.dequantize_groups(codes, scales)[0], 2 * grid)


def test_dequant_error_bound():
    # |v - q s| <= s * half grid gap at v' (0.25 below 2, 0.5 below 4, 1 up to 6),
    # plus the fp32 rounding of v' = v * (1/s).
    rng = np.random.default_rng(13)
    g = rng.normal(0, 1, (512, 256)).astype(np.float32)
    codes, scales = C.quantize_groups(g)
    deq = C.dequantize_groups(codes, scales)
    s = np.repeat(F.e4m3_decode(scales), 16, axis=1)
    vp = np.abs(g / s)
    half_gap = np.where(vp <= 2, 0.25, np.where(vp <= 4, 0.5, 1.0))
    over = np.maximum(vp - 6, 0)                  # saturation excess
    assert np.all(np.abs(g - deq) <= s * (half_gap + over) * (1 + 1e-6) + 1e-30)


def test_pack_nibble_order():
    codes = np.array([[1, 2, 0xF, 0x8]], np.uint8)
    np.testing.assert_array_equal(C.pack_codes(codes), [[0x21, 0x8F]])
    np.testing.assert_array_equal(C.unpack_codes(C.pack_codes(codes)), codes)


def test_scale_atom_layout_hand_offsets_and_roundtrip():
    rows, kb = 200, 8
    s = np.zeros((rows, kb), np.uint8)
    s[33, 5] = 7       # atom (0, 1): 512 + (33%32)*16 + (33//32)*4 + 5%4 = 533
    s[130, 2] = 9      # atom (1, 0): 2*512 + 2*16 + 0*4 + 2 = 1058
    s[199, 7] = 11     # atom (1, 1): 3*512 + 7*16 + 2*4 + 3 = 1659
    flat = C.scales_to_atoms(s)
    assert flat.size == 256 * kb
    assert flat[533] == 7 and flat[1058] == 9 and flat[1659] == 11
    assert np.count_nonzero(flat) == 3
    rng = np.random.default_rng(14)
    s = rng.integers(0, 256, (rows, kb)).astype(np.uint8)
    flat = C.scales_to_atoms(s)
    np.testing.assert_array_equal(C.atoms_to_scales(flat, rows, kb), s)
    assert np.all(C.atoms_to_scales(flat, 256, kb)[rows:] == 0)   # padded rows are zero
    # bijective on the padded index space: every one-hot lands on its own byte
    seen = set()
    for m in range(256):
        for j in range(kb):
            one = np.zeros((256, kb), np.uint8)
            one[m, j] = 1
            seen.add(int(np.flatnonzero(C.scales_to_atoms(one))[0]))
    assert seen == set(range(256 * kb))
