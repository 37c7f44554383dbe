"""Number formats of the SVDQuant NVFP4 path, written out from their bit definitions.

TEST INFRASTRUCTURE ONLY: this module belongs to the CPU oracle.  Only the
tests, the smoke check and the benchmark's CPU baseline may import it; the
library never does.

Formats (SVDQuant, paperlayer.ai summary of arXiv 2411.05007v4):
  * E2M1 ("4-bit floating point with a 1-bit mantissa and 2-bit exponent, qmax
    is 6"; §3 Quantization Preliminary).  1 sign bit, 2 exponent bits with bias
    1, 1 mantissa bit; exponent field 0 encodes the subnormals 0 and 0.5.
  * E4M3 ("NVFP4 uses group size 16 with FP8 scales"; App. D Implementation
    details).  1 sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent
    field 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; no infinities,
    so the largest finite value is 448.
  * bf16 (the 16-bit format of the low-rank branch, §4.2): the top 16 bits of
    an IEEE fp32 value.

Rounding is round-to-nearest, ties to the even significand, with saturation to
the largest finite magnitude ("satfinite").  Values are computed in float64,
where every comparison below is exact.
"""

from __future__ import annotations

import numpy as np


def e2m1_decode(codes) -> np.ndarray:
    """Value of each 4-bit E2M1 code (0..15) as float64."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.exp2(e - 1.0))
    return sign * mag


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 byte (0..255) as float64 (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def _positive_table(decode, nbits_mag):
    codes = np.arange(1 << nbits_mag)
    vals = decode(codes)
    ok = np.isfinite(vals)
    codes, vals = codes[ok], vals[ok]
    order = np.argsort(vals, kind="stable")
    return vals[order], codes[order]


_E2M1_VALS, _E2M1_CODES = _positive_table(e2m1_decode, 3)   # 0 .. 6
_E4M3_VALS, _E4M3_CODES = _positive_table(e4m3_decode, 7)   # 0 .. 448


def _encode_rne_satfinite(x, vals, codes):
    """Nearest representable magnitude, ties to the even code, clamp to max."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input to the 4/8-bit encoder")
    a = np.minimum(np.abs(x), vals[-1])
    hi_i = np.searchsorted(vals, a, side="left")          # first vals >= a
    hi_i = np.minimum(hi_i, len(vals) - 1)
    lo_i = np.where(vals[hi_i] == a, hi_i, np.maximum(hi_i - 1, 0))
    lo, hi = vals[lo_i], vals[hi_i]
    two_a, mid2 = 2.0 * a, lo + hi                        # exact in float64
    pick_hi = (two_a > mid2) | ((two_a == mid2) & (codes[hi_i] % 2 == 0) & (lo_i != hi_i))
    code = np.where(pick_hi, codes[hi_i], codes[lo_i])
    return code.astype(np.int64), np.signbit(x)


def e2m1_encode(x) -> np.ndarray:
    """E2M1 code of each value: RNE, satfinite at 6.  A value whose rounded
    magnitude is 0 gets the code +0 (0x0) whatever its sign."""
    mag_code, neg = _encode_rne_satfinite(x, _E2M1_VALS, _E2M1_CODES)
    code = np.where(neg & (mag_code != 0), mag_code | 0x8, mag_code)
    return code.astype(np.uint8)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 byte of each value: RNE, satfinite at 448 (sign kept, -0 -> 0x80)."""
    mag_code, neg = _encode_rne_satfinite(x, _E4M3_VALS, _E4M3_CODES)
    code = np.where(neg, mag_code | 0x80, mag_code)
    return code.astype(np.uint8)


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 (or float64 via float32, which rounds correctly here since
    24 >= 2*8+2 bits) to bf16, ties to even; returns the uint16 bit patterns."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if not np.all(np.isfinite(f)):
        raise ValueError("non-finite input to bf16 rounding")
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f64(bits) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """float64 value of bf16(x)."""
    return bf16_bits_to_f64(f32_to_bf16_bits(x))
