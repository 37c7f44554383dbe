"""NVFP4 group codec and the block-scale storage layout.

TEST INFRASTRUCTURE ONLY: part of the CPU oracle (see ``oracle/__init__.py``).

Codec (SVDQuant, paperlayer.ai summary of arXiv 2411.05007v4): per-group
symmetric quantization (App. D Implementation details), NVFP4 group size 16
with FP8 (E4M3) scales (App. D), FP4 qmax = 6 (§3 Quantization Preliminary),
and dequantization as "low-bit tensor times its scaling factor" (§3; also
Q(R) = s_R * Q_R in App. A.2).  For each group of 16 consecutive values v
along K:

  amax = max |v|                          (fp32, exact)
  s    = E4M3_rne_satfinite(fp32(amax / 6))
  if s decodes to 0: every code is +0, the scale byte is 0x00
  else: r = fp32(1 / s);  v' = fp32(v * r);  q = E2M1_rne_satfinite(v')

Each fp32 operation is one IEEE round-to-nearest operation (numpy float32
arithmetic).  The reciprocal-then-multiply order and the +0 code for values
that round to zero are readings of steps the pages leave open.

Packing: two codes per byte, element 2i in the low nibble and 2i+1 in the high
nibble; row-major, K contiguous.

Block-scale layout (a hardware contract of the Blackwell block-scaled MMA, not
in the pages): the [rows, K/16] scale matrix is cut into atoms of 128 rows x 4
scale columns (512 bytes).  Atoms are ordered K-atom fastest, then row-atom.
Inside an atom, row m (0..127) and column j (0..3) sit at byte
(m mod 32) * 16 + (m div 32) * 4 + j.  Rows are padded to a multiple of 128
with zero scales.
"""

from __future__ import annotations

import numpy as np

from .formats import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode

GROUP = 16
QMAX = 6.0


def quantize_groups(v) -> tuple:
    """Quantize float32 rows [R, K] (K % 16 == 0) group-wise along K.

    Returns (codes uint8 [R, K] one code per element, scales uint8 [R, K/16])."""
    v = np.asarray(v, dtype=np.float32)
    R, K = v.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 16")
    if not np.all(np.isfinite(v)):
        raise ValueError("non-finite input to the codec")
    g = v.reshape(R, K // GROUP, GROUP)
    amax = np.abs(g).max(axis=-1)                                    # exact
    s_code = e4m3_encode(amax / np.float32(QMAX))                    # fp32 div, then RNE
    s_val = e4m3_decode(s_code).astype(np.float32)                   # exact in fp32
    nz = s_val > 0
    recip = np.where(nz, np.float32(1.0) / np.where(nz, s_val, np.float32(1.0)),
                     np.float32(0.0)).astype(np.float32)
    vp = (g * recip[..., None]).astype(np.float32)                   # fp32 multiply
    codes = e2m1_encode(vp)
    codes = np.where(nz[..., None], codes, np.uint8(0)).astype(np.uint8)
    return codes.reshape(R, K), s_code.astype(np.uint8)


def dequantize_groups(codes, scales) -> np.ndarray:
    """float64 [R, K] values e2m1(code) * e4m3(scale)."""
    codes = np.asarray(codes)
    R, K = codes.shape
    vals = e2m1_decode(codes).reshape(R, K // GROUP, GROUP)
    return (vals * e4m3_decode(scales)[..., None]).reshape(R, K)


def pack_codes(codes) -> np.ndarray:
    """[R, K] codes -> [R, K/2] bytes, even element in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def padded_rows(rows: int) -> int:
    return -(-rows // 128) * 128


def scales_to_atoms(scales) -> np.ndarray:
    """Plain [R, K/16] scales -> flat atom-layout bytes of size padded_rows(R)*K/16."""
    s = np.asarray(scales, dtype=np.uint8)
    R, KB = s.shape
    if KB % 4:
        raise ValueError("K/16 must be a multiple of 4 (K % 64 == 0)")
    Rp = padded_rows(R)
    full = np.zeros((Rp, KB), dtype=np.uint8)
    full[:R] = s
    # rows m = ((mb*4 + m1)*32 + m0), columns kb = kq*4 + j
    t = full.reshape(Rp // 128, 4, 32, KB // 4, 4)          # mb, m1, m0, kq, j
    t = t.transpose(0, 3, 2, 1, 4)                            # mb, kq, m0, m1, j
    return np.ascontiguousarray(t).reshape(-1)


def atoms_to_scales(flat, rows: int, kb: int) -> np.ndarray:
    """Inverse of scales_to_atoms: flat atom bytes -> plain [rows, kb] scales."""
    Rp = padded_rows(rows)
    t = np.asarray(flat, dtype=np.uint8).reshape(Rp // 128, kb // 4, 32, 4, 4)
    t = t.transpose(0, 3, 2, 1, 4)                            # mb, m1, m0, kq, j
    return np.ascontiguousarray(t).reshape(Rp, kb)[:rows]
