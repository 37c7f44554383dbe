"""Helpers shared by the GPU parity tests: build library weights from the
oracle's factors (so both sides quantize the same residual), run the two
kernels, and compare with the oracle."""

from __future__ import annotations

import numpy as np
import torch

from oracle import codec as OC
from oracle import svdquant as OS
from synth import f32_to_bf16_bits

REL_FRO_TOL = 2e-3       # relative Frobenius error of Y against the oracle
ELEM_TOL = 1e-2          # per element |dY| <= ELEM_TOL * max(1, |Y_ref|)


def lib():
    import rank_outlier_gemm_b200 as L
    return L


def weights_from_oracle(prep: OS.Prepared):
    """Library handle holding exactly the oracle's split (before any LoRA)."""
    L = lib()
    r = prep.rank - prep.lora_rank
    L1p = f32_to_bf16_bits(prep.L1p[:, :r].astype(np.float32)) if r else None
    L2 = f32_to_bf16_bits(prep.L2b[:r].astype(np.float32)) if r else None
    return L.svdq_weights_from_factors(prep.N, prep.K, r, prep.inv_lam, L1p, L2, prep.R,
                                       prep.bias.astype(np.float32))


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def run_act(w, X_bits: np.ndarray):
    L = lib()
    M = X_bits.shape[0]
    X = to_dev_bf16(X_bits)
    xq, xsf, T = L.act_buffers(w, M)
    L.svdq_quantize_act_lowrank_down(w, X, xq, xsf, T)
    assert L.svdq_check_device_errors() == 0
    return X, xq, xsf, T


def run_layer(w, X_bits: np.ndarray):
    L = lib()
    X, xq, xsf, T = run_act(w, X_bits)
    M = X_bits.shape[0]
    Y = torch.empty((M, w.info["N"]), dtype=torch.bfloat16, device="cuda")
    L.svdq_linear_w4a4(w, xq, xsf, T, M, Y)
    assert L.svdq_check_device_errors() == 0
    return Y.float().cpu().numpy().astype(np.float64), (xq, xsf, T)


def check_codes(xq: torch.Tensor, xsf: torch.Tensor, X: np.ndarray, inv_lam, rows=None):
    """Activation codes and scales bit-exact against the oracle (optionally for a row sample)."""
    M, K = X.shape
    q = xq.cpu().numpy().reshape(M, K // 2)
    sf = OC.atoms_to_scales(xsf.cpu().numpy(), M, K // 16)
    idx = np.arange(M) if rows is None else np.asarray(rows)
    codes, scales = OS.quantize_activations(X[idx], inv_lam)
    np.testing.assert_array_equal(q[idx], OC.pack_codes(codes))
    np.testing.assert_array_equal(sf[idx], scales)
    if rows is None:  # padded rows of the last atom carry zero scales
        full = xsf.cpu().numpy()
        ref = OC.scales_to_atoms(scales)
        np.testing.assert_array_equal(full, ref)


def check_T(T: torch.Tensor, X: np.ndarray, prep: OS.Prepared, rows=None):
    """T_hi + T_lo against X L1' in float64 (fp32 accumulation tolerance)."""
    if T is None:
        return
    M = X.shape[0]
    idx = np.arange(M) if rows is None else np.asarray(rows)
    r = prep.rank
    rp = T.shape[1] // 2
    t = T.float().cpu().numpy().astype(np.float64)[idx]
    hi = np.concatenate([t[:, 32 * c: 32 * c + 16] for c in range(rp // 16)], axis=1)
    lo = np.concatenate([t[:, 32 * c + 16: 32 * c + 32] for c in range(rp // 16)], axis=1)
    got = (hi + lo)[:, :r]
    ref = X[idx].astype(np.float64) @ prep.L1p
    bound = 1e-4 * (np.abs(X[idx]).astype(np.float64) @ np.abs(prep.L1p)) + 1e-6
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))
    assert np.all((hi + lo)[:, r:] == 0)


def check_Y(Y: np.ndarray, ref: np.ndarray):
    rel = np.linalg.norm(Y - ref) / np.linalg.norm(ref)
    el = np.max(np.abs(Y - ref) / np.maximum(1.0, np.abs(ref)))
    assert np.all(np.isfinite(Y))
    assert rel <= REL_FRO_TOL, f"relative Frobenius error {rel:.3e}"
    assert el <= ELEM_TOL, f"max per-element error {el:.3e}"
    return rel, el
