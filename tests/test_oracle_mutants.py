"""The oracle's pins against planted mistakes.

Each mutant below is one plausible slip in the oracle: a flipped tie rule, a
swapped index or operand, a dropped term, a wrong constant.  It is planted in
a copy of ``oracle/`` (on the CPU, in a temporary directory); the pin tests of
the affected module then run against that copy and must fail.  A mutant that
every pin lets through would mean a step of the oracle that nothing outside it
checks, so the test lists the survivors.

Edits are textual and each must match its source exactly once, so a change to
the oracle that moves a line makes the mutant fail loudly here instead of
silently testing nothing."""

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FMT = ["test_oracle_formats.py", "test_oracle_codec.py"]
COD = ["test_oracle_codec.py", "test_oracle_svdquant.py"]
SVD = ["test_oracle_svdquant.py"]
I4 = ["test_oracle_int4.py"]
NRM = ["test_oracle_norm.py"]

# (name, file under oracle/, [(text, replacement), ...], pin files to run)
MUTANTS = [
    # number formats
    ("ties_to_odd", "formats.py", [("(codes[hi_i] % 2 == 0)", "(codes[hi_i] % 2 == 1)")], FMT),
    ("ties_away_from_zero", "formats.py",
     [("((two_a == mid2) & (codes[hi_i] % 2 == 0) & (lo_i != hi_i))", "((two_a == mid2) & (lo_i != hi_i))")], FMT),
    ("e4m3_exponent_bias_8", "formats.py", [("np.exp2(e - 7.0)", "np.exp2(e - 8.0)")], FMT),
    ("e4m3_subnormal_step", "formats.py", [("(m / 8.0) * 2.0 ** -6", "(m / 8.0) * 2.0 ** -7")], FMT),
    ("e2m1_subnormal_value", "formats.py", [("m * 0.5, (1.0 + m / 2.0)", "m * 0.25, (1.0 + m / 2.0)")], FMT),
    ("e2m1_negative_zero_code", "formats.py",
     [("np.where(neg & (mag_code != 0), mag_code | 0x8, mag_code)", "np.where(neg, mag_code | 0x8, mag_code)")], FMT),
    ("bf16_truncates", "formats.py", [("((u + 0x7FFF + lsb) >> 16)", "(u >> 16)")], FMT),
    ("bf16_ties_up", "formats.py", [("((u + 0x7FFF + lsb) >> 16)", "((u + 0x8000) >> 16)")], FMT),
    ("e4m3_nan_as_480", "formats.py", [("mag = np.where((e == 15) & (m == 7), np.nan, mag)", "mag = mag")], FMT),
    ("e2m1_exponent_bias_2", "formats.py", [("np.exp2(e - 1.0)", "np.exp2(e - 2.0)")], FMT),
    # NVFP4 group codec and scale layout
    ("codec_qmax_7", "codec.py", [("QMAX = 6.0", "QMAX = 7.0")], COD),
    ("codec_scale_by_reciprocal", "codec.py",
     [("e4m3_encode(amax / np.float32(QMAX))", "e4m3_encode(amax * np.float32(1.0 / QMAX))")], COD),
    ("codec_divides_by_scale", "codec.py",
     [("vp = (g * recip[..., None]).astype(np.float32)",
       "vp = (g / np.where(nz, s_val, np.float32(1.0))[..., None]).astype(np.float32)")], COD),
    ("codec_scale_rounded_up", "codec.py",
     [("s_code = e4m3_encode(amax / np.float32(QMAX))",
       "s_code = e4m3_encode(np.nextafter(amax / np.float32(QMAX), np.float32(np.inf)))")], COD),
    ("codec_nibble_order", "codec.py",
     [("(c[:, 0::2] | (c[:, 1::2] << 4))", "(c[:, 1::2] | (c[:, 0::2] << 4))")], COD),
    ("atom_rows_swapped", "codec.py",
     [("t = t.transpose(0, 3, 2, 1, 4)                            # mb, kq, m0, m1, j",
       "t = t.transpose(0, 3, 1, 2, 4)                            # mb, kq, m0, m1, j")], COD),
    # SVDQuant steps
    ("smoothing_exponents_swapped", "svdquant.py",
     [("ax[ok] ** alpha / wx[ok] ** (1.0 - alpha)", "ax[ok] ** (1.0 - alpha) / wx[ok] ** alpha")], SVD),
    ("smoothing_inverted", "svdquant.py",
     [("ax[ok] ** alpha / wx[ok] ** (1.0 - alpha)", "wx[ok] ** (1.0 - alpha) / ax[ok] ** alpha")], SVD),
    ("smoothing_zero_weight_channel", "svdquant.py", [("ok = (ax > 0) & (wx > 0)", "ok = (ax > 0)")], SVD),
    ("inv_lam_from_the_f64_lambda", "svdquant.py",
     [("inv32 = (1.0 / lam32.astype(np.float64)).astype(np.float32)", "inv32 = (1.0 / lam).astype(np.float32)")], SVD),
    ("l1_rounded_before_the_fold", "svdquant.py", [("round_bf16(L1 * inv64)", "round_bf16(L1) * inv64")], SVD),
    ("l2_not_rounded", "svdquant.py", [("round_bf16(L1 * inv64), round_bf16(L2)", "round_bf16(L1 * inv64), L2")], SVD),
    ("activations_not_smoothed", "svdquant.py",
     [("return quantize_groups(smooth_activations(X, inv_lam))", "return quantize_groups(np.asarray(X, np.float32))")],
     SVD),
    ("lora_on_smoothed_x", "svdquant.py",
     [("L1p = np.concatenate([prep.L1p, A], axis=1)",
       "L1p = np.concatenate([prep.L1p, A * prep.inv_lam.astype(np.float64)[:, None]], axis=1)")], SVD),
    ("svd_sigma_dropped", "svdquant.py", [("L1 = vt[:r].T * s[:r][None, :]", "L1 = vt[:r].T")], SVD),
    ("residual_sign", "svdquant.py", [("R = (W_hat - low.T)", "R = (W_hat + low.T)")], SVD),
    ("residual_ignores_smoothing", "svdquant.py",
     [("low = (L1p / inv64[:, None]) @ L2b", "low = L1p @ L2b")], SVD),
    ("weight_factor_floor", "svdquant.py",
     [("ceil_log2 = int(e) - 1 if frac == 0.5 else int(e)", "ceil_log2 = int(e) - 1")], SVD),
    ("weight_factor_doubles_powers", "svdquant.py",
     [("ceil_log2 = int(e) - 1 if frac == 0.5 else int(e)", "ceil_log2 = int(e)")], SVD),
    ("linear_drops_alpha_w", "svdquant.py", [("return prep.alpha_w * main +", "return main +")], SVD),
    ("linear_drops_bias", "svdquant.py",
     [("lowrank_down(X, prep) @ L2[:, c] + prep.bias[None, c]", "lowrank_down(X, prep) @ L2[:, c]")], SVD),
    ("linear_drops_lowrank", "svdquant.py",
     [("main + lowrank_down(X, prep) @ L2[:, c] + prep.bias", "main + prep.bias")], SVD),
    ("lowrank_on_smoothed_x", "svdquant.py",
     [("return np.asarray(X, np.float64) @ prep.L1p",
       "return smooth_activations(X, prep.inv_lam).astype(np.float64) @ prep.L1p")], SVD),
    ("lora_scale_dropped", "svdquant.py",
     [("round_bf16(scale * B)", "round_bf16(B)"), ("scale * B], axis=0)", "B], axis=0)")], SVD),
    ("lora_reference_uses_rounded_factor", "svdquant.py",
     [("L2 = prep.L2b if prep.lora_B_exact is None else prep.lora_B_exact", "L2 = prep.L2b")], SVD),
    ("smooth_weight_multiplies", "svdquant.py",
     [("return np.asarray(W, np.float64) / np.asarray(inv_lam, np.float64)[None, :]",
       "return np.asarray(W, np.float64) * np.asarray(inv_lam, np.float64)[None, :]")], SVD),
    ("residual_not_divided_by_alpha_w", "svdquant.py",
     [("Rp = (R.astype(np.float64) / aw).astype(np.float32)  # exact: power of two",
       "Rp = R.astype(np.float32)")], SVD),
    ("fake_quantize_drops_alpha_w", "svdquant.py",
     [("return dequantize_groups(codes, scales) * aw", "return dequantize_groups(codes, scales)")], SVD),
    ("alpha_search_picks_the_worst", "svdquant.py",
     [("return errs, int(np.argmin(errs))", "return errs, int(np.argmax(errs))")], SVD),
    ("refinement_keeps_last", "svdquant.py",
     [("if best is None or errors[-1] < min(errors[:-1]):", "if True:")], SVD),
    ("refinement_repeats_the_split", "svdquant.py", [("        A = W_hat - Q\n", "        A = W_hat - prep.R\n")], SVD),
    ("prop41_drops_a_term", "svdquant.py",
     [("f(X) * dW + f(X - QX) * (f(W) + dW)", "f(X) * dW + f(X - QX) * f(W)")], SVD),
    # INT4 variant
    ("int4_qmax_8", "int4.py", [("QMAX = 7\n", "QMAX = 8\n")], I4),
    ("int4_ties_up", "int4.py", [("np.clip(np.rint(t), -QMAX, QMAX)", "np.clip(np.floor(t + 0.5), -QMAX, QMAX)")], I4),
    ("int4_scale_not_bf16", "int4.py",
     [("s = round_bf16((amax / np.float32(QMAX)).astype(np.float32))",
       "s = (amax / np.float32(QMAX)).astype(np.float32).astype(np.float64)")], I4),
    ("int4_pack_order", "int4.py",
     [("word |= (c[..., 2 * k].astype(np.uint64) << np.uint64(4 * k)) | \\\n"
       "                (c[..., 2 * k + 1].astype(np.uint64) << np.uint64(16 + 4 * k))",
       "word |= (c[..., 2 * k].astype(np.uint64) << np.uint64(8 * k)) | \\\n"
       "                (c[..., 2 * k + 1].astype(np.uint64) << np.uint64(8 * k + 4))")], I4),
    ("int4_no_sign_extension", "int4.py", [("return np.where(out >= 8, out - 16, out).astype(np.int8)",
                                            "return out.astype(np.int8)")], I4),
    ("int4_linear_drops_lowrank", "int4.py",
     [("return main + S.lowrank_down(X, b) @ L2[:, c] + b.bias[None, c]", "return main + b.bias[None, c]")], I4),
    ("int4_dequant_ignores_scale", "int4.py",
     [("return (codes.reshape(R, K // GROUP, GROUP) * s[..., None]).reshape(R, K)",
       "return codes.reshape(R, K).astype(np.float64)")], I4),
    ("int4_lora_dropped", "int4.py",
     [("return dataclasses.replace(prep, base=S.attach_lora(prep.base, A, B, scale))", "return prep")], I4),
    # LayerNorm front end
    ("norm_mean_over_tokens", "norm.py", [("mu = Z.mean(axis=1)", "mu = Z.mean(axis=1) * 0.0 + Z.mean()")], NRM),
    ("norm_steps_in_float64", "norm.py",
     [("d = (Z - mu).astype(np.float32)\n    n = (d * rstd).astype(np.float32)",
       "d = Z.astype(np.float64) - mu\n    n = d * rstd")], NRM),
    ("norm_eps_dropped", "norm.py", [("1.0 / np.sqrt(var + eps)", "1.0 / np.sqrt(var)")], NRM),
    ("norm_sample_variance", "norm.py",
     [("var = ((Z - mu[:, None]) ** 2).mean(axis=1)", "var = ((Z - mu[:, None]) ** 2).sum(axis=1) / (Z.shape[1] - 1)")],
     NRM),
    ("norm_shift_and_scale_swapped", "norm.py",
     [("x = ((n * np.asarray(a, np.float32)[None, :]).astype(np.float32) + np.asarray(c, np.float32)[None, :])",
       "x = ((n * np.asarray(c, np.float32)[None, :]).astype(np.float32) + np.asarray(a, np.float32)[None, :])")],
     NRM),
    ("norm_not_rounded_to_bf16", "norm.py",
     [("return round_bf16(x.astype(np.float32)).astype(np.float32)", "return x.astype(np.float32)")], NRM),
]


def _plant(base: str, mutant) -> tuple:
    name, fname, edits, pins = mutant
    d = os.path.join(base, name)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"))
    shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(d, "synth"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(d, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    for f in ["conftest.py", *pins]:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(d, "tests", f))
    path = os.path.join(d, "oracle", fname)
    src = open(path).read()
    for old, new in edits:
        if src.count(old) != 1:
            return name, -1, f"edit text found {src.count(old)} times in oracle/{fname}: {old[:60]!r}"
        src = src.replace(old, new)
    open(path, "w").write(src)
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1", OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1",
               MKL_NUM_THREADS="1")
    env.pop("PYTHONPATH", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *[os.path.join("tests", p) for p in pins]],
                       cwd=d, env=env, capture_output=True, text=True, timeout=900)
    return name, r.returncode, r.stdout[-400:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda m: _plant(str(tmp_path), m), MUTANTS))
    bad_edit = [(n, out) for n, rc, out in results if rc == -1]
    assert not bad_edit, bad_edit
    # pytest exits 1 when tests ran and some failed; anything else (0 = all
    # passed, 2+ = the copy did not even import) is not a caught mutant
    survivors = [n for n, rc, _ in results if rc == 0]
    assert not survivors, f"mistakes no pin catches: {survivors}"
    broken = [(n, rc, out) for n, rc, out in results if rc != 1]
    assert not broken, broken
