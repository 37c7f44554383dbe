"""The C ABI loads, exports every entry point that include/svdq.h declares, and
validates arguments on the host (no GPU needed for these checks)."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svdq.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ["svdq_prepare_weights", "svdq_quantize_act_lowrank_down", "svdq_linear_w4a4",
                 "svdq_attach_lora"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    from rank_outlier_gemm_b200 import binding
    lib = ctypes.CDLL(binding.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared()) == set(binding.EXPORTED)


def test_host_only_helpers():
    from rank_outlier_gemm_b200 import binding as B
    assert B.svdq_act_codes_bytes(7, 128) == 7 * 64
    assert B.svdq_act_sf_bytes(1, 3072) == 128 * 192
    assert B.svdq_act_sf_bytes(129, 64) == 256 * 4
    o = B.svdq_prepare_opts_default()
    assert (o.alpha, o.rank, o.power_iters, o.oversample, o.refine_iters) == (0.5, 32, 4, 16, 1)
    assert o.format == B.FORMATS["nvfp4"] == 0 and B.FORMATS["int4"] == 1
    assert "sm_100a" in B.svdq_version()


def test_invalid_arguments_rejected_before_gpu():
    from rank_outlier_gemm_b200 import binding as B
    W = np.zeros((32, 96), np.uint16)          # K % 64 != 0
    with pytest.raises(B.SvdqError) as e:
        B.svdq_prepare_weights(W, np.ones(96, np.float32), rank=4)
    assert e.value.status == 1 and "multiple of 64" in str(e.value)
    W = np.zeros((24, 64), np.uint16)          # N % 16 != 0
    with pytest.raises(B.SvdqError) as e:
        B.svdq_prepare_weights(W, np.ones(64, np.float32), rank=4)
    assert e.value.status == 1
    W = np.zeros((32, 64), np.uint16)
    with pytest.raises(B.SvdqError) as e:   # rank above min(N, K)
        B.svdq_prepare_weights(W, np.ones(64, np.float32), rank=40)
    assert e.value.status == 1
    with pytest.raises(B.SvdqError) as e:   # refinement needs at least one split
        B.svdq_prepare_weights(W, np.ones(64, np.float32), rank=4, refine_iters=0)
    assert e.value.status == 1 and "refine_iters" in str(e.value)
    with pytest.raises(B.SvdqError) as e:   # refinement is NVFP4-only
        B.svdq_prepare_weights(W, np.ones(64, np.float32), rank=4, fmt="int4", refine_iters=2)
    assert e.value.status == 1 and "NVFP4 only" in str(e.value)
    import ctypes
    h = ctypes.c_void_p()
    R0 = np.zeros((32, 64), np.float32)
    st = B._lib.svdq_weights_from_factors_fmt(32, 64, 0, np.ones(64, np.float32).ctypes.data, None, None,
                                              R0.ctypes.data, None, 7, None, ctypes.byref(h))
    assert st == 1 and b"format" in B._lib.svdq_last_error()
    bad = np.ones(64, np.float32)
    bad[3] = np.nan
    with pytest.raises(B.SvdqError) as e:
        B.svdq_prepare_weights(W, bad, rank=4)
    assert e.value.status == 1
    R = np.zeros((32, 64), np.float32)
    R[0, 0] = np.inf
    with pytest.raises(B.SvdqError) as e:
        B.svdq_weights_from_factors(32, 64, 0, np.ones(64, np.float32), None, None, R)
    assert e.value.status == 1


def _prototypes():
    """name -> (return type, parameter count) of every function the header declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"([A-Za-z_][\w\s\*]*?)\b(svdq_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        ret = " ".join(m.group(1).split())
        params = m.group(3).strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        out[m.group(2)] = (ret, n)
    return out


def test_binding_signatures_match_the_header():
    """Every ctypes signature of the binding has the header's parameter count and
    a return type of the matching kind (status and int -> c_int, size_t ->
    c_size_t, const char* -> c_char_p, void -> None)."""
    import ctypes
    from rank_outlier_gemm_b200 import binding as B
    protos = _prototypes()
    assert set(protos) == set(B._SIGS)
    kinds = {"svdq_status": ctypes.c_int, "int": ctypes.c_int, "size_t": ctypes.c_size_t,
             "const char*": ctypes.c_char_p, "const char *": ctypes.c_char_p, "void": None}
    for name, (ret, n) in protos.items():
        res, args = B._SIGS[name]
        assert len(args) == n, (name, len(args), n)
        assert kinds[ret] is res, (name, ret, res)

