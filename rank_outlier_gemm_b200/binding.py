"""ctypes binding of ``libsvdq.so`` (declared in ``include/svdq.h``).

Each function has the name of the C entry point it calls and only marshals
arguments: host arrays become pointers to their data, CUDA tensors become
device pointers, and the CUDA stream is PyTorch's current stream unless one is
given.  Every step of the layer runs in the library's kernels; there is no
fallback path, and importing this module fails if the library is not built.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsvdq.so")

SVDQ_OK = 0
STATUS_NAMES = {0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_UNSUPPORTED_DEVICE",
                3: "SVDQ_ERR_CUDA", 4: "SVDQ_ERR_OOM", 5: "SVDQ_ERR_TIMEOUT",
                6: "SVDQ_ERR_DEVICE_CHECK"}


class SvdqError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        self.status = status
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")


class PrepareOpts(ctypes.Structure):
    _fields_ = [("alpha", ctypes.c_float), ("rank", ctypes.c_int), ("power_iters", ctypes.c_int),
                ("oversample", ctypes.c_int), ("seed", ctypes.c_uint64), ("keep_residual", ctypes.c_int),
                ("refine_iters", ctypes.c_int), ("format", ctypes.c_int)]


FORMATS = {"nvfp4": 0, "int4": 1}


_vp, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
_SIGS = {
    "svdq_prepare_opts_default": (None, [ctypes.POINTER(PrepareOpts)]),
    "svdq_prepare_weights": (_i, [_vp, _vp, _vp, _i, _i, ctypes.POINTER(PrepareOpts), _vp, ctypes.POINTER(_vp)]),
    "svdq_weights_from_factors": (_i, [_i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(_vp)]),
    "svdq_weights_from_factors_fmt": (_i, [_i, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _vp, ctypes.POINTER(_vp)]),
    "svdq_weights_format": (_i, [_vp, ctypes.POINTER(_i)]),
    "svdq_weights_sf_bytes": (_sz, [_vp]),
    "svdq_attach_lora": (_i, [_vp, _vp, _vp, _i, _f, _vp]),
    "svdq_quantize_act_lowrank_down": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _vp]),
    "svdq_linear_w4a4": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _vp]),
    "svdq_forward": (_i, [_vp, _vp, _i, _vp, _vp, _sz, _vp]),
    "svdq_forward_host": (_i, [_vp, _vp, _i, _vp, _vp, _sz, _vp]),
    "svdq_forward_noalloc": (_i, [_vp, _vp, _i, _vp, _vp]),
    "svdq_act_row_stats": (_i, [_vp, _i, _i, _f, _vp, _vp]),
    "svdq_norm_quantize_act_lowrank_down": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "svdq_forward_norm": (_i, [_vp, _vp, _i, _vp, _vp, _f, _vp, _vp, _sz, _vp]),
    "svdq_forward_norm_workspace_bytes": (_sz, [_vp, _i]),
    "svdq_act_codes_bytes": (_sz, [_i, _i]),
    "svdq_act_sf_bytes": (_sz, [_i, _i]),
    "svdq_lowrank_bytes": (_sz, [_vp, _i]),
    "svdq_forward_workspace_bytes": (_sz, [_vp, _i]),
    "svdq_forward_host_workspace_bytes": (_sz, [_vp, _i]),
    "svdq_weights_rank": (_i, [_vp]),
    "svdq_weights_info": (_i, [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i),
                               ctypes.POINTER(_i), ctypes.POINTER(_f)]),
    "svdq_weights_export": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "svdq_weights_destroy": (_i, [_vp]),
    "svdq_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "svdq_check_device_errors": (_i, [_vp]),
    "svdq_selftest_codec": (_i, [ctypes.POINTER(ctypes.c_uint)]),
    "svdq_weights_refine_errors": (_i, [_vp, ctypes.POINTER(ctypes.c_double), _i, ctypes.POINTER(_i)]),
    "svdq_search_alpha": (_i, [_vp, _vp, _i, _vp, _i, _i, _vp, _i, ctypes.POINTER(PrepareOpts), _vp,
                               ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i)]),
    "svdq_debug_launch_stalled_act": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _vp]),
    "svdq_debug_linear_w4a4_ksplit": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _vp]),
    "svdq_debug_forward_small_m": (_i, [_vp, _vp, _i, _vp, _i, _vp]),
    "svdq_last_error": (ctypes.c_char_p, []),
    "svdq_version": (ctypes.c_char_p, []),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m rank_outlier_gemm_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
EXPORTED = tuple(_SIGS)


def _check(status: int, fn: str):
    if status != SVDQ_OK:
        raise SvdqError(status, fn, _lib.svdq_last_error().decode())


def _host(a, dtype) -> tuple:
    """(pointer, keep-alive) of a contiguous host array of the given numpy dtype."""
    if a is None:
        return None, None
    if isinstance(a, torch.Tensor):
        if a.is_cuda:
            raise ValueError("expected a host array")
        if a.dtype == torch.bfloat16:
            a = a.view(torch.int16)
        a = a.numpy()
    arr = np.ascontiguousarray(a)
    if arr.dtype != np.dtype(dtype):
        if np.dtype(dtype) == np.uint16 and arr.dtype == np.int16:
            arr = arr.view(np.uint16)
        else:
            arr = arr.astype(dtype)
    return arr.ctypes.data, arr


def _dev(t: Optional[torch.Tensor], name: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Weights:
    """Owns an svdq_weights handle; destroyed with the object."""

    def __init__(self, handle: int):
        self.handle = handle

    @property
    def info(self) -> dict:
        N, K, r, rp, aw = _i(), _i(), _i(), _i(), _f()
        _check(_lib.svdq_weights_info(self.handle, ctypes.byref(N), ctypes.byref(K), ctypes.byref(r),
                                      ctypes.byref(rp), ctypes.byref(aw)), "svdq_weights_info")
        fmt = _i()
        _check(_lib.svdq_weights_format(self.handle, ctypes.byref(fmt)), "svdq_weights_format")
        return {"N": N.value, "K": K.value, "rank": r.value, "r_pad": rp.value, "alpha_w": aw.value,
                "format": {v: k for k, v in FORMATS.items()}[fmt.value]}

    def __del__(self):
        # at interpreter exit the module globals may already be gone
        if getattr(self, "handle", None) and _lib is not None:
            _lib.svdq_weights_destroy(self.handle)
            self.handle = None


def svdq_prepare_opts_default() -> PrepareOpts:
    o = PrepareOpts()
    _lib.svdq_prepare_opts_default(ctypes.byref(o))
    return o


def svdq_prepare_weights(W_bf16, act_absmax, bias_bf16=None, rank: int = 32, alpha: float = 0.5,
                         power_iters: int = 4, oversample: int = 16, seed: int = 0,
                         keep_residual: bool = False, refine_iters: int = 1, fmt: str = "nvfp4",
                         stream=None) -> Weights:
    Wp, Wk = _host(W_bf16, np.uint16)
    N, K = Wk.shape
    ap, ak = _host(act_absmax, np.float32)
    bp, bk = _host(bias_bf16, np.uint16)
    o = svdq_prepare_opts_default()
    o.alpha, o.rank, o.power_iters, o.oversample, o.seed = alpha, rank, power_iters, oversample, seed
    o.keep_residual = int(keep_residual)
    o.refine_iters = int(refine_iters)
    o.format = FORMATS[fmt]
    h = _vp()
    _check(_lib.svdq_prepare_weights(Wp, ap, bp, N, K, ctypes.byref(o), _stream(stream), ctypes.byref(h)),
           "svdq_prepare_weights")
    return Weights(h.value)


def svdq_weights_from_factors(N: int, K: int, rank: int, inv_lam, L1p_bf16, L2_bf16, R, bias=None,
                              stream=None, fmt: str = "nvfp4") -> Weights:
    ip, ik = _host(inv_lam, np.float32)
    lp, lk = _host(L1p_bf16, np.uint16) if rank else (None, None)
    l2p, l2k = _host(L2_bf16, np.uint16) if rank else (None, None)
    rp, rk = _host(R, np.float32)
    bp, bk = _host(bias, np.float32)
    h = _vp()
    _check(_lib.svdq_weights_from_factors_fmt(N, K, rank, ip, lp, l2p, rp, bp, FORMATS[fmt], _stream(stream),
                                              ctypes.byref(h)), "svdq_weights_from_factors_fmt")
    return Weights(h.value)


def svdq_attach_lora(w: Weights, A_bf16, B_bf16, scale: float = 1.0, stream=None) -> None:
    Ap, Ak = _host(A_bf16, np.uint16)
    Bp, Bk = _host(B_bf16, np.uint16)
    _check(_lib.svdq_attach_lora(w.handle, Ap, Bp, Ak.shape[1], scale, _stream(stream)), "svdq_attach_lora")


def svdq_quantize_act_lowrank_down(w: Weights, X: torch.Tensor, xq: torch.Tensor, xsf: torch.Tensor,
                                   T: Optional[torch.Tensor], stream=None) -> None:
    _check(_lib.svdq_quantize_act_lowrank_down(w.handle, _dev(X, "X"), X.shape[0], _dev(xq, "xq"),
                                               _dev(xsf, "xsf"), _dev(T, "T"), _stream(stream)),
           "svdq_quantize_act_lowrank_down")


def svdq_debug_launch_stalled_act(w: Weights, X, xq, xsf, T, stream=None) -> None:
    _check(_lib.svdq_debug_launch_stalled_act(w.handle, _dev(X, "X"), X.shape[0], _dev(xq, "xq"),
                                              _dev(xsf, "xsf"), _dev(T, "T"), _stream(stream)),
           "svdq_debug_launch_stalled_act")


def svdq_linear_w4a4(w: Weights, xq, xsf, T, M: int, Y: torch.Tensor, stream=None) -> None:
    _check(_lib.svdq_linear_w4a4(w.handle, _dev(xq, "xq"), _dev(xsf, "xsf"), _dev(T, "T"), M, _dev(Y, "Y"),
                                 _stream(stream)), "svdq_linear_w4a4")


def svdq_debug_linear_w4a4_ksplit(w: Weights, xq, xsf, T, M: int, Y: torch.Tensor, ksplit: int,
                                  stream=None) -> None:
    _check(_lib.svdq_debug_linear_w4a4_ksplit(w.handle, _dev(xq, "xq"), _dev(xsf, "xsf"), _dev(T, "T"), M,
                                              _dev(Y, "Y"), ksplit, _stream(stream)),
           "svdq_debug_linear_w4a4_ksplit")


def svdq_debug_forward_small_m(w: Weights, X: torch.Tensor, Y: torch.Tensor, ksplit: int = 0, stream=None) -> None:
    _check(_lib.svdq_debug_forward_small_m(w.handle, _dev(X, "X"), X.shape[0], _dev(Y, "Y"), ksplit, _stream(stream)),
           "svdq_debug_forward_small_m")


def svdq_forward(w: Weights, X: torch.Tensor, Y: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    _check(_lib.svdq_forward(w.handle, _dev(X, "X"), X.shape[0], _dev(Y, "Y"), _dev(workspace, "workspace"),
                             workspace.numel() * workspace.element_size(), _stream(stream)), "svdq_forward")


def svdq_forward_host(w: Weights, X_host: torch.Tensor, Y_host: torch.Tensor, workspace: torch.Tensor,
                      stream=None) -> None:
    if X_host.is_cuda or Y_host.is_cuda:
        raise ValueError("X_host and Y_host must be host tensors")
    _check(_lib.svdq_forward_host(w.handle, X_host.data_ptr(), X_host.shape[0], Y_host.data_ptr(),
                                  _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                  _stream(stream)), "svdq_forward_host")


def svdq_forward_noalloc(w: Weights, X: torch.Tensor, Y: torch.Tensor, stream=None) -> None:
    """svdq_forward with the intermediates in the library's static device block (no allocation)."""
    _check(_lib.svdq_forward_noalloc(w.handle, _dev(X, "X"), X.shape[0], _dev(Y, "Y"), _stream(stream)),
           "svdq_forward_noalloc")


def svdq_act_row_stats(Z: torch.Tensor, eps: float, stats: torch.Tensor, stream=None) -> None:
    """(mu, rstd) per row of a CUDA bf16 [M, K] tensor into a CUDA float32 [M, 2] tensor."""
    _check(_lib.svdq_act_row_stats(_dev(Z, "Z"), Z.shape[0], Z.shape[1], float(eps), _dev(stats, "stats"),
                                   _stream(stream)), "svdq_act_row_stats")


def svdq_norm_quantize_act_lowrank_down(w: Weights, Z: torch.Tensor, stats: torch.Tensor, norm_a: torch.Tensor,
                                        norm_c: torch.Tensor, xq, xsf, T, stream=None) -> None:
    _check(_lib.svdq_norm_quantize_act_lowrank_down(w.handle, _dev(Z, "Z"), Z.shape[0], _dev(stats, "stats"),
                                                    _dev(norm_a, "norm_a"), _dev(norm_c, "norm_c"), _dev(xq, "xq"),
                                                    _dev(xsf, "xsf"), _dev(T, "T"), _stream(stream)),
           "svdq_norm_quantize_act_lowrank_down")


def svdq_forward_norm(w: Weights, Z: torch.Tensor, norm_a: torch.Tensor, norm_c: torch.Tensor, eps: float,
                      Y: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    _check(_lib.svdq_forward_norm(w.handle, _dev(Z, "Z"), Z.shape[0], _dev(norm_a, "norm_a"), _dev(norm_c, "norm_c"),
                                  float(eps), _dev(Y, "Y"), _dev(workspace, "workspace"),
                                  workspace.numel() * workspace.element_size(), _stream(stream)), "svdq_forward_norm")


def svdq_forward_norm_workspace_bytes(w: Weights, M: int) -> int:
    return _lib.svdq_forward_norm_workspace_bytes(w.handle, M)


def svdq_act_codes_bytes(M: int, K: int) -> int:
    return _lib.svdq_act_codes_bytes(M, K)


def svdq_act_sf_bytes(M: int, K: int) -> int:
    return _lib.svdq_act_sf_bytes(M, K)


def svdq_lowrank_bytes(w: Weights, M: int) -> int:
    return _lib.svdq_lowrank_bytes(w.handle, M)


def svdq_forward_workspace_bytes(w: Weights, M: int) -> int:
    return _lib.svdq_forward_workspace_bytes(w.handle, M)


def svdq_forward_host_workspace_bytes(w: Weights, M: int) -> int:
    return _lib.svdq_forward_host_workspace_bytes(w.handle, M)


def svdq_weights_info(w: Weights) -> dict:
    return w.info


def svdq_weights_rank(w: Weights) -> int:
    return int(_lib.svdq_weights_rank(w.handle))


def svdq_weights_export(w: Weights, residual: bool = False) -> dict:
    i = w.info
    N, K, r = i["N"], i["K"], i["rank"]
    out = {"codes": np.empty((N, K // 2), np.uint8), "sf": np.empty(_lib.svdq_weights_sf_bytes(w.handle), np.uint8),
           "L1p": np.empty((K, r), np.uint16), "L2": np.empty((r, N), np.uint16),
           "inv_lam": np.empty(K, np.float32), "bias": np.empty(N, np.float32)}
    if residual:
        out["residual"] = np.empty((N, K), np.float32)
    _check(_lib.svdq_weights_export(w.handle, out["codes"].ctypes.data, out["sf"].ctypes.data,
                                    out["L1p"].ctypes.data if r else None, out["L2"].ctypes.data if r else None,
                                    out["inv_lam"].ctypes.data, out["bias"].ctypes.data,
                                    out["residual"].ctypes.data if residual else None), "svdq_weights_export")
    out.update(i)
    return out


def svdq_set_wait_limit_ns(ns: int) -> None:
    _lib.svdq_set_wait_limit_ns(int(ns))


def svdq_search_alpha(W_bf16, X_bf16, bias_bf16=None, alphas=(0.3, 0.4, 0.5, 0.6, 0.7, 0.8), rank: int = 32,
                      refine_iters: int = 1, fmt: str = "nvfp4", stream=None):
    """(relative output error per alpha, index of the best) on the calibration batch X."""
    Wp, Wk = _host(W_bf16, np.uint16)
    Xp, Xk = _host(X_bf16, np.uint16)
    bp, bk = _host(bias_bf16, np.uint16)
    N, K = Wk.shape
    a = np.ascontiguousarray(np.asarray(alphas, np.float32))
    o = svdq_prepare_opts_default()
    o.rank, o.refine_iters = rank, refine_iters
    o.format = FORMATS[fmt]
    err = (ctypes.c_double * len(a))()
    best = ctypes.c_int(0)
    _check(_lib.svdq_search_alpha(Wp, Xp, Xk.shape[0], bp, N, K, a.ctypes.data, len(a), ctypes.byref(o),
                                  _stream(stream), err, ctypes.byref(best)), "svdq_search_alpha")
    return [float(err[i]) for i in range(len(a))], int(best.value)


def svdq_weights_refine_errors(w: Weights) -> list:
    """Residual quantization error of each split prepare tried (the kept one is the smallest)."""
    n = ctypes.c_int(0)
    _check(_lib.svdq_weights_refine_errors(w.handle, None, 0, ctypes.byref(n)), "svdq_weights_refine_errors")
    buf = (ctypes.c_double * max(1, n.value))()
    _check(_lib.svdq_weights_refine_errors(w.handle, buf, n.value, ctypes.byref(n)), "svdq_weights_refine_errors")
    return [float(buf[i]) for i in range(n.value)]


def svdq_selftest_codec() -> int:
    """Mismatch count of the encoder's exact division/reciprocal shortcuts on the current device."""
    out = ctypes.c_uint(0)
    _check(_lib.svdq_selftest_codec(ctypes.byref(out)), "svdq_selftest_codec")
    return int(out.value)


def svdq_check_device_errors(stream=None) -> int:
    """Returns the device error status (0 = none) after synchronizing the stream."""
    return _lib.svdq_check_device_errors(_stream(stream))


def svdq_last_error() -> str:
    return _lib.svdq_last_error().decode()


def svdq_version() -> str:
    return _lib.svdq_version().decode()


# ---------------------------------------------------------------- helpers
def act_buffers(w: Weights, M: int, device="cuda"):
    """Device buffers (xq, xsf, T) for one activation batch of M rows."""
    i = w.info
    xq = torch.empty(max(1, svdq_act_codes_bytes(M, i["K"])), dtype=torch.uint8, device=device)
    xsf = torch.empty(svdq_act_sf_bytes(M, i["K"]), dtype=torch.uint8, device=device)
    T = torch.empty((M, 2 * i["r_pad"]), dtype=torch.bfloat16, device=device) if i["r_pad"] else None
    return xq, xsf, T


def linear(w: Weights, X: torch.Tensor, stream=None) -> torch.Tensor:
    """Y = layer(X) for a CUDA bf16 X of shape [M, K] (both kernels)."""
    M = X.shape[0]
    xq, xsf, T = act_buffers(w, M, X.device)
    Y = torch.empty((M, w.info["N"]), dtype=torch.bfloat16, device=X.device)
    svdq_quantize_act_lowrank_down(w, X, xq, xsf, T, stream)
    svdq_linear_w4a4(w, xq, xsf, T, M, Y, stream)
    return Y
