"""The allocation-free forward (svdq_forward_noalloc) against svdq_forward.

Some callers cannot call cudaMalloc: code running inside a caching
allocator's callbacks (an allocation there re-enters the allocator or fails
against its reserve) and serving loops whose device memory is reserved up
front.  For them the library keeps the layer's intermediates (activation
codes, scales, T) in one static 32 MiB block per device that every call
reuses.  Both entry points run the same kernels on the same inputs, so their
outputs must be equal bit for bit, call after call; the output must also
follow the oracle.  The first call on a device loads the block; later calls
must leave the device's free memory unchanged, a layer too large for the block
is rejected before any GPU work, and the path's own error word is read and
cleared by svdq_check_device_errors.

This file is collected last (its name sorts after every other test file), so
a run that stops at the first failure has run every other test first; one
test starts a fresh process so that the first call on the device is covered
whatever ran before."""

import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

from oracle import int4 as OI
from oracle import svdquant as OS
from synth import config_cases, f32_to_bf16_bits, make_layer_inputs
from tests import gpu_common as G

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _forward_with_workspace(L, w, X):
    M = X.shape[0]
    Y = torch.empty((M, w.info["N"]), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.svdq_forward_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward(w, X, Y, ws)
    return Y


def _noalloc(L, w, X):
    Y = torch.full((X.shape[0], w.info["N"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.svdq_forward_noalloc(w, X, Y)
    return Y


def _handle(kind: str, t, prep: OS.Prepared):
    """(library handle, oracle preparation, oracle layer function) of one kind:
    the NVFP4 layer at rank 32, the INT4 variant of the same split, or the
    NVFP4 layer without a low-rank branch (no T at all)."""
    L = G.lib()
    if kind == "rank0":
        K, N = prep.K, prep.N
        p0 = OS.prepare_from_factors(OS.smooth_weight(t.W, prep.inv_lam), prep.inv_lam, np.zeros((K, 0)),
                                     np.zeros((0, N)), t.bias)
        return G.weights_from_oracle(p0), p0, OS.linear
    if kind == "int4":
        w = L.svdq_weights_from_factors(prep.N, prep.K, prep.rank, prep.inv_lam,
                                        f32_to_bf16_bits(prep.L1p.astype(np.float32)),
                                        f32_to_bf16_bits(prep.L2b.astype(np.float32)), prep.R,
                                        prep.bias.astype(np.float32), fmt="int4")
        return w, OI.from_base(prep), OI.linear
    return G.weights_from_oracle(prep), prep, OS.linear


@pytest.mark.parametrize("kind", ["nvfp4", "int4", "rank0"])
def test_forward_noalloc_matches_forward_on_two_calls(kind):
    L = G.lib()
    case = [c for c in config_cases("pixart") if c.name == "mlp_up"][0]
    t = make_layer_inputs(case, M=300)
    w, prep, linear = _handle(kind, t, OS.prepare(t.W, t.act_absmax, t.bias, case.rank))
    rng = np.random.default_rng(5)
    rows2 = rng.permutation(300)[:200]
    for X_bits, X in ((t.X_bits, t.X), (t.X_bits[rows2], t.X[rows2])):
        Xd = G.to_dev_bf16(X_bits)
        ref = _forward_with_workspace(L, w, Xd)
        Y = _noalloc(L, w, Xd)
        assert L.svdq_check_device_errors() == 0
        assert torch.equal(Y, ref)
        G.check_Y(Y.float().cpu().numpy().astype(np.float64), linear(prep, X))


def test_forward_noalloc_leaves_free_memory_unchanged():
    """After the first call on the device, calls allocate nothing: the
    device's free memory (cudaMemGetInfo) is the same before and after."""
    L = G.lib()
    case = [c for c in config_cases("flux") if c.name == "attn_out"][0]
    t = make_layer_inputs(case, M=1000)
    w = G.weights_from_oracle(OS.prepare(t.W, t.act_absmax, t.bias, case.rank))
    X = G.to_dev_bf16(t.X_bits)
    Y = torch.empty((1000, case.N), dtype=torch.bfloat16, device="cuda")
    L.svdq_forward_noalloc(w, X, Y)               # the block is loaded by now
    torch.cuda.synchronize()
    before = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        L.svdq_forward_noalloc(w, X, Y)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == before
    assert L.svdq_check_device_errors() == 0


def test_forward_noalloc_first_call_in_a_fresh_process():
    """A fresh process whose first layer call is svdq_forward_noalloc: the call
    looks up (and so loads) the static block on the device, its output equals
    svdq_forward's bit for bit, and a second call allocates nothing."""
    code = textwrap.dedent("""
        import sys
        sys.path.insert(0, %r)
        import numpy as np, torch
        import rank_outlier_gemm_b200 as L
        from oracle import svdquant as OS
        from synth import config_cases, make_layer_inputs
        from tests import gpu_common as G
        case = [c for c in config_cases("sdxl") if c.name == "r32_attn"][0]
        t = make_layer_inputs(case, M=257)
        prep = OS.prepare(t.W, t.act_absmax, t.bias, case.rank)
        w = G.weights_from_oracle(prep)
        X = G.to_dev_bf16(t.X_bits)
        Y1 = torch.empty((257, case.N), dtype=torch.bfloat16, device="cuda")
        Y2 = torch.empty_like(Y1)
        ws = torch.empty(L.svdq_forward_workspace_bytes(w, 257), dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()
        L.svdq_forward_noalloc(w, X, Y1)
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        L.svdq_forward_noalloc(w, X, Y1)
        torch.cuda.synchronize()
        free2 = torch.cuda.mem_get_info()[0]
        assert L.svdq_check_device_errors() == 0
        L.svdq_forward(w, X, Y2, ws)
        torch.cuda.synchronize()
        assert torch.equal(Y1, Y2), "noalloc differs from svdq_forward"
        G.check_Y(Y1.float().cpu().numpy().astype(np.float64), OS.linear(prep, t.X))
        assert free1 == free2, (free1, free2)
        print("fresh-process ok")
    """ % ROOT)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "fresh-process ok" in r.stdout


def test_forward_noalloc_rejects_layers_beyond_its_block():
    L = G.lib()
    case = [c for c in config_cases("flux") if c.name == "mlp_down"][0]   # K = 12288
    t = make_layer_inputs(case, M=8)
    K = case.K
    prep = OS.prepare_from_factors(t.W[:64], np.ones(K, np.float32), np.zeros((K, 0)), np.zeros((0, 64)), None)
    w = G.weights_from_oracle(prep)
    M = 8192                                  # 8192 x 12288 / 2 bytes of codes alone exceed 32 MiB
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((M, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.SvdqError) as e:
        L.svdq_forward_noalloc(w, X, Y)
    assert e.value.status == 1 and "allocation-free" in str(e.value)
    torch.cuda.synchronize()
    assert torch.isnan(Y.float()).all()        # rejected before any GPU work
