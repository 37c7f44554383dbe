"""The allocation-free forward (svdq_forward_noalloc) against svdq_forward.

Callers that cannot allocate device memory (allocator callbacks, captures
whose pool forbids allocation, fully reserved serving pools) use this entry
point; it keeps the layer's intermediates in a static device block that every
call reuses.  Two calls in a row on different inputs must each match the
workspace-based svdq_forward within the layer tolerance, and a layer too large
for the block must be rejected up front."""

import numpy as np
import pytest
import torch

from oracle import svdquant as OS
from synth import config_cases, make_layer_inputs
from tests import gpu_common as G

pytestmark = pytest.mark.gpu


def _forward_with_workspace(L, w, X):
    M = X.shape[0]
    Y = torch.empty((M, w.info["N"]), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.svdq_forward_workspace_bytes(w, M), dtype=torch.uint8, device="cuda")
    L.svdq_forward(w, X, Y, ws)
    return Y


def test_forward_noalloc_matches_forward_on_two_calls():
    L = G.lib()
    case = [c for c in config_cases("pixart") if c.name == "mlp_up"][0]
    t1 = make_layer_inputs(case, M=300)
    prep = OS.prepare(t1.W, t1.act_absmax, t1.bias, case.rank)
    w = G.weights_from_oracle(prep)
    rng = np.random.default_rng(5)
    X1 = G.to_dev_bf16(t1.X_bits)
    X2 = G.to_dev_bf16(t1.X_bits[rng.permutation(300)[:200]])
    for X in (X1, X2):
        ref = _forward_with_workspace(L, w, X).float().cpu().numpy().astype(np.float64)
        Y = torch.empty((X.shape[0], case.N), dtype=torch.bfloat16, device="cuda")
        L.svdq_forward_noalloc(w, X, Y)
        assert L.svdq_check_device_errors() == 0
        G.check_Y(Y.float().cpu().numpy().astype(np.float64), ref)


def test_forward_noalloc_rejects_layers_beyond_its_block():
    L = G.lib()
    case = [c for c in config_cases("flux") if c.name == "mlp_down"][0]   # K = 12288
    t = make_layer_inputs(case, M=8)
    K = case.K
    prep = OS.prepare_from_factors(t.W[:64], np.ones(K, np.float32), np.zeros((K, 0)), np.zeros((0, 64)), None)
    w = G.weights_from_oracle(prep)
    M = 8192                                  # 8192 x 12288 / 2 bytes of codes alone exceed 32 MiB
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((M, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.SvdqError) as e:
        L.svdq_forward_noalloc(w, X, Y)
    assert e.value.status == 1 and "allocation-free" in str(e.value)
