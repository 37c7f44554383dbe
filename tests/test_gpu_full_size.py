"""Every output of a full-size FLUX.1 layer against the oracle.

The benchmark's configuration exactly: M = 4608 tokens, weights prepared by
the library's own host SVD at rank 32, both kernels as the benchmark launches
them (the activation kernel's K-split and the persistent GEMM over all 148
SMs).  The oracle takes the library's exported split (smoothing multipliers,
16-bit factors and residual; SVDQuant §4.2) and evaluates the layer in float64:
every activation code and scale (including the zero scales of padding rows),
every weight code and scale, every element of T within the fp32 accumulation
bound, and every element of Y within the layer tolerance.  attn_out runs
3072 -> 3072 (36 x 12 output tiles, three per CTA); mlp_down runs the
K = 12288 path (48 K tiles per output tile)."""

import numpy as np
import pytest

from oracle import codec as OC
from oracle import formats as OF
from oracle import svdquant as OS
from synth import config_cases, make_layer_inputs
from tests import gpu_common as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["attn_out", "mlp_down"])
def test_bench_configuration_every_element(name):
    L = G.lib()
    case = [c for c in config_cases("flux") if c.name == name][0]
    t = make_layer_inputs(case)
    w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=case.rank, keep_residual=True)
    ex = L.svdq_weights_export(w, residual=True)
    Y, (xq, xsf, T) = G.run_layer(w, t.X_bits)
    N, K = case.N, case.K
    inv = ex["inv_lam"]
    Rp = ex["residual"]
    codes, scales = OC.quantize_groups(Rp)
    np.testing.assert_array_equal(ex["codes"], OC.pack_codes(codes))
    np.testing.assert_array_equal(ex["sf"], OC.scales_to_atoms(scales))
    prep = OS.Prepared(N, K, ex["rank"], (1.0 / inv.astype(np.float64)).astype(np.float32), inv,
                       OF.bf16_bits_to_f64(ex["L1p"]), OF.bf16_bits_to_f64(ex["L2"]),
                       (Rp.astype(np.float64) * ex["alpha_w"]).astype(np.float32), ex["alpha_w"], Rp, codes,
                       scales, ex["bias"].astype(np.float64))
    G.check_codes(xq, xsf, t.X, inv)
    G.check_T(T, t.X, prep)
    G.check_Y(Y, OS.linear(prep, t.X))
