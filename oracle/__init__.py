"""CPU oracle for the SVDQuant W4A4 + low-rank linear layer.

TEST INFRASTRUCTURE ONLY.  A plain, slow, float64 NumPy restatement of what the
layer computes, written from the SVDQuant pages (paperlayer.ai summary of
arXiv 2411.05007v4).  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import it.  It shares no code with the CUDA
library and never imports it.

Modules:
  formats   E2M1 / E4M3 / bf16 encode and decode from their bit definitions
  codec     NVFP4 group-16 codec, nibble packing, block-scale atom layout
  svdquant  smoothing, SVD split, residual, weight factor, output, LoRA
  int4      INT4 variant: group-64 codec with bf16 scales, nibble packing, output
  norm      LayerNorm + per-channel modulation in front of the layer (fused path)

Parity status: every function is pinned by a CPU test against library casts,
brute force, closed forms or invariants (tests/test_oracle_*.py).
"""

from . import codec, formats, int4, norm, svdquant  # noqa: F401
