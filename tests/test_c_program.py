"""The boundary from C: include/svdq.h compiles as strict C99 (no C++ types in
any signature) and a C program linked against the library runs its host-only
entry points and the host-side argument checks, with no GPU."""

import ctypes
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "rank_outlier_gemm_b200")

C_SRC = r"""
#include <stddef.h>
#include <stdio.h>
#include <string.h>
#include "svdq.h"

int main(void) {
  svdq_prepare_opts o;
  svdq_prepare_opts_default(&o);
  if (o.rank != 32 || o.alpha != 0.5f || o.format != SVDQ_FORMAT_NVFP4) return 10;
  if (svdq_act_codes_bytes(7, 128) != 7 * 64) return 11;
  if (svdq_act_sf_bytes(129, 64) != 256 * 4) return 12;
  if (strstr(svdq_version(), "sm_100a") == NULL) return 13;

  /* K = 96 is not a multiple of 64: rejected on the host, no handle made */
  static uint16_t W[32 * 96];
  float amax[96];
  for (int i = 0; i < 96; ++i) amax[i] = 1.0f;
  svdq_weights* w = NULL;
  svdq_status st = svdq_prepare_weights(W, amax, NULL, 32, 96, &o, NULL, &w);
  if (st != SVDQ_ERR_INVALID_ARG || w != NULL) return 20;
  if (strstr(svdq_last_error(), "multiple of 64") == NULL) return 21;

  /* a null weights handle is an invalid argument for every call that takes one
     (sizes: 0), and the check comes before any GPU work */
  const svdq_weights* nw = NULL;
  double errs[4];
  int n = 0, k = 0, r = 0, rp = 0, fmt = 0;
  float aw = 0.0f;
  svdq_status got[] = {
      svdq_linear_w4a4(nw, NULL, NULL, NULL, 1, NULL, NULL),
      svdq_weights_refine_errors(nw, errs, 4, &n),
      svdq_weights_format(nw, &fmt),
      svdq_attach_lora(NULL, NULL, NULL, 16, 1.0f, NULL),
      svdq_quantize_act_lowrank_down(nw, NULL, 1, NULL, NULL, NULL, NULL),
      svdq_norm_quantize_act_lowrank_down(nw, NULL, 1, NULL, NULL, NULL, NULL, NULL, NULL, NULL),
      svdq_forward_norm(nw, NULL, 1, NULL, NULL, 1e-6f, NULL, NULL, 0, NULL),
      svdq_forward(nw, NULL, 1, NULL, NULL, 0, NULL),
      svdq_forward_host(nw, NULL, 1, NULL, NULL, 0, NULL),
      svdq_forward_noalloc(nw, NULL, 1, NULL, NULL),
      svdq_weights_info(nw, &n, &k, &r, &rp, &aw),
      svdq_weights_export(nw, NULL, NULL, NULL, NULL, NULL, NULL, NULL),
      svdq_debug_launch_stalled_act(nw, NULL, 1, NULL, NULL, NULL, NULL),
      svdq_debug_linear_w4a4_ksplit(nw, NULL, NULL, NULL, 1, NULL, 2, NULL),
      svdq_debug_forward_small_m(nw, NULL, 1, NULL, 0, NULL),
      svdq_act_row_stats(NULL, 1, 64, 1e-6f, NULL, NULL),
      svdq_search_alpha(NULL, NULL, 1, NULL, 16, 64, NULL, 0, &o, NULL, errs, &n),
      svdq_selftest_codec(NULL),
  };
  for (unsigned i = 0; i < sizeof(got) / sizeof(got[0]); ++i)
    if (got[i] != SVDQ_ERR_INVALID_ARG) {
      printf("call %u returned %d\n", i, (int)got[i]);
      return 30;
    }
  if (svdq_weights_sf_bytes(nw) != 0 || svdq_lowrank_bytes(nw, 8) != 0 ||
      svdq_forward_workspace_bytes(nw, 8) != 0 || svdq_forward_norm_workspace_bytes(nw, 8) != 0 ||
      svdq_forward_host_workspace_bytes(nw, 8) != 0)
    return 31;
  if (svdq_weights_destroy(NULL) != SVDQ_OK) return 32;
  if (svdq_weights_rank(nw) != -1) return 33;
  printf("layout %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(svdq_prepare_opts),
         offsetof(svdq_prepare_opts, alpha), offsetof(svdq_prepare_opts, rank),
         offsetof(svdq_prepare_opts, power_iters), offsetof(svdq_prepare_opts, oversample),
         offsetof(svdq_prepare_opts, seed), offsetof(svdq_prepare_opts, keep_residual),
         offsetof(svdq_prepare_opts, refine_iters), offsetof(svdq_prepare_opts, format));
  printf("ok %s\n", svdq_version());
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_a_c_program_links_and_runs(tmp_path):
    lib = os.path.join(LIBDIR, "libsvdq.so")
    assert os.path.exists(lib), "build the library first (__graft_entry__.build())"
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", f"-I{ROOT}/include",
                    str(src), "-o", str(exe), f"-L{LIBDIR}", "-lsvdq", f"-Wl,-rpath,{LIBDIR}"],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    layout, ok = r.stdout.splitlines()
    assert ok.startswith("ok ")
    # the Python binding's copy of svdq_prepare_opts has the C layout
    from rank_outlier_gemm_b200.binding import PrepareOpts
    P = PrepareOpts
    want = [ctypes.sizeof(P)] + [getattr(P, f).offset for f in
                                 ["alpha", "rank", "power_iters", "oversample", "seed", "keep_residual",
                                  "refine_iters", "format"]]
    assert [int(v) for v in layout.split()[1:]] == want
