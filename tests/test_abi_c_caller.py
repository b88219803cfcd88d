"""The boundary is a plain C interface: a C99 program that includes only include/starkv.h
compiles without a C++ compiler, links against the built library, and calls the host-only
entry points (layout, sizes) without a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "rank_quantized_kv_decode_b200")

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "starkv.h"

int main(void) {
  starkv_config cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.n_q_heads = 32;
  cfg.n_kv_heads = 8;
  cfg.head_dim = 128;
  cfg.d_model = 4096;
  cfg.key_rank = 256;
  for (int g = 0; g < 8; ++g) cfg.value_rank[g] = 32;
  cfg.fmt = STARKV_FMT_MIXED;
  cfg.page_tokens = 64;
  cfg.rope_theta = 500000.0;
  starkv_layout lay;
  if (starkv_layout_init(&cfg, &lay) != STARKV_OK) {
    printf("layout: %s\n", starkv_last_error());
    return 1;
  }
  starkv_sizes sz;
  if (starkv_alloc(&lay, 100, 2, 8, 16, &sz) != STARKV_OK) return 2;
  int64_t rows = 0;
  size_t scratch = 0;
  if (starkv_absorbed_sizes(&lay, 2, 4096, &rows, &scratch) != STARKV_OK) return 3;
  /* the hybrid assignment: a key latent per KV head, one joint value latent */
  starkv_hybrid_config hc;
  memset(&hc, 0, sizeof hc);
  hc.n_q_heads = 32;
  hc.n_kv_heads = 8;
  hc.head_dim = 128;
  hc.d_model = 4096;
  for (int g = 0; g < 8; ++g) hc.key_rank[g] = 16 * (1 + g % 3);
  hc.value_rank = 256;
  hc.fmt = STARKV_FMT_MIXED;
  hc.page_tokens = 64;
  hc.rope_theta = 500000.0;
  starkv_layout hl;
  if (starkv_hybrid_layout_init(&hc, &hl) != STARKV_OK) return 4;
  if (hl.assignment != STARKV_ASSIGN_HYBRID || hl.n_latents != 9) return 5;
  starkv_sizes hs;
  if (starkv_alloc(&hl, 100, 2, 8, 16, &hs) != STARKV_OK) return 6;
  /* a joint-key call refuses the hybrid layout before touching the device */
  if (starkv_absorbed_sizes(&hl, 2, 4096, &rows, &scratch) != STARKV_ERR_UNSUPPORTED) return 7;
  printf("%lld %lld %lld %d %d %lld\n", (long long)lay.page_bytes, (long long)sz.cache_bytes,
         (long long)rows, starkv_version(), hl.proj_cols, (long long)hs.cache_bytes);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c99_caller_compiles_links_and_runs_host_calls(tmp_path):
    lib = os.path.join(LIB_DIR, "libstarkv.so")
    if not os.path.exists(lib):
        from rank_quantized_kv_decode_b200.build import build
        build()
    src = tmp_path / "caller.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "caller"
    proc = subprocess.run(
        ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
         "-o", str(exe), "-L", LIB_DIR, "-lstarkv", "-Wl,-rpath," + LIB_DIR,
         "-Wl,--unresolved-symbols=ignore-in-shared-libs"],
        capture_output=True, text=True)
    assert proc.returncode == 0, proc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True,
                         env=dict(os.environ, LD_LIBRARY_PATH=LIB_DIR + ":" +
                                  os.environ.get("LD_LIBRARY_PATH", "")))
    if run.returncode != 0 and "error while loading shared libraries" in run.stderr:
        pytest.skip("the CUDA runtime the library links is not on the loader path here")
    assert run.returncode == 0, run.stdout + run.stderr
    page_bytes, cache_bytes, rows, version, hproj, hcache = (int(v) for v in run.stdout.split())
    assert cache_bytes == 100 * page_bytes and rows == 4 * 8 * 32 and version > 0
    assert hproj == sum(16 * (1 + g % 3) for g in range(8)) + 256 and hcache % 100 == 0
