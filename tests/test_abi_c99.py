"""include/stem.h is a plain C header: a C99 program that includes it, takes the address of
every entry point and calls the host-only ones links against libstem.so and agrees with
the oracle's budget plan.  No GPU call is made."""
import os
import shutil
import subprocess

import pytest

from block_sparse_attention_oam_b200 import build as B
from block_sparse_attention_oam_b200 import stem as S
from oracle import stem_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "stem.h"

typedef void (*any_fn)(void);

int main(void) {
  /* every entry point the header declares, by address */
  any_fn fns[] = {
    (any_fn)stem_query_sizes, (any_fn)stem_workspace_size, (any_fn)stem_tpd_plan, (any_fn)stem_score,
    (any_fn)stem_select, (any_fn)stem_score_select, (any_fn)bsa_prefill, (any_fn)bsa_dense_prefill, (any_fn)stem_attention,
    (any_fn)stem_attention_host, (any_fn)stem_attention_noalloc, (any_fn)stem_query_status,
    (any_fn)stem_reset_status, (any_fn)stem_debug_inject, (any_fn)stem_status_string, (any_fn)stem_last_error};
  for (unsigned i = 0; i < sizeof(fns) / sizeof(fns[0]); ++i)
    if (fns[i] == 0) return 10;

  double r = 0.0;
  int64_t total = 0;
  if (stem_tpd_plan(1024, 0.25, 0.7, &r, &total) != STEM_OK) return 11;
  printf("plan %.17g %lld\n", r, (long long)total);

  int32_t cu[3] = {0, 300, 2412};
  stem_problem_t p = {0};
  p.num_seqs = 2; p.cu_seqlens = cu; p.num_q_heads = 8; p.num_kv_heads = 2; p.head_dim = 128;
  p.block_size = 128; p.dtype = STEM_DT_BF16; p.q_scale = p.k_scale = p.v_scale = 1.0f;
  p.softmax_scale = 0.0f; p.beta = 0.2f; p.keep = 0.25; p.mu = 0.7; p.shared_lists = 0;
  stem_sizes_t sz;
  if (stem_query_sizes(&p, &sz) != STEM_OK) return 12;
  if (stem_workspace_size(&p) != sz.workspace_bytes) return 13;
  printf("sizes %lld %lld %lld %lld %lld\n", (long long)sz.num_rows, (long long)sz.scores_per_head,
         (long long)sz.nnz_per_head, (long long)sz.total_tokens, (long long)sz.list_heads);

  /* refused on the host, before any CUDA call */
  if (stem_attention(NULL, 0, 0, 0, NULL, 0, NULL, NULL, NULL, 0, 0, NULL) != STEM_ERR_INVALID) return 14;
  if (stem_last_error()[0] == '\0') return 15;
  p.num_kv_heads = 3;
  if (stem_query_sizes(&p, &sz) != STEM_ERR_INVALID) return 16;
  printf("status %s\n", stem_status_string(STEM_ERR_TIMEOUT));
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib_dir():
    B.build()
    S.lib()
    return os.path.dirname(S.LIB_PATH)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_c99_and_links(lib_dir):
    work = os.path.join(lib_dir, "_build", "c99")
    os.makedirs(work, exist_ok=True)
    src, exe = os.path.join(work, "abi.c"), os.path.join(work, "abi")
    with open(src, "w") as f:
        f.write(PROGRAM)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", src, "-I",
                         os.path.join(ROOT, "include"), "-L", lib_dir, "-lstem", "-Wl,-rpath," + lib_dir, "-o", exe],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    out = dict((ln.split(" ", 1)[0], ln.split(" ", 1)[1]) for ln in run.stdout.splitlines())
    r, total = out["plan"].split()
    r_o, _, k_o = O.tpd_plan(1024, 0.25, 0.7)
    assert float(r) == r_o and int(total) == int(sum(k_o))
    rows, spc, nnz, tokens, lists = map(int, out["sizes"].split())
    assert (rows, tokens, lists) == (3 + 17, 2412, 8)
    assert spc == 3 * 4 // 2 + 17 * 18 // 2
    assert out["status"] == "device pipeline wait timed out"
