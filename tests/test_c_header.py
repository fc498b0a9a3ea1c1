"""include/moe.h as a plain C interface (no GPU needed): a C99 program that
includes it compiles with gcc -Wall -Wextra -Werror, links against the
library, and runs the entry points that stop before any device call. The
struct layouts it prints match the Python binding's ctypes structures, so
the binding marshals the same bytes the C callers do."""
import ctypes
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stddef.h>
#include <stdio.h>
#include <string.h>
#include "moe.h"

int main(void) {
  moe_config_t c;
  if (moe_config_init_k2(&c) != MOE_OK) return 1;
  if (c.hidden_size != 7168 || c.n_routed_experts != 384 || c.num_experts_per_tok != 8) return 2;
  if (moe_config_init_k2(NULL) != MOE_ERR_INVALID_ARG) return 3;
  c.n_group = 64; /* rejected before any device call */
  moe_handle_t* h = NULL;
  if (moe_create(&c, 0, &h) != MOE_ERR_UNSUPPORTED || h != NULL) return 4;
  if (strcmp(moe_status_string(MOE_OK), "ok") != 0) return 5;
  if (moe_forward(NULL, NULL, 0, NULL, NULL, NULL) != MOE_ERR_INVALID_ARG) return 6;
  printf("config %zu %zu %zu %zu %zu\n", sizeof(moe_config_t),
         offsetof(moe_config_t, routed_scaling_factor), offsetof(moe_config_t, weight_block_size),
         offsetof(moe_config_t, max_tokens), offsetof(moe_config_t, single_launch_max_tokens));
  printf("weights %zu %zu\n", sizeof(moe_weights_t), offsetof(moe_weights_t, shared_down_scale));
  printf("opts %zu %zu %zu %zu\n", sizeof(moe_forward_opts_t), offsetof(moe_forward_opts_t, flags),
         offsetof(moe_forward_opts_t, pair_rows_out), offsetof(moe_forward_opts_t, wait_limit_ns));
  return 0;
}
"""


@pytest.fixture(scope="module")
def smoe():
    import __graft_entry__
    __graft_entry__.build()
    import sparse_moe_sigmoid_b200 as m
    return m


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_c99_and_layouts_match_the_binding(smoe, tmp_path):
    src = tmp_path / "use_moe.c"
    exe = tmp_path / "use_moe"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(smoe.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(smoe.LIB_PATH),
           "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    got = {line.split()[0]: [int(v) for v in line.split()[1:]] for line in r.stdout.splitlines()}
    C, W, O = smoe.moe_config_t, smoe.moe_weights_t, smoe.moe_forward_opts_t
    assert got["config"] == [ctypes.sizeof(C), C.routed_scaling_factor.offset,
                             C.weight_block_size.offset, C.max_tokens.offset,
                             C.single_launch_max_tokens.offset]
    assert got["weights"] == [ctypes.sizeof(W), W.shared_down_scale.offset]
    assert got["opts"] == [ctypes.sizeof(O), O.flags.offset, O.pair_rows_out.offset,
                           O.wait_limit_ns.offset]
