"""A plain C program compiled against include/nsa.h and linked to libnsa_b200.so.

Shows the boundary is a C ABI usable without Python: the program calls the entry points
that need no GPU (version, error strings, workspace sizes, argument validation) and
prints what they return.
"""
import os
import shutil
import subprocess

import pytest

from sparse_attention_long_fwd_b200 import nsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include "nsa.h"

int main(void) {
  nsa_params_t p = {0};
  p.n_tokens = 4096; p.n_video = 4096; p.num_q_heads = 28; p.num_kv_heads = 4; p.head_dim = 128;
  p.cmp_block = 32; p.cmp_stride = 16; p.sel_block = 64; p.top_n = 16; p.window = 512;
  p.softmax_scale = 0.0f; p.out_dtype = NSA_OUT_F32; p.batch = 2;
  printf("version %s\n", nsa_version());
  printf("invalid %s\n", nsa_error_string(NSA_ERR_INVALID_ARG));
  printf("ws_prefill %zu\n", nsa_workspace_size(&p, 0));
  printf("ws_decode %zu\n", nsa_workspace_size(&p, 1));
  printf("ws_backward %zu\n", nsa_backward_workspace_size(&p));
  printf("ws_pooled %zu\n", nsa_gate_mlp_pooled_workspace_size(2, 4096, 28, 128));
  printf("prefill_null %d\n", nsa_prefill(0, 0, 0, 0, &p, 0, 0, 0, 0, 0));
  printf("gate_dim %d\n", nsa_gate_mlp((void*)0x100000, (void*)0x100000, (float*)0x100000, (float*)0x100000,
                                        (float*)0x100000, 10, 96, (float*)0x100000, 0));
  p.head_dim = 96;
  printf("ws_bad %zu\n", nsa_workspace_size(&p, 0));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_calls_the_abi(tmp_path):
    lib = nsa.load_library()._name
    libdir = os.path.dirname(lib)
    src = tmp_path / "consumer.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "consumer"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                           "-L", libdir, "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    vals = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert vals["version"].startswith("nsa-b200")
    assert vals["invalid"] == nsa.nsa_error_string(nsa.NSA_ERR_INVALID_ARG)
    p = nsa.make_params(4096, 4096, 28, 4, 128, batch=2)
    assert int(vals["ws_prefill"]) == nsa.nsa_workspace_size(p, False) > 0
    assert int(vals["ws_decode"]) == nsa.nsa_workspace_size(p, True) > 0
    assert int(vals["ws_backward"]) == nsa.nsa_backward_workspace_size(p) > 0
    assert int(vals["ws_pooled"]) == nsa.nsa_gate_mlp_pooled_workspace_size(2, 4096, 28, 128) > 0
    assert int(vals["prefill_null"]) == nsa.NSA_ERR_INVALID_ARG
    assert int(vals["gate_dim"]) == nsa.NSA_ERR_UNSUPPORTED
    assert int(vals["ws_bad"]) == 0
