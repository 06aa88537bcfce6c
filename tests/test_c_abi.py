"""The boundary from C: every public header compiles as C99 (gcc, strict), and
a C program linked against libdynconv.so calls the host-side entry points
(status strings, variant choice, workspace sizes, argument refusals, the loud
failure with no device) and gets the values the Python binding gets."""
import os
import subprocess

import pytest

import dynamic_convolution_b200 as dc
from dynamic_convolution_b200 import build as dcbuild
from dynamic_convolution_b200 import synth

INCLUDE = os.path.join(dcbuild.ROOT, "include")
HEADERS = ("dynconv.h", "dynconv_backward.h", "dynconv_cells.h")

PROGRAM = r"""
#include <stdio.h>
#include "dynconv.h"
#include "dynconv_backward.h"
#include "dynconv_cells.h"

int main(void) {
  dynconv_desc d = {64, 128, 28, 28, 128, 3, 3, 1, 1, 1, 4, DYNCONV_BF16, DYNCONV_VARIANT_AUTO};
  printf("status %s|%s\n", dynconv_status_string(DYNCONV_OK),
         dynconv_status_string(DYNCONV_ERR_WORKSPACE));
  printf("variant %d\n", dynconv_select_variant(&d, dynconv_workspace_size(&d)));
  printf("ws %zu %zu\n", dynconv_workspace_size(&d), dynconv_backward_workspace_size(&d));
  dynconv_desc c = d;
  c.n = 128;
  printf("cells %zu\n", dynconv_cells_workspace_size(&c, 16));
  dynconv_desc bad = d;
  bad.groups = 3;
  printf("bad %d\n", dynconv_forward(&bad, (void*)256, (void*)256, (float*)256, 0, (void*)256, 0, 0, 0));
  printf("nodev %d\n", dynconv_route(&d, (void*)256, (float*)256, 0, DYNCONV_SOFTMAX, 1.0f,
                                     (float*)256, 0));
  return 0;
}
"""


@pytest.mark.parametrize("header", HEADERS)
def test_header_compiles_as_c(tmp_path, header):
    src = tmp_path / "inc.c"
    src.write_text(f'#include "{header}"\nint main(void) {{ return 0; }}\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    f"-I{INCLUDE}", "-I/usr/local/cuda/include", "-fsyntax-only", str(src)],
                   check=True)


def test_c_program_against_the_library(tmp_path):
    lib = dcbuild.build()
    src = tmp_path / "prog.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "prog"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", f"-I{INCLUDE}", str(src), "-o", str(exe),
                    lib, f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    lines = dict(line.split(" ", 1) for line in out.strip().splitlines())
    d = dc.desc_from_config(synth.CONFIGS["resnet18_3x3"])
    assert lines["status"] == f"{dc.dynconv_status_string(dc.OK)}|" \
                              f"{dc.dynconv_status_string(dc.ERR_WORKSPACE)}"
    assert int(lines["variant"]) == dc.dynconv_select_variant(d, dc.dynconv_workspace_size(d))
    assert lines["ws"].split() == [str(dc.dynconv_workspace_size(d)),
                                   str(dc.dynconv_backward_workspace_size(d))]
    c = dc.desc_from_config(synth.CONFIGS["resnet18_3x3"])
    c.n = 128
    assert int(lines["cells"]) == dc.dynconv_cells_workspace_size(c, 16) > 0
    assert int(lines["bad"]) == dc.ERR_INVALID_ARG
    assert int(lines["nodev"]) == dc.ERR_CUDA
