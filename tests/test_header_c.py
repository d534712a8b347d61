"""The C ABI from C: include/situ_glu.h compiles as C11 with warnings as
errors, a C program that takes the address of every declared function links
against libsitu_glu.so, and running it calls the entry points that need no
GPU (version, status strings, an argument error, the workspace query)."""
import os
import re
import shutil
import subprocess

import pytest

from ffn_gated_activation_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "situ_glu.h")


def declared():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(situ_(?:glu|attn_res)_\w+)\s*\(", text, flags=re.M)))


PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "situ_glu.h"

int main(void) {
  const void *fns[] = { %(fns)s };
  for (size_t i = 0; i < sizeof fns / sizeof fns[0]; ++i)
    if (fns[i] == NULL) return 10;
  if (situ_glu_abi_version() != SITU_GLU_ABI_VERSION) return 11;
  if (strlen(situ_glu_status_string(SITU_ERR_INVALID_ARG)) == 0) return 12;
  /* a negative token count is rejected on the host, before any CUDA call */
  if (situ_glu_fwd(NULL, SITU_DTYPE_BF16, -1, 64, 128, NULL, SITU_DTYPE_F32, SITU_RW_NONE, 1, 4.0, 1, 25.0,
                   NULL, 64, NULL) != SITU_ERR_INVALID_ARG) return 13;
  if (strlen(situ_glu_last_error()) == 0) return 14;
  if (situ_glu_bwd_workspace_bytes(1024, 256, SITU_RW_SCALAR, 1) == 0) return 15;
  printf("%%d\n", situ_glu_abi_version());
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_and_links_from_c(native_lib_path, tmp_path):
    names = declared()
    assert len(names) >= 15
    src = tmp_path / "use_abi.c"
    src.write_text(PROGRAM % {"fns": ", ".join(f"(const void *)&{n}" for n in names)})
    exe = tmp_path / "use_abi"
    lib_dir = os.path.dirname(native_lib_path)
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I",
           os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", lib_dir, "-lsitu_glu",
           f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert int(run.stdout.strip()) == abi.ABI_VERSION
