"""The boundary is a C ABI: a plain C99 program includes include/attn.h, links
libattn.so and calls the entry points that need no GPU (error text, workspace
sizes, the split heuristic, argument validation)."""
import shutil
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "attn.h"

int main(void) {
  if (strlen(attn_strerror(ATTN_ERR_INVALID)) == 0) return 1;
  if (attn_bwd_workspace_size(2, 32, 8192, 128) != (size_t)2 * 8192 * 32 * 128 * 4 + (size_t)2 * 32 * 8192 * 4)
    return 2;
  if (attn_splitkv_num_splits(2, 32, 8192, 8192) != 1) return 3;
  if (attn_splitkv_workspace_size(1, 4, 128, 64, 0) != 0) return 4;
  /* invalid arguments are rejected before anything is launched */
  if (attn_fwd(NULL, NULL, NULL, NULL, 0, NULL, NULL, 1, 4, 2, 128, 128, 128, 0.1f, 0, ATTN_BF16, NULL) !=
      ATTN_ERR_INVALID)
    return 5;
  if (attn_fwd_dv(NULL, NULL, NULL, NULL, NULL, 1, 4, 4, 64, 64, 128, 96, 0.1f, 0, ATTN_BF16, NULL) !=
      ATTN_ERR_UNSUPPORTED)
    return 6;
  if (attn_launch_count(0) != 0) return 7;
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_plain_c_and_links(tmp_path):
    from exact_io_aware_57_b200 import attn

    lib = Path(attn.LIB_PATH)
    src = tmp_path / "use_attn.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_attn"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", str(ROOT / "include"), str(src),
                         "-o", str(exe), str(lib), f"-Wl,-rpath,{lib.parent}"], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)
