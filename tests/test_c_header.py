"""include/fia.h is a plain C header: a C11 program compiles against it with
warnings as errors, links libfia.so and calls it (no GPU needed: the calls
below are rejected before any device work)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "fia.h"

int main(void) {
    uint64_t ws = 1;
    fia_op *op = (fia_op *)&ws;
    fia_plan_info info;
    /* every argument NULL: rejected before anything is read */
    fia_status st = fia_get_workspace_size(NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, 0, 0, 0,
                                           0.0f, NULL, NULL, &ws, &op);
    if (st != FIA_ERR_NULLPTR || ws != 0 || op != NULL) return 1;
    if (fia_run(NULL, 0, NULL, NULL) != FIA_ERR_NULLPTR) return 2;
    if (fia_op_get_plan_info(NULL, &info) != FIA_ERR_NULLPTR) return 3;
    if (fia_decode_run_static(NULL, NULL) != FIA_ERR_NULLPTR) return 4;
    if (strlen(fia_status_string(FIA_ERR_SHAPE)) == 0) return 5;
    uint32_t word = 7;
    if (fia_decode_static_error_word(NULL, &word) != FIA_ERR_NULLPTR) return 6;
    if (fia_op_set_wait_limit(NULL, 0, 0) != FIA_ERR_NULLPTR) return 7;
    printf("%s\n", fia_status_string(FIA_OK));
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_links(tmp_path):
    import __graft_entry__
    lib = __graft_entry__.load_builder().build()
    src = tmp_path / "use_fia.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "use_fia"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(lib),
           "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.strip()
