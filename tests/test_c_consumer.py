"""The boundary as a C program sees it: include/rosa.h compiles as C99 with
warnings as errors, a program links against the in-tree library, and its
host-only calls answer without a GPU (sizes, launch counts, status names,
argument errors returned before anything is enqueued)."""
import os
import shutil
import subprocess

import pytest

from tests.conftest import ROOT

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "rosa.h"

int main(void) {
    /* workspace sizes grow with the problem and are 0 for invalid sizes */
    size_t a = rosa_match_workspace_size(4, 1000, 256);
    size_t b = rosa_match_workspace_size(8, 1000, 256);
    if (a == 0 || b <= a) { printf("workspace %zu %zu\n", a, b); return 1; }
    if (rosa_match_workspace_size(-1, 10, 4) != 0) return 2;
    if (rosa_match_workspace_size(1, 10, 0) != 0) return 3;
    /* launch counts: -1 for invalid sizes, 0 for empty work, positive otherwise */
    if (rosa_match_launch_count(1, 10, 0, 1) != -1) return 4;
    if (rosa_match_launch_count(0, 10, 4, 1) != 0) return 5;
    if (rosa_match_launch_count(2, 4096, 2, 1) <= 0) return 6;
    /* argument errors come back before any device work */
    int32_t dummy = 0;
    if (rosa_match(NULL, NULL, NULL, 2, 16, 300, 2, &dummy, &dummy, &dummy, NULL, 0, NULL)
        != ROSA_ERR_INVALID_ARG) return 7;
    if (rosa_discretize(NULL, 1, 4, 6, 4, NULL, NULL) != ROSA_ERR_INVALID_ARG) return 8;
    if (strlen(rosa_status_string(ROSA_ERR_WORKSPACE)) == 0) return 9;
    printf("ok %zu %d\n", a, rosa_match_launch_count(2, 4096, 2, 1));
    return 0;
}
"""


def _cuda_include():
    for root in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if root and os.path.exists(os.path.join(root, "include", "cuda_runtime_api.h")):
            return os.path.join(root, "include")
    nvcc = shutil.which("nvcc")
    if nvcc:
        inc = os.path.join(os.path.dirname(os.path.dirname(nvcc)), "include")
        if os.path.exists(os.path.join(inc, "cuda_runtime_api.h")):
            return inc
    return None


def test_c_program_links_and_calls_host_entry_points(tmp_path):
    gcc, inc = shutil.which("gcc"), _cuda_include()
    if not gcc or not inc:
        pytest.skip("gcc or the CUDA headers are missing")
    from suffix_automaton_retrieval_b200 import build
    lib = build.build()
    libdir = os.path.dirname(lib)
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", inc,
           str(src), "-o", str(exe), "-L", libdir, "-lrosa_b200", f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.startswith("ok ")
