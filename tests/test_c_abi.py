"""The C ABI used from plain C, with no Python in between.

include/streamkl.h must compile as C99 and as C++ (it is included by C and
C++ callers alike), and a C program linked against libstreamkl.so must be able
to call the host-side entry points: the version, the error strings, the
workspace size, and argument checking that rejects a bad call before any CUDA
call (so this runs on a machine without a GPU).  The ctypes tests
(tests/test_abi.py) check the same entry points through Python; this one shows
that the header, the exported names and the calling convention agree for a C
caller.
"""
import os
import shutil
import subprocess

import pytest

from attention_kl_divergence_attn_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "streamkl.h"

int main(void) {
    const void *p = (const void *)16;            /* aligned, never dereferenced */
    float *f = (float *)16;
    char ws[256];
    if (streamkl_version() <= 0) return 10;
    if (streamkl_workspace_size(1, 32, 8192, 8192, 128, 128, 1) < 256) return 11;
    if (strlen(streamkl_strerror(STREAMKL_ERR_INVALID_ARG)) == 0) return 12;
    if (strlen(streamkl_strerror(STREAMKL_ERR_BOUNDS)) == 0) return 13;
    /* rejected before any CUDA call: a head dimension the kernels do not cover */
    if (streamkl_fwd(p, p, p, p, 1, 1, 128, 128, 96, 64, 0.1f, 0.1f, 0, f, f, f, NULL,
                     ws, sizeof ws, NULL) != STREAMKL_ERR_UNSUPPORTED) return 14;
    /* causal with more queries than keys */
    if (streamkl_fwd(p, p, p, p, 1, 1, 200, 100, 64, 64, 0.1f, 0.1f, 1, f, f, f, NULL,
                     ws, sizeof ws, NULL) != STREAMKL_ERR_INVALID_ARG) return 15;
    /* no workspace */
    if (streamkl_fwd(p, p, p, p, 1, 1, 128, 128, 64, 64, 0.1f, 0.1f, 0, f, f, f, NULL,
                     NULL, 0, NULL) != STREAMKL_ERR_WORKSPACE) return 16;
    /* a teacher gradient pair must be complete */
    if (streamkl_bwd(p, p, p, p, 1, 1, 128, 128, 64, 64, 0.1f, 0.1f, 0, f, f, f, NULL, 1.0f,
                     f, f, f, NULL, ws, sizeof ws, NULL) != STREAMKL_ERR_INVALID_ARG) return 17;
    printf("ok\n");
    return 0;
}
"""


def _compiler(name):
    path = shutil.which(name)
    if path is None:
        pytest.skip(f"{name} not available")
    return path


@pytest.mark.parametrize("lang", ["c99", "c++11"])
def test_header_compiles(tmp_path, lang):
    cc = _compiler("gcc" if lang == "c99" else "g++")
    src = tmp_path / ("h.c" if lang == "c99" else "h.cpp")
    src.write_text('#include "streamkl.h"\nint main(void) { return streamkl_version() > 0 ? 0 : 1; }\n')
    subprocess.run([cc, f"-std={lang}", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", INCLUDE, "-c",
                    str(src), "-o", str(tmp_path / "h.o")], check=True)


def test_a_c_program_calls_the_library(tmp_path):
    cc = _compiler("gcc")
    lib = build.build()
    src = tmp_path / "prog.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "prog"
    libdir = os.path.dirname(lib)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, str(src), "-o", str(exe),
                    lib, f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.strip() == "ok"
