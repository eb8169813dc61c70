"""The C ABI from C (no GPU needed).

include/la.h must compile as strict C99 and as C++11, and a C program must
link against libla.so and call it: the boundary is usable without Python.
The program only calls entry points that need no device (feature dimensions,
status strings, workspace sizes, kernel plans, argument errors).
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "la.h"

int main(void)
{
    char names[256];
    int fails = 0;
    if (la_feature_dim(LA_FMAP_TAYLOR2, 16) != 273) ++fails;
    if (la_feature_dim(LA_FMAP_TAYLOR2_SYM, 16) != 153) ++fails;
    if (la_feature_dim(LA_FMAP_ELU1, 64) != 64) ++fails;
    if (strcmp(la_status_string(LA_ERR_INVALID_ARG), "LA_ERR_INVALID_ARG") != 0) ++fails;
    /* the headline forward plans two launches and needs a workspace */
    if (la_kernel_plan(0, 4, 8, 4096, 64, 64, LA_FMAP_ELU1, LA_BF16, names, sizeof names) != 2) ++fails;
    if (strstr(names, "fwd_split_out_kernel") == NULL) ++fails;
    if (la_forward_workspace_bytes(4, 8, 4096, 64, 64, LA_FMAP_ELU1, LA_BF16) == 0) ++fails;
    /* argument errors come back before anything touches a device */
    if (la_forward(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, 1, 16, 64, 64, LA_FMAP_ELU1, LA_BF16, NULL)
        != LA_ERR_INVALID_ARG) ++fails;
    if (la_decode_step(NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, 16, 64, LA_FMAP_TAYLOR2, LA_F32, NULL)
        != LA_ERR_INVALID_ARG) ++fails;
    printf("%d\n", fails);
    return fails != 0;
}
"""


def _cc(name):
    path = shutil.which(name)
    if path is None:
        pytest.skip(f"{name} not installed")
    return path


@pytest.mark.parametrize("std,compiler,lang", [("c99", "gcc", "c"), ("c++11", "g++", "c++")])
def test_header_compiles_strictly(tmp_path, std, compiler, lang):
    src = tmp_path / "use.c"
    src.write_text('#include "la.h"\nint main(void) { return (int)sizeof(la_status) + LA_FMAP_TAYLOR2_SYM - 6; }\n')
    subprocess.run([_cc(compiler), f"-std={std}", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", INCLUDE,
                    "-x", lang, "-c", str(src), "-o", str(tmp_path / "use.o")], check=True)


def test_c_program_links_and_calls_the_library(tmp_path):
    from causal_kernelized_sequence_b200 import build
    lib = build.build()
    src = tmp_path / "prog.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "prog"
    subprocess.run([_cc("gcc"), "-std=c99", "-Wall", "-Werror", "-I", INCLUDE, str(src), "-o", str(exe),
                    lib, f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "0"
