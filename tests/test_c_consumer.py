"""The boundary is a C ABI: a plain C11 program (and the same file built as
C++) compiles against include/ipe.h with every warning an error, links
libipe.so and calls the host-only entry points without a GPU."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import interpolated_position_encoding_b200 as ipe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "ipe.h"

int main(void)
{
    float inv[32];
    int i;
    if (ipe_rope_inv_freq(64, 1e7, inv) != IPE_OK) return 1;
    if (ipe_rope_inv_freq(7, 1e4, inv + 16) != IPE_EINVAL) return 2;
    if (strlen(ipe_last_error()) == 0) return 3;
    printf("%d\n", ipe_version());
    for (i = 0; i < 32; ++i) printf("%.9e\n", (double)inv[i]);
    return 0;
}
"""


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-std=c11"]), ("g++", ["-x", "c++", "-std=c++17"])])
def test_c_program_uses_the_abi(compiler, flags, tmp_path, orc):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not available")
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    libdir = os.path.dirname(ipe.lib()._name)
    exe = tmp_path / "consumer"
    cmd = [compiler, *flags, "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-x", "none", "-L", libdir, "-lipe", f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    p = subprocess.run(cmd, capture_output=True, text=True)
    assert p.returncode == 0, p.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stderr)
    lines = r.stdout.split()
    assert int(lines[0]) == ipe.lib().ipe_version()
    got = np.array([float(v) for v in lines[1:]], np.float32)
    assert np.array_equal(got.view(np.uint32), orc.rope_inv_freq(64, 1e7).view(np.uint32))
