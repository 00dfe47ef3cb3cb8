"""The boundary is a C ABI: a plain C program (tests/c_abi/abi_from_c.c),
compiled with gcc against include/flce.h and linked to libflce.so, calls the
entry points that need no GPU.  Runs on the CPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "lm_head_projection_flce_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_links_and_calls_the_abi(tmp_path):
    from lm_head_projection_flce_b200 import build
    build.build()
    exe = tmp_path / "abi_from_c"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", f"-I{os.path.join(ROOT, 'include')}",
                    os.path.join(ROOT, "tests", "c_abi", "abi_from_c.c"), f"-L{LIB_DIR}", "-lflce",
                    f"-Wl,-rpath,{LIB_DIR}", "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    assert "C ABI ok" in res.stdout
