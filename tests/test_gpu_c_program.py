"""A plain C program (tests/c_abi/zero_head_from_c.c) allocates device memory
with the CUDA runtime, runs forward and backward through the C ABI and checks
the closed form of a zero head (lse = log V, loss = #valid * log V, dhidden =
0, dW[v] = #valid/V - #labels equal to v, with all-ones hidden)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "lm_head_projection_flce_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

pytestmark = pytest.mark.gpu


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_on_the_gpu_matches_the_zero_head_closed_form(tmp_path):
    from lm_head_projection_flce_b200 import build
    build.build()
    exe = tmp_path / "zero_head_from_c"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", f"-I{os.path.join(ROOT, 'include')}",
                    f"-I{os.path.join(CUDA, 'include')}",
                    os.path.join(ROOT, "tests", "c_abi", "zero_head_from_c.c"), f"-L{LIB_DIR}",
                    "-lflce", f"-L{os.path.join(CUDA, 'lib64')}", "-lcudart", "-lm",
                    f"-Wl,-rpath,{LIB_DIR}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}",
                    "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "zero head from C ok" in res.stdout
