"""The C ABI from plain C: include/flce.h compiles as C99 (CPU), and a C program linked
against libflce.so runs the fused forward on the GPU."""
import os
import subprocess

import pytest

from lm_head_linear_gemm_b200 import _abi
from lm_head_linear_gemm_b200 import build as flce_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "flce_c_smoke.c")
CUDA_INC = "/usr/local/cuda/include"


def test_header_is_plain_c():
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I",
                    os.path.join(ROOT, "include"), "-I", CUDA_INC, SRC], check=True)


@pytest.mark.gpu
def test_c_program_runs_on_gpu(tmp_path, cuda_device):
    flce_build.build(quiet=True)
    exe = tmp_path / "flce_c_smoke"
    libdir = os.path.dirname(_abi.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-O2", "-I", os.path.join(ROOT, "include"), "-I", CUDA_INC,
                    SRC, "-o", str(exe), "-L", libdir, "-lflce", "-L", "/usr/local/cuda/lib64",
                    "-lcudart", "-lm", f"-Wl,-rpath,{libdir}",
                    "-Wl,-rpath,/usr/local/cuda/lib64"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    print(out.stdout, out.stderr)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "status 0" in out.stdout
