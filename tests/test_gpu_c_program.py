"""The C ABI from a plain C program on the GPU: fa_build_basis, fa_compress and fa_decode on
device buffers allocated with the CUDA runtime, checked inside the program against the
oracle values stored in tests/golden/c_abi_gpu_case.txt."""
import os
import subprocess

import pytest

import fourier_basis_attention_b200 as fa

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def build_c_program(out_path):
    libdir = os.path.dirname(fa.LIB_PATH)
    cudalib = os.path.join(CUDA_HOME, "lib64")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA_HOME, "include"),
                    os.path.join(ROOT, "tests", "c_abi_gpu.c"), "-o", str(out_path),
                    "-L", libdir, "-lfourier_attention", "-L", cudalib, "-lcudart", "-lm",
                    f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{cudalib}"], check=True)


def test_c_program_compresses_and_decodes_on_the_gpu(tmp_path):
    exe = tmp_path / "c_abi_gpu"
    build_c_program(exe)
    out = subprocess.run([str(exe), os.path.join(ROOT, "tests", "golden", "c_abi_gpu_case.txt")],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
