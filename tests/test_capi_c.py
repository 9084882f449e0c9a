"""The C ABI used from a plain C program (tests/c/capi_from_c.c) through the
public header alone: compiled with gcc against the built library (and, for
the GPU mode, the CUDA runtime and the CPU oracle) and run as a separate
process."""
import os
import subprocess

import pytest
import torch

import oracle
import residual_add_rmsnorm_rms_b200 as rn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "capi_from_c.c")
CUDA_LIB = "/usr/local/cuda/lib64"


def _build(tmp_path):
    lib_dir = os.path.dirname(rn.LIB_PATH)
    oracle_lib = oracle.build()
    exe = str(tmp_path / "capi_from_c")
    cmd = ["gcc", "-O1", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           SRC, "-o", exe, rn.LIB_PATH, oracle_lib, "-L", CUDA_LIB, "-lcudart", "-lm",
           f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{os.path.dirname(oracle_lib)}",
           f"-Wl,-rpath,{CUDA_LIB}"]
    subprocess.check_call(cmd)
    return exe


def test_c_program_host_logic(tmp_path):
    exe = _build(tmp_path)
    res = subprocess.run([exe, "host"], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr + res.stdout
    assert "ok (host)" in res.stdout


@pytest.mark.gpu
def test_c_program_on_the_gpu(tmp_path):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    exe = _build(tmp_path)
    res = subprocess.run([exe, "gpu"], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr + res.stdout
    assert "ok (gpu)" in res.stdout
