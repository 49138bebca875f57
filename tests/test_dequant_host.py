"""The tensor-core kernel's dequantisation routines (csrc/dequant.cuh),
compiled for the CPU and checked against a plain unpack for every bitwidth."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_dequant_routines_on_cpu(tmp_path):
    exe = str(tmp_path / "dequant_selftest")
    subprocess.check_call(["g++", "-std=c++17", "-O1", os.path.join(HERE, "dequant_selftest.cpp"),
                           "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
