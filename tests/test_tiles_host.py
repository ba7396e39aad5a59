"""The tile enumeration shared by the tensor-core / SIMT product kernels and
the host planner (dm_tiles.cuh), compiled for the host with g++ and checked
exhaustively over many shapes: symmetric products must visit exactly the
tiles meeting the upper triangle, once each; the others every tile once, in
their documented order."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.isdir(CUDA_INC),
                    reason="needs g++ and the CUDA headers")
def test_tile_enumeration(tmp_path):
    exe = tmp_path / "tiles_check"
    cmd = ["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "dimuon_optimizer_b200", "csrc"), "-I", CUDA_INC,
           os.path.join(ROOT, "tests", "tiles_check.cpp"), "-o", str(exe)]
    build = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert build.returncode == 0, build.stderr[-3000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stdout[-3000:]
    assert "0 failures" in run.stdout
