"""The tile and mask logic the kernels share (csrc/tiles.cuh), compiled for the host and
checked against brute force: which tiles a mask leaves visible, the per-row column
ranges that replace the element-wise test inside a tile, and the coverage of the
persistent schedule (tests/tiles_check.cpp)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "exact_attention_126_b200", "csrc")


def test_tile_logic_matches_brute_force(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = tmp_path / "tiles_check"
    subprocess.run([cxx, "-O2", "-std=c++17", "-I", CSRC, os.path.join(HERE, "tiles_check.cpp"),
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "OK", out.stdout + out.stderr
