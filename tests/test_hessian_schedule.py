"""Host logic of the persistent Hessian kernel's schedule (no GPU): the tile order and the
(tile, token segment) unit map, compiled from the same header the kernel includes."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "post_weight_quantization_layer_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs a host C++ compiler")
def test_schedule_covers_every_tile_and_segment_once(tmp_path):
    exe = tmp_path / "hessian_schedule_check"
    src = os.path.join(ROOT, "tests", "hessian_schedule_check.cpp")
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, src, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs a host C++ compiler")
def test_factor_plan_reserves_every_nodes_scratch(tmp_path):
    """Host logic of the factor's recursion plan (the header factor.cu includes): every node's
    products fit the per-depth scratch, int8 nodes stay within the int8 kernel's K range."""
    exe = tmp_path / "factor_plan_check"
    src = os.path.join(ROOT, "tests", "factor_plan_check.cpp")
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, src, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout
