"""The small-M kernel's shared-memory addressing, checked on the host: the
kernel's own functions (csrc/small_m_layout.cuh, compiled for the host by
nvcc) against the packed layout's and the TMA box swizzle's definitions, for
every format, rows-per-CTA choice, piece size, step, quad thread and row.
And its launch planner (csrc/small_m_plan.h, compiled by g++) against the
ordering it states, with the launch shapes of the FLUX linears pinned."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "weight_quantised_gemm_b200", "csrc")
HARNESS = os.path.join(ROOT, "tests", "native", "small_m_addressing.cu")
PLAN_HARNESS = os.path.join(ROOT, "tests", "native", "small_m_plan.cpp")


def _nvcc():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    p = os.path.join(cuda, "bin", "nvcc")
    return p if os.path.exists(p) else shutil.which("nvcc")


def test_small_m_addressing_matches_the_layout(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc is not installed")
    exe = str(tmp_path / "small_m_addressing")
    build = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1", "-I", CSRC,
                            HARNESS, "-o", exe],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout
    last = run.stdout.strip().splitlines()[-1].split()
    assert last[0] == "checked" and int(last[1]) > 100000 and last[2:] == ["mismatches", "0"], run.stdout


def test_small_m_planner_matches_its_definition(tmp_path):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ is not installed")
    exe = str(tmp_path / "small_m_plan")
    build = subprocess.run([gxx, "-std=c++17", "-O1", "-Wall", "-Wextra", "-I", CSRC, PLAN_HARNESS, "-o", exe],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout
    last = run.stdout.strip().splitlines()[-1].split()
    assert last[0] == "checked" and int(last[1]) > 50000 and last[2:] == ["mismatches", "0"], run.stdout
