"""The library's work plans (csrc/plan.h) under SM counts other than a full
B200's: the device's SM count is queried at run time, so a partial GPU (fewer
SMs) must still get splits that cover every token, with no empty piece and no
more record slots than the workspace was sized for. Checked on the CPU by a
host program built from the plan header alone."""

import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kernelized_linear_attention_phi_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "cuda", "plan_check.cpp")
BUILD = os.path.join(ROOT, "tests", "_build")


@pytest.fixture(scope="module")
def plan_check():
    os.makedirs(BUILD, exist_ok=True)
    exe = os.path.join(BUILD, "plan_check")
    cmd = ["g++", "-std=c++17", "-O1", "-Wall", f"-I{CSRC}", f"-I{os.path.join(ROOT, 'include')}",
           "-I/usr/local/cuda/include", SRC, "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_plans_cover_every_token_for_any_sm_count(plan_check):
    r = subprocess.run([plan_check], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-4000:]
    assert r.stdout.strip().splitlines()[-1].startswith("checked ")
