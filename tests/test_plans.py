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


def test_bench_mirror_of_the_block_plan(plan_check):
    """bench.py counts the bytes of a KV pass that skips the last block from
    its own copy of the block plan: it must agree with the library's."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for B, H, N, d, dt in [(1, 16, 131072, 128, 1), (2, 8, 4096, 64, 1), (8, 8, 2048, 64, 1), (1, 3, 1000, 128, 1),
                           (64, 32, 2048, 128, 1), (1, 1, 300, 64, 0), (4, 16, 16384, 64, 1)]:
        for sms in (148, 132, 100, 16, 1):
            out = subprocess.run([plan_check, "plan", str(B), str(H), str(N), str(d), str(dt), str(sms)],
                                 capture_output=True, text=True, check=True).stdout.split()
            want = (int(out[0]), int(out[1]))
            assert bench.block_plan(B, H, N, d, "bf16" if dt == 1 else "f32", sms) == want, (B, H, N, d, dt, sms)
