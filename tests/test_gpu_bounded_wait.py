"""Failure detection without a GPU fault: a wait that nothing satisfies must
run out within its limit, report through the error word and leave the CUDA
context usable. The probe kernel (tests/cuda/wait_timeout.cu) uses the
library's own wait primitive and abort flag."""

import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def probe():
    from kernelized_linear_attention_phi_b200 import build
    out_dir = os.path.join(HERE, "_build")
    os.makedirs(out_dir, exist_ok=True)
    so = os.path.join(out_dir, "libwait_timeout_probe.so")
    src = os.path.join(HERE, "cuda", "wait_timeout.cu")
    cmd = [build.nvcc(), *build.ARCH, "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           f"-I{build.CSRC}", f"-I{build.INCLUDE}", src, "-o", so]
    subprocess.run(cmd, check=True, capture_output=True)
    lib = ctypes.CDLL(so)
    lib.wait_timeout_probe.restype = ctypes.c_int
    lib.wait_timeout_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    return lib


def test_unsatisfied_wait_times_out_and_releases_the_cta(probe):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = torch.zeros(4, dtype=torch.int64, device="cuda")
    assert probe.wait_timeout_probe(ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(res.data_ptr())) == 0
    torch.cuda.synchronize()
    ok0, ns0, ok1, ns1 = (int(x) for x in res.cpu())
    assert int(err.item()) == 2          # the timeout bit (FLAG_TIMEOUT), nothing else
    assert ok0 == 0 and ok1 == 0          # both waits reported failure
    assert 1.9e9 <= ns0 <= 4e9            # warp 0 waited its full limit (2 s), not forever
    assert ns1 < 1.8e9                    # warp 1 left early through the abort flag
    # the context is still usable
    x = torch.arange(1000, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 499500.0
