"""la_kv_summary_static, the KV summary for callers that cannot allocate
device memory (its scratch is a fixed device array inside the library), must
give what la_kv_summary gives. Collected last, so that a run that stops at the
first failure has run every other test; it must also pass on its own in a
fresh process (the first call sets up the array's device address)."""

import ctypes

import pytest
import torch

import oracle
from kernelized_linear_attention_phi_b200 import binding as la
from kernelized_linear_attention_phi_b200 import workloads as W

from gpu_util import f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kernelized_linear_attention_phi_b200 import build
    build.build()
    la.lib()


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("bf16", 128), ("f32", 64)])
def test_static_scratch_matches_workspace_entry_point(dtype, d):
    """Two calls in a row on different inputs, each against la_kv_summary."""
    B, H, N = 2, 4, 3000
    for seed in (1, 2):
        _, k, v = W.qkv(B, H, N, d, 1.0, seed, dtype, "cuda")
        S_ref, z_ref = la.la_kv_summary(k, v)
        S = torch.full((B, H, d, d), float("nan"), device="cuda")
        z = torch.full((B, H, d), float("nan"), device="cuda")
        la.la_kv_summary_static(k, v, S, z)
        torch.cuda.synchronize()
        assert oracle.max_row_rel_err(f64(S), f64(S_ref)) < 1e-5
        assert oracle.max_row_rel_err(f64(z)[..., None, :], f64(z_ref)[..., None, :]) < 1e-5


def test_static_scratch_rejects_problems_beyond_its_size():
    """A problem whose scratch would exceed the fixed array is refused
    before anything is launched."""
    desc = la.make_desc(64, 32, 128, 128, torch.bfloat16)  # 2048 heads: many partial records
    assert la.la_workspace_size(desc, "kv_summary") > (32 << 20)
    P = ctypes.c_void_p(1 << 20)
    st = la.lib().la_kv_summary_static(ctypes.byref(desc), P, P, P, P, None)
    assert la.STATUS_NAMES[st] == "LA_ERR_WORKSPACE"
