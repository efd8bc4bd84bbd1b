"""la_kv_summary_static, the KV summary for callers that cannot allocate
device memory (its scratch is a fixed device array inside the library), must
give what la_kv_summary gives, and what the oracle gives. Collected last, so
that a run that stops at the first failure has run every other test; it must
also pass on its own in a fresh process (the first call in a context looks up
the array's device address)."""

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


# S and z are fp32 sums. bf16 inputs with relu+1: exact features, so only
# fp32 accumulation error. fp32 inputs: S is formed on the tensor cores from
# two-part bf16 splits of the fp32 operands (about 1e-5) and is held to the
# fp32 bar of 1e-4; z is summed in fp32 on the CUDA cores.
TOL = 1e-5
TOL_S = {"bf16": 1e-5, "f32": 1e-4}


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("bf16", 128), ("f32", 64)])
def test_static_scratch_matches_workspace_entry_point_and_oracle(dtype, d):
    """Two calls in a row on different inputs, each against la_kv_summary
    and against the oracle's KV summary; the calls allocate nothing through
    torch's allocator."""
    B, H, N = 2, 4, 3000
    for seed in (1, 2):
        _, k, v = W.qkv(B, H, N, d, 1.0, seed, dtype, "cuda")
        S_ref, z_ref = la.la_kv_summary(k, v)
        S = torch.full((B, H, d, d), float("nan"), device="cuda")
        z = torch.full((B, H, d), float("nan"), device="cuda")
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated()
        la.la_kv_summary_static(k, v, S, z)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        assert oracle.max_row_rel_err(f64(S), f64(S_ref)) < TOL
        assert oracle.max_row_rel_err(f64(z)[..., None, :], f64(z_ref)[..., None, :]) < TOL
        S_o, z_o = oracle.kv_summary_batched(f64(k), f64(v))
        assert oracle.max_row_rel_err(f64(S), S_o) < TOL_S[dtype]
        assert oracle.max_row_rel_err(f64(z)[..., None, :], z_o[..., None, :]) < TOL


def test_static_scratch_rejects_problems_beyond_its_size():
    """A problem whose scratch would exceed the fixed array is refused
    before anything is launched."""
    desc = la.make_desc(64, 32, 128, 128, torch.bfloat16)  # 2048 heads: many partial records
    assert la.la_workspace_size(desc, "kv_summary") > (32 << 20)
    P = ctypes.c_void_p(1 << 20)
    st = la.lib().la_kv_summary_static(ctypes.byref(desc), P, P, P, P, None)
    assert la.STATUS_NAMES[st] == "LA_ERR_WORKSPACE"
