"""The per-kernel timing hook (la_timing_enable / la_timing_read): one
duration per kernel the call launches, for direct calls and for replays of a
captured CUDA graph."""

import pytest
import torch

from kernelized_linear_attention_phi_b200 import binding as la
from tests.gpu_util import qkv

pytestmark = pytest.mark.gpu

# kernels per call on the bf16 tensor-core path at this size (8 heads of
# 1024 tokens, d = 64): KV summary and non-causal: one thread-block-cluster
# kernel (a cluster per head reduces the summary); causal: block states
# scanned inside a cluster per head, sweep; prefix mask: the same plus the
# binning; decode: one; gradients: forward states (non-causal: the cluster
# kernel without its readout; causal: scanned in-cluster), dq sweep, (G, h)
# reduction or reverse scan, dk/dv sweep
TC_LAUNCHES = {"kv_summary": 1, "noncausal": 1, "causal": 2, "prefix": 3, "decode": 1, "noncausal_bwd": 4,
               "causal_bwd": 4}


@pytest.fixture
def timing():
    la.la_timing_enable(True)
    yield
    la.la_timing_enable(False)


def _calls(dev):
    B, H, N, d = 2, 4, 1024, 64
    q, k, v = qkv(B, H, N, d, "bf16", seed=41)
    m = torch.randint(0, N, (B, N), dtype=torch.int32, device=dev)
    S = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    z = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    q1, k1, v1 = (t[:, :, :1].contiguous() for t in (q, k, v))
    out1 = torch.empty_like(q1)
    desc = la._desc_of(q, "relu1", True)
    ws = {op: la.workspace(desc, op, 64, dev)
          for op in ("kv_summary", "noncausal", "causal", "prefix", "noncausal_bwd", "causal_bwd")}
    dout = torch.randn_like(q)
    return {
        "kv_summary": lambda: la.la_kv_summary(k, v, S, z, ws=ws["kv_summary"]),
        "noncausal": lambda: la.la_noncausal(q, k, v, out, ws=ws["noncausal"]),
        "causal": lambda: la.la_causal_chunked(q, k, v, out, 64, ws=ws["causal"]),
        "prefix": lambda: la.la_prefix_mask(q, k, v, m, out, 64, ws=ws["prefix"]),
        "decode": lambda: la.la_decode_step(q1, k1, v1, S, z, out1),
        "noncausal_bwd": lambda: la.la_noncausal_backward(q, k, v, dout, ws=ws["noncausal_bwd"]),
        "causal_bwd": lambda: la.la_causal_backward(q, k, v, dout, ws=ws["causal_bwd"]),
    }


@pytest.mark.parametrize("op", list(TC_LAUNCHES))
def test_direct_call_times_each_kernel(timing, op):
    fn = _calls(torch.device("cuda", 0))[op]
    fn()
    ms = la.la_timing_read()
    assert len(ms) == TC_LAUNCHES[op]
    assert all(0.0 < t < 100.0 for t in ms)


def test_graph_replay_times_each_kernel(timing):
    fn = _calls(torch.device("cuda", 0))["causal"]
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(3):
        g.replay()
        ms = la.la_timing_read()
        assert len(ms) == TC_LAUNCHES["causal"]
        assert all(0.0 < t < 100.0 for t in ms)


def test_disabled_records_nothing_new():
    la.la_timing_enable(True)
    calls = _calls(torch.device("cuda", 0))
    calls["causal"]()
    assert len(la.la_timing_read()) == TC_LAUNCHES["causal"]
    la.la_timing_enable(False)
    calls["decode"]()
    # the last timed call is still the causal one
    assert len(la.la_timing_read()) == TC_LAUNCHES["causal"]
