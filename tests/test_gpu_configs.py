"""The five workloads at full size, in the launch configuration bench.py uses
(the library's work plans depend only on the problem shape), against the
fp64 oracle: every row where the oracle's O(N d^2) form is quick, sampled rows
(block edges, whole chunks, random rows; by the recurrence) for the long
causal sequence, 64 heads over all 1024 steps for the decode workload."""

import numpy as np
import pytest
import torch

import oracle
from kernelized_linear_attention_phi_b200 import binding as la
from kernelized_linear_attention_phi_b200 import workloads as W

from gpu_util import DT, TOL, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kernelized_linear_attention_phi_b200 import build
    build.build()
    la.lib()


def _inputs(wl, dtype):
    return W.qkv(wl.B, wl.H, wl.N, wl.d, wl.sigma, wl.seed, dtype, "cuda")


def test_single_head_fp32():
    wl = W.WORKLOADS["single_head"]
    q, k, v = _inputs(wl, "f32")
    out = la.la_noncausal(q, k, v)
    ref = oracle.batched(oracle.noncausal, f64(q), f64(k), f64(v))
    assert oracle.max_row_rel_err(f64(out), ref) < 1e-4


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_multi_head(dt):
    wl = W.WORKLOADS["multi_head"]
    q, k, v = _inputs(wl, dt)
    Q, K, V = f64(q), f64(k), f64(v)
    out = la.la_noncausal(q, k, v)
    ref = oracle.batched(oracle.noncausal, Q, K, V)
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[DT[dt]]
    out = la.la_causal_chunked(q, k, v, chunk=wl.chunk)
    ref = oracle.batched(oracle.causal, Q, K, V)
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[DT[dt]]


@pytest.mark.parametrize("mask", ["uniform", "arange"])
def test_prefix_mask_workload(mask):
    wl = W.WORKLOADS["prefix_mask"]
    q, k, v = _inputs(wl, "bf16")
    m = (W.prefix_mask_uniform(wl.B, wl.N, wl.seed, "cuda") if mask == "uniform"
         else W.prefix_mask_arange(wl.B, wl.N, "cuda"))
    out = la.la_prefix_mask(q, k, v, m, chunk=wl.chunk, phi=wl.phi, normalize=wl.normalize)
    ref = oracle.batched(oracle.prefix_mask, f64(q), f64(k), f64(v), m=m.cpu().numpy(),
                         phi_kind=wl.phi, normalize=wl.normalize)
    assert oracle.max_row_rel_err(f64(out), ref) < 2e-2


def test_long_noncausal():
    wl = W.WORKLOADS["long_noncausal"]
    q, k, v = _inputs(wl, "bf16")
    out = la.la_noncausal(q, k, v)
    got = f64(out)
    errs = []
    for b in range(wl.B):
        for h in range(wl.H):
            ref = oracle.noncausal(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]))[0]
            errs.append(oracle.max_row_rel_err(got[b, h], ref))
    assert max(errs) < 2e-2


def _block_starts(wl, sms):
    """Token starts of the blocks the library's block plan cuts a head into
    on a device with `sms` SMs (one wave of CTAs; d = 128 bf16 sweeps one
    CTA per SM; blocks of at least 256 tokens in multiples of 128)."""
    per_sm = 1 if wl.d == 128 else 2
    target = max(1, per_sm * sms // (wl.B * wl.H))
    bt = max(256, -(-(-(-wl.N // target)) // 128) * 128)
    return list(range(0, wl.N, bt))


def test_long_causal_sampled_rows():
    """Every head: the first and last token of every block and every token
    of one 64-token chunk per block (with the tokens on either side of it),
    the first 130 and last 2 tokens of the head, and random rows, against the
    oracle's recurrence."""
    wl = W.WORKLOADS["long_causal"]
    q, k, v = _inputs(wl, "bf16")
    out = la.la_causal_chunked(q, k, v, chunk=wl.chunk)
    starts = _block_starts(wl, torch.cuda.get_device_properties(0).multi_processor_count)
    ends = starts[1:] + [wl.N]
    rng = np.random.default_rng(0)
    errs = []
    for h in range(wl.H):
        rows = set(range(130)) | {wl.N - 2, wl.N - 1}
        for s0, s1 in zip(starts, ends):
            rows |= {s0, s1 - 1}
            c0 = s0 + 64 * int(rng.integers(0, (s1 - s0) // 64))  # one chunk of the block
            rows |= set(range(max(0, c0 - 1), min(wl.N, c0 + 65)))
        rows |= set(rng.integers(0, wl.N, size=16).tolist())
        rows = sorted(rows)
        ref = oracle.causal_rows(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), rows)
        errs.append(oracle.max_row_rel_err(f64(out[0, h, rows]), ref))
    assert max(errs) < 2e-2


def test_decode_workload():
    wl = W.WORKLOADS["decode"]
    B, H, d, N0, T = wl.B, wl.H, wl.d, wl.N, wl.decode_steps
    _, k0, v0 = W.qkv(B, H, N0, d, wl.sigma, wl.seed, "bf16", "cuda")
    S, z = la.la_kv_summary(k0, v0)
    S0_sample = {}
    # 64 heads: every sequence, its head spread over H
    heads = [(b, (7 * b + 3) % H) for b in range(B)]
    for b, h in heads:
        S0_sample[(b, h)] = (f64(S[b, h]), f64(z[b, h]))
    qs, ks, vs = W.decode_tokens(T, B, H, d, wl.sigma, wl.seed + 1, "bf16", "cuda")
    outs = torch.empty(T, B, H, 1, d, dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        la.la_decode_step(qs[t], ks[t], vs[t], S, z, out=outs[t])
    torch.cuda.synchronize()
    for b, h in heads:
        # the prefill itself against the oracle
        S_ref, z_ref = oracle.kv_summary(f64(k0[b, h]), f64(v0[b, h]))
        assert oracle.max_row_rel_err(S0_sample[(b, h)][0], S_ref) < 1e-5
        Sr, zr = S_ref, z_ref
        ref = np.empty((T, d))
        Qh, Kh, Vh = f64(qs[:, b, h, 0]), f64(ks[:, b, h, 0]), f64(vs[:, b, h, 0])
        for t in range(T):
            ref[t], Sr, zr = oracle.decode_step(Sr, zr, Qh[t], Kh[t], Vh[t])
        assert oracle.max_row_rel_err(f64(outs[:, b, h, 0]), ref) < 2e-2
        assert oracle.max_row_rel_err(f64(S[b, h]), Sr) < 1e-5
        np.testing.assert_allclose(f64(z[b, h]), zr, rtol=1e-5)
