"""Gradients on the GPU (la_noncausal_backward, la_causal_backward) against
the fp64 gradient oracle, which differentiates the forward definition
(oracle/backward.py, pinned by finite differences and autograd)."""

import numpy as np
import pytest
import torch

import oracle
from kernelized_linear_attention_phi_b200 import binding as la

from gpu_util import DT, TOL, f64, qkv

pytestmark = pytest.mark.gpu

MODES = [("relu1", True), ("relu1", False), ("identity", False), ("elu1", True)]
FN = {"noncausal": la.la_noncausal_backward, "causal": la.la_causal_backward}


def plain_err_where_not_cancelling(got, ref, scale):
    """The plain relative row error, over the rows whose exact value is not
    small against their rounding scale (norm at least a tenth of it): the
    scale floor of max_row_grad_err relaxes only rows that really cancel."""
    r = ref.reshape(-1, ref.shape[-1])
    keep = np.linalg.norm(r, axis=1) >= 0.1 * np.asarray(scale).reshape(-1)
    if not keep.any():
        return 0.0
    return oracle.max_row_rel_err(got.reshape(-1, ref.shape[-1])[keep], r[keep])


def _case(form, dt, d, N, phi, normalize, B=1, H=2, seed=0):
    sigma = 1.0 if phi != "identity" else d ** -0.5
    q, k, v = qkv(B, H, N, d, dt, seed=seed, sigma=sigma)
    g = torch.Generator(device="cpu").manual_seed(seed + 1000)
    dout = torch.randn(B, H, N, d, generator=g).to(device="cuda", dtype=q.dtype)
    dq, dk, dv = FN[form](q, k, v, dout, phi=phi, normalize=normalize)
    ref = oracle.backward_batched(f64(q), f64(k), f64(v), f64(dout), form, phi_kind=phi, normalize=normalize,
                                  scales=True)
    return (dq, dk, dv), ref


@pytest.mark.parametrize("form", ["noncausal", "causal"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("N", [2, 100, 700])
@pytest.mark.parametrize("phi,normalize", MODES)
def test_gradients_match_oracle(form, dt, d, N, phi, normalize):
    got, ref = _case(form, dt, d, N, phi, normalize, seed=N + d)
    for name, gt, rf, sc in zip(("dq", "dk", "dv"), got, ref[:3], ref[3:]):
        err = oracle.max_row_grad_err(f64(gt), rf, sc)
        assert err < TOL[DT[dt]], (name, err)
        err = plain_err_where_not_cancelling(f64(gt), rf, sc)
        assert err < TOL[DT[dt]], (name, "plain", err)


@pytest.mark.parametrize("form", ["noncausal", "causal"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("phi", ["relu1", "elu1"])
def test_single_token_normalized(form, dt, phi):
    """One key: the normalized output is v whatever q and k are, so dq and dk
    vanish (the kernels form them as differences of ordinary-size terms and
    return rounding noise: fp32 noise on the CUDA cores, bf16-operand noise,
    of order 2^-9 of the terms, on the tensor cores) and dv equals dout."""
    q, k, v = qkv(2, 3, 1, 64, dt, seed=3)
    g = torch.Generator(device="cpu").manual_seed(4)
    dout = torch.randn(q.shape, generator=g).to(device=q.device, dtype=q.dtype)
    dq, dk, dv = FN[form](q, k, v, dout, phi=phi)
    if dt == "f32":
        assert float(dq.abs().max()) < 1e-5 and float(dk.abs().max()) < 1e-5
    # both terms of each row are proportional to g . v, which a draw can make
    # arbitrarily small; the oracle's rounding scale (the product with the
    # state in absolute values, here |b| (|gn| . |v| + |gden|)) is not
    ref = oracle.backward_batched(f64(q), f64(k), f64(v), f64(dout), form, phi_kind=phi, scales=True)
    for gt, rf, sc in ((dq, ref[0], ref[3]), (dk, ref[1], ref[4])):
        assert float(abs(rf).max()) < 1e-12  # the definition: exactly zero
        assert oracle.max_row_grad_err(f64(gt), rf, sc) < TOL[DT[dt]]
    assert oracle.max_row_rel_err(f64(dv), f64(dout)) < TOL[DT[dt]]


def test_gradients_several_heads_and_sequences():
    got, ref = _case("causal", "bf16", 64, 1500, "relu1", True, B=2, H=3, seed=5)
    for gt, rf, sc in zip(got, ref[:3], ref[3:]):
        assert oracle.max_row_grad_err(f64(gt), rf, sc) < TOL[torch.bfloat16]
        assert plain_err_where_not_cancelling(f64(gt), rf, sc) < TOL[torch.bfloat16]


def test_gradients_are_deterministic():
    q, k, v = qkv(1, 2, 900, 64, "bf16", seed=8)
    dout = torch.randn_like(q)
    for fn in FN.values():
        a, b = fn(q, k, v, dout), fn(q, k, v, dout)
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_causal_gradient_of_last_row_touches_every_key():
    """A loss on the last output row only: every key and value of the head
    gets a gradient (the last query sees them all), and dq is zero except in
    that row."""
    B, H, N, d = 1, 1, 300, 32
    q, k, v = qkv(B, H, N, d, "f32", seed=9)
    dout = torch.zeros_like(q)
    dout[0, 0, -1] = 1.0
    dq, dk, dv = la.la_causal_backward(q, k, v, dout)
    assert torch.count_nonzero(dq[0, 0, :-1]) == 0
    assert bool((dv[0, 0].abs().sum(dim=1) > 0).all())
    ref = oracle.backward_batched(f64(q), f64(k), f64(v), f64(dout), "causal", scales=True)
    for gt, rf, sc in zip((dq, dk, dv), ref[:3], ref[3:]):
        assert oracle.max_row_grad_err(f64(gt), rf, sc) < TOL[torch.float32]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("phi,normalize", [("relu1", True), ("elu1", True), ("identity", False)])
def test_noncausal_gradients_split_across_heads(d, phi, normalize):
    """16 heads of 2500 tokens: the tensor-core gradient kernels split the
    (head, 128-token tile) pairs into contiguous ranges that cross heads, so
    a CTA sums G and h over several tiles of one head and then starts the
    next head's records and operands."""
    got, ref = _case("noncausal", "bf16", d, 2500, phi, normalize, B=2, H=8, seed=11)
    for name, gt, rf, sc in zip(("dq", "dk", "dv"), got, ref[:3], ref[3:]):
        err = oracle.max_row_grad_err(f64(gt), rf, sc)
        assert err < TOL[torch.bfloat16], (name, err)
        err = plain_err_where_not_cancelling(f64(gt), rf, sc)
        assert err < TOL[torch.bfloat16], (name, "plain", err)


def test_causal_gradients_with_two_blocks_per_cta():
    """15 heads of 2500 tokens (10 blocks each): 15 clusters of 10 CTAs would
    not all be resident, so the forward block states are formed and scanned
    with two blocks per CTA (clusters of 5)."""
    got, ref = _case("causal", "bf16", 64, 2500, "relu1", True, B=1, H=15, seed=12)
    for name, gt, rf, sc in zip(("dq", "dk", "dv"), got, ref[:3], ref[3:]):
        err = oracle.max_row_grad_err(f64(gt), rf, sc)
        assert err < TOL[torch.bfloat16], (name, err)
        err = plain_err_where_not_cancelling(f64(gt), rf, sc)
        assert err < TOL[torch.bfloat16], (name, "plain", err)

