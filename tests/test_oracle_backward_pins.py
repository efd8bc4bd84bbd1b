"""Pins for the gradient oracle (oracle/backward.py): central finite
differences of the forward definition (itself pinned in test_oracle_pins.py)
and torch's automatic differentiation of the same definition in float64."""

import numpy as np
import pytest
import torch

import oracle as la
from oracle import backward as bw

MODES = [(la.PHI_RELU1, True), (la.PHI_RELU1, False), (la.PHI_IDENTITY, False), (la.PHI_ELU1, True)]


def _inputs(n, d, seed, phi_kind):
    rng = np.random.default_rng(seed)
    # keep relu+1 inputs away from its kink at 0 (finite differences straddle it)
    def draw(shape):
        x = rng.normal(size=shape)
        if phi_kind == la.PHI_RELU1:
            x = np.sign(x) * (np.abs(x) + 0.1)
        return x
    Q, K, V, G = draw((n, d)), draw((n, d)), rng.normal(size=(n, d)), rng.normal(size=(n, d))
    if phi_kind == la.PHI_IDENTITY:
        Q += 2.0  # keeps the unnormalized case far from cancellation; harmless
    m = rng.integers(0, n, size=n)
    return Q, K, V, G, m


def _fd_grads(Q, K, V, G, form, m, phi_kind, normalize, h=1e-6):
    def loss(Qx, Kx, Vx):
        return float((G * la.attention_dense(Qx, Kx, Vx, form, m, phi_kind, normalize)).sum())
    grads = []
    for which in range(3):
        X = [Q.copy(), K.copy(), V.copy()]
        g = np.zeros_like(X[which])
        for idx in np.ndindex(*g.shape):
            Xp = [x.copy() for x in X]
            Xm = [x.copy() for x in X]
            Xp[which][idx] += h
            Xm[which][idx] -= h
            g[idx] = (loss(*Xp) - loss(*Xm)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("form", la.FORMS)
@pytest.mark.parametrize("phi_kind,normalize", MODES)
@pytest.mark.parametrize("n,d", [(1, 2), (5, 3), (8, 4)])
def test_backward_matches_finite_differences(form, phi_kind, normalize, n, d):
    Q, K, V, G, m = _inputs(n, d, 7 * n + d, phi_kind)
    mm = m if form == la.FORM_PREFIX else None
    got = bw.backward_dense(Q, K, V, G, form, mm, phi_kind, normalize)
    want = _fd_grads(Q, K, V, G, form, mm, phi_kind, normalize)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=1e-6, atol=1e-7)


def _torch_forward(Q, K, V, form, m, phi_kind, normalize):
    if phi_kind == la.PHI_RELU1:
        A, B = torch.relu(Q) + 1, torch.relu(K) + 1
    elif phi_kind == la.PHI_ELU1:
        A, B = torch.nn.functional.elu(Q) + 1, torch.nn.functional.elu(K) + 1
    else:
        A, B = Q, K
    n = Q.shape[0]
    vis = torch.from_numpy(la.visible(n, form, m))
    W = torch.where(vis, A @ B.T, torch.zeros((), dtype=Q.dtype))
    num = W @ V
    return num / W.sum(dim=1, keepdim=True) if normalize else num


@pytest.mark.parametrize("form", la.FORMS)
@pytest.mark.parametrize("phi_kind,normalize", MODES)
def test_backward_matches_autograd(form, phi_kind, normalize):
    n, d = 23, 6
    Q, K, V, G, m = _inputs(n, d, 99, phi_kind)
    mm = m if form == la.FORM_PREFIX else None
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V)]
    out = _torch_forward(*ts, form, mm, phi_kind, normalize)
    out.backward(torch.tensor(G))
    got = bw.backward_dense(Q, K, V, G, form, mm, phi_kind, normalize)
    for g, t in zip(got, ts):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_phi_grad_values():
    x = np.array([-2.0, -0.0, 0.0, 0.5])
    np.testing.assert_array_equal(bw.phi_grad(x, la.PHI_RELU1), [0, 0, 0, 1])
    np.testing.assert_array_equal(bw.phi_grad(x, la.PHI_IDENTITY), [1, 1, 1, 1])
    np.testing.assert_allclose(bw.phi_grad(x, la.PHI_ELU1), [np.exp(-2.0), 1, 1, 1], rtol=1e-15)


def test_finite_difference_pin_catches_a_dropped_denominator_term():
    """A planted mistake: the gradient through the denominator left out. The
    finite-difference pin must reject it."""
    Q, K, V, G, _ = _inputs(6, 3, 5, la.PHI_RELU1)
    # gradient of the normalized output computed as if unnormalized: the
    # 1/den scaling and the dden term are both missing
    got = bw.backward_dense(Q, K, V, G, la.FORM_CAUSAL, None, la.PHI_RELU1, normalize=False)
    want = _fd_grads(Q, K, V, G, la.FORM_CAUSAL, None, la.PHI_RELU1, True)
    assert any(not np.allclose(g, w, rtol=1e-6, atol=1e-7) for g, w in zip(got, want))


def test_gradient_metric_and_scales():
    """max_row_grad_err judges a row against the larger of its own norm and
    its term scale; the oracle's scale of a structurally zero row (one visible
    key, normalized) is the size of its two cancelling terms, which are
    equal."""
    from oracle.metrics import max_row_grad_err
    ref = np.array([[3.0, 4.0], [0.0, 0.0]])
    got = ref + np.array([[0.05, 0.0], [0.0, 0.01]])
    assert abs(max_row_grad_err(got, ref, [5.0, 0.02]) - 0.5) < 1e-12  # row 1: 0.01 / 0.02
    assert abs(max_row_grad_err(got, ref, [5.0, 2.0]) - 0.01) < 1e-12  # row 0: 0.05 / 5
    Q, K, V, G, _ = _inputs(4, 3, 11, la.PHI_RELU1)
    dq, dk, dv, tq, tk, tv = bw.backward_dense(Q, K, V, G, la.FORM_CAUSAL, scales=True)
    assert np.linalg.norm(dq[0]) < 1e-12 < tq[0]        # row 0 sees one key
    assert np.all(tq >= np.linalg.norm(dq, axis=1) - 1e-12)
    assert np.all(tk >= np.linalg.norm(dk, axis=1) - 1e-12)
    assert np.all(tv >= np.linalg.norm(dv, axis=1) - 1e-12)


@pytest.mark.parametrize("form", [la.FORM_NONCAUSAL, la.FORM_CAUSAL])
def test_gradient_scale_bounds_terms_and_keeps_power(form):
    """The rounding scale of a gradient row (its product with the states it
    sees, in absolute values) dominates the norm of each exact term of the
    row, and a row with a term dropped (planted here, in the oracle's own
    arithmetic) still fails the metric by far more than the bf16 tolerance."""
    from oracle.metrics import max_row_grad_err
    rng = np.random.default_rng(21)
    n, d = 300, 16
    Q, K, V, G = (rng.standard_normal((n, d)) for _ in range(4))
    dq, dk, dv, tq, tk, tv = bw.backward_dense(Q, K, V, G, form, scales=True)
    A, B = la.phi(Q), la.phi(K)
    vis = la.visible(n, form, None)
    W = np.where(vis, A @ B.T, 0.0)
    den = W.sum(axis=1)
    out = (W @ V) / den[:, None]
    gn, gden = G / den[:, None], -(G * out).sum(axis=1) / den
    pq = bw.phi_grad(Q)
    t1 = pq * (np.where(vis, gn @ V.T, 0.0) @ B)          # the gn . v term of dq
    t2 = pq * (np.where(vis, gden[:, None], 0.0) @ B)     # the gden term of dq
    assert np.allclose(t1 + t2, dq, atol=1e-10)
    assert np.all(tq >= np.linalg.norm(t1, axis=1) - 1e-12)
    assert np.all(tq >= np.linalg.norm(t2, axis=1) - 1e-12)
    assert max_row_grad_err(t1, dq, tq) > 0.2             # gden term dropped
    assert max_row_grad_err(t2, dq, tq) > 0.2             # gn . v term dropped
