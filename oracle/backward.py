"""Plain fp64 CPU oracle for the gradients of kernelized linear attention.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only the tests,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may use it.

The pages list a backward pass ("lineartile 1.0.1", "Project Structure":
``core/kernels/backward.py`` and the ``test_backward`` suite) without giving
its formulas. It is the derivative of the forward definition, written out
here from that definition and nothing else:

    a_i = phi(q_i), b_j = phi(k_j), w_ij = a_i . b_j for visible j (else 0),
    num_i = sum_j w_ij v_j, den_i = sum_j w_ij, out_i = num_i / den_i
    (out_i = num_i when unnormalized).

With g_i = dL/dout_i:

    dnum_i = g_i / den_i,   dden_i = -(g_i . out_i) / den_i     (normalized)
    dnum_i = g_i,           dden_i = 0                          (unnormalized)
    dw_ij  = dnum_i . v_j + dden_i          for visible j, else 0
    dV     = W^T dnum
    da_i   = sum_j dw_ij b_j,   db_j = sum_i dw_ij a_i
    dQ = phi'(Q) * dA,  dK = phi'(K) * dB   (elementwise)

phi' is 1 where x > 0 and 0 elsewhere for relu+1 (the derivative of relu is
taken as 0 at 0, the usual convention), 1 for the identity, and 1 where
x > 0, exp(x) elsewhere for elu+1. Everything is O(N^2 d) and float64; it is
pinned by tests against finite differences of the forward definition and
against torch's automatic differentiation of the same definition.
"""

from __future__ import annotations

import numpy as np

from .linear_attention import (FORM_CAUSAL, FORM_NONCAUSAL, PHI_ELU1, PHI_IDENTITY, PHI_RELU1, phi,
                               visible)


def phi_grad(x, kind=PHI_RELU1):
    """d phi / dx, elementwise (see the module docstring for the value at 0)."""
    x = np.asarray(x, dtype=np.float64)
    if kind == PHI_RELU1:
        return np.where(x > 0, 1.0, 0.0)
    if kind == PHI_IDENTITY:
        return np.ones_like(x)
    if kind == PHI_ELU1:
        return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))
    raise ValueError(f"unknown feature map {kind!r}")


def backward_dense(Q, K, V, dO, form=FORM_NONCAUSAL, m=None, phi_kind=PHI_RELU1,
                   normalize=True, scales=False):
    """(dQ, dK, dV) of one head by the definition above. With scales=True
    also (tq, tk, tv), per row the size of what rounding acts on. The rows
    are products with the states a query or key sees,
        dq_i = phi'(q_i) (S_i dnum_i + dden_i z_i),   S_i = sum_{j vis i} b_j v_j^T,
        dk_j = phi'(k_j) (G_j v_j + h_j),   dv_j = G_j^T b_j,
                                   G_j = sum_{i sees j} a_i dnum_i^T,
    and the scale of each is the same product with every factor replaced by
    its absolute value, the states summed exactly first (|S_i| |dnum_i| +
    |dden_i| z_i, and so on): a product of rounded operands errs by at most
    the unit roundoff times the product of the absolute values, and the
    states are what a chunked computation rounds, not their single terms.
    The norms of the exact terms are not such a scale (an inner product of
    them can cancel while their rounding does not); a sum of absolute values
    over keys would be one, but loose by a factor that grows with N."""
    Q, K, V, dO = (np.asarray(t, dtype=np.float64) for t in (Q, K, V, dO))
    n = Q.shape[0]
    A, Bk = phi(Q, phi_kind), phi(K, phi_kind)
    W = np.where(visible(n, form, m), A @ Bk.T, 0.0)
    num = W @ V
    if normalize:
        den = W.sum(axis=1)
        out = num / den[:, None]
        dnum = dO / den[:, None]
        dden = -(dO * out).sum(axis=1) / den
    else:
        dnum = dO
        dden = np.zeros(n)
    dW = np.where(visible(n, form, m), dnum @ V.T + dden[:, None], 0.0)
    dV = W.T @ dnum
    dA = dW @ Bk
    dB = dW.T @ A
    grads = (phi_grad(Q, phi_kind) * dA, phi_grad(K, phi_kind) * dB, dV)
    if not scales:
        return grads
    vis = visible(n, form, m).astype(np.float64)
    # per-row states: S_i, z_i over the keys query i sees; G_j, h_j over the
    # queries that see key j
    Sx = Bk[:, :, None] * V[:, None, :]      # b_j v_j^T
    Gx = A[:, :, None] * dnum[:, None, :]    # a_i dnum_i^T
    if form == FORM_NONCAUSAL:
        S = np.broadcast_to(Sx.sum(0), Sx.shape)
        z = np.broadcast_to(Bk.sum(0), Bk.shape)
        G = np.broadcast_to(Gx.sum(0), Gx.shape)
        h = np.broadcast_to((A * dden[:, None]).sum(0), A.shape)
    elif form == FORM_CAUSAL:
        S, z = np.cumsum(Sx, 0), np.cumsum(Bk, 0)
        G = np.cumsum(Gx[::-1], 0)[::-1]
        h = np.cumsum((A * dden[:, None])[::-1], 0)[::-1]
    else:
        S, z = np.einsum("ij,jkv->ikv", vis, Sx), vis @ Bk
        G, h = np.einsum("ij,ikv->jkv", vis, Gx), vis.T @ (A * dden[:, None])
    pq, pk = np.abs(phi_grad(Q, phi_kind)), np.abs(phi_grad(K, phi_kind))
    tq = np.linalg.norm(pq * (np.einsum("ikv,iv->ik", np.abs(S), np.abs(dnum)) + np.abs(dden)[:, None] * np.abs(z)),
                        axis=1)
    tk = np.linalg.norm(pk * (np.einsum("jkv,jv->jk", np.abs(G), np.abs(V)) + np.abs(h)), axis=1)
    tv = np.linalg.norm(np.einsum("jkv,jk->jv", np.abs(G), np.abs(Bk)), axis=1)
    return grads + (tq, tk, tv)


def backward_batched(Q, K, V, dO, form=FORM_NONCAUSAL, m=None, **kw):
    """backward_dense over every (b, h) of [B, H, N, d] arrays; m is [B, N]
    (one mask per sequence) or None. Returns (dQ, dK, dV) as [B, H, N, d]
    (and with scales=True the per-row scales as [B, H, N])."""
    Q, K, V, dO = (np.asarray(t, dtype=np.float64) for t in (Q, K, V, dO))
    out = [np.empty_like(Q), np.empty_like(K), np.empty_like(V)]
    if kw.get("scales"):
        out += [np.empty(Q.shape[:3]) for _ in range(3)]
    for b in range(Q.shape[0]):
        for h in range(Q.shape[1]):
            res = backward_dense(Q[b, h], K[b, h], V[b, h], dO[b, h], form,
                                 None if m is None else m[b], **kw)
            for o, r in zip(out, res):
                o[b, h] = r
    return tuple(out)
