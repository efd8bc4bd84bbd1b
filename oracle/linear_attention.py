"""Plain fp64 CPU oracle for kernelized linear attention.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import this module. The product
path (the CUDA library and its Python binding) never calls it and shares no
code with it.

Everything is numpy float64. Callers pass arrays that already hold the exact
input values (bf16 and fp32 tensors upcast losslessly). One head is a matrix
``[n_tokens, head_dim]``; the batched helpers at the bottom loop over the
leading ``[B, H]`` axes.

What is computed, and where it is stated:

* feature map ``phi``: relu(x)+1 -- "nx_f32_linear_attention.nx source",
  function ``la_phi`` (a value whose sign bit is set becomes 0, then 1 is
  added); identity -- "trim-transformer 0.1.0", introduction
  (Attn(Q,K,V) = Q K^T V); elu(x)+1 -- "lineartile 1.0.1", "How It Works"
  (the page names ELU without its parameter; read as the usual alpha = 1:
  x + 1 for x > 0, exp(x) otherwise).
* KV summary ``S = sum_j phi(K_j) (x) V_j`` (d_k x d_v, row-major ``S[a, b]``)
  and ``z = sum_j phi(K_j)`` -- nx source, header comment and the
  "accumulate KV-summary" loop.
* readout ``out_i = (phi(Q_i) S) / (phi(Q_i) . z)`` with no epsilon and no
  1/sqrt(d) scale -- nx source, header comment and the "per-query" loop (the
  denominator is formed first, then each output column is its numerator
  divided by it).
* unnormalized form ``out_i = phi(Q_i) S`` -- trim-transformer 0.1.0,
  introduction.
* key sets: non-causal (every key), causal (keys 0..i, inclusive) and prefix
  mask (keys 0..m_i, inclusive) -- trim-transformer 0.1.0, "Masking"
  (torch.arange(n) is the causal mask; [2, 0, 1] is the 2-D mask
  [[F,F,F],[F,T,T],[F,F,T]] with True meaning "set to 0").
* decode step: the stored state is updated with the new token, then the new
  token reads out from it -- trim-transformer 0.1.0, "Key-value caching"
  (``use_kv_cache`` reads the stored state, ``update_kv_cache`` adds the new
  token's key and value, and the call runs with ``is_causal=True``, whose key
  set includes the token itself).

Two forms are given for each attention variant:

* the *definition* (``attention_dense`` / ``attention_rows``): weights
  ``w_ij = phi(q_i) . phi(k_j)`` over the key set, then ``sum_j w_ij v_j``,
  divided by ``sum_j w_ij`` when normalized. O(N^2 d) for all rows, O(i d)
  for one row.
* the *recurrence* the nx source describes (``noncausal``, ``causal``,
  ``prefix_mask``, ``decode_step``): build (S, z) as running sums over keys in
  order, then read out. O(N d^2).

Each is pinned by tests against values the pages print, closed forms and each
other; see tests/test_oracle_pins.py.
"""

from __future__ import annotations

import numpy as np

PHI_RELU1 = "relu1"
PHI_IDENTITY = "identity"
PHI_ELU1 = "elu1"
PHI_KINDS = (PHI_RELU1, PHI_IDENTITY, PHI_ELU1)

FORM_NONCAUSAL = "noncausal"
FORM_CAUSAL = "causal"
FORM_PREFIX = "prefix"
FORMS = (FORM_NONCAUSAL, FORM_CAUSAL, FORM_PREFIX)


def _f64(x):
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Feature map
# ---------------------------------------------------------------------------

def phi(x, kind=PHI_RELU1):
    """Elementwise feature map.

    relu1: nx source, ``la_phi``. The relu is decided by the sign bit, so
    -0.0 maps to 0 + 1 = 1, like +0.0.
    identity: trim-transformer 0.1.0 introduction, where the attention kernel
    is Q K^T V with no feature map.
    elu1: lineartile 1.0.1, "How It Works": elu(x) + 1 with alpha = 1, that
    is x + 1 where x > 0 and exp(x) - 1 + 1 = exp(x) elsewhere.
    """
    x = _f64(x)
    if kind == PHI_RELU1:
        return np.where(np.signbit(x), 0.0, x) + 1.0
    if kind == PHI_IDENTITY:
        return x.copy()
    if kind == PHI_ELU1:
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    raise ValueError(f"unknown feature map {kind!r}")


# ---------------------------------------------------------------------------
# Key sets
# ---------------------------------------------------------------------------

def key_limits(n, form, m=None):
    """Index of the last key each query sees (inclusive), shape [n].

    noncausal: n-1 for every query. causal: i (trim-transformer 0.1.0,
    "Masking": the causal mask is torch.arange(n)). prefix: m_i, an integer
    in [0, n-1] (same section).
    """
    if form == FORM_NONCAUSAL:
        return np.full(n, n - 1, dtype=np.int64)
    if form == FORM_CAUSAL:
        return np.arange(n, dtype=np.int64)
    if form == FORM_PREFIX:
        m = np.asarray(m, dtype=np.int64)
        if m.shape != (n,):
            raise ValueError(f"mask must have shape ({n},), got {m.shape}")
        if n and (m.min() < 0 or m.max() > n - 1):
            raise ValueError("mask values must lie in [0, n-1]")
        return m.copy()
    raise ValueError(f"unknown form {form!r}")


def visible(n, form, m=None):
    """Dense boolean matrix: visible[i, j] is True when query i sees key j."""
    lim = key_limits(n, form, m)
    return np.arange(n)[None, :] <= lim[:, None]


def torch_convention_mask(m):
    """The 2-D mask trim-transformer 0.1.0 ("Masking") pairs with an integer
    prefix mask m: entry [i, j] is True when it is set to 0, i.e. j > m_i."""
    m = np.asarray(m, dtype=np.int64)
    return ~visible(m.shape[0], FORM_PREFIX, m)


# ---------------------------------------------------------------------------
# The definition: weights times values
# ---------------------------------------------------------------------------

def attention_dense(Q, K, V, form=FORM_NONCAUSAL, m=None, phi_kind=PHI_RELU1,
                    normalize=True):
    """All rows by the definition. w_ij = phi(q_i).phi(k_j) for visible j;
    out_i = sum_j w_ij v_j, divided by sum_j w_ij when normalized."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    n = Q.shape[0]
    W = phi(Q, phi_kind) @ phi(K, phi_kind).T
    W = np.where(visible(n, form, m), W, 0.0)
    num = W @ V
    if not normalize:
        return num
    return num / W.sum(axis=1)[:, None]


def attention_rows(Q, K, V, rows, form=FORM_NONCAUSAL, m=None,
                   phi_kind=PHI_RELU1, normalize=True):
    """Selected rows by the definition, one row at a time (O(i d) per row).

    Used for large inputs, where the full O(N^2) matrix is out of reach."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    n = Q.shape[0]
    lim = key_limits(n, form, m)
    pk = phi(K, phi_kind)
    out = np.empty((len(rows), V.shape[1]))
    for r, i in enumerate(rows):
        last = int(lim[i])
        w = pk[: last + 1] @ phi(Q[i], phi_kind)
        num = w @ V[: last + 1]
        out[r] = num / w.sum() if normalize else num
    return out


# ---------------------------------------------------------------------------
# The recurrence (nx source): KV summary, then readout
# ---------------------------------------------------------------------------

def kv_summary(K, V, phi_kind=PHI_RELU1):
    """S[a, b] = sum_j phi(K_j)[a] V_j[b] and z[a] = sum_j phi(K_j)[a].

    nx source, "accumulate KV-summary": the sum over tokens j of the outer
    product phi(K_j) (x) V_j, and of phi(K_j). phi(K)^T V is that same sum."""
    pk = phi(K, phi_kind)
    return pk.T @ _f64(V), pk.sum(axis=0)


def readout(Q, S, z, phi_kind=PHI_RELU1, normalize=True):
    """out_i[b] = (sum_a phi(Q_i)[a] S[a, b]) / (sum_a phi(Q_i)[a] z[a]).

    nx source, "per-query": the denominator phi(Q_i).z, then each column's
    numerator divided by it. Unnormalized: the numerator alone."""
    pq = phi(Q, phi_kind)
    num = pq @ _f64(S)
    if not normalize:
        return num
    return num / (pq @ _f64(z))[..., None]


def noncausal(Q, K, V, phi_kind=PHI_RELU1, normalize=True):
    """Non-causal attention as the nx source computes it. Returns (out, S, z)."""
    S, z = kv_summary(K, V, phi_kind)
    return readout(Q, S, z, phi_kind, normalize), S, z


def decode_step(S, z, q, k, v, phi_kind=PHI_RELU1, normalize=True):
    """One recurrent step on a cached state, for one head.

    S += phi(k) (x) v; z += phi(k); out = phi(q) S / (phi(q) . z).
    The update comes first, so the token sees itself (trim-transformer 0.1.0,
    "Key-value caching", with the inclusive causal mask of "Masking").
    Returns (out, S_new, z_new); the inputs are not modified."""
    pk = phi(k, phi_kind)
    S_new = _f64(S) + np.outer(pk, _f64(v))
    z_new = _f64(z) + pk
    return readout(q, S_new, z_new, phi_kind, normalize), S_new, z_new


def causal(Q, K, V, phi_kind=PHI_RELU1, normalize=True, S0=None, z0=None):
    """Causal attention as the running recurrence: for i = 0..n-1, add key i
    to (S, z), then read out query i. Optionally starts from a cached state.
    Returns (out, S_final, z_final)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    dk, dv = K.shape[1], V.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else _f64(S0)
    z = np.zeros(dk) if z0 is None else _f64(z0)
    out = np.empty((Q.shape[0], dv))
    for i in range(Q.shape[0]):
        out[i], S, z = decode_step(S, z, Q[i], K[i], V[i], phi_kind, normalize)
    return out, S, z


def prefix_mask(Q, K, V, m, phi_kind=PHI_RELU1, normalize=True):
    """Prefix-mask attention (query i sees keys 0..m_i) as a recurrence: keys
    are added to (S, z) in order, and each query reads out once the running
    sum holds exactly keys 0..m_i."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    n = Q.shape[0]
    lim = key_limits(n, FORM_PREFIX, m)
    pk = phi(K, phi_kind)
    S = np.zeros((K.shape[1], V.shape[1]))
    z = np.zeros(K.shape[1])
    out = np.empty((n, V.shape[1]))
    added = 0  # keys 0..added-1 are in (S, z)
    for i in np.argsort(lim, kind="stable"):
        while added <= lim[i]:
            S += np.outer(pk[added], V[added])
            z += pk[added]
            added += 1
        out[i] = readout(Q[i], S, z, phi_kind, normalize)
    return out


def causal_rows(Q, K, V, rows, phi_kind=PHI_RELU1, normalize=True):
    """Selected rows of causal attention by the nx recurrence, for long
    sequences: keys are added to (S, z) in order, the keys between two
    requested rows as one KV summary of that stretch (the same sum over j,
    grouped), and each requested row i reads out once (S, z) holds keys
    0..i. O(N d^2) for any number of rows, against O(i d) per row for
    ``attention_rows``."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    rows = np.asarray(rows, dtype=np.int64)
    S = np.zeros((K.shape[1], V.shape[1]))
    z = np.zeros(K.shape[1])
    out = np.empty((len(rows), V.shape[1]))
    added = 0  # keys 0..added-1 are in (S, z)
    for r in np.argsort(rows, kind="stable"):
        i = int(rows[r])
        if i + 1 > added:
            dS, dz = kv_summary(K[added:i + 1], V[added:i + 1], phi_kind)
            S, z = S + dS, z + dz
            added = i + 1
        out[r] = readout(Q[i], S, z, phi_kind, normalize)
    return out


# ---------------------------------------------------------------------------
# Batched helpers over [B, H, N, d]
# ---------------------------------------------------------------------------

def batched(fn, Q, K, V, *args, m=None, **kw):
    """Apply a one-head function to every (b, h) of [B, H, N, d] arrays.

    ``m`` is [B, N] (one mask per sequence, shared by its heads) or None.
    ``fn`` returns either the output or a tuple whose first item is it."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H = Q.shape[:2]
    out = np.empty(Q.shape[:3] + (V.shape[3],))
    for b in range(B):
        for h in range(H):
            extra = () if m is None else (np.asarray(m)[b],)
            r = fn(Q[b, h], K[b, h], V[b, h], *extra, *args, **kw)
            out[b, h] = r[0] if isinstance(r, tuple) else r
    return out


def kv_summary_batched(K, V, phi_kind=PHI_RELU1):
    """(S, z) for every head: S [B, H, d_k, d_v], z [B, H, d_k]."""
    K, V = _f64(K), _f64(V)
    B, H = K.shape[:2]
    S = np.empty((B, H, K.shape[3], V.shape[3]))
    z = np.empty((B, H, K.shape[3]))
    for b in range(B):
        for h in range(H):
            S[b, h], z[b, h] = kv_summary(K[b, h], V[b, h], phi_kind)
    return S, z
