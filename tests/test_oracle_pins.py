"""Pins for the fp64 oracle: values the pages print, closed forms, invariants
and brute force. None of these tests needs a GPU, and none compares the oracle
with itself by retyping its formula: each one checks it against something the
pages or the mathematics fix independently."""

import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import linear_attention as la


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# Feature map (nx source, la_phi)
# ---------------------------------------------------------------------------

def test_phi_relu1_sign_bit():
    x = np.array([-0.0, 0.0, -1.5, 2.5, -1e-30, 1e-30])
    got = la.phi(x, la.PHI_RELU1)
    np.testing.assert_array_equal(got, [1.0, 1.0, 1.0, 3.5, 1.0, 1.0 + 1e-30])


def test_phi_elu1_matches_torch_elu():
    """lineartile's map elu(x) + 1 (alpha = 1), against torch's own elu in
    float64: x + 1 above zero, exp(x) at and below zero (so -0.0 and +0.0 map
    to 1), strictly positive everywhere."""
    import torch
    x = np.array([-30.0, -3.5, -1.0, -1e-3, -0.0, 0.0, 1e-3, 0.5, 1.0, 7.25])
    want = torch.nn.functional.elu(torch.tensor(x, dtype=torch.float64), alpha=1.0).numpy() + 1.0
    got = la.phi(x, la.PHI_ELU1)
    # torch forms expm1(x) + 1, which cancels far below zero: an absolute
    # tolerance there (a wrong map misses by orders of magnitude more)
    np.testing.assert_allclose(got, want, rtol=1e-15, atol=1e-16)
    assert got[4] == 1.0 and got[5] == 1.0 and np.all(got > 0)


def test_phi_identity_is_identity():
    x = np.array([-2.0, -0.0, 0.0, 3.25])
    np.testing.assert_array_equal(la.phi(x, la.PHI_IDENTITY), x)


# ---------------------------------------------------------------------------
# The pages' worked examples
# ---------------------------------------------------------------------------

def test_nx_gate1_uniform_gives_mean(golden_dir):
    g = _load(golden_dir, "nx_gate1.json")
    Q, K, V = (np.array(g[k], dtype=np.float64) for k in "QKV")
    want = np.array(g["out"], dtype=np.float64)
    out, _, _ = la.noncausal(Q, K, V)
    assert np.max(np.abs(out - want)) < g["abs_tol"]
    np.testing.assert_array_equal(out, want)  # exact in fp64
    np.testing.assert_array_equal(la.attention_dense(Q, K, V), want)


def test_nx_gate2_worked_example(golden_dir):
    g = _load(golden_dir, "nx_gate2.json")
    Q, K, V = (np.array(g[k], dtype=np.float64) for k in "QKV")
    np.testing.assert_array_equal(la.phi(K), np.array(g["phi_K"], float))
    S, z = la.kv_summary(K, V)
    np.testing.assert_array_equal(S, np.array(g["S"], float))
    np.testing.assert_array_equal(z, np.array(g["z"], float))
    num = np.array(g["out_numerator"], float)
    den = np.array(g["out_denominator"], float)[:, None]
    want = num / den
    for out in (la.noncausal(Q, K, V)[0], la.attention_dense(Q, K, V),
                la.attention_rows(Q, K, V, [0, 1])):
        assert np.max(np.abs(out - want)) < g["abs_tol"]
        np.testing.assert_array_equal(out, want)


def test_nx_gate2_causal_and_prefix_derived(golden_dir):
    """Derived from the worked example: causally, row 0 sees only key 0, so
    its output is v_0 exactly; row 1 sees both keys, so it equals the
    non-causal row 1, [38, 56]/9. The prefix mask m = [0, 1] is the same."""
    g = _load(golden_dir, "nx_gate2.json")
    Q, K, V = (np.array(g[k], dtype=np.float64) for k in "QKV")
    want = np.array([[2.0, 4.0], [38.0 / 9.0, 56.0 / 9.0]])
    for out in (la.causal(Q, K, V)[0],
                la.attention_dense(Q, K, V, la.FORM_CAUSAL),
                la.prefix_mask(Q, K, V, [0, 1]),
                la.attention_dense(Q, K, V, la.FORM_PREFIX, m=[0, 1])):
        np.testing.assert_array_equal(out, want)
    # m = [1, 0]: row 0 sees both keys (non-causal row 0), row 1 sees key 0.
    want2 = np.array([[34.0 / 9.0, 52.0 / 9.0], [2.0, 4.0]])
    np.testing.assert_array_equal(la.prefix_mask(Q, K, V, [1, 0]), want2)
    np.testing.assert_array_equal(
        la.attention_dense(Q, K, V, la.FORM_PREFIX, m=[1, 0]), want2)


def test_nx_gate2_exact_rational_brute_force(golden_dir):
    """The worked example recomputed in exact rationals with Python loops, for
    every key set on two tokens: an independent check of the weighting."""
    g = _load(golden_dir, "nx_gate2.json")
    Q, K, V = (np.array(g[k], dtype=np.float64) for k in "QKV")

    def frac_phi(x):
        return Fraction(0) if x <= 0 else Fraction(x)

    for m in itertools.product(range(2), repeat=2):
        for i in range(2):
            w = [sum((frac_phi(Q[i, a]) + 1) * (frac_phi(K[j, a]) + 1)
                     for a in range(2)) for j in range(m[i] + 1)]
            num = [sum(w[j] * Fraction(V[j, b]) for j in range(m[i] + 1))
                   for b in range(2)]
            exact = [float(x / sum(w)) for x in num]
            got = la.prefix_mask(Q, K, V, list(m))[i]
            np.testing.assert_array_equal(got, exact)


def test_trim_mask_example(golden_dir):
    g = _load(golden_dir, "trim_mask_example.json")
    want = np.array(g["mask_true_means_zeroed"], dtype=bool)
    np.testing.assert_array_equal(la.torch_convention_mask(g["m"]), want)
    # causal is arange(n): lower triangle with diagonal visible.
    for n in (1, 3, 8):
        np.testing.assert_array_equal(
            la.visible(n, la.FORM_PREFIX, np.arange(n)),
            np.tril(np.ones((n, n), dtype=bool)))
        np.testing.assert_array_equal(la.visible(n, la.FORM_CAUSAL),
                                      np.tril(np.ones((n, n), dtype=bool)))
        assert la.visible(n, la.FORM_NONCAUSAL).all()


def test_mask_range_is_checked():
    with pytest.raises(ValueError):
        la.key_limits(3, la.FORM_PREFIX, [0, 3, 1])
    with pytest.raises(ValueError):
        la.key_limits(3, la.FORM_PREFIX, [0, -1, 1])


# ---------------------------------------------------------------------------
# Closed forms
# ---------------------------------------------------------------------------

def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("phi_kind", la.PHI_KINDS)
def test_uniform_keys_give_mean_of_visible_values(phi_kind):
    """If every key row is the same vector k, every weight of query i is the
    same number phi(q_i).phi(k), so a normalized output is the plain mean of
    the visible values, whatever Q is (nx source, gate 1's principle)."""
    rng = _rng(1)
    n, d = 13, 5
    Q = rng.normal(size=(n, d)) + (2.0 if phi_kind == la.PHI_IDENTITY else 0)
    k = np.abs(rng.normal(size=d)) + 0.5
    K = np.tile(k, (n, 1))
    V = rng.normal(size=(n, d))
    m = rng.integers(0, n, size=n)
    csum = np.cumsum(V, axis=0)
    mean_nc = np.tile(V.mean(axis=0), (n, 1))
    mean_c = csum / np.arange(1, n + 1)[:, None]
    mean_m = csum[m] / (m + 1)[:, None]
    for form, want, mm in ((la.FORM_NONCAUSAL, mean_nc, None),
                           (la.FORM_CAUSAL, mean_c, None),
                           (la.FORM_PREFIX, mean_m, m)):
        got = la.attention_dense(Q, K, V, form, mm, phi_kind)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(la.noncausal(Q, K, V, phi_kind)[0], mean_nc,
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(la.causal(Q, K, V, phi_kind)[0], mean_c,
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(la.prefix_mask(Q, K, V, m, phi_kind), mean_m,
                               rtol=1e-12, atol=1e-12)


def test_identity_unnormalized_associativity():
    """Unnormalized identity-map attention is Q (K^T V) = (Q K^T) V
    (trim-transformer 0.1.0 introduction). The recurrence takes the first
    order, the definition the second; a transposed operand breaks one."""
    rng = _rng(2)
    n, dk, dv = 11, 4, 3
    Q, K, V = rng.normal(size=(n, dk)), rng.normal(size=(n, dk)), rng.normal(size=(n, dv))
    ref = np.empty((n, dv))
    for i in range(n):              # textbook loops, no matrix routines
        for b in range(dv):
            ref[i, b] = sum(sum(Q[i, a] * K[j, a] for a in range(dk)) * V[j, b]
                            for j in range(n))
    np.testing.assert_allclose(la.noncausal(Q, K, V, la.PHI_IDENTITY, False)[0],
                               ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(
        la.attention_dense(Q, K, V, phi_kind=la.PHI_IDENTITY, normalize=False),
        ref, rtol=1e-12, atol=1e-12)


def test_masked_identity_matches_triple_loop():
    """Masked unnormalized identity attention against plain Python loops over
    the 2-D mask of trim-transformer's convention (True = set to 0)."""
    rng = _rng(3)
    n, d = 9, 3
    Q, K, V = (rng.normal(size=(n, d)) for _ in range(3))
    m = rng.integers(0, n, size=n)
    zeroed = la.torch_convention_mask(m)
    ref = np.zeros((n, d))
    for i in range(n):
        for j in range(n):
            if zeroed[i, j]:
                continue
            w = sum(Q[i, a] * K[j, a] for a in range(d))
            for b in range(d):
                ref[i, b] += w * V[j, b]
    for got in (la.prefix_mask(Q, K, V, m, la.PHI_IDENTITY, False),
                la.attention_dense(Q, K, V, la.FORM_PREFIX, m, la.PHI_IDENTITY, False),
                la.attention_rows(Q, K, V, range(n), la.FORM_PREFIX, m,
                                  la.PHI_IDENTITY, False)):
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_kv_summary_against_token_loop():
    """S and z against the nx source's loop order written out element by
    element (token j, then row a, then column b)."""
    rng = _rng(4)
    n, dk, dv = 7, 3, 4
    K, V = rng.normal(size=(n, dk)), rng.normal(size=(n, dv))
    S = [[0.0] * dv for _ in range(dk)]
    z = [0.0] * dk
    for j in range(n):
        for a in range(dk):
            pk = (K[j, a] if K[j, a] > 0 else 0.0) + 1.0
            z[a] += pk
            for b in range(dv):
                S[a][b] += pk * V[j, b]
    S2, z2 = la.kv_summary(K, V)
    np.testing.assert_allclose(S2, S, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(z2, z, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------
# Brute force: recurrence vs definition on random tiny inputs
# ---------------------------------------------------------------------------

CASES = [(n, d) for n in (1, 2, 5, 17, 64) for d in (2, 4, 16)]


@pytest.mark.parametrize("n,d", CASES)
@pytest.mark.parametrize("phi_kind,normalize",
                         [(la.PHI_RELU1, True), (la.PHI_RELU1, False),
                          (la.PHI_IDENTITY, False)])
def test_recurrence_matches_definition(n, d, phi_kind, normalize):
    rng = _rng(100 * n + d)
    Q, K, V = (rng.normal(size=(n, d)) for _ in range(3))
    m = rng.integers(0, n, size=n)
    kw = dict(phi_kind=phi_kind, normalize=normalize)
    pairs = [
        (la.noncausal(Q, K, V, **kw)[0], la.attention_dense(Q, K, V, la.FORM_NONCAUSAL, **kw)),
        (la.causal(Q, K, V, **kw)[0], la.attention_dense(Q, K, V, la.FORM_CAUSAL, **kw)),
        (la.prefix_mask(Q, K, V, m, **kw), la.attention_dense(Q, K, V, la.FORM_PREFIX, m, **kw)),
    ]
    for fast, dense in pairs:
        np.testing.assert_allclose(fast, dense, rtol=1e-10, atol=1e-10)
    rows = sorted(set([0, n - 1, n // 2]))
    np.testing.assert_allclose(
        la.attention_rows(Q, K, V, rows, la.FORM_PREFIX, m, **kw),
        la.attention_dense(Q, K, V, la.FORM_PREFIX, m, **kw)[rows],
        rtol=1e-10, atol=1e-10)


def test_prefix_mask_extremes():
    """m = n-1 everywhere is non-causal; m = arange(n) is causal
    (trim-transformer 0.1.0, "Masking")."""
    rng = _rng(5)
    n, d = 33, 8
    Q, K, V = (rng.normal(size=(n, d)) for _ in range(3))
    np.testing.assert_allclose(la.prefix_mask(Q, K, V, np.full(n, n - 1)),
                               la.noncausal(Q, K, V)[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(la.prefix_mask(Q, K, V, np.arange(n)),
                               la.causal(Q, K, V)[0], rtol=1e-12, atol=1e-12)
    # m = 0 everywhere: every query sees key 0 only, so a normalized output is v_0.
    np.testing.assert_allclose(la.prefix_mask(Q, K, V, np.zeros(n, int)),
                               np.tile(V[0], (n, 1)), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Decode (KV cache)
# ---------------------------------------------------------------------------

def test_decode_steps_reproduce_causal_rows():
    rng = _rng(6)
    n, d = 20, 6
    Q, K, V = (rng.normal(size=(n, d)) for _ in range(3))
    ref = la.attention_dense(Q, K, V, la.FORM_CAUSAL)
    S, z = np.zeros((d, d)), np.zeros(d)
    for t in range(n):
        out, S, z = la.decode_step(S, z, Q[t], K[t], V[t])
        np.testing.assert_allclose(out, ref[t], rtol=1e-12, atol=1e-12)


def test_decode_from_prefill_state():
    """A prefill's (S, z) is phi(K)^T V and sum phi(K); decoding on from it
    equals causal attention over the whole sequence for the new tokens."""
    rng = _rng(7)
    n0, n1, d = 25, 6, 4
    Q, K, V = (rng.normal(size=(n0 + n1, d)) for _ in range(3))
    _, S, z = la.noncausal(Q[:n0], K[:n0], V[:n0])
    pk = np.where(K[:n0] > 0, K[:n0], 0) + 1
    np.testing.assert_allclose(S, sum(np.outer(pk[j], V[j]) for j in range(n0)),
                               rtol=1e-12)
    np.testing.assert_allclose(z, pk.sum(axis=0), rtol=1e-12)
    ref = la.attention_dense(Q, K, V, la.FORM_CAUSAL)
    for t in range(n0, n0 + n1):
        out, S, z = la.decode_step(S, z, Q[t], K[t], V[t])
        np.testing.assert_allclose(out, ref[t], rtol=1e-12, atol=1e-12)
    out_c, S_c, z_c = la.causal(Q[n0:], K[n0:], V[n0:],
                                S0=la.noncausal(Q[:n0], K[:n0], V[:n0])[1],
                                z0=pk.sum(axis=0))
    np.testing.assert_allclose(out_c, ref[n0:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S_c, S, rtol=1e-12)


def test_decode_does_not_modify_inputs():
    S, z = np.ones((2, 2)), np.ones(2)
    la.decode_step(S, z, [1.0, 2.0], [3.0, -1.0], [0.5, 0.5])
    np.testing.assert_array_equal(S, np.ones((2, 2)))
    np.testing.assert_array_equal(z, np.ones(2))


# ---------------------------------------------------------------------------
# Invariants
# ---------------------------------------------------------------------------

def test_linear_in_values():
    rng = _rng(8)
    n, d = 15, 4
    Q, K, V1, V2 = (rng.normal(size=(n, d)) for _ in range(4))
    m = rng.integers(0, n, size=n)
    for form, mm in ((la.FORM_NONCAUSAL, None), (la.FORM_CAUSAL, None),
                     (la.FORM_PREFIX, m)):
        f = lambda V: la.attention_dense(Q, K, V, form, mm)
        np.testing.assert_allclose(f(2.0 * V1 - 3.0 * V2), 2.0 * f(V1) - 3.0 * f(V2),
                                   rtol=1e-11, atol=1e-11)


def test_normalized_output_is_convex_combination():
    """With phi = relu+1 every weight is positive, so each normalized output
    column lies between the smallest and largest visible value."""
    rng = _rng(9)
    n, d = 30, 5
    Q, K, V = (rng.normal(size=(n, d)) for _ in range(3))
    out = la.causal(Q, K, V)[0]
    for i in range(n):
        lo, hi = V[: i + 1].min(axis=0), V[: i + 1].max(axis=0)
        assert np.all(out[i] >= lo - 1e-12) and np.all(out[i] <= hi + 1e-12)


def test_noncausal_key_permutation_invariance():
    rng = _rng(10)
    n, d = 21, 6
    Q, K, V = (rng.normal(size=(n, d)) for _ in range(3))
    p = rng.permutation(n)
    np.testing.assert_allclose(la.noncausal(Q, K[p], V[p])[0], la.noncausal(Q, K, V)[0],
                               rtol=1e-12, atol=1e-12)


def test_batched_helpers_match_per_head():
    rng = _rng(11)
    B, H, n, d = 2, 3, 10, 4
    Q, K, V = (rng.normal(size=(B, H, n, d)) for _ in range(3))
    m = rng.integers(0, n, size=(B, n))
    got = la.batched(la.prefix_mask, Q, K, V, m=m)
    for b in range(B):
        for h in range(H):
            np.testing.assert_array_equal(got[b, h], la.prefix_mask(Q[b, h], K[b, h], V[b, h], m[b]))
    S, z = la.kv_summary_batched(K, V)
    np.testing.assert_array_equal(S[1, 2], la.kv_summary(K[1, 2], V[1, 2])[0])
    np.testing.assert_array_equal(z[0, 1], la.kv_summary(K[0, 1], V[0, 1])[1])


def test_metric():
    r = np.array([[3.0, 4.0], [1.0, 0.0]])
    assert oracle.max_row_rel_err(r, r) == 0.0
    g = r + np.array([[0.0, 0.5], [0.0, 0.0]])
    assert oracle.max_row_rel_err(g, r) == pytest.approx(0.1)
    g2 = r.copy()
    g2[1, 0] = np.nan
    assert oracle.max_row_rel_err(g2, r) == float("inf")


# ---------------------------------------------------------------------------
# The pins catch planted mistakes (planted in a copy of the oracle, on the CPU)
# ---------------------------------------------------------------------------

def _gate2_ok(golden_dir, fn):
    g = _load(golden_dir, "nx_gate2.json")
    Q, K, V = (np.array(g[k], dtype=np.float64) for k in "QKV")
    want = np.array(g["out_numerator"], float) / 9.0
    return np.allclose(fn(Q, K, V), want, rtol=0, atol=g["abs_tol"])


def test_planted_mistakes_fail_the_worked_example(golden_dir, monkeypatch):
    assert _gate2_ok(golden_dir, lambda Q, K, V: la.noncausal(Q, K, V)[0])
    # dropped +1 in phi
    no_plus_one = lambda x, kind=la.PHI_RELU1: np.maximum(np.asarray(x, float), 0.0)
    monkeypatch.setattr(la, "phi", no_plus_one)
    with np.errstate(divide="ignore", invalid="ignore"):
        assert not _gate2_ok(golden_dir, lambda Q, K, V: la.noncausal(Q, K, V)[0])
    monkeypatch.undo()
    # transposed S in the readout
    def transposed(Q, K, V):
        S, z = la.kv_summary(K, V)
        return la.readout(Q, S.T, z)
    assert not _gate2_ok(golden_dir, transposed)
    # denominator taken over S's row sums instead of z
    def wrong_den(Q, K, V):
        S, z = la.kv_summary(K, V)
        return la.readout(Q, S, S.sum(axis=1))
    assert not _gate2_ok(golden_dir, wrong_den)


@pytest.mark.parametrize("phi_kind,normalize", [("relu1", True), ("identity", False), ("elu1", True)])
def test_causal_rows_match_definition(phi_kind, normalize):
    """causal_rows (segment sums of the KV summary between requested rows)
    gives the definition's rows, in any order and with repeats."""
    rng = np.random.default_rng(21)
    n, d = 300, 8
    Q, K, V = (rng.standard_normal((n, d)) for _ in range(3))
    rows = [299, 0, 5, 5, 64, 63, 127, 128, 1, 250]
    got = la.causal_rows(Q, K, V, rows, phi_kind, normalize)
    ref = la.attention_rows(Q, K, V, rows, la.FORM_CAUSAL, phi_kind=phi_kind, normalize=normalize)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    dense = la.attention_dense(Q, K, V, la.FORM_CAUSAL, phi_kind=phi_kind, normalize=normalize)
    np.testing.assert_allclose(got, dense[rows], rtol=1e-12, atol=1e-12)
