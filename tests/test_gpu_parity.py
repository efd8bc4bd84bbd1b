"""GPU results against the fp64 oracle, element by element, at sizes the
oracle finishes in seconds: several tiles, ragged tails, every head size and
element type, and the edge cases (N = 1, degenerate masks, empty cache,
out-of-range mask values)."""

import numpy as np
import pytest
import torch

import oracle
from kernelized_linear_attention_phi_b200 import binding as la
from kernelized_linear_attention_phi_b200 import workloads

from gpu_util import DT, TOL, f64, qkv

pytestmark = pytest.mark.gpu

DS = (16, 32, 64, 128)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kernelized_linear_attention_phi_b200 import build
    build.build()
    la.lib()


def _modes():
    return [("relu1", True), ("relu1", False), ("identity", False), ("elu1", True)]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", DS)
@pytest.mark.parametrize("N", [1, 77, 1000])
@pytest.mark.parametrize("phi,normalize", _modes())
def test_noncausal(dt, d, N, phi, normalize):
    sigma = 1.0 if phi == "relu1" else d ** -0.5
    q, k, v = qkv(2, 3, N, d, dt, seed=N + d, sigma=sigma)
    S = torch.empty(2, 3, d, d, device="cuda")
    z = torch.empty(2, 3, d, device="cuda")
    out = la.la_noncausal(q, k, v, S_out=S, z_out=z, phi=phi, normalize=normalize)
    Q, K, V = f64(q), f64(k), f64(v)
    ref = oracle.batched(oracle.noncausal, Q, K, V, phi_kind=phi, normalize=normalize)
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[DT[dt]]
    S_ref, z_ref = oracle.kv_summary_batched(K, V, phi)
    assert oracle.max_row_rel_err(f64(S), S_ref) < _state_tol(dt, phi)
    assert oracle.max_row_rel_err(f64(z)[..., None, :], z_ref[..., None, :]) < _state_tol(dt, phi)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32])
@pytest.mark.parametrize("B,H,N", [(3, 5, 64), (3, 5, 256), (3, 5, 257), (3, 5, 2500), (4, 80, 200)])
def test_noncausal_short_heads_in_one_launch(dt, d, B, H, N):
    """d <= 32: heads of at most 256 tokens run in one launch (one CTA per head
    forms S and z, then reads out its queries); longer heads through the split
    partials, their reduction and the readout. The launch count says which
    path ran, and both match the oracle, S and z included."""
    q, k, v = qkv(B, H, N, d, dt, seed=7 * N + d)
    S = torch.empty(B, H, d, d, device="cuda")
    z = torch.empty(B, H, d, device="cuda")
    la.la_timing_enable(True)
    try:
        out = la.la_noncausal(q, k, v, S_out=S, z_out=z)
        launches = len(la.la_timing_read())
    finally:
        la.la_timing_enable(False)
    assert launches == (1 if N <= 256 else 3)
    Q, K, V = f64(q), f64(k), f64(v)
    ref = oracle.batched(oracle.noncausal, Q, K, V, phi_kind="relu1", normalize=True)
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[DT[dt]]
    S_ref, z_ref = oracle.kv_summary_batched(K, V, "relu1")
    assert oracle.max_row_rel_err(f64(S), S_ref) < _state_tol(dt, "relu1")
    assert oracle.max_row_rel_err(f64(z)[..., None, :], z_ref[..., None, :]) < _state_tol(dt, "relu1")
    # without S_out / z_out the outputs are the same, bit for bit
    assert torch.equal(la.la_noncausal(q, k, v), out)


def _state_tol(dt, phi):
    """Tolerance on a KV summary. bf16 inputs: relu+1 and the identity are
    exact in bf16 (relu(K) and K are bf16 values; the +1 is added exactly in
    fp32), so S and z carry only fp32 accumulation error; elu+1 has no such
    split (phi(K) is rounded to bf16) and is held to the bf16 output
    tolerance. fp32 inputs: the fp32 bar on every result, 1e-4 (the tensor-core
    path forms each product from two-part bf16 splits of its fp32 operands,
    within about 3 * 2^-16 of exact, so S carries about 1e-5)."""
    if dt == "f32":
        return TOL[DT[dt]]
    return TOL[DT[dt]] if phi == "elu1" else 1e-5


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", DS)
@pytest.mark.parametrize("N", [1, 300, 777])
def test_kv_summary(dt, d, N):
    _, k, v = qkv(1, 2, N, d, dt, seed=7 * N + d)
    S, z = la.la_kv_summary(k, v)
    S_ref, z_ref = oracle.kv_summary_batched(f64(k), f64(v))
    assert oracle.max_row_rel_err(f64(S), S_ref) < _state_tol(dt, "relu1")
    np.testing.assert_allclose(f64(z), z_ref, rtol=1e-5)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", DS)
@pytest.mark.parametrize("N", [1, 63, 130, 700])
@pytest.mark.parametrize("chunk", [64, 128])
@pytest.mark.parametrize("phi,normalize", [("relu1", True), ("identity", False)])
def test_causal(dt, d, N, chunk, phi, normalize):
    sigma = 1.0 if phi == "relu1" else d ** -0.5
    q, k, v = qkv(1, 3, N, d, dt, seed=3 * N + d, sigma=sigma)
    out = la.la_causal_chunked(q, k, v, chunk=chunk, phi=phi, normalize=normalize)
    ref = oracle.batched(oracle.causal, f64(q), f64(k), f64(v), phi_kind=phi, normalize=normalize)
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[DT[dt]]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", DS)
@pytest.mark.parametrize("N", [1, 129, 640])
@pytest.mark.parametrize("phi,normalize", [("relu1", True), ("identity", False)])
def test_prefix_mask_uniform(dt, d, N, phi, normalize):
    sigma = 1.0 if phi == "relu1" else d ** -0.5
    B = 2
    q, k, v = qkv(B, 2, N, d, dt, seed=5 * N + d, sigma=sigma)
    m = workloads.prefix_mask_uniform(B, N, seed=N, device="cuda")
    ws = la.workspace(la._desc_of(q, phi, normalize), "prefix", 64)
    out = la.la_prefix_mask(q, k, v, m, phi=phi, normalize=normalize, ws=ws)
    assert la.la_last_error(ws) == (0, 0)
    ref = oracle.batched(oracle.prefix_mask, f64(q), f64(k), f64(v), phi_kind=phi,
                         normalize=normalize, m=m.cpu().numpy())
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[DT[dt]]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("kind", ["zeros", "last", "arange", "blocks"])
def test_prefix_mask_degenerate(dt, kind):
    B, H, N, d = 2, 2, 300, 64
    q, k, v = qkv(B, H, N, d, dt, seed=11)
    if kind == "zeros":
        m = torch.zeros(B, N, dtype=torch.int32, device="cuda")
    elif kind == "last":
        m = torch.full((B, N), N - 1, dtype=torch.int32, device="cuda")
    elif kind == "arange":
        m = workloads.prefix_mask_arange(B, N, device="cuda")
    else:  # every query's limit at a chunk edge, including -1 partial chunks
        m = (torch.arange(N, device="cuda", dtype=torch.int32) // 64 * 64 + 63).clamp(max=N - 1)
        m = m.repeat(B, 1).contiguous()
    out = la.la_prefix_mask(q, k, v, m)
    ref = oracle.batched(oracle.prefix_mask, f64(q), f64(k), f64(v), m=m.cpu().numpy())
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[DT[dt]]
    if kind == "last":
        nc = la.la_noncausal(q, k, v)
        assert oracle.max_row_rel_err(f64(out), f64(nc)) < TOL[DT[dt]]
    if kind == "arange":
        c = la.la_causal_chunked(q, k, v)
        assert oracle.max_row_rel_err(f64(out), f64(c)) < TOL[DT[dt]]


def test_prefix_mask_out_of_range_is_clamped_and_flagged():
    B, H, N, d = 1, 2, 200, 32
    q, k, v = qkv(B, H, N, d, "f32", seed=12)
    m = workloads.prefix_mask_uniform(B, N, seed=3, device="cuda")
    m[0, 5] = -4
    m[0, 9] = N + 10
    ws = la.workspace(la._desc_of(q, "relu1", True), "prefix", 64)
    out = la.la_prefix_mask(q, k, v, m, ws=ws)
    status, flags = la.la_last_error(ws)
    assert status == 6 and flags == 1
    assert la.la_last_error(ws) == (0, 0)  # cleared by the read
    mc = m.clamp(0, N - 1).cpu().numpy()
    ref = oracle.batched(oracle.prefix_mask, f64(q), f64(k), f64(v), m=mc)
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[torch.float32]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", DS)
def test_decode_from_prefill(dt, d):
    B, H, N0, T = 2, 3, 150, 20
    q, k, v = qkv(B, H, N0 + T, d, dt, seed=d)
    S, z = la.la_kv_summary(k[:, :, :N0].contiguous(), v[:, :, :N0].contiguous())
    outs = []
    for t in range(N0, N0 + T):
        sl = lambda x: x[:, :, t:t + 1].contiguous()
        outs.append(la.la_decode_step(sl(q), sl(k), sl(v), S, z))
    got = torch.cat(outs, dim=2)
    Q, K, V = f64(q), f64(k), f64(v)
    ref = np.empty(got.shape)
    for b in range(B):
        for h in range(H):
            S0, z0 = oracle.kv_summary(K[b, h, :N0], V[b, h, :N0])
            ref[b, h] = oracle.causal(Q[b, h, N0:], K[b, h, N0:], V[b, h, N0:], S0=S0, z0=z0)[0]
    assert oracle.max_row_rel_err(f64(got), ref) < TOL[DT[dt]]
    S_ref, z_ref = oracle.kv_summary_batched(K, V)
    assert oracle.max_row_rel_err(f64(S), S_ref) < _state_tol(dt, "relu1")


def test_decode_from_empty_cache_equals_causal():
    B, H, N, d = 1, 2, 40, 64
    q, k, v = qkv(B, H, N, d, "f32", seed=13)
    S = torch.zeros(B, H, d, d, device="cuda")
    z = torch.zeros(B, H, d, device="cuda")
    got = torch.cat([la.la_decode_step(q[:, :, t:t + 1].contiguous(), k[:, :, t:t + 1].contiguous(),
                                       v[:, :, t:t + 1].contiguous(), S, z) for t in range(N)], dim=2)
    causal = la.la_causal_chunked(q, k, v)
    ref = oracle.batched(oracle.causal, f64(q), f64(k), f64(v))
    assert oracle.max_row_rel_err(f64(got), ref) < 1e-4
    assert oracle.max_row_rel_err(f64(causal), ref) < 1e-4


def test_results_are_deterministic():
    q, k, v = qkv(2, 4, 1500, 64, "bf16", seed=21)
    m = workloads.prefix_mask_uniform(2, 1500, seed=21, device="cuda")
    for fn in (lambda: la.la_noncausal(q, k, v), lambda: la.la_causal_chunked(q, k, v),
               lambda: la.la_prefix_mask(q, k, v, m)):
        a, b = fn(), fn()
        assert torch.equal(a, b)


def test_chunk_size_does_not_change_the_result():
    q, k, v = qkv(1, 2, 1000, 128, "bf16", seed=22)
    a = la.la_causal_chunked(q, k, v, chunk=64)
    b = la.la_causal_chunked(q, k, v, chunk=128)
    ref = oracle.batched(oracle.causal, f64(q), f64(k), f64(v))
    assert oracle.max_row_rel_err(f64(a), ref) < 2e-2
    assert oracle.max_row_rel_err(f64(b), ref) < 2e-2


def test_worked_example_on_gpu(golden_dir):
    """The nx source's gate 2 (Q = K = I2, V = [[2,4],[6,8]]) padded to the
    smallest supported head size: extra feature dimensions are 0 in Q and K
    and add phi = 1 to every weight, so the padded case is checked against
    the oracle rather than the printed numbers; the unpadded values are
    pinned in the oracle tests."""
    d = 16
    Q = torch.zeros(1, 1, 2, d)
    Q[0, 0, 0, 0] = 1
    Q[0, 0, 1, 1] = 1
    V = torch.zeros(1, 1, 2, d)
    V[0, 0, :, :2] = torch.tensor([[2.0, 4.0], [6.0, 8.0]])
    q, k, v = Q.cuda(), Q.cuda(), V.cuda()
    out = la.la_noncausal(q, k, v)
    ref = oracle.batched(oracle.noncausal, f64(q), f64(k), f64(v))
    assert oracle.max_row_rel_err(f64(out), ref) < 1e-6


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("chunk", [64, 128])
def test_prefix_mask_many_query_tiles_per_bin(d, chunk):
    """Masks whose values cluster on a few positions put hundreds of queries
    into one bin, so a chunk answers many query tiles back to back; repeated
    calls exercise the pipelining of those tiles."""
    B, H, N = 2, 3, 1500
    q, k, v = qkv(B, H, N, d, "bf16", seed=31 + d)
    gen = torch.Generator().manual_seed(5)
    choices = torch.tensor([0, 63, 64, 127, 128, 700, N - 1], dtype=torch.int32)
    m = choices[torch.randint(0, len(choices), (B, N), generator=gen)].contiguous().cuda()
    ref = oracle.batched(oracle.prefix_mask, f64(q), f64(k), f64(v), m=m.cpu().numpy())
    ws = la.workspace(la._desc_of(q, "relu1", True), "prefix", chunk)
    for _ in range(10):
        out = la.la_prefix_mask(q, k, v, m, chunk=chunk, ws=ws)
        assert oracle.max_row_rel_err(f64(out), ref) < 2e-2


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,H,N", [(4, 40, 300), (8, 50, 1), (2, 100, 129), (1, 3, 20000)])
def test_balanced_split_ranges_cross_heads(d, B, H, N):
    """The KV summary and readout split the flattened (head, 128-token tile)
    sequence evenly over the SMs, so one CTA's range can cover the end of
    one head and the start of the next, or several whole heads."""
    q, k, v = qkv(B, H, N, d, "bf16", seed=B * H + N)
    S = torch.empty(B, H, d, d, device="cuda")
    z = torch.empty(B, H, d, device="cuda")
    out = la.la_noncausal(q, k, v, S_out=S, z_out=z)
    Q, K, V = f64(q), f64(k), f64(v)
    S_ref, z_ref = oracle.kv_summary_batched(K, V)
    assert oracle.max_row_rel_err(f64(S), S_ref) < 1e-5
    np.testing.assert_allclose(f64(z), z_ref, rtol=1e-5)
    ref = np.einsum("bhna,bhac->bhnc", oracle.phi(Q), S_ref) / \
        np.einsum("bhna,bha->bhn", oracle.phi(Q), z_ref)[..., None]
    assert oracle.max_row_rel_err(f64(out), ref) < 2e-2


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("phi", ["relu1", "elu1"])
def test_causal_prefill_then_decode(dt, d, phi):
    """la_causal_prefill: the causal outputs (bit for bit those of
    la_causal_chunked) and the state after the last token, from which decode
    steps continue the sequence as the oracle's causal recurrence does."""
    B, H, N0, T = 2, 3, 1100, 12
    q, k, v = qkv(B, H, N0 + T, d, dt, seed=40 + d)
    pre = lambda x: x[:, :, :N0].contiguous()
    out, S, z = la.la_causal_prefill(pre(q), pre(k), pre(v), phi=phi)
    assert torch.equal(out, la.la_causal_chunked(pre(q), pre(k), pre(v), phi=phi))
    Q, K, V = f64(q), f64(k), f64(v)
    S_ref, z_ref = oracle.kv_summary_batched(K[:, :, :N0], V[:, :, :N0], phi)
    assert oracle.max_row_rel_err(f64(S), S_ref) < _state_tol(dt, phi)
    assert oracle.max_row_rel_err(f64(z)[..., None, :], z_ref[..., None, :]) < _state_tol(dt, phi)
    steps = []
    for t in range(N0, N0 + T):
        sl = lambda x: x[:, :, t:t + 1].contiguous()
        steps.append(la.la_decode_step(sl(q), sl(k), sl(v), S, z, phi=phi))
    got = torch.cat(steps, dim=2)
    ref = oracle.batched(oracle.causal, Q, K, V, phi_kind=phi)[:, :, N0:]
    assert oracle.max_row_rel_err(f64(got), ref) < TOL[DT[dt]]
    ref_pre = oracle.batched(oracle.causal, Q[:, :, :N0], K[:, :, :N0], V[:, :, :N0], phi_kind=phi)
    assert oracle.max_row_rel_err(f64(out), ref_pre) < TOL[DT[dt]]


@pytest.mark.parametrize("B,H,N", [(1, 16, 4096), (1, 16, 3800), (1, 2, 2300), (4, 37, 512), (1, 1, 64)])
def test_causal_and_prefix_block_counts(B, H, N):
    """bf16, d = 64 with 16, 15, 9, 2 and 1 blocks per head (148 heads of 2
    blocks fill the wave). The KV pass scans the block states inside a
    cluster per head: one block per CTA up to the non-portable cluster size 9
    here, two blocks per CTA for 16 heads of 16 or 15 blocks (the last CTA
    then takes one, partial block). 64- and 128-token chunks agree with each
    other and with the oracle, the prefill's outputs are those of the causal
    call and its state is the KV summary."""
    d = 64
    q, k, v = qkv(B, H, N, d, "bf16", seed=B + H + N)
    ref = oracle.batched(oracle.causal, f64(q), f64(k), f64(v))
    out = la.la_causal_chunked(q, k, v, chunk=64)
    assert oracle.max_row_rel_err(f64(out), ref) < 2e-2
    assert oracle.max_row_rel_err(f64(out), f64(la.la_causal_chunked(q, k, v, chunk=128))) < 2e-2
    out_p, S, z = la.la_causal_prefill(q, k, v, chunk=64)
    assert torch.equal(out_p, out)
    S_ref, z_ref = oracle.kv_summary_batched(f64(k), f64(v))
    assert oracle.max_row_rel_err(f64(S), S_ref) < 1e-4
    np.testing.assert_allclose(f64(z), z_ref, rtol=1e-4)
    m = workloads.prefix_mask_uniform(B, N, seed=N, device="cuda")
    ws = la.workspace(la._desc_of(q, "relu1", True), "prefix", 64)
    out_m = la.la_prefix_mask(q, k, v, m, chunk=64, ws=ws)
    assert la.la_last_error(ws) == (0, 0)
    ref_m = oracle.batched(oracle.prefix_mask, f64(q), f64(k), f64(v), m=m.cpu().numpy())
    assert oracle.max_row_rel_err(f64(out_m), ref_m) < 2e-2
