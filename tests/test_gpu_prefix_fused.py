"""Prefix-mask attention through the one-kernel path (bf16, d = 64, at most
4096 tokens: a thread-block cluster per head, the queries binned inside the
kernel by the 128-key sub-block that holds m_i, tiles of 128 sorted queries
that may span sub-blocks) against the fp64 oracle, over cluster sizes 1-8,
masks that fill one block or one sub-block, ragged lengths and every feature
map; and the multi-kernel path that longer sequences take."""

import pytest
import torch

import oracle
from kernelized_linear_attention_phi_b200 import binding as la
from kernelized_linear_attention_phi_b200 import workloads

from gpu_util import TOL, f64, qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kernelized_linear_attention_phi_b200 import build
    build.build()
    la.lib()


def _mask(kind, B, N, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    if kind == "uniform":
        m = torch.randint(0, N, (B, N), generator=g, dtype=torch.int32)
    elif kind == "arange":
        m = torch.arange(N, dtype=torch.int32).repeat(B, 1)
    elif kind == "reverse":
        m = (N - 1 - torch.arange(N, dtype=torch.int32)).repeat(B, 1)
    elif kind == "last":  # every query in the last block: its tiles fill the kernel's table
        m = torch.full((B, N), N - 1, dtype=torch.int32)
    elif kind == "zeros":
        m = torch.zeros(B, N, dtype=torch.int32)
    elif kind == "narrow":  # every limit inside one 128-key sub-block
        lo = N // 2
        m = torch.randint(lo, min(N, lo + 100), (B, N), generator=g, dtype=torch.int32)
    elif kind == "sparse":  # few queries per sub-block: tiles span several sub-blocks
        m = (torch.randint(0, max(1, N // 300), (B, N), generator=g, dtype=torch.int32) * 300).clamp(max=N - 1)
    else:
        raise ValueError(kind)
    return m.contiguous().cuda()


def _check(B, H, N, kind, phi="relu1", normalize=True, seed=0):
    sigma = 1.0 if phi != "identity" else 64 ** -0.5
    q, k, v = qkv(B, H, N, 64, "bf16", seed=seed, sigma=sigma)
    m = _mask(kind, B, N, seed)
    ws = la.workspace(la._desc_of(q, phi, normalize), "prefix", 64)
    out = la.la_prefix_mask(q, k, v, m, phi=phi, normalize=normalize, ws=ws)
    assert la.la_last_error(ws) == (0, 0)
    ref = oracle.batched(oracle.prefix_mask, f64(q), f64(k), f64(v), phi_kind=phi, normalize=normalize,
                         m=m.cpu().numpy())
    err = oracle.max_row_rel_err(f64(out), ref)
    assert err < TOL[torch.bfloat16], err
    return out


@pytest.mark.parametrize("B,H,N", [(1, 1, 1), (1, 1, 128), (1, 3, 129), (2, 4, 1000), (1, 16, 4096), (3, 37, 700),
                                   (2, 2, 2049)])
@pytest.mark.parametrize("kind", ["uniform", "arange", "last", "narrow", "sparse"])
def test_fused_prefix_mask_shapes_and_masks(B, H, N, kind):
    _check(B, H, N, kind, seed=B * 1000 + N)


@pytest.mark.parametrize("phi,normalize", [("relu1", True), ("identity", False), ("elu1", True),
                                           ("relu1", False)])
@pytest.mark.parametrize("kind", ["uniform", "reverse", "zeros"])
def test_fused_prefix_mask_feature_maps(phi, normalize, kind):
    _check(2, 8, 2048, kind, phi, normalize, seed=3)


def test_fused_prefix_mask_is_deterministic():
    q, k, v = qkv(2, 8, 3000, 64, "bf16", seed=9)
    m = _mask("uniform", 2, 3000, 9)
    a = la.la_prefix_mask(q, k, v, m)
    b = la.la_prefix_mask(q, k, v, m)
    assert torch.equal(a, b)


def test_fused_prefix_mask_out_of_range_is_clamped_and_flagged():
    B, H, N = 2, 4, 777
    q, k, v = qkv(B, H, N, 64, "bf16", seed=12)
    m = workloads.prefix_mask_uniform(B, N, seed=3, device="cuda")
    m[0, 5] = -4
    m[1, 9] = N + 10
    ws = la.workspace(la._desc_of(q, "relu1", True), "prefix", 64)
    out = la.la_prefix_mask(q, k, v, m, ws=ws)
    status, flags = la.la_last_error(ws)
    assert status == 6 and flags == 1
    mc = m.clamp(0, N - 1).cpu().numpy()
    ref = oracle.batched(oracle.prefix_mask, f64(q), f64(k), f64(v), m=mc)
    assert oracle.max_row_rel_err(f64(out), ref) < TOL[torch.bfloat16]


@pytest.mark.parametrize("N", [4097, 6000])
def test_longer_sequences_take_the_multi_kernel_path(N):
    """Past 4096 tokens the binning kernel, the block states and the gather
    sweep answer the prefix mask."""
    _check(1, 4, N, "uniform", seed=N)
    _check(1, 2, N, "arange", phi="identity", normalize=False, seed=N + 1)
