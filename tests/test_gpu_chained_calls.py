"""Calls whose inputs are the outputs of the call just before them on the
same stream, with no other kernel in between: every kernel lets the next one
launch early (programmatic dependent launch), so the first kernel of a call
must not read its inputs before the previous kernel has finished. Each chain
is run back to back and again with a device synchronization between the
calls; the library is deterministic, so the two must agree bit for bit."""

import pytest
import torch

from kernelized_linear_attention_phi_b200 import binding as la

from gpu_util import qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kernelized_linear_attention_phi_b200 import build
    build.build()
    la.lib()


def _chain(q, k, v, m, sync):
    """causal -> non-causal (its keys) -> KV summary (its values) -> prefix
    mask (its queries) -> causal (its keys)."""
    s = (lambda: torch.cuda.synchronize()) if sync else (lambda: None)
    a = la.la_causal_chunked(q, k, v)
    s()
    b = la.la_noncausal(q, a, v)
    s()
    S, z = la.la_kv_summary(k, b)
    s()
    c = la.la_prefix_mask(b, k, v, m)
    s()
    d = la.la_causal_chunked(q, c, v)
    torch.cuda.synchronize()
    return a, b, S, z, c, d


@pytest.mark.parametrize("B,H,N,d", [(2, 8, 4096, 64), (1, 4, 2048, 128), (2, 8, 1024, 64)])
def test_back_to_back_calls_match_synchronized_calls(B, H, N, d):
    q, k, v = qkv(B, H, N, d, "bf16", seed=40 + d)
    m = torch.randint(0, N, (B, N), dtype=torch.int32, device="cuda",
                      generator=torch.Generator(device="cuda").manual_seed(7))
    ref = _chain(q, k, v, m, sync=True)
    for _ in range(3):
        got = _chain(q, k, v, m, sync=False)
        for x, y in zip(got, ref):
            assert torch.equal(x, y)
