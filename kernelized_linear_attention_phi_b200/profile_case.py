"""Runs one library call on one synthetic problem a few times and exits: the
command to put under a profiler (ncu) when studying a single kernel.

    python -m kernelized_linear_attention_phi_b200.profile_case \\
        --op noncausal --B 1 --H 16 --N 16384 --d 64 --iters 3

``--op`` is one of kv_summary, noncausal, causal, prefix, decode,
noncausal_bwd, causal_bwd. Inputs come from the seeded generators in
``workloads``; nothing is checked or timed.
"""

from __future__ import annotations

import argparse

import torch

from . import binding as la
from . import workloads as W


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", required=True, choices=["kv_summary", "noncausal", "causal", "prefix", "decode",
                                                      "noncausal_bwd", "causal_bwd"])
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--N", type=int, default=16384)
    ap.add_argument("--d", type=int, default=64)
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--phi", default="relu1", choices=["relu1", "identity", "elu1"])
    ap.add_argument("--unnormalized", action="store_true")
    ap.add_argument("--chunk", type=int, default=64)
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    from . import build
    build.build()
    dev = torch.device("cuda", 0)
    sigma = a.d ** -0.5 if a.phi == "identity" else 1.0
    norm = not a.unnormalized
    q, k, v = W.qkv(a.B, a.H, a.N, a.d, sigma, 1, a.dtype, dev)
    desc = la._desc_of(q, a.phi, norm)
    if a.op == "decode":
        S = torch.zeros(a.B, a.H, a.d, a.d, device=dev)
        z = torch.zeros(a.B, a.H, a.d, device=dev)
        q1, k1, v1 = (t[0].contiguous() for t in W.decode_tokens(1, a.B, a.H, a.d, sigma, 1, a.dtype, dev))
        out = torch.empty_like(q1)
        fn = lambda: la.la_decode_step(q1, k1, v1, S, z, out, a.phi, norm)
    elif a.op.endswith("_bwd"):
        ws = la.workspace(desc, a.op, a.chunk, dev)
        dout = W.upstream_grad(a.B, a.H, a.N, a.d, 1, a.dtype, dev)
        grads = [torch.empty_like(q) for _ in range(3)]
        bwd = la.la_noncausal_backward if a.op == "noncausal_bwd" else la.la_causal_backward
        fn = lambda: bwd(q, k, v, dout, *grads, phi=a.phi, normalize=norm, ws=ws)
    else:
        ws = la.workspace(desc, a.op, a.chunk, dev)
        out = torch.empty_like(q)
        m = W.prefix_mask_uniform(a.B, a.N, 1, dev)
        fn = {
            "kv_summary": lambda: la.la_kv_summary(k, v, phi=a.phi, ws=ws),
            "noncausal": lambda: la.la_noncausal(q, k, v, out, phi=a.phi, normalize=norm, ws=ws),
            "causal": lambda: la.la_causal_chunked(q, k, v, out, a.chunk, a.phi, norm, ws),
            "prefix": lambda: la.la_prefix_mask(q, k, v, m, out, a.chunk, a.phi, norm, ws),
        }[a.op]
    for _ in range(a.iters):
        fn()
    torch.cuda.synchronize()


if __name__ == "__main__":
    main()
