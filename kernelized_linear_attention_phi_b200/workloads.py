"""Seeded synthetic inputs: the workloads the pages describe, with their shapes.

This module only draws random numbers and describes shapes. It holds none of
the attention arithmetic, so both the CUDA path (bench, tests) and the fp64
oracle (tests) can take their inputs from it.

Shapes follow the pages:

* ``single_head``: one head, N=256, d=16, fp32 -- the scale of the nx
  source's worked examples grown to several tiles.
* ``multi_head``: B=2, H=8, N=4096, d=64 (d_model 512 in 8 heads) -- the
  lineartile 1.0.1 "Quick Start" input x[2, 4096, 512].
* ``prefix_mask``: B=8, H=8, N=2048, d=64, identity map, unnormalized, values
  ~ N(0, 1/d) -- the trim-transformer 0.1.0 "Quickstart" input x[8, 2048, 512]
  and its "Masking" section.
* ``long_noncausal``: B=4, H=16, N=16384 (128x128 latent tokens), d=64 --
  the DiT/SANA motivation in the nx source header.
* ``long_causal``: B=1, H=16, N=131072, d=128, causal.
* ``decode``: 64 sequences, H=32, d=128, prefilled from 2048 tokens, then
  1024 one-token steps -- trim-transformer 0.1.0 "Key-value caching".
"""

from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtypes: tuple
    phi: str            # "relu1" or "identity"
    normalize: bool
    forms: tuple        # subset of ("noncausal", "causal", "prefix", "decode",
                        # "noncausal_bwd", "causal_bwd")
    sigma: float        # standard deviation of Q, K, V entries
    seed: int
    chunk: int = 64
    decode_steps: int = 0
    note: str = ""


WORKLOADS = {
    "single_head": Workload("single_head", 1, 1, 256, 16, ("f32",), "relu1", True,
                            ("noncausal",), 1.0, 1),
    "multi_head": Workload("multi_head", 2, 8, 4096, 64, ("bf16", "f32"), "relu1", True,
                           ("noncausal", "causal"), 1.0, 2, chunk=64),
    "prefix_mask": Workload("prefix_mask", 8, 8, 2048, 64, ("bf16",), "identity", False,
                            ("prefix",), 64 ** -0.5, 3, chunk=64),
    "long_noncausal": Workload("long_noncausal", 4, 16, 16384, 64, ("bf16",), "relu1", True,
                               ("noncausal",), 1.0, 4),
    "long_causal": Workload("long_causal", 1, 16, 131072, 128, ("bf16",), "relu1", True,
                            ("causal",), 1.0, 5, chunk=128),
    "decode": Workload("decode", 64, 32, 2048, 128, ("bf16",), "relu1", True,
                       ("decode",), 1.0, 6, decode_steps=1024),
    # the gradients of the multi-head forms, for an upstream gradient
    # dout ~ N(0, 1) (upstream_grad)
    "multi_head_bwd": Workload("multi_head_bwd", 2, 8, 4096, 64, ("bf16", "f32"), "relu1", True,
                               ("noncausal_bwd", "causal_bwd"), 1.0, 2, chunk=64),
}

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, sigma=1.0, seed=0, dtype="bf16", device="cpu"):
    """Gaussian N(0, sigma^2) entries, drawn in fp32 then cast to ``dtype``."""
    g = generator(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(TORCH_DTYPES.get(dtype, dtype))


def qkv(B, H, N, d, sigma=1.0, seed=0, dtype="bf16", device="cpu"):
    """Three independent [B, H, N, d] tensors (seeds seed*3 + 0, 1, 2)."""
    return tuple(normal((B, H, N, d), sigma, 3 * seed + i, dtype, device)
                 for i in range(3))


def prefix_mask_uniform(B, N, seed=0, device="cpu"):
    """int32 [B, N], each m_i uniform in [0, N-1] (one mask per sequence)."""
    g = generator(10_000 + seed, device)
    return torch.randint(0, N, (B, N), generator=g, device=device, dtype=torch.int32)


def prefix_mask_arange(B, N, device="cpu"):
    """The causal mask m_i = i, for every sequence."""
    return torch.arange(N, device=device, dtype=torch.int32).repeat(B, 1)


def decode_tokens(steps, B, H, d, sigma=1.0, seed=0, dtype="bf16", device="cpu"):
    """q, k, v for ``steps`` one-token steps: three [steps, B, H, 1, d] tensors."""
    return tuple(normal((steps, B, H, 1, d), sigma, 20_000 + 3 * seed + i, dtype, device)
                 for i in range(3))


def upstream_grad(B, H, N, d, seed, dtype="bf16", device="cpu"):
    """dL/dout for the gradient workloads: N(0, 1) entries, generator seed
    30000 + seed."""
    return normal((B, H, N, d), 1.0, 30_000 + seed, dtype, device)
