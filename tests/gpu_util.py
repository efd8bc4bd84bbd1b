"""Helpers for the GPU parity tests: inputs from the seeded generators, exact
upcast to float64 for the oracle, and the tolerances."""

import numpy as np
import torch

from kernelized_linear_attention_phi_b200 import workloads

# Maximum relative row error against the fp64 oracle: 1e-4 for fp32 inputs,
# 2e-2 for bf16 inputs with fp32 accumulation.
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy (bf16 and fp32 values are representable)."""
    return t.detach().to(torch.float64).cpu().numpy()


def qkv(B, H, N, d, dtype, seed, sigma=1.0):
    return workloads.qkv(B, H, N, d, sigma=sigma, seed=seed, dtype=dtype, device="cuda")
