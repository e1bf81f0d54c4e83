"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and lays them out in the shapes,
dtypes and value distributions of the workloads; it holds none of the
quantization or matmul arithmetic, so the oracle and the CUDA library can
both be fed from it without sharing any of the method's code.

Recipe (the same for every consumer):

* The tiny case draws with NumPy ``default_rng(0)``: W [16, 259] ~ N(0, 1)
  fp32, then row 3 columns 128..255 set to 0 (one all-zero group at
  group 128), then x [4, 259] ~ N(0, 1) fp32.
* Every other tensor is drawn with a ``torch.Generator`` seeded per tensor on
  the device it will live on, in fp32, then rounded to the stored dtype by
  round-to-nearest-even (``Tensor.to``).
* Heavy-tailed weights are Student-t with 3 degrees of freedom, drawn as
  z0 / sqrt((z1^2 + z2^2 + z3^2) / 3) from four standard normals, times 0.02.
* "1% of groups all-zero" draws a Bernoulli(0.01) mask over the (row, group)
  grid from the same generator and zeroes each selected group, the partial
  last group included.
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

__all__ = [
    "tiny_case",
    "make_weights",
    "make_activations",
    "Layer",
    "DISTILGPT2_LINEARS",
    "LLAMA7B_DECODE_LINEARS",
    "PREFILL_LINEARS",
    "BULK_QUANTIZE_LINEARS",
]


def tiny_case():
    """W [16, 259] fp32, x [4, 259] fp32, group 128, with one all-zero group."""
    rng = np.random.default_rng(0)
    w = rng.normal(size=(16, 259)).astype(np.float32)
    w[3, 128:256] = 0.0
    x = rng.normal(size=(4, 259)).astype(np.float32)
    return {"w": w, "x": x, "group": 128}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_weights(N: int, K: int, *, seed: int, device="cpu", dtype=torch.float32,
                 dist: str = "normal", std: float = 0.02,
                 zero_group_frac: float = 0.0, group: int = 128) -> torch.Tensor:
    """Weight matrix [N, K] in ``dtype`` on ``device`` (see the module recipe)."""
    g = _gen(seed, device)
    if dist == "normal":
        w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std
    elif dist == "student_t3":
        z0 = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
        chi = torch.zeros((N, K), device=device, dtype=torch.float32)
        for _ in range(3):
            z = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
            chi.addcmul_(z, z)
            del z
        w = z0.div_(torch.sqrt_(chi.div_(3.0))).mul_(std)
        del chi
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    if zero_group_frac > 0.0:
        G = -(-K // group)
        mask = torch.rand((N, G), generator=g, device=device) < zero_group_frac
        keep = (~mask).repeat_interleave(group, dim=1)[:, :K]
        w.mul_(keep)
        del keep
    return w.to(dtype)


def make_activations(M: int, K: int, *, seed: int, device="cpu",
                     dtype=torch.bfloat16) -> torch.Tensor:
    """Activations x [M, K] ~ N(0, 1) in ``dtype`` on ``device``."""
    g = _gen(seed, device)
    return torch.randn((M, K), generator=g, device=device, dtype=torch.float32).to(dtype)


@dataclasses.dataclass(frozen=True)
class Layer:
    """One weight matrix of a workload: W [N, K] with its group size."""
    name: str
    N: int
    K: int
    group: int


# distilgpt2's quantized linears, shaped [out, in]: c_attn, mlp c_fc, mlp c_proj.
DISTILGPT2_LINEARS = [Layer(f"{n}_g{g}", N, K, g)
                      for (n, N, K) in (("c_attn", 2304, 768), ("c_fc", 3072, 768),
                                        ("c_proj", 768, 3072))
                      for g in (32, 64)]

# Llama-7B-shaped linears used for the skinny decode matmul (M = 1, 4, 16).
LLAMA7B_DECODE_LINEARS = [Layer("qkvo", 4096, 4096, 128), Layer("up", 11008, 4096, 128),
                          Layer("down", 4096, 11008, 128)]

# Large linears used for the tensor-core prefill matmul (M = 2048, 8192).
PREFILL_LINEARS = [Layer("square", 8192, 8192, 128), Layer("wide", 28672, 8192, 128)]

# Bulk quantize/pack + unpack: heavy-tailed bf16 weights, 1% all-zero groups.
BULK_QUANTIZE_LINEARS = [Layer(f"{n}_g{g}", N, K, g)
                         for (n, N, K) in (("wide", 28672, 8192), ("oddK", 8192, 28673))
                         for g in (32, 64, 128)]
