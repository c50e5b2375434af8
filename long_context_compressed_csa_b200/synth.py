"""Seeded synthetic inputs shared by the tests, the bench and the oracle harness.

Holds none of the method's arithmetic: only random draws, their storage dtype and the
workload shapes.  Projected quantities (C, Z streams, queries, indexer queries and
weights, compressed caches) are drawn directly as N(0, 1): that is the distribution a
projection of N(0, 1) hidden states by N(0, 1/fan_in) weights produces, and the pages
give no trained weights or model width.  bf16 tensors are the fp32 draws rounded by
torch's bf16 conversion, so the CPU oracle and the GPU see identical values.
"""
from __future__ import annotations

import torch

# Production settings of V4-Pro ("DeepSeek-V4 Hybrid Attention: CSA and HCA from
# Scratch", running-example parameter list and section 12.2).
C = 512        # compressed entry width c
M = 4          # CSA compression ratio m
M_PRIME = 128  # HCA compression ratio m'
TOPK = 1024    # CSA selection budget k
N_H = 128      # query heads n_h
N_HI = 64      # indexer heads n_h^I
C_I = 128      # indexer head width c^I

WORKLOADS = {
    "csa_decode_8k": dict(B=1, n=8192, m=M, c=C, cI=C_I, k=512, n_h=N_H, n_hI=N_HI),
    "hca_decode_b16_128k": dict(B=16, n=131072, m_prime=M_PRIME, c=C, n_h=N_H),
    "csa_prefill_decode_b4_256k": dict(B=4, n=262144, m=M, c=C, cI=C_I, k=TOPK, n_h=N_H,
                                       n_hI=N_HI, decode_steps=64),
    "hybrid_1m_decode": dict(B=1, n=1 << 20, m=M, m_prime=M_PRIME, c=C, cI=C_I, k=TOPK,
                             n_h=N_H, n_hI=N_HI, decode_steps=256),
}


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn(shape, seed: int, dtype=torch.bfloat16, device="cpu", scale: float = 1.0) -> torch.Tensor:
    """N(0, scale^2) draws of ``shape`` from a dedicated generator, stored as ``dtype``."""
    g = generator(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def randint_values(shape, seed: int, low: int, high: int, dtype=torch.bfloat16, device="cpu"):
    """Small integers in [low, high) stored as ``dtype`` (exact in bf16 and fp32)."""
    g = generator(seed, device)
    return torch.randint(low, high, tuple(shape), generator=g, device=device).to(dtype)


def to_f64(x: torch.Tensor):
    """float64 numpy copy of a (CPU or CUDA) tensor, for the oracle."""
    return x.detach().to("cpu", torch.float64).numpy()
