"""Seeded synthetic query / key projection weights for the head classifier.

Input construction only: draws weights with a chosen spectral shape and
computes no effective rank or classification; it imports neither the oracle
nor the CUDA library.

Each d_head x d_model head block is W = diag(s) G / sqrt(d_model) with G
standard normal and s_k = (k + 1)^(-alpha): for d_model >> d_head the rows of
G are nearly orthogonal, so alpha sets how concentrated the block's spectrum
is.  Every KV group draws a steepness alpha_g ~ U[alpha_lo, alpha_hi]; its
query heads take alpha_g + N(0, 0.05^2) and its key block a flatter
alpha_g / 3.  Values are drawn in float32 and rounded to bf16.

Default sizes are Llama-3.1-8B's attention projections: 32 layers, d_model
4096, 32 query and 8 KV heads of 128 (the model the AoH page reports on).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass
class ProjectionWeights:
    w_q: torch.Tensor          # bf16 [L, Hq * d_head, d_model]
    w_k: torch.Tensor          # bf16 [L, Hkv * d_head, d_model]
    num_layers: int
    d_model: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    alpha_q: torch.Tensor      # float32 [L, Hq]
    alpha_k: torch.Tensor      # float32 [L, Hkv]


def make_projections(device="cuda", seed: int = 7, num_layers: int = 32, d_model: int = 4096,
                     num_q_heads: int = 32, num_kv_heads: int = 8, head_dim: int = 128,
                     alpha_lo: float = 0.1, alpha_hi: float = 1.5) -> ProjectionWeights:
    G = num_q_heads // num_kv_heads
    gen = torch.Generator(device=device)
    gen.manual_seed(seed * 1000 + 11)
    a_g = alpha_lo + (alpha_hi - alpha_lo) * torch.rand((num_layers, num_kv_heads), generator=gen, device=device)
    a_q = (a_g.repeat_interleave(G, dim=1)
           + 0.05 * torch.randn((num_layers, num_q_heads), generator=gen, device=device)).clamp_min(0.0)
    a_k = a_g / 3.0
    k = torch.arange(1, head_dim + 1, device=device, dtype=torch.float32)
    w_q = torch.empty((num_layers, num_q_heads * head_dim, d_model), dtype=torch.bfloat16, device=device)
    w_k = torch.empty((num_layers, num_kv_heads * head_dim, d_model), dtype=torch.bfloat16, device=device)
    for layer in range(num_layers):
        s_q = k[None, :] ** (-a_q[layer][:, None])                 # [Hq, d_head]
        s_k = k[None, :] ** (-a_k[layer][:, None])
        gq = torch.randn((num_q_heads * head_dim, d_model), generator=gen, device=device) / math.sqrt(d_model)
        gk = torch.randn((num_kv_heads * head_dim, d_model), generator=gen, device=device) / math.sqrt(d_model)
        w_q[layer] = (gq * s_q.reshape(-1, 1)).to(torch.bfloat16)
        w_k[layer] = (gk * s_k.reshape(-1, 1)).to(torch.bfloat16)
    return ProjectionWeights(w_q, w_k, num_layers, d_model, num_q_heads, num_kv_heads, head_dim,
                             a_q.float(), a_k.float())
