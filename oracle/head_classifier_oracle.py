"""Plain float64 CPU definition of the data-free head classifier.

TEST INFRASTRUCTURE ONLY: the oracle that the CUDA classifier is checked
against.  It may be imported only by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``.  It shares no code with
the CUDA path.

Source: [AoH] "Autonomy-of-Heads: Data-Free Sparse Attention from Frozen
Query-Key Geometry", gist.science/ar/paper/2608.06849, Methodology:
  §1  the kernel attention operator of head h, M_h = W_K^T W_Q (d_model x
      d_model); a concentrated spectrum marks a retrieval head, a diffuse
      one a streaming head;
  §2  the effective rank, exp of the Shannon entropy of the normalised
      singular values of M_h; low ER -> retrieval, high ER -> streaming;
  §3  the nonzero singular values of M_h follow from the d_head x d_head
      matrix C_h = (W_Q W_Q^T)(W_K W_K^T) (Sylvester's determinant identity);
  §4  heads ranked by ER, the k lowest become retrieval heads; under GQA the
      head scores are mean-pooled to the group.

Readings taken where the page is silent or garbled:
  * W_Q^h is the d_head x d_model block of rows h*d_head .. (h+1)*d_head - 1
    of the query projection weight [Hq*d_head, d_model] (q = W x), and W_K^g
    likewise of the key projection; head h pairs with KV head g = h // (Hq/Hkv);
  * §3's garbled relation read as: the eigenvalues of C_h are the squares of
    the nonzero singular values of M_h, so sigma_k = sqrt(lambda_k(C_h));
  * r_h, the number of nonzero singular values, applies the usual
    numerical-rank threshold to the quantity each route computes: sigma >
    sigma_max * d_model * eps for the SVD of M_h, lambda > lambda_max * d_head
    * eps for the eigenvalues of C_h (an eigenvalue of C_h is known to about
    eps * lambda_max, so its square root only to about sqrt(eps) * sigma_max);
  * a head with no nonzero singular value has ER = exp(0) = 1 (the empty sum);
  * §4's "k lowest" is a count of GQA groups given by the caller; equal pooled
    scores go to the lower group index; a NaN score ranks after every number;
    the pooled mean sums the group's heads in head order, then divides.

Pins (``tests/test_classifier_pins.py``): closed forms of the entropy, weights
built with a known spectrum (equal singular values, rank one, a prescribed
spectrum through an orthonormal basis), and the two routes of §1-2 and §3
against each other on random weights.
"""

from __future__ import annotations

import math
from typing import Sequence

import numpy as np

__all__ = [
    "effective_rank_of_spectrum",
    "kernel_operator",
    "singular_values_direct",
    "singular_values_sylvester",
    "head_block",
    "layer_effective_ranks",
    "classify_groups",
]


def effective_rank_of_spectrum(sigma) -> float:
    """[AoH] §2: ER = exp(-sum_k s_k log s_k), s_k = sigma_k / sum sigma over
    the r_h nonzero singular values (``sigma`` holds those only)."""
    s = np.asarray(sigma, dtype=np.float64)
    if s.size == 0 or s.sum() == 0.0:
        return 1.0
    p = s / s.sum()
    return float(np.exp(-np.sum(p * np.log(p))))


def _nonzero(sigma, shape) -> np.ndarray:
    sigma = np.asarray(sigma, dtype=np.float64)
    if sigma.size == 0 or sigma.max() <= 0.0:
        return sigma[:0]
    tol = sigma.max() * max(shape) * np.finfo(np.float64).eps
    return sigma[sigma > tol]


def kernel_operator(wq_h, wk_g) -> np.ndarray:
    """[AoH] §1: M_h = W_K^T W_Q, from the d_head x d_model blocks."""
    return np.asarray(wk_g, dtype=np.float64).T @ np.asarray(wq_h, dtype=np.float64)


def singular_values_direct(wq_h, wk_g) -> np.ndarray:
    """Nonzero singular values of M_h by a full SVD of the d_model x d_model
    matrix ([AoH] §1-2 as written)."""
    m = kernel_operator(wq_h, wk_g)
    return _nonzero(np.linalg.svd(m, compute_uv=False), m.shape)


def singular_values_sylvester(wq_h, wk_g) -> np.ndarray:
    """Nonzero singular values of M_h from the eigenvalues of C_h =
    (W_Q W_Q^T)(W_K W_K^T), d_head x d_head ([AoH] §3)."""
    q = np.asarray(wq_h, dtype=np.float64)
    k = np.asarray(wk_g, dtype=np.float64)
    c = (q @ q.T) @ (k @ k.T)
    lam = _nonzero(np.linalg.eigvals(c).real, c.shape)
    return np.sqrt(lam)


def head_block(w, head: int, head_dim: int) -> np.ndarray:
    """Rows head*head_dim .. (head+1)*head_dim - 1 of a projection weight."""
    return np.asarray(w)[head * head_dim:(head + 1) * head_dim]


def layer_effective_ranks(w_q, w_k, num_q_heads: int, num_kv_heads: int, head_dim: int,
                          route: str = "sylvester") -> np.ndarray:
    """ER of every query head of one layer: w_q [Hq*d_head, d_model], w_k
    [Hkv*d_head, d_model] (float arrays holding the weights' values)."""
    group = num_q_heads // num_kv_heads
    sv = singular_values_sylvester if route == "sylvester" else singular_values_direct
    out = np.empty(num_q_heads, dtype=np.float64)
    for h in range(num_q_heads):
        wq_h = head_block(w_q, h, head_dim)
        wk_g = head_block(w_k, h // group, head_dim)
        out[h] = effective_rank_of_spectrum(sv(wq_h, wk_g))
    return out


def classify_groups(eff_rank: Sequence[float], num_kv_heads: int, num_retrieval_groups: int) -> np.ndarray:
    """[AoH] §4: mean-pool the heads' ER to their GQA group, rank the groups by
    pooled ER (ties: lower group first), mark the heads of the
    ``num_retrieval_groups`` lowest as retrieval (1), the rest streaming (0)."""
    er = np.asarray(eff_rank, dtype=np.float64)
    group = er.size // num_kv_heads
    pooled = []
    for g in range(num_kv_heads):
        total = 0.0
        for h in range(g * group, (g + 1) * group):    # in head order, one rounding per add
            total += float(er[h])
        pooled.append(total / group)
    # a NaN (no converged spectrum) ranks after every number
    order = sorted(range(num_kv_heads), key=lambda g: (math.isnan(pooled[g]),
                                                       0.0 if math.isnan(pooled[g]) else pooled[g], g))
    chosen = set(order[:num_retrieval_groups])
    return np.array([1 if h // group in chosen else 0 for h in range(er.size)], dtype=np.int32)
