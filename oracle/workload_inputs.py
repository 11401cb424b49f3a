"""Conversion of a synthetic workload (torch tensors, any device) into the
oracle's plain numpy inputs.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: used by ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``.  It copies
bytes and relabels storage; it holds none of the method's arithmetic.
"""

from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

from .sparse_decode_oracle import OracleConfig

__all__ = ["bf16_bits", "oracle_config", "oracle_inputs"]


def bf16_bits(t) -> np.ndarray:
    """Raw bf16 bit patterns (uint16) of a bf16 torch tensor."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_config(w) -> OracleConfig:
    """The oracle's configuration of a workload (same heads, modes and scales)."""
    return OracleConfig(w.num_q_heads, w.num_kv_heads, w.head_dim, w.index_dim, w.page_size,
                        list(w.head_is_retrieval), w.window, w.num_sinks, w.mode, top_p=w.top_p,
                        top_k=w.top_k, top_k_frac=w.top_k_frac,
                        attn_scale=w.attn_scale or None, index_scale=w.index_scale or None)


def oracle_inputs(w, seqs: Optional[Sequence[int]] = None):
    """numpy inputs of the oracle for the sequences `seqs` (all by default).

    Only the pages of those sequences are copied; they are renumbered in a
    compact pool and the page table is remapped accordingly (a relabelling of
    storage, which the page-table indirection makes invisible)."""
    import torch
    if seqs is None:
        seqs = list(range(w.batch))
    seqs = list(seqs)
    lens = w.seq_lens.cpu().numpy()
    pt = w.page_table.cpu().numpy()
    pages = []
    new_pt = -np.ones((len(seqs), pt.shape[1]), np.int64)
    for i, b in enumerate(seqs):
        m = math.ceil(int(lens[b]) / w.page_size)
        ids = pt[b, :m].astype(np.int64)
        new_pt[i, :m] = np.arange(len(pages), len(pages) + m)
        pages.extend(ids.tolist())
    idx = torch.tensor(pages, dtype=torch.long, device=w.k_cache.device)
    if len(pages):
        kc = bf16_bits(w.k_cache.index_select(0, idx))
        vc = bf16_bits(w.v_cache.index_select(0, idx))
    else:
        kc = np.zeros((0,) + tuple(w.k_cache.shape[1:]), np.uint16)
        vc = np.zeros_like(kc)
    sel = torch.tensor(seqs, dtype=torch.long, device=w.q.device)
    return dict(proj=w.proj.float().cpu().numpy(),
                q_pre=w.q_pre.index_select(0, sel).float().cpu().numpy(),
                q=w.q.index_select(0, sel).float().cpu().numpy(),
                k_cache=kc, v_cache=vc, page_table=new_pt, seq_lens=lens[seqs])
