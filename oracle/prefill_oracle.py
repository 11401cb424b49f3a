"""Plain float64 CPU definition of head-wise prefill attention.

TEST INFRASTRUCTURE ONLY: the oracle that the CUDA prefill is checked against.
It may be imported only by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py``.  It shares no code with the
CUDA path.

Sources:
[RTP] "Full attention strikes back: moving full attention to sparse attention
      within hundreds of training steps", gist.science/ar/paper/2605.16928,
      Methodology §1: heads split into retrieval and local heads; during
      inference the local heads use a sliding window with attention sinks,
      while the retrieval heads keep their full KV through the prefill phase
      and move to dynamic sparse selection only when decoding.  Results: the
      prefill speed-up over dense FlashAttention-2 grows with the context.
[AoH] "Autonomy-of-Heads: Data-Free Sparse Attention from Frozen Query-Key
      Geometry", gist.science/ar/paper/2608.06849, Methodology §4: streaming
      heads keep a sink prefix plus a recent window; the split works with
      standard chunked prefill.

Prefill of a chunk: sequence b holds N_b tokens in the cache; its last T_b are
the chunk, whose queries sit at positions N_b - T_b .. N_b - 1.  The query at
position i of head h attends, causally, to

    retrieval head:  keys 0 .. i                         (dense causal)
    local head:      keys [0, num_sinks) U [i - window + 1, i], within [0, i]

Readings: the window counts the query's own position,
so a local head's keys at position i are the decode local set at length
i + 1; the chunk's own keys and values are already in the cache; earlier
chunks' keys are read from the cache like any other.

Pins (``tests/test_prefill_pins.py``): torch's float64 scaled-dot-product
attention with its causal flag (retrieval heads) and with a boolean band mask
built by broadcasting (local heads); chunk invariance; a one-token chunk equals
the decode oracle's output.
"""

from __future__ import annotations

from typing import Dict, Iterable, Optional, Tuple

import numpy as np

from .sparse_decode_oracle import attend_set, gather_rows, local_positions

__all__ = ["prefill_positions", "prefill_reference"]


def prefill_positions(pos: int, is_retrieval: bool, window: int, num_sinks: int) -> np.ndarray:
    """Keys the query at position ``pos`` attends to ([RTP] §1, [AoH] §4)."""
    if is_retrieval:
        return np.arange(pos + 1, dtype=np.int64)
    return local_positions(pos + 1, window, num_sinks)


def prefill_reference(cfg, q, k_cache, v_cache, page_table, seq_lens, q_starts,
                      pairs: Optional[Iterable[Tuple[int, int]]] = None) -> Dict[Tuple[int, int], np.ndarray]:
    """Outputs of the chunk's queries: q [total_q, Hq, d] packed by sequence
    (sequence b's queries are rows q_starts[b] .. q_starts[b+1] - 1), caches
    paged as for decode.  Returns {(row, h): out[d]} for the (row, h) pairs
    asked (default: all)."""
    Hq, Hkv = cfg.num_q_heads, cfg.num_kv_heads
    G = Hq // Hkv
    attn_scale, _ = cfg.scales()
    starts = [int(x) for x in q_starts]
    B = len(starts) - 1
    row_seq = {}
    for b in range(B):
        for r in range(starts[b], starts[b + 1]):
            row_seq[r] = b
    if pairs is None:
        pairs = [(r, h) for r in range(starts[-1]) for h in range(Hq)]
    out = {}
    cache: Dict[Tuple[int, int], Tuple[np.ndarray, np.ndarray]] = {}
    for r, h in pairs:
        b = row_seq[r]
        n = int(seq_lens[b])
        t = starts[b + 1] - starts[b]
        pos = n - t + (r - starts[b])
        g = h // G
        if (b, g) not in cache:
            cache[(b, g)] = (gather_rows(k_cache, page_table[b], n, g, cfg.page_size),
                             gather_rows(v_cache, page_table[b], n, g, cfg.page_size))
        K, V = cache[(b, g)]
        S = prefill_positions(pos, bool(cfg.head_is_retrieval[h]), cfg.window, cfg.num_sinks)
        out[(r, h)] = attend_set(q[r, h], K, V, S, attn_scale)
    return out
