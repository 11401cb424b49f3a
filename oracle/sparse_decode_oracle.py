"""Plain float64 CPU definition of head-wise sparse decode attention.

TEST INFRASTRUCTURE ONLY: the oracle that the CUDA library is checked against.
It may be imported only by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py``.  It shares no code with the
CUDA path (no common helpers, tables or constants) and is written for a reader
who checks it against the pages by eye: no blocking, fusion or reordering
beyond what each definition states.

Sources (gist.science summary pages; cited below by the short tag):

[RTP] "Full attention strikes back: moving full attention to sparse attention
      within hundreds of training steps" (RTPurbo), gist.science/ar/paper/2605.16928.
      Methodology §1 head specialisation (retrieval heads vs local heads with a
      sliding window and attention sinks), §2 low-dimensional token indexing
      (an r << d, r = 16, projection of pre-RoPE q and k), §3 dynamic top-p
      (accumulate attention mass in the low-dimensional space until the
      cumulative threshold p) versus fixed top-k.
[ICS] "Inference-time context sparsity: illusion or opportunity?",
      gist.science/ar/paper/2605.24168.  §2 Methodology ("Oracle Top-K": exact
      selection of the k highest tokens), §3a (50x sparsity = ~2% of tokens),
      §3c (sparse decode moves O(N d) memory traffic to O(k d)).
[NHA] "Native Hybrid Attention for Efficient Sequence Modeling",
      gist.science/ar/paper/2510.07019.  §2 unified softmax: one softmax over
      the union of the key sets; §2.3: a window equal to the full sequence is
      full attention.
[AoH] "Autonomy-of-Heads: Data-Free Sparse Attention from Frozen Query-Key
      Geometry", gist.science/ar/paper/2608.06849.  Methodology §4 deployment:
      streaming (local) heads keep a fixed sink prefix plus a recent window.

Readings taken where the pages are silent:
  * one projection P_g of shape [d, r] per KV head g, shared by the keys of
    that head and the queries of its GQA group;
  * the index cache stores k~ = P_g^T k rounded to bf16 (round to nearest
    even, from the exact value);
  * index score s_j = c * <q~, k~_j> with c = index_scale (default sqrt(d)/r);
  * top-p keeps every token whose score ties the threshold score;
  * p and top-k's frac are the float32 values the configuration stores;
  * top-k breaks ties by the lower position;
  * p >= 1 keeps every token;
  * the attention logit scale is attn_scale (default 1/sqrt(d)).

Arrays: caches may be given as float32 arrays holding bf16 values, or as
uint16 arrays holding raw bf16 bit patterns; both are widened exactly to
float64 before any arithmetic.

Parity pins: every function below is pinned by ``tests/test_oracle_pins.py``
against closed forms, brute force or an independent library routine.  The
end-to-end composition (``decode_reference``) is pinned on constructed cases:
the degenerate settings that reduce to dense attention, and planted needles
under a coordinate-selection projection, whose selected set is known by
construction (compared with float64 SDPA over that set).  On general inputs
the composition has no pin beyond those of its parts ("parity unpinned").
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "BF16_MAX",
    "bf16_round",
    "widen",
    "index_keys",
    "query_index",
    "index_scores",
    "exact_scores",
    "select_top_p",
    "stored_top_p",
    "select_top_k",
    "top_k_budget",
    "local_positions",
    "local_slot",
    "compact_local_rows",
    "attend_set",
    "gather_rows",
    "OracleConfig",
    "decode_reference",
    "mass_retained",
]

# Largest finite bfloat16: (2 - 2^-7) * 2^127.
BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


# --------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits and float32's exponent range.  The value
    is rounded once, from the exact float64 input (never through float32),
    as the index-cache reading requires ([RTP] §2 gives the index, the pages
    give no storage precision; bf16 is the reading).  Returns float64 arrays
    holding bf16-representable values; overflow goes to +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0.0)
    xv = x[fin]
    _, e = np.frexp(xv)                      # xv = m * 2**e, 0.5 <= |m| < 1
    # quantum of a bf16 value in [2**(e-1), 2**e) is 2**(e-8); below the
    # smallest normal (2**-126) the subnormal quantum 2**-133 applies.
    q = np.maximum(e - 8, -133)
    r = np.rint(np.ldexp(xv, -q))            # exact scaling, then ties-to-even
    y = np.ldexp(r, q)
    y = np.where(np.abs(y) > BF16_MAX, np.copysign(np.inf, y), y)
    out[fin] = y
    return out


def widen(a) -> np.ndarray:
    """Exact float64 view of bf16 data given as float32 values or uint16 bits."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# --------------------------------------------------------------------------
# Index ([RTP] §2)
# --------------------------------------------------------------------------

def index_keys(proj_g, k_rows) -> np.ndarray:
    """Index entries of keys of one KV head: bf16(P_g^T k) for each row.

    proj_g: [d, r] projection of the KV head (bf16 values).
    k_rows: [n, d] pre-RoPE keys (bf16 values).
    Returns [n, r] float64 holding bf16 values.  [RTP] §2: the r-dim index is
    a projection of the pre-RoPE keys.
    """
    P = widen(proj_g)
    K = widen(k_rows)
    return bf16_round(K @ P)


def query_index(proj_g, q_row) -> np.ndarray:
    """Low-dimensional query q~ = P_g^T q (float64, not rounded).  [RTP] §2."""
    return widen(q_row) @ widen(proj_g)


def index_scores(q_idx, k_idx, index_scale: float) -> np.ndarray:
    """Index scores s_j = c * <q~, k~_j> for every cached token j.  [RTP] §2."""
    return float(index_scale) * (np.asarray(k_idx, np.float64) @ np.asarray(q_idx, np.float64))


def exact_scores(q, K, attn_scale: float) -> np.ndarray:
    """Exact attention logits l_j = attn_scale * <q, k_j> of one query against
    every cached key (post-RoPE q and the cached keys).  [ICS] §2: "Oracle
    Top-K" selects the tokens by these true attention scores instead of an
    approximate index."""
    return float(attn_scale) * (widen(K) @ widen(q))


# --------------------------------------------------------------------------
# Selection ([RTP] §3, [ICS] §2)
# --------------------------------------------------------------------------

def select_top_p(scores, p: float) -> np.ndarray:
    """Dynamic top-p set of one (sequence, head), as ascending positions.

    [RTP] §3: attention mass in the low-dimensional space, softmax over the
    index scores, is accumulated in descending score order until it reaches
    the cumulative threshold p.  The threshold score tau is the score at the
    first position (descending order) where the cumulative mass reaches p;
    every token with score >= tau is kept (ties at tau are all kept).  p >= 1
    keeps every token, as does a cumulative sum that never reaches p through
    rounding.
    """
    s = np.asarray(scores, dtype=np.float64)
    n = s.shape[0]
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    if p >= 1.0:
        return np.arange(n, dtype=np.int64)
    w = np.exp(s - s.max())
    w = w / w.sum()
    order = np.argsort(-s, kind="stable")
    cum = np.cumsum(w[order])
    first = int(np.searchsorted(cum, p, side="left"))   # first cum >= p
    if first >= n:
        return np.arange(n, dtype=np.int64)
    tau = s[order[first]]
    return np.flatnonzero(s >= tau).astype(np.int64)


def stored_top_p(p: float) -> float:
    """The mass p a top-p head must reach, as the float32 value the
    configuration stores (the C interface holds p as a float; [RTP] §3 gives p,
    e.g. 0.9, with no precision).  p and float32(p) differ by up to ~3e-8 of p;
    near p = 1 that can move the threshold by a token whose score lies far
    outside any tolerance band around it."""
    return float(np.float32(p))


def top_k_budget(n: int, top_k: int, top_k_frac: float) -> int:
    """Number of tokens a top-k head keeps for a context of n tokens.

    k = top_k when top_k > 0, else max(1, floor(frac * n)) with frac taken as
    the float32 value the configuration stores ([ICS] §3a: 50x sparsity keeps
    ~2% of tokens); never more than n.
    """
    if top_k > 0:
        k = int(top_k)
    else:
        k = max(1, int(math.floor(float(np.float32(top_k_frac)) * n)))
    return min(k, n)


def select_top_k(scores, k: int) -> np.ndarray:
    """Fixed-budget set: the k highest index scores, ties to the lower
    position, as ascending positions.  [ICS] §2 ("Oracle Top-K" is exact top-k);
    [RTP] §3 (fixed top-k budget)."""
    s = np.asarray(scores, dtype=np.float64)
    n = s.shape[0]
    k = min(int(k), n)
    order = np.lexsort((np.arange(n), -s))   # primary -s, secondary position
    return np.sort(order[:k]).astype(np.int64)


def local_positions(n: int, window: int, num_sinks: int) -> np.ndarray:
    """Positions a local head attends to: sinks [0, n_sink) union the recent
    window [n - w, n), clamped to [0, n).  [RTP] §1 (sliding window plus
    attention sinks), [AoH] §4 (sink prefix plus recent window)."""
    sinks = np.arange(min(num_sinks, n))
    win = np.arange(max(0, n - window), n)
    return np.union1d(sinks, win).astype(np.int64)


def local_slot(pos: int, window: int, num_sinks: int) -> int:
    """Row of position ``pos`` in a compacted local-head cache of
    num_sinks + window rows: a sink keeps its own row, every later position
    cycles through a ring of ``window`` rows; -1 when the position is kept
    nowhere (window 0).  Storage reading: the pages fix only which positions a
    local head attends to ([RTP] §1, [AoH] §4); keeping just those rows is the
    KV saving that [AoH] §4 attributes to streaming heads."""
    if pos < num_sinks:
        return int(pos)
    if window == 0:
        return -1
    return int(num_sinks + pos % window)


def compact_local_rows(rows, window: int, num_sinks: int) -> np.ndarray:
    """Compacted cache of one (sequence, local KV head) after the rows of
    positions 0..n-1 (``rows[j]``, n = len(rows)) were written in position
    order, each to its ``local_slot``; a row never written stays zero.  Keeps
    the dtype of ``rows`` (raw bf16 bit patterns stay bit patterns)."""
    rows = np.asarray(rows)
    out = np.zeros((num_sinks + window,) + rows.shape[1:], dtype=rows.dtype)
    for j in range(rows.shape[0]):
        s = local_slot(j, window, num_sinks)
        if s >= 0:
            out[s] = rows[j]
    return out


# --------------------------------------------------------------------------
# Attention over a set ([ICS] §3c, [NHA] §2)
# --------------------------------------------------------------------------

def attend_set(q, K, V, positions, attn_scale: float) -> np.ndarray:
    """Exact softmax attention of one query over the rows ``positions``.

    logits l_j = attn_scale * <q, k_j>; o = sum_j e^{l_j - max l} v_j /
    sum_j e^{l_j - max l}.  One softmax over the whole set ([NHA] §2); only
    the selected rows are read ([ICS] §3c).  An empty set gives zeros.
    """
    pos = np.asarray(positions, dtype=np.int64)
    d = np.asarray(V).shape[-1]
    if pos.size == 0:
        return np.zeros(d, dtype=np.float64)
    Ks = widen(np.asarray(K)[pos])
    Vs = widen(np.asarray(V)[pos])
    logits = float(attn_scale) * (Ks @ widen(q))
    e = np.exp(logits - logits.max())
    return (e @ Vs) / e.sum()


def gather_rows(cache, page_table_row, n: int, g: int, page_size: int) -> np.ndarray:
    """Rows 0..n-1 of KV head g of one sequence from a paged cache
    [num_pages, Hkv, page_size, width]; position j lives in page
    page_table_row[j // page_size], slot j % page_size.  Returns the raw rows
    (caller widens)."""
    j = np.arange(n)
    pages = np.asarray(page_table_row)[j // page_size]
    return np.asarray(cache)[pages, g, j % page_size]


# --------------------------------------------------------------------------
# Whole decode step
# --------------------------------------------------------------------------

@dataclass
class OracleConfig:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    index_dim: int
    page_size: int
    head_is_retrieval: Sequence[int]
    window: int
    num_sinks: int
    mode: str                      # "top_p" or "top_k"
    top_p: float = 0.9
    top_k: int = 0
    top_k_frac: float = 0.0
    attn_scale: Optional[float] = None
    index_scale: Optional[float] = None
    score: str = "index"           # "index" (r-dim index, [RTP] §2) or "exact" ([ICS] §2)

    def scales(self) -> Tuple[float, float]:
        a = self.attn_scale if self.attn_scale else 1.0 / math.sqrt(self.head_dim)
        c = self.index_scale if self.index_scale else math.sqrt(self.head_dim) / self.index_dim
        return float(a), float(c)


@dataclass
class OracleResult:
    sets: Dict[Tuple[int, int], np.ndarray] = field(default_factory=dict)
    scores: Dict[Tuple[int, int], np.ndarray] = field(default_factory=dict)
    out: Dict[Tuple[int, int], np.ndarray] = field(default_factory=dict)


def decode_reference(cfg: OracleConfig, proj, q_pre, q, k_cache, v_cache,
                     page_table, seq_lens, pairs: Optional[Iterable[Tuple[int, int]]] = None,
                     sets_override: Optional[Dict[Tuple[int, int], np.ndarray]] = None,
                     keep_scores: bool = False) -> OracleResult:
    """One decode step of head-wise sparse attention for the (b, h) pairs asked.

    For a retrieval head ([RTP] §1-§3): build the index of the sequence's keys
    of its KV head, score every cached token, select by top-p or top-k, attend
    exactly over the selected rows.  With cfg.score == "exact" the tokens are
    scored by the exact attention logits instead of the index ([ICS] §2).  For a local head ([RTP] §1, [AoH] §4):
    attend over sinks plus the recent window.  Head h uses KV head
    h // (Hq / Hkv) (GQA).  ``sets_override`` replaces the selection of the
    given retrieval pairs (used to test attention alone).
    """
    Hq, Hkv = cfg.num_q_heads, cfg.num_kv_heads
    G = Hq // Hkv
    attn_scale, index_scale = cfg.scales()
    B = len(seq_lens)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hq)]
    pairs = list(pairs)
    res = OracleResult()
    index_cache: Dict[Tuple[int, int], np.ndarray] = {}
    for b, h in pairs:
        n = int(seq_lens[b])
        g = h // G
        K = gather_rows(k_cache, page_table[b], n, g, cfg.page_size)
        V = gather_rows(v_cache, page_table[b], n, g, cfg.page_size)
        if cfg.head_is_retrieval[h]:
            if sets_override is not None and (b, h) in sets_override:
                S = np.asarray(sets_override[(b, h)], dtype=np.int64)
            else:
                if cfg.score == "exact":
                    s = exact_scores(q[b, h], K, attn_scale)
                else:
                    if (b, g) not in index_cache:
                        index_cache[(b, g)] = index_keys(proj[g], K)
                    qi = query_index(proj[g], q_pre[b, h])
                    s = index_scores(qi, index_cache[(b, g)], index_scale)
                if cfg.mode == "top_p":
                    S = select_top_p(s, stored_top_p(cfg.top_p))
                else:
                    S = select_top_k(s, top_k_budget(n, cfg.top_k, cfg.top_k_frac))
                if keep_scores:
                    res.scores[(b, h)] = s
            res.sets[(b, h)] = S
        else:
            S = local_positions(n, cfg.window, cfg.num_sinks)
        res.out[(b, h)] = attend_set(q[b, h], K, V, S, attn_scale)
    return res


def mass_retained(q, K, positions, attn_scale: float) -> float:
    """Diagnostic: share of the full-attention softmax mass that falls on the
    kept positions ([RTP] results report the retained attention mass)."""
    logits = float(attn_scale) * (widen(K) @ widen(q))
    w = np.exp(logits - logits.max())
    w = w / w.sum()
    return float(w[np.asarray(positions, dtype=np.int64)].sum())
