"""Shared test plumbing: moving a synthetic workload to the oracle's numpy
arrays, running the CUDA path through the C ABI, and the parity comparisons
(set equality with the threshold band, output max-abs and relative L2)."""

from __future__ import annotations

import math
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np
import torch

import oracle as O
from oracle.workload_inputs import bf16_bits, oracle_config, oracle_inputs  # noqa: F401
from workloads import Workload, keys_at, slots_of

# Tolerances stated for the path: sets bit-exact except tokens whose oracle
# score lies within 1e-5 (relative) of the threshold; outputs within 2e-3
# max-abs and 1e-3 relative L2 of the float64 oracle.
BAND_REL = 1e-5
OUT_MAX_ABS = 2e-3
OUT_REL_L2 = 1e-3


def make_step(w: Workload, build_index: bool = True):
    from head_wise_sparse_02_b200.decode import DecodeStep
    st = DecodeStep(k_cache=w.k_cache, v_cache=w.v_cache, page_table=w.page_table,
                    seq_lens=w.seq_lens, proj=w.proj, num_q_heads=w.num_q_heads,
                    head_is_retrieval=w.head_is_retrieval, window=w.window, num_sinks=w.num_sinks,
                    mode=w.mode, top_p=w.top_p, top_k=w.top_k, top_k_frac=w.top_k_frac,
                    attn_scale=w.attn_scale, index_scale=w.index_scale)
    if build_index:
        slots = slots_of(w)
        st.build_index(slots, keys_at(w, slots))
    return st


def retrieval_rows(w: Workload) -> Dict[int, int]:
    """q head -> row of sel_idx (rank among retrieval heads)."""
    rows, r = {}, 0
    for h, x in enumerate(w.head_is_retrieval):
        if x:
            rows[h] = r
            r += 1
    return rows


def gpu_sets(st, w: Workload, pairs: Iterable[Tuple[int, int]]) -> Dict[Tuple[int, int], np.ndarray]:
    rows = retrieval_rows(w)
    cnt = st.sel_count.cpu().numpy()
    out = {}
    sel = st.sel_idx
    for b, h in pairs:
        r = rows[h]
        n = int(cnt[b, r])
        out[(b, h)] = sel[b, r, :n].cpu().numpy().astype(np.int64)
    return out


def compare_set(got: np.ndarray, want: np.ndarray, scores: np.ndarray) -> Tuple[bool, int, str]:
    """Set parity with the threshold band.  Returns (ok, n_band_tokens, msg).

    got must be strictly ascending; every token in the symmetric difference
    must have an oracle score within BAND_REL * max(|tau|, max|s|) of the
    oracle threshold tau (the lowest score in the oracle set)."""
    if got.size > 1 and not np.all(np.diff(got) > 0):
        return False, 0, "positions not strictly ascending"
    if np.array_equal(got, want):
        return True, 0, ""
    diff = np.setxor1d(got, want)
    if want.size == 0:
        return False, diff.size, "oracle set empty but GPU set is not"
    tau = scores[want].min()
    scale = max(abs(tau), np.abs(scores).max())
    dev = np.abs(scores[diff] - tau)
    bad = diff[dev > BAND_REL * scale]
    if bad.size:
        return False, diff.size, (f"{bad.size} tokens outside the band: e.g. pos {bad[:5].tolist()} "
                                  f"score {scores[bad[:5]].tolist()} tau {tau} |S| gpu {got.size} oracle {want.size}")
    return True, diff.size, ""


def compare_out(got: np.ndarray, want: np.ndarray) -> Tuple[float, float]:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    max_abs = float(np.abs(got - want).max()) if got.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(got - want) / den) if den > 0 else float(np.linalg.norm(got - want))
    return max_abs, rel


def assert_out_close(got, want, what=""):
    max_abs, rel = compare_out(got, want)
    assert max_abs <= OUT_MAX_ABS and rel <= OUT_REL_L2, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"
