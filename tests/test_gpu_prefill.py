"""GPU parity of head-wise prefill (through the C ABI) against the float64
oracle: retrieval heads dense causal, local heads sinks + window ending at
their own position ([RTP] Methodology §1, [AoH] Methodology §4).  Outputs
within the path's output tolerance (2e-3 max-abs, 1e-3 relative L2 per
(query, head)); full chunks and later chunks, ragged and permuted pages,
group shapes, tile edges."""

import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import assert_out_close, oracle_config, oracle_inputs
from workloads import make_workload, prefill_inputs

pytestmark = pytest.mark.gpu


def _ctx(w):
    from head_wise_sparse_02_b200.sparse_decode import SparseDecode
    return SparseDecode(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                        head_is_retrieval=w.head_is_retrieval, num_pages=int(w.k_cache.shape[0]),
                        max_batch=w.batch, max_pages_per_seq=int(w.page_table.shape[1]), proj=w.proj,
                        window=w.window, num_sinks=w.num_sinks, mode=w.mode, top_p=w.top_p, top_k=w.top_k,
                        top_k_frac=w.top_k_frac)


def _run(w, chunk_lens, seed=0, rows=None, label=""):
    sd = _ctx(w)
    q, starts = prefill_inputs(w, chunk_lens, seed=seed)
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    sd.prefill(q, w.k_cache, w.v_cache, w.page_table, w.seq_lens, starts, out)
    torch.cuda.synchronize()
    assert sd.error_word() == 0
    inp = oracle_inputs(w)
    cfg = oracle_config(w)
    qn = q.float().cpu().numpy()
    total = int(starts[-1])
    rows = range(total) if rows is None else rows
    pairs = [(r, h) for r in rows for h in range(w.num_q_heads)]
    ref = O.prefill_reference(cfg, qn, inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"],
                              starts.cpu().numpy(), pairs=pairs)
    got = out.cpu().numpy()
    for (r, h), o in ref.items():
        assert_out_close(got[r, h], o, f"{label} row={r} h={h}")
    sd.close()


@pytest.mark.parametrize("N", [1, 15, 16, 17, 63, 64, 65, 130, 200])
def test_full_prefill_tiny(N):
    w = make_workload("tiny_ref", "cuda", N=N, permute=True, seed=N)
    _run(w, [N], label=f"N={N}")


@pytest.mark.parametrize("N", [1, 17, 64, 65, 128, 129, 200])
def test_full_prefill_d128(N):
    """d = 128 (the tcgen05 kernel) at the edges of its 128-row query tile and
    64-key tile: one retrieval and one local head per KV group, so each CTA
    holds two heads, and a group whose second head slot is empty."""
    from workloads.synthetic import _base
    w = _base("d128", N, "cuda", [N], 6, 2, 128, [1, 0, 0, 1, 1, 0], 40, 3, "top_p", permute=True)
    _run(w, [N], seed=N, label=f"d128 N={N}")


def test_empty_chunk_between_sequences_d128():
    """Three sequences, the middle one with an empty chunk (no query rows): the
    query tiles of the others map to the right sequences and positions."""
    from workloads.synthetic import _base
    w = _base("emptychunk", 8, "cuda", [150, 90, 300], 8, 2, 128, [1, 0, 1, 1, 0, 0, 1, 0], 50, 2, "top_p",
              permute=True)
    _run(w, [150, 0, 130], seed=2, label="empty chunk")


def test_later_chunks_ragged_permuted():
    from workloads.synthetic import _base
    w = _base("chunks", 5, "cuda", [300, 1000, 77], 8, 2, 128, [1, 1, 0, 0, 0, 1, 0, 0], 96, 4, "top_p",
              permute=True)
    _run(w, [100, 33, 77], label="chunks")


@pytest.mark.parametrize("case", [
    ("g16", [700], 32, 2, 128, [1] * 16 + [0] * 16, 200, 4),
    ("d64", [513, 222], 8, 2, 64, [1, 0, 1, 0, 0, 0, 1, 1], 100, 2),
    ("mha", [300], 4, 4, 128, [1, 0, 0, 1], 64, 0),
    ("sinks_only", [260], 4, 2, 128, [0, 0, 1, 0], 0, 5),
    ("window_covers", [180], 4, 2, 128, [0, 0, 1, 1], 4096, 2),
    ("no_local_set", [90], 4, 2, 128, [0, 1, 0, 0], 0, 0),
], ids=lambda c: c[0])
def test_group_shapes(case):
    from workloads.synthetic import _base
    name, lens, Hq, Hkv, d, retr, window, sinks = case
    w = _base(name, 9, "cuda", lens, Hq, Hkv, d, retr, window, sinks, "top_p", permute=True)
    _run(w, lens, seed=3, label=name)


def test_llama3_8b_shapes_sampled_rows():
    """One 4096-token prefill with the llama3_8b_topp head split (8 retrieval
    heads, window 1024 + 4 sinks): sampled query rows, every head."""
    w = make_workload("llama3_8b_topp", "cuda", B=1, N=4096, permute=True)
    rng = np.random.default_rng(1)
    rows = sorted(set(rng.integers(0, 4096, size=24).tolist()) | {0, 1023, 1024, 1025, 4095})
    _run(w, [4096], rows=rows, label="llama3 4096")


def test_prefill_32k_sampled_rows():
    """The bench's prefill at full size (prefill_llama3_8b: one 32768-token
    chunk, 8 retrieval + 24 local heads, window 1024 + 4 sinks, d = 128, the
    tcgen05 kernel), every head of sampled rows: tile edges, the window edge and
    the longest key ranges at the end of the sequence."""
    w = make_workload("llama3_8b_topp", "cuda", B=1, N=32768, permute=True, seed=1)
    rng = np.random.default_rng(7)
    rows = sorted(set(rng.integers(0, 32768, size=10).tolist())
                  | {0, 1, 63, 64, 127, 128, 1023, 1024, 1028, 16383, 32640, 32766, 32767})
    _run(w, [32768], seed=5, rows=rows, label="32K")


@pytest.mark.parametrize("scale", [0.25, 4.0, 48.0])
def test_peaked_and_flat_softmax(scale):
    """Query scales that make the softmax nearly flat (0.25) or sharply peaked
    with row maxima jumping between key tiles (4.0; 48.0: logits spread over
    hundreds of log2 units, so later tiles' weights against the row's first
    reference overflow it, the reference moves and the partial outputs are
    rescaled), 700 positions, ragged pages."""
    from workloads.synthetic import _base
    w = _base("scaled", 12, "cuda", [700, 300], 8, 2, 128, [1, 1, 0, 0, 1, 0, 0, 1], 160, 4, "top_p", permute=True)
    sd = _ctx(w)
    q, starts = prefill_inputs(w, [700, 250], seed=4, scale=scale)
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    sd.prefill(q, w.k_cache, w.v_cache, w.page_table, w.seq_lens, starts, out)
    torch.cuda.synchronize()
    assert sd.error_word() == 0
    inp = oracle_inputs(w)
    ref = O.prefill_reference(oracle_config(w), q.float().cpu().numpy(), inp["k_cache"], inp["v_cache"],
                              inp["page_table"], inp["seq_lens"], starts.cpu().numpy())
    got = out.cpu().numpy()
    for (r, h), o in ref.items():
        assert_out_close(got[r, h], o, f"scale {scale} row={r} h={h}")
    sd.close()


def test_inconsistent_chunk_sets_error_word_without_fault():
    from head_wise_sparse_02_b200.sparse_decode import SD_EBIT_SEQLEN
    w = make_workload("tiny_ref", "cuda", N=100)
    sd = _ctx(w)
    q = torch.zeros((40, w.num_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((40, w.num_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
    starts = torch.tensor([0, 40], dtype=torch.int32, device="cuda")
    bad_lens = torch.tensor([30], dtype=torch.int32, device="cuda")          # chunk longer than the sequence
    sd.prefill(q, w.k_cache, w.v_cache, w.page_table, bad_lens, starts, out)
    torch.cuda.synchronize()
    assert sd.error_word() & SD_EBIT_SEQLEN
    assert float(out.abs().sum()) == 0.0                                     # nothing written
    sd.close()


@pytest.mark.parametrize("d", [64, 128])
def test_bad_page_ids_error_word_without_fault(d):
    """Page-table entries outside the pool (past its end, negative) inside a
    sequence's range: the kernel reads zeros in their place, sets the page
    error bit and leaves every output finite."""
    from head_wise_sparse_02_b200.sparse_decode import SD_EBIT_PAGE
    from workloads.synthetic import _base
    w = _base("badpage", 3, "cuda", [300], 4, 2, d, [1, 0, 0, 1], 64, 2, "top_p", permute=True)
    pt = w.page_table.clone()
    pt[0, 5] = int(w.k_cache.shape[0]) + 7
    pt[0, 9] = -3
    sd = _ctx(w)
    q, starts = prefill_inputs(w, [300], seed=2)
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    sd.prefill(q, w.k_cache, w.v_cache, pt, w.seq_lens, starts, out)
    torch.cuda.synchronize()
    assert sd.error_word() & SD_EBIT_PAGE
    assert bool(torch.isfinite(out).all())
    sd.close()


def test_bounded_wait_runs_out_and_is_reported():
    """A device-side wait that cannot end (the testing switch makes the MMA warp
    of every CTA wait on an mbarrier that nothing arrives at) runs out after its
    bound; the other roles stop, the outputs are zero, the error word reports
    SD_EBIT_TIMEOUT, and the next call on the same context is correct."""
    import time

    from head_wise_sparse_02_b200 import sparse_decode as S
    from workloads.synthetic import _base
    w = _base("stall", 65, "cuda", [65], 6, 2, 128, [1, 0, 0, 1, 1, 0], 40, 3, "top_p", permute=True)
    sd = _ctx(w)
    q, starts = prefill_inputs(w, [65], seed=1)
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    S.sparse_decode_testing_stall_prefill(True)
    try:
        t0 = time.time()
        sd.prefill(q, w.k_cache, w.v_cache, w.page_table, w.seq_lens, starts, out)
        torch.cuda.synchronize()
        took = time.time() - t0
    finally:
        S.sparse_decode_testing_stall_prefill(False)
    assert sd.error_word() & S.SD_EBIT_TIMEOUT
    assert float(out.abs().sum()) == 0.0
    assert took < 60.0
    # the context and the GPU stay usable: the same call again, checked against the oracle
    out.fill_(float("nan"))
    sd.prefill(q, w.k_cache, w.v_cache, w.page_table, w.seq_lens, starts, out)
    torch.cuda.synchronize()
    assert sd.error_word() == 0
    inp = oracle_inputs(w)
    ref = O.prefill_reference(oracle_config(w), q.float().cpu().numpy(), inp["k_cache"], inp["v_cache"],
                              inp["page_table"], inp["seq_lens"], starts.cpu().numpy())
    got = out.cpu().numpy()
    for (r, h), o in ref.items():
        assert_out_close(got[r, h], o, f"after stall row={r} h={h}")
    sd.close()
