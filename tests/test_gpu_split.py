"""GPU parity of the split cache layout (through the C ABI): paged caches of the
retrieval KV groups only, plus compacted sink + window caches of the local
groups.

  * local_append: the compacted caches bit-exact against the oracle's
    compaction of the same rows (written in position order, over several
    calls, so the ring wraps);
  * attend_split / select_attend_split: outputs identical to the full layout's
    (same rows, same tiles) and within the output tolerance of the oracle.
"""

import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import assert_out_close, bf16_bits, gpu_sets, make_step, oracle_config, oracle_inputs
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _groups(w):
    G = w.num_q_heads // w.num_kv_heads
    r = [g for g in range(w.num_kv_heads) if any(w.head_is_retrieval[g * G:(g + 1) * G])]
    l = [g for g in range(w.num_kv_heads) if not all(w.head_is_retrieval[g * G:(g + 1) * G])]
    return r, l


def _mixed(name, lens, Hq, Hkv, retr, window, sinks, seed=21, mode="top_p", **kw):
    from workloads.synthetic import _base, _gen, _plant_needles
    w = _base(name, seed, "cuda", lens, Hq, Hkv, 128, retr, window, sinks, mode, permute=True, **kw)
    if mode == "top_p":
        _plant_needles(w, {b: [3] * sum(retr) for b in range(w.batch)}, _gen("cuda", seed, 6))
    return w


# KV groups holding both kinds of heads, and retrieval groups whose rank
# differs from their KV head (ranks 0, 1 <-> KV heads 0, 3)
MIXED = [
    ("two_mixed_groups", [1300, 517], 8, 2, [1, 1, 0, 0, 1, 0, 0, 0], 96, 4),
    ("ranks_differ", [2049, 40, 999], 8, 4, [1, 1, 0, 0, 0, 0, 1, 0], 64, 2),
    ("no_sinks", [800], 8, 2, [1, 0, 0, 0, 1, 1, 0, 0], 128, 0),
    ("sinks_only", [700, 3], 8, 2, [0, 0, 1, 0, 0, 0, 0, 1], 0, 5),
    ("all_local", [900, 1200], 4, 2, [0, 0, 0, 0], 200, 4),
]


def _mixed_case(case):
    name, lens, Hq, Hkv, retr, window, sinks = case
    return _mixed(name, lens, Hq, Hkv, retr, window, sinks)


def _check_compaction(st, w, label):
    """Each (sequence, local group) cache against the oracle's compaction of
    that group's rows 0..N-1, bit for bit."""
    _, loc = _groups(w)
    kb, vb = bf16_bits(w.k_cache), bf16_bits(w.v_cache)
    pt = w.page_table.cpu().numpy()
    lk = st.local_k.cpu().view(torch.int16).numpy().view(np.uint16)
    lv = st.local_v.cpu().view(torch.int16).numpy().view(np.uint16)
    for b, n in enumerate(w.seq_lens.tolist()):
        for li, g in enumerate(loc):
            want_k = O.compact_local_rows(O.gather_rows(kb, pt[b], n, g, 16), w.window, w.num_sinks)
            want_v = O.compact_local_rows(O.gather_rows(vb, pt[b], n, g, 16), w.window, w.num_sinks)
            assert np.array_equal(lk[b, li], want_k), f"{label} K b={b} group={g}"
            assert np.array_equal(lv[b, li], want_v), f"{label} V b={b} group={g}"


def _append_streaming(st, w, chunk):
    """Every position of every sequence, in position order, `chunk` positions
    per sequence per call (interleaved across sequences)."""
    st.local_k, st.local_v = st.sd.local_cache()
    lens = w.seq_lens.tolist()
    dev = w.k_cache.device
    for c0 in range(0, max(lens), chunk):
        seq, pos = [], []
        for b, n in enumerate(lens):
            p = list(range(c0, min(n, c0 + chunk)))
            seq += [b] * len(p)
            pos += p
        if not pos:
            continue
        seq_t = torch.tensor(seq, dtype=torch.int32, device=dev)
        pos_t = torch.tensor(pos, dtype=torch.int32, device=dev)
        page = w.page_table[seq_t.long(), (pos_t // 16).long()].long()
        off = (pos_t % 16).long()
        k_new = w.k_cache[page, :, off].contiguous()
        v_new = w.v_cache[page, :, off].contiguous()
        st.sd.local_append(k_new, v_new, seq_t, pos_t, st.local_k, st.local_v)


@pytest.mark.parametrize("case", MIXED, ids=[c[0] for c in MIXED])
def test_local_append_streaming_matches_oracle_compaction(case):
    w = _mixed_case(case)
    st = make_step(w, build_index=False)
    chunk = max(1, min(w.window, 50)) if w.window else 37
    _append_streaming(st, w, chunk)
    torch.cuda.synchronize()
    assert st.error_word() == 0
    _check_compaction(st, w, case[0])
    st.close()


def test_local_append_prefill_of_the_local_positions_matches_oracle_compaction():
    w = make_workload("llama3_8b_topp", "cuda", B=3, N=5000, permute=True, window=100)
    st = make_step(w, build_index=False)
    st.make_split()
    torch.cuda.synchronize()
    assert st.error_word() == 0
    _check_compaction(st, w, "prefill")
    st.close()


def _split_vs_full(w, label, oracle_seqs=None):
    st = make_step(w)
    st.make_split()
    # separate calls
    st.select(w.q_pre)
    full = st.attend(w.q).clone()
    split = st.attend_split(w.q).clone()
    torch.cuda.synchronize()
    assert st.error_word() == 0
    assert torch.equal(full, split), f"{label}: attend_split differs from attend"
    sets_idx, sets_cnt = st.sel_idx.clone(), st.sel_count.clone()
    # joined calls
    full_j = st.select_attend(w.q_pre, w.q).clone()
    if any(w.head_is_retrieval):                      # without retrieval heads nothing is selected
        st.sel_count.fill_(-7)
    split_j = st.select_attend_split(w.q_pre, w.q).clone()
    torch.cuda.synchronize()
    assert st.error_word() == 0
    assert torch.equal(st.sel_count, sets_cnt), label
    for b in range(w.batch):
        for r in range(st.sel_count.shape[1]):
            n = int(sets_cnt[b, r])
            assert torch.equal(st.sel_idx[b, r, :n], sets_idx[b, r, :n]), f"{label} b={b} row={r}"
    assert torch.equal(full_j, split_j), f"{label}: select_attend_split differs from select_attend"
    # against the oracle over the selected sets
    seqs = list(range(w.batch)) if oracle_seqs is None else list(oracle_seqs)
    retr = [(i, h) for i in range(len(seqs)) for h in range(w.num_q_heads) if w.head_is_retrieval[h]]
    got = gpu_sets(st, w, [(seqs[i], h) for i, h in retr]) if retr else {}
    ref = O.decode_reference(oracle_config(w), **oracle_inputs(w, seqs),
                             sets_override={(i, h): got[(seqs[i], h)] for i, h in retr})
    for (i, h), o in ref.out.items():
        assert_out_close(split_j[seqs[i], h].cpu().numpy(), o, f"{label} oracle b={seqs[i]} h={h}")
    st.close()


@pytest.mark.parametrize("case", MIXED, ids=[c[0] for c in MIXED])
def test_split_layout_equals_full_layout_mixed_groups(case):
    _split_vs_full(_mixed_case(case), case[0])


SPLIT = [
    ("tiny_ref", dict()),
    ("tiny_ref", dict(N=67, permute=True, seed=5)),
    ("llama3_8b_topp", dict(B=3, N=5000, permute=True, window=100)),
    ("llama3_8b_topp", dict(B=40, N=3000, permute=True, window=100)),   # union built in the selection
    ("ragged_paged", dict(B=5, N_min=1, N_max=3000, window=200)),
]


@pytest.mark.parametrize("name,kw", SPLIT, ids=[f"{n}-{i}" for i, (n, _) in enumerate(SPLIT)])
def test_split_layout_equals_full_layout(name, kw):
    w = make_workload(name, "cuda", **kw)
    _split_vs_full(w, f"split {name}{kw}", oracle_seqs=[0, w.batch - 1])


def test_local_append_bad_sequence_or_position_sets_error_word_without_fault():
    from head_wise_sparse_02_b200.sparse_decode import SD_EBIT_SLOT
    w = _mixed_case(MIXED[0])
    st = make_step(w, build_index=False)
    st.local_k, st.local_v = st.sd.local_cache()
    T = 3
    k_new = torch.ones((T, w.num_kv_heads, 128), dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([0, w.batch, 1], dtype=torch.int32, device="cuda")      # w.batch is out of range
    pos = torch.tensor([5, 5, -1], dtype=torch.int32, device="cuda")
    st.sd.local_append(k_new, k_new, seq, pos, st.local_k, st.local_v)
    torch.cuda.synchronize()
    assert st.error_word() & SD_EBIT_SLOT
    # the valid token landed, the others were skipped
    assert float(st.local_k[0, 0, O.local_slot(5, w.window, w.num_sinks)].float().sum()) == 128.0
    assert float(st.local_k[1].float().abs().sum()) == 0.0
    st.close()


def test_split_host_side_argument_errors():
    from head_wise_sparse_02_b200.sparse_decode import SD_ERR_INVALID_ARG, SparseDecodeError
    w = _mixed_case(MIXED[0])
    st = make_step(w)
    st.make_split()
    st.select(w.q_pre)
    with pytest.raises(ValueError):                                  # local caches of the wrong shape
        st.sd.attend_split(w.q, st.k_ret, st.v_ret, st.local_k[:, :1], st.local_v, w.page_table, w.seq_lens,
                           st.sel_idx, st.sel_count, st.out, st.workspace)
    with pytest.raises(SparseDecodeError) as e:                      # local caches missing
        st.sd.attend_split(w.q, st.k_ret, st.v_ret, None, None, w.page_table, w.seq_lens, st.sel_idx,
                           st.sel_count, st.out, st.workspace)
    assert e.value.status == SD_ERR_INVALID_ARG
    flat = torch.empty(st.local_k.numel() + 8, dtype=torch.bfloat16, device="cuda")
    mis = flat[1:1 + st.local_k.numel()].view(st.local_k.shape)   # 2 bytes off a 16-byte boundary
    with pytest.raises(SparseDecodeError) as e:
        st.sd.attend_split(w.q, st.k_ret, st.v_ret, mis, st.local_v, w.page_table, w.seq_lens, st.sel_idx,
                           st.sel_count, st.out, st.workspace)
    assert e.value.status == SD_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert st.error_word() == 0
    st.close()
