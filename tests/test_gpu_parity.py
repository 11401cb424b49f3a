"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle.

Stage-wise:
  * index_keys: bf16 index entries bit-exact against the oracle's;
  * select:     sets equal to the oracle's except tokens whose oracle score is
                within 1e-5 (relative) of the threshold;
  * attend:     fed the oracle's own sets, outputs within 2e-3 max-abs and
                1e-3 relative L2;
  * end to end: select + attend against the oracle's outputs.
Small cases span several tiles and ragged tails; full-size workloads are
checked on sampled (sequence, head) pairs in the launch configuration the
bench times.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import (assert_out_close, bf16_bits, compare_set, gpu_sets, make_step,
                           oracle_config, oracle_inputs)
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _pairs(w, seqs, heads=None):
    heads = range(w.num_q_heads) if heads is None else heads
    return [(b, h) for b in seqs for h in heads]


def check_workload(w, seqs=None, heads=None, label=""):
    """Run select + attend on the GPU and compare with the oracle on the given
    sequences / heads.  Returns the number of band tokens reported."""
    st = make_step(w)
    st.select(w.q_pre)
    out_e2e = st.attend(w.q).clone()
    torch.cuda.synchronize()
    assert st.error_word() == 0
    seqs = list(range(w.batch)) if seqs is None else list(seqs)
    cfg = oracle_config(w)
    inp = oracle_inputs(w, seqs)
    local_pairs = _pairs(w, range(len(seqs)), heads)
    ref = O.decode_reference(cfg, **inp, pairs=local_pairs, keep_scores=True)
    retr = [(i, h) for (i, h) in local_pairs if w.head_is_retrieval[h]]
    got_sets = gpu_sets(st, w, [(seqs[i], h) for (i, h) in retr])
    band = 0
    for (i, h) in retr:
        ok, nb, msg = compare_set(got_sets[(seqs[i], h)], ref.sets[(i, h)], ref.scores[(i, h)])
        assert ok, f"{label} set b={seqs[i]} h={h}: {msg}"
        band += nb
    # attend alone, on the oracle's sets
    if retr:
        sel = torch.zeros_like(st.sel_idx)
        cnt = torch.zeros_like(st.sel_count)
        rows = {h: r for r, h in enumerate([h for h in range(w.num_q_heads) if w.head_is_retrieval[h]])}
        for (i, h) in retr:
            s = torch.tensor(ref.sets[(i, h)], dtype=torch.int32)
            sel[seqs[i], rows[h], :s.numel()] = s.to(sel.device)
            cnt[seqs[i], rows[h]] = s.numel()
        out_att = st.attend(w.q, sel_idx=sel, sel_count=cnt).clone()
    else:
        out_att = out_e2e
    torch.cuda.synchronize()
    assert st.error_word() == 0
    for (i, h) in local_pairs:
        b = seqs[i]
        assert_out_close(out_att[b, h].cpu().numpy(), ref.out[(i, h)], f"{label} attend b={b} h={h}")
        assert_out_close(out_e2e[b, h].cpu().numpy(), ref.out[(i, h)], f"{label} e2e b={b} h={h}")
    st.close()
    return band


# ------------------------------------------------------------------ index keys

@pytest.mark.parametrize("name,kw", [
    ("tiny_ref", dict()),
    ("llama3_8b_topp", dict(B=2, N=3000)),
    ("long_zipf", dict(N=5000)),
])
def test_index_keys_bit_exact(name, kw):
    w = make_workload(name, "cuda", **kw)
    st = make_step(w)
    torch.cuda.synchronize()
    assert st.error_word() == 0
    inp = oracle_inputs(w)
    idx = bf16_bits(st.index_cache)
    pt = w.page_table.cpu().numpy()
    for b in range(w.batch):
        n = int(w.seq_lens[b])
        for g in range(w.num_kv_heads):
            K = O.gather_rows(inp["k_cache"], inp["page_table"][b], n, g, 16)
            want = O.index_keys(inp["proj"][g], K)
            got = O.widen(O.gather_rows(idx, pt[b], n, g, 16))
            mism = int((got != want).sum())
            assert mism == 0, f"b={b} g={g}: {mism} index entries differ"
    st.close()


# ------------------------------------------------------------------ small cases

SMALL = [
    ("tiny_ref", dict()),
    ("tiny_ref", dict(permute=True, seed=5)),
    ("tiny_ref", dict(N=1)),
    ("tiny_ref", dict(N=15)),
    ("tiny_ref", dict(N=16)),
    ("tiny_ref", dict(N=17)),
    ("tiny_ref", dict(N=63)),
    ("tiny_ref", dict(N=64)),
    ("tiny_ref", dict(N=67)),
    ("tiny_ref", dict(N=68)),
    ("tiny_ref", dict(N=69)),
    ("tiny_ref", dict(N=100, needles=0)),
    ("tiny_ref", dict(N=2000, needles=1, seed=3)),
    ("llama3_8b_topp", dict(B=2, N=3000, window=256)),
    ("llama3_8b_topp", dict(B=3, N=5000, permute=True, window=100, sinks=0)),
    ("topk_128k", dict(B=2, N=8192, permute=True)),
    ("topk_128k", dict(B=1, N=4100, top_k=5)),
    ("topk_128k", dict(B=2, N=3001, top_k_frac=0.3)),
    ("long_zipf", dict(N=20000, top_p=0.5, alpha=1.2)),
    ("long_zipf", dict(N=20000, top_p=0.99, alpha=0.8, window=333)),
    ("ragged_paged", dict(B=5, N_min=300, N_max=3000, window=200)),
]


@pytest.mark.parametrize("name,kw", SMALL, ids=[f"{n}-{i}" for i, (n, _) in enumerate(SMALL)])
def test_small_parity(name, kw):
    w = make_workload(name, "cuda", **kw)
    check_workload(w, label=f"{name}{kw}")


def test_top_p_one_is_dense_attention():
    w = make_workload("tiny_ref", "cuda", N=700)
    w.top_p = 1.0
    st = make_step(w)
    st.select(w.q_pre)
    out = st.attend(w.q).cpu().numpy()
    assert st.error_word() == 0
    cnt = st.sel_count.cpu().numpy()
    assert (cnt == 700).all()
    inp = oracle_inputs(w)
    for h in (0, 1):
        K = O.widen(O.gather_rows(inp["k_cache"], inp["page_table"][0], 700, 0, 16))
        V = O.widen(O.gather_rows(inp["v_cache"], inp["page_table"][0], 700, 0, 16))
        qt = torch.tensor(inp["q"][0, h], dtype=torch.float64)[None, None, None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, torch.tensor(K)[None, None], torch.tensor(V)[None, None], scale=1 / 8)[0, 0, 0].numpy()
        assert_out_close(out[0, h], ref, f"dense h={h}")
    st.close()


def test_empty_sequence_gives_empty_sets_and_zero_output():
    w = make_workload("llama3_8b_topp", "cuda", B=3, N=600, window=64)
    w.seq_lens[1] = 0
    st = make_step(w, build_index=False)
    from workloads import keys_at, slots_of
    slots = slots_of(w)
    st.build_index(slots, keys_at(w, slots))
    st.select(w.q_pre)
    out = st.attend(w.q)
    torch.cuda.synchronize()
    assert st.error_word() == 0
    assert (st.sel_count[1] == 0).all()
    assert (out[1] == 0).all()
    check = check_workload(w, seqs=[0, 2], label="with empty")
    assert check >= 0


def test_bad_page_id_sets_error_word_without_fault():
    w = make_workload("tiny_ref", "cuda")
    st = make_step(w)
    st.page_table = w.page_table.clone()
    st.page_table[0, 3] = w.num_pages + 7       # out of the pool: kernels must skip it
    st.select(w.q_pre)
    st.attend(w.q)
    from head_wise_sparse_02_b200.sparse_decode import SD_EBIT_PAGE
    word = st.error_word()
    assert word & SD_EBIT_PAGE
    assert st.error_word() == 0                  # reading clears it
    st.close()


def test_host_side_argument_errors():
    from head_wise_sparse_02_b200.sparse_decode import SD_ERR_WORKSPACE, SparseDecodeError
    w = make_workload("tiny_ref", "cuda")
    st = make_step(w)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(SparseDecodeError) as e:
        st.sd.select(w.q_pre, st.index_cache, w.page_table, w.seq_lens, st.sel_idx, st.sel_count, small)
    assert e.value.status == SD_ERR_WORKSPACE
    with pytest.raises(TypeError):
        st.sd.select(w.q_pre.float(), st.index_cache, w.page_table, w.seq_lens, st.sel_idx,
                     st.sel_count, st.workspace)
    st.close()


# ------------------------------------------------------------------ full sizes

FULL = [
    ("llama3_8b_topp", dict(), [0, 3]),
    ("topk_128k", dict(), [0, 9, 15]),
    ("long_zipf", dict(top_p=0.9, alpha=1.2), [0]),
    ("long_zipf", dict(top_p=0.99, alpha=0.8), [0]),
    ("ragged_paged", dict(), [0, 17, 63]),
]


@pytest.mark.parametrize("name,kw,seqs", FULL, ids=[f"{n}-{i}" for i, (n, _, _) in enumerate(FULL)])
def test_full_size_sampled(name, kw, seqs):
    w = make_workload(name, "cuda", **kw)
    G = w.num_q_heads // w.num_kv_heads
    # every retrieval head of two groups plus two local heads per sampled sequence
    retr = [h for h in range(w.num_q_heads) if w.head_is_retrieval[h]]
    loc = [h for h in range(w.num_q_heads) if not w.head_is_retrieval[h]]
    heads = sorted(set(retr[:G] + retr[-G:] + loc[:1] + loc[-1:]))
    check_workload(w, seqs=seqs, heads=heads, label=name)
    del w
    torch.cuda.empty_cache()
