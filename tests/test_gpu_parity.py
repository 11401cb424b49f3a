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


def check_workload(w, seqs=None, heads=None, label="", score="index"):
    """Run select + attend on the GPU and compare with the oracle on the given
    sequences / heads.  Returns the number of band tokens reported.  With
    score="exact" the sets come from the exact attention logits on both sides."""
    st = make_step(w)
    if score == "exact":
        st.select_exact(w.q)
    else:
        st.select(w.q_pre)
    out_e2e = st.attend(w.q).clone()
    torch.cuda.synchronize()
    assert st.error_word() == 0
    seqs = list(range(w.batch)) if seqs is None else list(seqs)
    cfg = oracle_config(w)
    cfg.score = score
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
    # a set that differs from the oracle's only inside the threshold band is
    # a correct set: the end-to-end output is then judged against the oracle's
    # attention over that same set
    e2e_ref = dict(ref.out)
    differ = {(i, h): np.asarray(got_sets[(seqs[i], h)]) for (i, h) in retr
              if not np.array_equal(got_sets[(seqs[i], h)], ref.sets[(i, h)])}
    if differ:
        alt = O.decode_reference(cfg, **inp, pairs=list(differ), sets_override=differ)
        e2e_ref.update(alt.out)
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
        assert_out_close(out_e2e[b, h].cpu().numpy(), e2e_ref[(i, h)], f"{label} e2e b={b} h={h}")
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


# ------------------------------------------------------------------ group shapes

# GQA group sizes and head dims beyond the named workloads: 16 heads per group
# (all 16 rows of the attention MMA), 8 per group in top-k, MHA (1 per group),
# d = 64 in top-k; ragged lengths, permuted pages
SHAPES = [
    ("g16_topk", [3001, 2500], 32, 2, 128, [1] * 32, 0, 0, "top_k", dict(top_k_frac=0.05)),
    ("g16_mixed_topp", [2900, 1700], 32, 2, 128, [1] * 16 + [0] * 16, 300, 4, "top_p", dict(top_p=0.9)),
    ("g8_topk", [4100, 777], 32, 4, 128, [1] * 32, 0, 0, "top_k", dict(top_k=100)),
    ("d64_topk", [2000, 3333], 8, 2, 64, [1] * 8, 0, 0, "top_k", dict(top_k_frac=0.03)),
    ("mha_mixed_topp", [1500, 2222], 8, 8, 128, [1, 0] * 4, 200, 2, "top_p", dict(top_p=0.8)),
]


@pytest.mark.parametrize("case", SHAPES, ids=[c[0] for c in SHAPES])
def test_group_shapes(case):
    from workloads.synthetic import _base, _gen, _plant_needles
    name, lens, Hq, Hkv, d, retr, window, sinks, mode, kw = case
    w = _base(name, 11, "cuda", lens, Hq, Hkv, d, retr, window, sinks, mode, permute=True, **kw)
    if mode == "top_p":
        _plant_needles(w, {b: [3] * sum(retr) for b in range(w.batch)}, _gen("cuda", 11, 6))
    check_workload(w, label=name)


# ------------------------------------------------------------------ top-k fallback

def _group_query_keys(w, b, n, gain, noise, seed):
    """[Hkv, n, d] bf16 keys along the mean pre-RoPE query of each GQA group
    (times `gain`) plus N(0, noise^2) noise: their index scores sit far above
    those of N(0, 1) keys."""
    G = w.num_q_heads // w.num_kv_heads
    qm = w.q_pre[b].float().view(w.num_kv_heads, G, w.head_dim).mean(1)
    qm = qm / qm.norm(dim=-1, keepdim=True) * math.sqrt(w.head_dim)
    gen = torch.Generator(device=w.k_cache.device)
    gen.manual_seed(seed)
    eps = torch.randn((w.num_kv_heads, n, w.head_dim), generator=gen, device=w.k_cache.device)
    return (gain * qm[:, None, :] + noise * eps).to(torch.bfloat16)


def _set_keys(w, b, positions, keys):
    """k_cache rows of sequence b at `positions` (all KV heads) := keys [Hkv, n, d]."""
    pos = torch.as_tensor(positions, device=w.page_table.device, dtype=torch.long)
    pages = w.page_table[b, pos // w.page_size].long()
    slots = pos % w.page_size
    for g in range(w.num_kv_heads):
        w.k_cache[pages, g, slots] = keys[g]


def _exact_sets(w, seqs, label):
    """Sets must equal the oracle's exactly (ties go to the lower position on
    both sides); outputs are checked by check_workload."""
    st = make_step(w)
    st.select(w.q_pre)
    torch.cuda.synchronize()
    assert st.error_word() == 0
    ref = O.decode_reference(oracle_config(w), **oracle_inputs(w, seqs),
                             pairs=_pairs(w, range(len(seqs))), keep_scores=True)
    retr = [h for h in range(w.num_q_heads) if w.head_is_retrieval[h]]
    got = gpu_sets(st, w, [(b, h) for b in seqs for h in retr])
    for i, b in enumerate(seqs):
        for h in retr:
            assert np.array_equal(got[(b, h)], np.asarray(ref.sets[(i, h)])), f"{label} b={b} h={h}"
    st.close()
    return ref


def test_topk_sample_overestimate_falls_back_to_exact():
    """High-scoring keys on every 8th page, the stride at which the score
    window samples a 2048-page context: the sample then puts the window above
    the k-th score, the streaming pass cannot resolve the budget, and the
    exact selector must produce the same sets."""
    w = make_workload("topk_128k", "cuda", B=2, N=32768)
    for b in range(w.batch):
        pos = [p * 16 + s for p in range(0, 2048, 8) for s in range(16)]
        _set_keys(w, b, pos, _group_query_keys(w, b, len(pos), 2.0, 0.5, 100 + b))
    ref = _exact_sets(w, [0, 1], "planted sample pages")
    # the construction: for many heads every selected token is a planted one
    # (keys follow the group's mean query, which some heads barely share), so
    # several groups take the exact path
    planted = set(p * 16 + s for p in range(0, 2048, 8) for s in range(16))
    inside = [set(int(x) for x in sset) <= planted for (i, h), sset in ref.sets.items()
              if w.head_is_retrieval[h]]
    assert sum(inside) * 4 >= len(inside)
    check_workload(w, seqs=[0, 1], heads=[0, 5, 31], label="planted sample pages")


def test_topk_heavy_ties_fall_back_to_exact():
    """Keys drawn from 6 distinct vectors besides 400 distinct high-scoring
    ones: the k-th score is shared by thousands of tokens, more than the
    streaming pass ranks exactly, so the exact selector takes over and must
    break the ties by position like the definition does."""
    w = make_workload("topk_128k", "cuda", B=1, N=40000)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    base = torch.randn((w.num_kv_heads, 6, w.head_dim), generator=gen, device="cuda").to(torch.bfloat16)
    pick = torch.randint(0, 6, (40000,), generator=gen, device="cuda")
    _set_keys(w, 0, list(range(40000)), base[:, pick])
    high = torch.randperm(40000, generator=gen, device="cuda")[:400].sort().values.cpu().tolist()
    _set_keys(w, 0, high, _group_query_keys(w, 0, 400, 2.0, 0.5, 11))
    ref = _exact_sets(w, [0], "heavy ties")
    for (i, h), sset in ref.sets.items():
        if w.head_is_retrieval[h]:
            assert len(sset) == math.floor(float(np.float32(0.02)) * 40000)   # 799
    check_workload(w, seqs=[0], heads=[0, 13, 31], label="heavy ties")


# ------------------------------------------------------------------ top-p fallback

@pytest.mark.parametrize("N", [20000, 40000])
def test_topp_heavy_ties(N):
    """Keys drawn from 6 distinct vectors: every head's index scores take 6
    values, each shared by N / 6 tokens, and the top-p threshold is one of
    them, so every token tied at it must be kept.  With N = 20000 the bin
    holding the threshold has about 3300 candidates and the streaming resolve
    takes them; with N = 40000 about 6700, more than it takes, and the exact
    selector must produce the sets."""
    w = make_workload("llama3_8b_topp", "cuda", B=1, N=N)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(8)
    base = torch.randn((w.num_kv_heads, 6, w.head_dim), generator=gen, device="cuda").to(torch.bfloat16)
    pick = torch.randint(0, 6, (N,), generator=gen, device="cuda")
    _set_keys(w, 0, list(range(N)), base[:, pick])
    check_workload(w, seqs=[0], label=f"top-p heavy ties N={N}")


def test_topp_weight_beyond_float_range_falls_back_to_exact():
    """One key per KV group along the group's mean query, 30 times its norm,
    on a page the score window does not sample (it takes pages 0, 8, 16, ...
    of 2048): for most heads its index score lies more than 80 above the
    sample maximum, beyond the range the mass pass takes weights in, so
    the mass pass flags the item and the exact selector (weights relative to
    the true maximum) produces the set, that single token."""
    w = make_workload("llama3_8b_topp", "cuda", B=1, N=32768)
    pos = [5 * 16 + 3]
    _set_keys(w, 0, pos, _group_query_keys(w, 0, 1, 30.0, 0.0, 3))
    ref = O.decode_reference(oracle_config(w), **oracle_inputs(w, [0]), pairs=_pairs(w, [0]), keep_scores=True)
    # the construction: for many heads the set is the planted token alone
    # and its score stands more than 80 above every other
    alone = 0
    for (i, h), sset in ref.sets.items():
        if w.head_is_retrieval[h]:
            sc = np.asarray(ref.scores[(i, h)])
            rest = np.delete(sc, pos[0])
            alone += list(sset) == pos and sc[pos[0]] - rest.max() > 80.0
    assert alone * 4 >= sum(w.head_is_retrieval)
    check_workload(w, seqs=[0], label="weight beyond float range")


def test_topp_threshold_below_window_falls_back_to_exact():
    """Keys of the sampled pages (0, 8, 16, ... of 2048) along the group's
    mean query at full norm, keys of all other pages at 0.8 of it: for heads
    aligned with that query the sample sees only the higher scores, the
    window starts near them, yet most of the softmax mass lies on the lower
    unsampled keys, so the threshold falls below the window, the mass pass
    cannot resolve it and the exact selector must produce the sets."""
    w = make_workload("llama3_8b_topp", "cuda", B=1, N=32768)
    sampled = [p * 16 + s for p in range(0, 2048, 8) for s in range(16)]
    others = [p * 16 + s for p in range(2048) if p % 8 for s in range(16)]
    _set_keys(w, 0, sampled, _group_query_keys(w, 0, len(sampled), 1.0, 0.05, 21))
    _set_keys(w, 0, others, _group_query_keys(w, 0, len(others), 0.8, 0.05, 22))
    ref = O.decode_reference(oracle_config(w), **oracle_inputs(w, [0]), pairs=_pairs(w, [0]), keep_scores=True)
    # the construction: for many heads the threshold lies below every
    # sampled score
    below = 0
    for (i, h), sset in ref.sets.items():
        if w.head_is_retrieval[h]:
            sc = np.asarray(ref.scores[(i, h)])
            below += sc[np.asarray(sset)].min() < sc[sampled].min()
    assert below * 4 >= sum(w.head_is_retrieval)
    check_workload(w, seqs=[0], label="threshold below window")


# ------------------------------------------------------------------ full sizes

def _spread(lens, n_seq=8):
    """n_seq sequences spread over the length range: the shortest, the
    longest and the ones between them at evenly spaced length ranks."""
    order = sorted(range(len(lens)), key=lambda b: lens[b])
    return sorted({order[round(i * (len(lens) - 1) / (n_seq - 1))] for i in range(n_seq)})


# Full-size workloads in the bench's launch configuration.  Every retrieval
# head of the listed sequences is compared (sets and outputs), plus the first
# and last local head; the long-context Zipf workload is run at every point of
# its top-p x alpha sweep.
FULL = [
    ("llama3_8b_topp", dict(), [0, 1, 2, 3]),
    ("topk_128k", dict(), [0, 9, 15]),
] + [("long_zipf", dict(top_p=p, alpha=a), [0]) for p in (0.5, 0.9, 0.99) for a in (0.8, 1.2)] + [
    ("ragged_paged", dict(), "spread"),
]


@pytest.mark.parametrize("name,kw,seqs", FULL, ids=[f"{n}-{i}" for i, (n, _, _) in enumerate(FULL)])
def test_full_size_all_retrieval_heads(name, kw, seqs):
    w = make_workload(name, "cuda", **kw)
    if seqs == "spread":
        lens = w.seq_lens.cpu().tolist()
        seqs = _spread(lens)
        picked = [lens[b] for b in seqs]
        assert len(seqs) == 8 and min(picked) == min(lens) and max(picked) == max(lens)
    retr = [h for h in range(w.num_q_heads) if w.head_is_retrieval[h]]
    loc = [h for h in range(w.num_q_heads) if not w.head_is_retrieval[h]]
    heads = sorted(set(retr + loc[:1] + loc[-1:]))
    band = check_workload(w, seqs=seqs, heads=heads, label=f"{name}{kw}")
    print(f"{name} {kw} seqs {seqs}: {len(retr) * len(seqs)} retrieval sets compared, "
          f"{band} tokens inside the threshold band")
    del w
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ exact-score selection

EXACT = [
    ("tiny_ref", dict()),
    ("tiny_ref", dict(N=69, permute=True, seed=4)),
    ("llama3_8b_topp", dict(B=2, N=3001, window=256)),
    ("topk_128k", dict(B=2, N=8192, permute=True)),
    ("topk_128k", dict(B=1, N=4100, top_k=5)),
    ("long_zipf", dict(N=20000, top_p=0.9, alpha=1.2)),
    ("ragged_paged", dict(B=4, N_min=300, N_max=5000, window=200)),
]


@pytest.mark.parametrize("name,kw", EXACT, ids=[f"{n}-{i}" for i, (n, _) in enumerate(EXACT)])
def test_exact_score_selection(name, kw):
    """Sets chosen by the exact attention logits (the reference selector of
    the ICS page) against the oracle in exact-score mode, then attention over
    them, for top-p and top-k workloads, ragged and permuted."""
    w = make_workload(name, "cuda", **kw)
    check_workload(w, label=f"exact {name}{kw}", score="exact")


def test_exact_score_selection_d64_and_group16():
    from workloads.synthetic import _base
    w = _base("d64_topk", 12, "cuda", [2000, 3333], 8, 2, 64, [1] * 8, 0, 0, "top_k", permute=True,
              top_k_frac=0.03)
    check_workload(w, label="exact d64", score="exact")
    w = _base("g16_topp", 13, "cuda", [2900, 1700], 32, 2, 128, [1] * 16 + [0] * 16, 300, 4, "top_p",
              permute=True, top_p=0.9)
    check_workload(w, label="exact g16", score="exact")


def test_exact_score_selection_full_size_128k():
    """The 128K fixed-budget workload in exact-score mode, in the launch
    configuration the bench times, on three sequences' heads."""
    w = make_workload("topk_128k", "cuda")
    check_workload(w, seqs=[0, 15], heads=list(range(0, 32, 3)), label="exact topk_128k", score="exact")
    del w
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ joined select + attend

# The joined call builds the union lists in the selection when the items
# ((sequence, retrieval group) pairs) fill at least half the GPU: the cases
# with 80 or more items take that path, the small ones the separate one.
JOINED = [
    ("tiny_ref", dict()),
    ("tiny_ref", dict(N=1)),
    ("tiny_ref", dict(N=67, permute=True, seed=5)),
    ("llama3_8b_topp", dict(B=3, N=5000, permute=True, window=100, sinks=0)),
    ("llama3_8b_topp", dict(B=40, N=3000, permute=True, window=100)),
    ("topk_128k", dict(B=2, N=8192, permute=True)),
    ("topk_128k", dict(B=10, N=8192, permute=True)),
    ("topk_128k", dict(B=10, N=3001, top_k_frac=0.3)),
    ("long_zipf", dict(N=20000, top_p=0.99, alpha=0.8, window=333)),
    ("ragged_paged", dict(B=5, N_min=300, N_max=3000, window=200)),
    ("ragged_paged", dict(B=40, N_min=1, N_max=4000, window=200)),
]


def _joined_vs_separate(w, label, oracle_seqs=None):
    """The joined call against select then attend: identical sets, outputs
    within the output tolerance of each other, and against the oracle over
    the selected sets."""
    st = make_step(w)
    st.select(w.q_pre)
    ref_out = st.attend(w.q).clone()
    ref_idx, ref_cnt = st.sel_idx.clone(), st.sel_count.clone()
    torch.cuda.synchronize()
    assert st.error_word() == 0
    st.sel_idx.fill_(-7)
    st.sel_count.fill_(-7)
    st.out.fill_(float("nan"))
    out = st.select_attend(w.q_pre, w.q).clone()
    torch.cuda.synchronize()
    assert st.error_word() == 0
    assert torch.equal(st.sel_count, ref_cnt), label
    for b in range(w.batch):
        for r in range(st.sel_count.shape[1]):
            n = int(ref_cnt[b, r])
            assert torch.equal(st.sel_idx[b, r, :n], ref_idx[b, r, :n]), f"{label} b={b} row={r}"
    # the same sets; the outputs are held to the output tolerance of each
    # other (they come out bit-identical today: same union lists, same tiles)
    got_o, ref_o = out.cpu().numpy(), ref_out.cpu().numpy()
    for b in range(w.batch):
        for h in range(w.num_q_heads):
            assert_out_close(got_o[b, h], ref_o[b, h], f"{label} joined vs separate b={b} h={h}")
    seqs = list(range(w.batch)) if oracle_seqs is None else list(oracle_seqs)
    retr = [(i, h) for i in range(len(seqs)) for h in range(w.num_q_heads) if w.head_is_retrieval[h]]
    got = gpu_sets(st, w, [(seqs[i], h) for i, h in retr])
    ref = O.decode_reference(oracle_config(w), **oracle_inputs(w, seqs),
                             sets_override={(i, h): got[(seqs[i], h)] for i, h in retr})
    for (i, h), o in ref.out.items():
        assert_out_close(out[seqs[i], h].cpu().numpy(), o, f"{label} oracle b={seqs[i]} h={h}")
    st.close()


@pytest.mark.parametrize("name,kw", JOINED, ids=[f"{n}-{i}" for i, (n, _) in enumerate(JOINED)])
def test_select_attend_joined(name, kw):
    w = make_workload(name, "cuda", **kw)
    _joined_vs_separate(w, f"joined {name}{kw}")


@pytest.mark.parametrize("case", SHAPES, ids=[c[0] for c in SHAPES])
def test_select_attend_joined_group_shapes(case):
    """Group shapes where the joined call builds the union in the selection
    (1, 2 and 4 retrieval heads per group) and where it falls back (8, 16)."""
    from workloads.synthetic import _base, _gen, _plant_needles
    name, lens, Hq, Hkv, d, retr, window, sinks, mode, kw = case
    w = _base(name, 11, "cuda", lens, Hq, Hkv, d, retr, window, sinks, mode, permute=True, **kw)
    if mode == "top_p":
        _plant_needles(w, {b: [3] * sum(retr) for b in range(w.batch)}, _gen("cuda", 11, 6))
    _joined_vs_separate(w, f"joined {name}")


def test_select_attend_joined_with_exact_fallback():
    """Planted keys on the sampled pages make the window miss for many groups
    (the construction of test_topk_sample_overestimate_falls_back_to_exact):
    those items are redone by the exact selector and planned by attend, the
    others come with their union lists from the selection."""
    w = make_workload("topk_128k", "cuda", B=10, N=32768)
    for b in range(w.batch):
        pos = [p * 16 + s for p in range(0, 2048, 8) for s in range(16)]
        _set_keys(w, b, pos, _group_query_keys(w, b, len(pos), 2.0, 0.5, 100 + b))
    _joined_vs_separate(w, "joined with fallback", oracle_seqs=[0, 5, 9])


def test_select_attend_joined_full_size_128k():
    w = make_workload("topk_128k", "cuda", B=10)
    _joined_vs_separate(w, "joined topk_128k B=10", oracle_seqs=[0, 9])
    del w
    torch.cuda.empty_cache()
