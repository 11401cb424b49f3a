"""The seeded synthetic workloads have the shapes, roles and planted structure
their recipes state (CPU, shrunken sizes).  Every parity case and the bench
draw their inputs here, so the recipe is checked on its own."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from workloads import make_workload
from workloads.synthetic import WORKLOAD_NAMES

SMALL = {
    "tiny_ref": dict(N=300),
    "llama3_8b_topp": dict(B=2, N=2000),
    "topk_128k": dict(B=1, N=2048),
    "long_zipf": dict(N=4096),
    "ragged_paged": dict(B=5, N_min=300, N_max=3000),
}

# (Hq, Hkv, d, retrieval heads, window, sinks, mode)
RECIPE = {
    "tiny_ref": (4, 2, 64, range(0, 2), 64, 4, "top_p"),
    "llama3_8b_topp": (32, 8, 128, range(0, 8), 1024, 4, "top_p"),
    "topk_128k": (32, 8, 128, range(0, 32), 0, 0, "top_k"),
    "long_zipf": (64, 8, 128, range(0, 16), 4096, 4, "top_p"),
    "ragged_paged": (32, 8, 128, range(0, 8), 2048, 4, "top_p"),
}


@pytest.mark.parametrize("name", WORKLOAD_NAMES)
def test_shapes_roles_and_determinism(name):
    w = make_workload(name, "cpu", **SMALL[name])
    Hq, Hkv, d, retr, window, sinks, mode = RECIPE[name]
    assert (w.num_q_heads, w.num_kv_heads, w.head_dim) == (Hq, Hkv, d)
    assert [h for h in range(Hq) if w.head_is_retrieval[h]] == list(retr)
    assert (w.window, w.num_sinks, w.mode) == (window, sinks, mode)
    B = w.batch
    assert tuple(w.q.shape) == (B, Hq, d) and w.q.dtype == torch.bfloat16
    assert tuple(w.proj.shape) == (Hkv, d, 16) and w.proj.dtype == torch.bfloat16
    assert tuple(w.k_cache.shape[1:]) == (Hkv, 16, d) and w.k_cache.shape == w.v_cache.shape
    again = make_workload(name, "cpu", **SMALL[name])
    for a, b in [(w.k_cache, again.k_cache), (w.v_cache, again.v_cache), (w.q, again.q), (w.proj, again.proj),
                 (w.page_table, again.page_table), (w.seq_lens, again.seq_lens)]:
        assert torch.equal(a, b)


@pytest.mark.parametrize("name,kw", [("ragged_paged", dict(B=6, N_min=300, N_max=3000)),
                                     ("tiny_ref", dict(N=300, permute=True)),
                                     ("llama3_8b_topp", dict(B=2, N=2000))])
def test_page_tables_give_each_sequence_its_own_pages(name, kw):
    w = make_workload(name, "cpu", **kw)
    pt = w.page_table.numpy()
    used = []
    for b in range(w.batch):
        m = math.ceil(int(w.seq_lens[b]) / 16)
        row = pt[b]
        assert np.all(row[:m] >= 0) and np.all(row[:m] < w.k_cache.shape[0])
        assert np.all(row[m:] == -1)
        used.extend(row[:m].tolist())
    assert len(used) == len(set(used)) == w.k_cache.shape[0]      # one shared pool, no page reused


def test_ragged_lengths_lie_in_their_range():
    w = make_workload("ragged_paged", "cpu", B=40, N_min=300, N_max=3000)
    lens = w.seq_lens.numpy()
    assert lens.min() >= 300 and lens.max() <= 3000 and len(set(lens.tolist())) > 20


@pytest.mark.parametrize("name,kw", [("tiny_ref", dict(N=300)), ("llama3_8b_topp", dict(B=2, N=2000))])
def test_needles_are_distinct_per_group_and_follow_their_head_query(name, kw):
    w = make_workload(name, "cpu", **kw)
    G = w.num_q_heads // w.num_kv_heads
    planted = w.notes["needles"]
    assert planted
    for b in range(w.batch):
        by_group = {}
        for (bb, h), pos in planted.items():
            if bb == b:
                by_group.setdefault(h // G, []).extend(pos)
        for g, pos in by_group.items():
            assert len(pos) == len(set(pos))                      # distinct across the group's heads
    for (b, h), pos in planted.items():
        q = w.q[b, h].float()
        qhat = q / q.norm()
        for p in pos:
            page = int(w.page_table[b, p // 16])
            k = w.k_cache[page, h // G, p % 16].float()
            # k = 0.8 sqrt(d) q / |q| + N(0, 0.1^2): the component along q is
            # 0.8 sqrt(d) up to the noise and bf16 rounding
            assert abs(float(k @ qhat) - 0.8 * math.sqrt(w.head_dim)) < 0.5
            assert float(k @ qhat) / float(k.norm()) > 0.95


def test_topk_query_scales_meet_their_entropy_targets():
    w = make_workload("topk_128k", "cpu", B=1, N=2048)
    tgt = w.notes["target_entropy_over_lnN"].numpy()
    got = w.notes["realised_entropy_over_lnN"].numpy()
    assert tgt.min() >= 0.2 and tgt.max() <= 0.9
    assert np.abs(got - tgt).max() < 0.02                        # bf16 rounding of the scaled query


@pytest.mark.parametrize("alpha", [0.8, 1.2])
def test_long_zipf_index_scores_follow_the_rank_profile(alpha):
    w = make_workload("long_zipf", "cpu", N=4096, alpha=alpha)
    G = w.num_q_heads // w.num_kv_heads
    c = math.sqrt(w.head_dim) / 16
    pages = w.page_table[0, torch.arange(4096) // 16].long()
    slots = torch.arange(4096) % 16
    for kvh in (0, 1):
        K = w.k_cache[pages, kvh, slots].float().numpy()
        rank = w.notes["rank"][kvh].numpy().astype(np.float64)
        kidx = O.index_keys(w.proj[kvh].float().numpy(), K)
        for h in (kvh * G, kvh * G + G - 1):
            s = O.index_scores(O.query_index(w.proj[kvh].float().numpy(), w.q[0, h].float().numpy()), kidx, c)
            want = -alpha * np.log(rank)
            # the head query is the group direction plus a 1 % perturbation;
            # keys and query are rounded to bf16
            assert np.corrcoef(s, want)[0, 1] > 0.99
            assert np.median(np.abs(s - want)) < 0.1 * alpha * np.log(4096)
