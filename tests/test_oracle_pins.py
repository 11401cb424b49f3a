"""Pins for the float64 oracle, each against something other than the oracle
itself: hand-derived cases (tests/golden), closed forms, brute force on tiny
inputs, exact rational arithmetic, and independent library routines (torch's
float32 -> bfloat16 cast, torch's float64 scaled_dot_product_attention,
numpy's argpartition).  CPU only.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_cases.json")


def _bf16_bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().astype(np.int64) & 0xFFFF


def _bf16_from_bits(bits):
    b = torch.tensor(np.asarray(bits, np.int64).astype(np.int16)).view(torch.bfloat16)
    return b.to(torch.float64).numpy()


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_cast_on_float32_inputs():
    rng = np.random.default_rng(1)
    mags = np.concatenate([
        rng.standard_normal(20000),
        rng.standard_normal(2000) * 1e-38,    # subnormal range
        rng.standard_normal(2000) * 1e-30,
        rng.uniform(-1.0, 1.0, 2000) * 3.3e38,  # near overflow
        rng.standard_normal(2000) * 1e6,
    ]).astype(np.float32)
    mags = mags[np.isfinite(mags)]
    ref = torch.tensor(mags).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(mags.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_round_ties_to_even_from_the_exact_value():
    # near 1.0 the bf16 quantum is 2^-7
    cases = {
        1.0 + 2.0 ** -8: 1.0,                              # tie -> even (1.0)
        1.0 + 3 * 2.0 ** -8: 1.0 + 2.0 ** -6,               # tie -> even mantissa
        1.0 + 2.0 ** -8 + 2.0 ** -30: 1.0 + 2.0 ** -7,      # just above the tie: up
        -(1.0 + 2.0 ** -8 + 2.0 ** -40): -(1.0 + 2.0 ** -7),
        1.0 + 2.0 ** -8 - 2.0 ** -40: 1.0,                 # just below the tie: down
    }
    for x, want in cases.items():
        assert O.bf16_round(np.array([x]))[0] == want, x
    # rounding through float32 first would turn 1 + 2^-8 + 2^-30 into the tie 1 + 2^-8
    # and then into 1.0; the oracle must not do that.
    assert np.float32(1.0 + 2.0 ** -8 + 2.0 ** -30) == np.float32(1.0 + 2.0 ** -8)


def test_bf16_round_special_values():
    x = np.array([0.0, -0.0, np.inf, -np.inf, 1e39, -1e39])
    y = O.bf16_round(x)
    assert y[0] == 0.0 and y[1] == 0.0 and np.signbit(y[1])
    assert np.isposinf(y[2]) and np.isneginf(y[3]) and np.isposinf(y[4]) and np.isneginf(y[5])


# ---------------------------------------------------------------- index keys

def test_index_keys_coordinate_selection_pins_operand_orientation():
    # P_g picks coordinate perm[j] of k for output j: k~_j = k[perm[j]] exactly.
    rng = np.random.default_rng(2)
    d, r = 16, 16
    perm = (3 * np.arange(r) + 1) % d           # not an involution
    P = np.zeros((d, r))
    P[perm, np.arange(r)] = 1.0
    k = O.bf16_round(rng.standard_normal((5, d)))
    got = O.index_keys(P, k)
    np.testing.assert_array_equal(got, k[:, perm])
    assert not np.array_equal(got, k[:, np.argsort(perm)])   # the transpose differs


def test_index_keys_is_the_nearest_bf16_of_the_exact_sum():
    rng = np.random.default_rng(3)
    d, r, n = 64, 16, 6
    P = O.bf16_round(rng.standard_normal((d, r)) / 8.0)
    K = O.bf16_round(rng.standard_normal((n, d)))
    got = O.index_keys(P, K)
    bits = _bf16_bits(got.astype(np.float32))
    assert np.array_equal(_bf16_from_bits(bits), got)        # representable in bf16
    lo, hi = _bf16_from_bits(bits - 1), _bf16_from_bits(bits + 1)   # bf16 neighbours
    for t in range(n):
        for j in range(r):
            exact = sum(Fraction(float(K[t, i])) * Fraction(float(P[i, j])) for i in range(d))
            err = abs(Fraction(float(got[t, j])) - exact)
            for nb in (lo[t, j], hi[t, j]):
                e_nb = abs(Fraction(float(nb)) - exact)
                assert err <= e_nb
                if err == e_nb:                                # a tie: even bit pattern
                    assert bits[t, j] % 2 == 0


def test_index_scores_with_identity_projection_are_full_dot_products():
    rng = np.random.default_rng(4)
    d = r = 16
    P = np.eye(d)
    q = O.bf16_round(rng.standard_normal(d))
    K = O.bf16_round(rng.standard_normal((40, d)))
    s = O.index_scores(O.query_index(P, q), O.index_keys(P, K), 0.25)
    want = np.array([0.25 * math.fsum(float(q[i]) * float(K[j, i]) for i in range(d)) for j in range(40)])
    np.testing.assert_allclose(s, want, rtol=0, atol=1e-12)


def test_query_index_uses_the_group_projection_columns():
    # q~_j = <q, P[:, j]>: with P = e_i e_j^T only output j is non-zero and equals q_i.
    d, r = 8, 4
    q = np.arange(1.0, d + 1)
    P = np.zeros((d, r)); P[5, 2] = 1.0
    np.testing.assert_array_equal(O.query_index(P, q), [0, 0, 6.0, 0])


# ---------------------------------------------------------------- golden cases

def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_top_p_hand_worked_cases():
    for c in _golden()["top_p"]:
        s = np.log(np.array(c["scores_ln"], dtype=np.float64))
        got = O.select_top_p(s, c["p"]).tolist()
        assert got == c["expected"], c


def test_top_k_hand_worked_cases():
    for c in _golden()["top_k"]:
        got = O.select_top_k(np.array(c["scores"], np.float64), c["k"]).tolist()
        assert got == c["expected"], c


def test_local_positions_hand_worked_cases():
    for c in _golden()["local"]:
        want = [j for a, b in c["expected_ranges"] for j in range(a, b)]
        assert O.local_positions(c["n"], c["window"], c["sinks"]).tolist() == want, c


# ---------------------------------------------------------------- compacted local cache

@pytest.mark.parametrize("sinks", [0, 1, 3, 8])
@pytest.mark.parametrize("window", [0, 1, 5, 16])
def test_compacted_local_rows_hold_exactly_the_local_positions(window, sinks):
    """After positions 0..n-1 are written in order, the compacted rows hold
    each position a local head attends to at length n exactly once and
    nothing else (marker rows: row j carries j + 1).  A ring that ignored the
    sinks, or a slot off by one, overwrites a kept row and fails here."""
    for n in range(0, 70):
        rows = (np.arange(n, dtype=np.int64) + 1)[:, None]
        comp = O.compact_local_rows(rows, window, sinks)
        assert comp.shape == (sinks + window, 1)
        held = sorted(int(x) - 1 for x in comp[:, 0] if x != 0)
        assert held == O.local_positions(n, window, sinks).tolist(), (n, window, sinks)


def test_local_slot_hand_cases():
    # sinks keep their rows; the ring starts after them and wraps every `window`
    assert [O.local_slot(p, 4, 2) for p in range(11)] == [0, 1, 4, 5, 2, 3, 4, 5, 2, 3, 4]
    assert [O.local_slot(p, 0, 2) for p in range(4)] == [0, 1, -1, -1]
    assert [O.local_slot(p, 3, 0) for p in range(5)] == [0, 1, 2, 0, 1]


def test_local_attention_over_compacted_rows_equals_the_paged_one():
    rng = np.random.default_rng(3)
    n, d, window, sinks = 57, 8, 16, 4
    K, V, q = rng.normal(size=(n, d)), rng.normal(size=(n, d)), rng.normal(size=d)
    keep = O.local_positions(n, window, sinks)
    ck = O.compact_local_rows(K, window, sinks)
    cv = O.compact_local_rows(V, window, sinks)
    slots = [O.local_slot(j, window, sinks) for j in keep]
    assert len(set(slots)) == len(slots)
    got = O.attend_set(q, ck, cv, slots, 0.3)
    want = O.attend_set(q, K, V, keep, 0.3)
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- top-p

def _mass(s):
    w = np.exp(s - s.max())
    return w / w.sum()


@pytest.mark.parametrize("seed", range(40))
def test_top_p_brute_force_over_all_subsets(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 11))
    s = rng.standard_normal(n) * rng.uniform(0.2, 4.0)      # distinct almost surely
    p = float(rng.uniform(0.05, 0.99))
    w = _mass(s)
    best = None
    for m in range(1, n + 1):
        reach = [T for T in itertools.combinations(range(n), m) if w[list(T)].sum() >= p]
        if reach:
            best = max(reach, key=lambda T: w[list(T)].sum())
            break
    assert best is not None
    assert O.select_top_p(s, p).tolist() == sorted(best)


@pytest.mark.parametrize("seed", range(10))
def test_top_p_defining_property(seed):
    rng = np.random.default_rng(200 + seed)
    n = int(rng.integers(50, 5000))
    s = rng.standard_normal(n) * rng.uniform(0.5, 6.0)
    p = float(rng.uniform(0.1, 0.99))
    S = O.select_top_p(s, p)
    w = _mass(s)
    inS = np.zeros(n, bool); inS[S] = True
    assert math.fsum(w[S]) >= p - 1e-12
    lowest = S[np.argmin(s[S])]
    assert math.fsum(w[S]) - w[lowest] < p + 1e-12          # minimal
    if (~inS).any():
        assert s[S].min() > s[~inS].max()                    # a prefix of the ranking


@pytest.mark.parametrize("alpha", [0.8, 1.2])
@pytest.mark.parametrize("p", [0.5, 0.9, 0.99])
def test_top_p_zipf_closed_form(alpha, p):
    # scores -alpha*ln(rank) give softmax masses proportional to rank^-alpha, so
    # |S| is the smallest n with sum_{r<=n} r^-alpha >= p * sum_{r<=N} r^-alpha.
    N = 262144
    rng = np.random.default_rng(7)
    rank = rng.permutation(N) + 1
    s = -alpha * np.log(rank.astype(np.float64))
    terms = [r ** -alpha for r in range(1, N + 1)]
    total = math.fsum(terms)
    acc, n_expect = 0.0, None
    partial = np.cumsum(np.array(terms))                     # monotone; exact check below
    n_expect = int(np.searchsorted(partial, p * total, side="left")) + 1
    # confirm the boundary with exact summation on both sides
    assert math.fsum(terms[:n_expect]) >= p * total
    assert math.fsum(terms[:n_expect - 1]) < p * total
    S = O.select_top_p(s, p)
    assert len(S) == n_expect
    assert set(rank[S].tolist()) == set(range(1, n_expect + 1))


def test_top_p_uses_the_float32_value_of_p():
    # two tokens whose first holds mass 0.990000005: p = 0.99 keeps it alone,
    # float32(0.99) = 0.99000000954 needs both; the configuration stores the
    # float32 value, and the decode step applies exactly that
    c1 = 0.990000005
    s = np.array([math.log(c1 / (1.0 - c1)), 0.0])
    assert O.select_top_p(s, 0.99).tolist() == [0]
    assert O.stored_top_p(0.99) == float(np.float32(0.99)) > 0.99
    assert O.select_top_p(s, O.stored_top_p(0.99)).tolist() == [0, 1]
    assert O.stored_top_p(1.0) == 1.0 and O.stored_top_p(0.5) == 0.5


def test_decode_step_applies_the_stored_top_p(monkeypatch):
    import oracle.sparse_decode_oracle as OM
    seen = []
    real = OM.select_top_p
    monkeypatch.setattr(OM, "select_top_p", lambda s, p: seen.append(p) or real(s, p))
    prob, Hq, Hkv, d, r = _tiny_problem(12, page_perm=False)
    cfg = O.OracleConfig(Hq, Hkv, d, r, 16, [1, 1, 0, 0], 8, 2, "top_p", top_p=0.99)
    O.decode_reference(cfg, **prob)
    assert seen and all(p == float(np.float32(0.99)) for p in seen)


def test_top_p_one_keeps_everything_and_scale_invariance_of_order():
    s = np.array([3.0, -1.0, 2.0])
    assert O.select_top_p(s, 1.0).tolist() == [0, 1, 2]
    assert O.select_top_p(s + 1000.0, 0.6).tolist() == O.select_top_p(s, 0.6).tolist()


# ---------------------------------------------------------------- top-k

@pytest.mark.parametrize("seed", range(20))
def test_top_k_brute_force_and_argpartition(seed):
    rng = np.random.default_rng(300 + seed)
    n = int(rng.integers(1, 10))
    s = rng.standard_normal(n)
    k = int(rng.integers(1, n + 1))
    best = max(itertools.combinations(range(n), k), key=lambda T: s[list(T)].sum())
    assert O.select_top_k(s, k).tolist() == sorted(best)
    big = rng.standard_normal(3000)
    kk = int(rng.integers(1, 3000))
    assert O.select_top_k(big, kk).tolist() == sorted(np.argpartition(-big, kk - 1)[:kk].tolist())


def test_top_k_budget():
    assert O.top_k_budget(131072, 0, 0.02) == 2621       # 2% of 128K, float32 fraction
    assert O.top_k_budget(100, 0, 0.001) == 1
    assert O.top_k_budget(100, 5000, 0.0) == 100
    assert O.top_k_budget(512, 7, 0.5) == 7


# ---------------------------------------------------------------- attention

def _sdpa64(q, K, V, scale):
    qt = torch.tensor(q, dtype=torch.float64)[None, None, None, :]
    Kt = torch.tensor(K, dtype=torch.float64)[None, None]
    Vt = torch.tensor(V, dtype=torch.float64)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)[0, 0, 0].numpy()


def test_attend_full_set_is_dense_sdpa():
    rng = np.random.default_rng(5)
    n, d = 300, 64
    q, K, V = (O.bf16_round(rng.standard_normal(sh)) for sh in [(d,), (n, d), (n, d)])
    got = O.attend_set(q, K, V, np.arange(n), 1 / 8)
    np.testing.assert_allclose(got, _sdpa64(q, K, V, 1 / 8), rtol=1e-12, atol=1e-13)


def test_attend_single_and_pair_closed_forms():
    rng = np.random.default_rng(6)
    d = 16
    q, K, V = rng.standard_normal(d), rng.standard_normal((5, d)), rng.standard_normal((5, d))
    np.testing.assert_array_equal(O.attend_set(q, K, V, [3], 0.3), V[3])
    l1, l4 = 0.3 * K[1] @ q, 0.3 * K[4] @ q
    a = 1.0 / (1.0 + math.exp(l4 - l1))
    np.testing.assert_allclose(O.attend_set(q, K, V, [1, 4], 0.3), a * V[1] + (1 - a) * V[4], rtol=1e-13)
    assert np.all(O.attend_set(q, K, V, [], 0.3) == 0)


def _tiny_problem(seed, page_perm=False, n_list=(37, 20), Hq=4, Hkv=2, d=32, r=16):
    rng = np.random.default_rng(seed)
    ps = 16
    B = len(n_list)
    pages_per = [math.ceil(n / ps) for n in n_list]
    total = sum(pages_per)
    ids = rng.permutation(total) if page_perm else np.arange(total)
    pt = -np.ones((B, max(pages_per)), np.int64)
    c = 0
    for b, m in enumerate(pages_per):
        pt[b, :m] = ids[c:c + m]
        c += m
    kc = O.bf16_round(rng.standard_normal((total, Hkv, ps, d)))
    vc = O.bf16_round(rng.standard_normal((total, Hkv, ps, d)))
    proj = O.bf16_round(rng.standard_normal((Hkv, d, r)) / math.sqrt(d))
    q = O.bf16_round(rng.standard_normal((B, Hq, d)))
    return dict(proj=proj, q_pre=q, q=q, k_cache=kc, v_cache=vc, page_table=pt,
                seq_lens=np.array(n_list)), Hq, Hkv, d, r


@pytest.mark.parametrize("mode", ["top_p1", "top_kN", "windowN"])
def test_decode_step_degenerate_cases_are_dense_sdpa(mode):
    # p = 1, k >= N and window >= N all reduce to dense attention ([NHA] §2.3:
    # a window as long as the sequence is full attention).
    prob, Hq, Hkv, d, r = _tiny_problem(11, page_perm=True)
    retr = [1, 1, 0, 0]
    if mode == "top_p1":
        cfg = O.OracleConfig(Hq, Hkv, d, r, 16, retr, 10 ** 6, 2, "top_p", top_p=1.0)
    elif mode == "top_kN":
        cfg = O.OracleConfig(Hq, Hkv, d, r, 16, retr, 10 ** 6, 2, "top_k", top_k=10 ** 6)
    else:
        cfg = O.OracleConfig(Hq, Hkv, d, r, 16, [0, 0, 0, 0], 10 ** 6, 0, "top_p")
    res = O.decode_reference(cfg, **prob)
    G = Hq // Hkv
    for (b, h), o in res.out.items():
        n = prob["seq_lens"][b]
        K = O.gather_rows(prob["k_cache"], prob["page_table"][b], n, h // G, 16)
        V = O.gather_rows(prob["v_cache"], prob["page_table"][b], n, h // G, 16)
        np.testing.assert_allclose(o, _sdpa64(prob["q"][b, h], K, V, 1 / math.sqrt(d)),
                                   rtol=1e-11, atol=1e-12)


def test_decode_step_page_table_permutation_invariance():
    # the same logical cache stored under a permuted page table gives the same result
    prob, Hq, Hkv, d, r = _tiny_problem(12, page_perm=False)
    cfg = O.OracleConfig(Hq, Hkv, d, r, 16, [1, 1, 0, 0], 8, 2, "top_p", top_p=0.7)
    a = O.decode_reference(cfg, **prob)
    rng = np.random.default_rng(0)
    total = prob["k_cache"].shape[0]
    perm = rng.permutation(total)           # new physical location of old page i
    kc = np.empty_like(prob["k_cache"]); kc[perm] = prob["k_cache"]
    vc = np.empty_like(prob["v_cache"]); vc[perm] = prob["v_cache"]
    pt = prob["page_table"].copy()
    pt[pt >= 0] = perm[pt[pt >= 0]]
    b_ = O.decode_reference(cfg, **{**prob, "k_cache": kc, "v_cache": vc, "page_table": pt})
    for key in a.out:
        np.testing.assert_array_equal(a.out[key], b_.out[key])
    for key in a.sets:
        np.testing.assert_array_equal(a.sets[key], b_.sets[key])


def test_widen_accepts_bf16_bit_patterns():
    x = O.bf16_round(np.random.default_rng(9).standard_normal(100))
    bits = _bf16_bits(x.astype(np.float32)).astype(np.uint16)
    np.testing.assert_array_equal(O.widen(bits), x)


# ---------------------------------------------------------------- composition

def _planted_problem(seed, n=200, d=32, needles=(17, 64, 130, 199), gain=40.0):
    """One sequence, Hq = 2 retrieval heads on KV head 0 plus 2 local heads on
    KV head 1.  The projection selects the first 16 coordinates, so a key's
    index entry is its first 16 coordinates.  Background keys are zero there
    (index score exactly 0); needle i points along the query with scores
    gain - 0.1 i (distinct, far above 0).  Pages are permuted."""
    rng = np.random.default_rng(seed)
    ps, r, Hq, Hkv = 16, 16, 4, 2
    pages = math.ceil(n / ps)
    perm = rng.permutation(pages)
    pt = perm[None, :].astype(np.int64)
    K = O.bf16_round(rng.standard_normal((n, Hkv, d)))
    V = O.bf16_round(rng.standard_normal((n, Hkv, d)))
    K[:, 0, :r] = 0.0
    q = O.bf16_round(rng.standard_normal((1, Hq, d)))
    # both retrieval heads share the first 16 query coordinates (unit-norm u)
    u = rng.standard_normal(r)
    u /= np.linalg.norm(u)
    q[0, 0, :r] = O.bf16_round(u)
    q[0, 1, :r] = O.bf16_round(u)
    c = math.sqrt(d) / r
    for i, j in enumerate(needles):
        # index score = c * <q~, k~> with k~ = a u  =>  a = target / (c <q[:r], u>)
        a = (gain - 0.1 * i) / (c * float(q[0, 0, :r] @ u))
        K[j, 0, :r] = O.bf16_round(a * u)
    kc = np.zeros((pages, Hkv, ps, d))
    vc = np.zeros((pages, Hkv, ps, d))
    for j in range(n):
        kc[perm[j // ps], :, j % ps] = K[j]
        vc[perm[j // ps], :, j % ps] = V[j]
    proj = np.zeros((Hkv, d, r))
    proj[:, :r, :] = np.eye(r)
    prob = dict(proj=proj, q_pre=q, q=q, k_cache=kc, v_cache=vc, page_table=pt, seq_lens=np.array([n]))
    return prob, K, V, Hq, Hkv, d, r


@pytest.mark.parametrize("mode", ["top_k", "top_p"])
def test_decode_step_composed_on_planted_needles(mode):
    # index keys -> scores -> selection -> attention on a case whose selected
    # set is known by construction; the output must equal float64 SDPA over
    # exactly that set, and the local heads SDPA over sinks + window
    needles = (17, 64, 130, 199)
    prob, K, V, Hq, Hkv, d, r = _planted_problem(21, needles=needles)
    retr = [1, 1, 0, 0]
    if mode == "top_k":
        cfg = O.OracleConfig(Hq, Hkv, d, r, 16, retr, 5, 2, "top_k", top_k=len(needles))
    else:
        # masses e^40, e^39.9, e^39.8, e^39.7 (cumulative 0.29, 0.55, 0.79, 1.0):
        # p = 0.9 needs all four; the 196 zero scores add ~1e-15 of the mass
        cfg = O.OracleConfig(Hq, Hkv, d, r, 16, retr, 5, 2, "top_p", top_p=0.9)
    res = O.decode_reference(cfg, **prob, keep_scores=True)
    for h in (0, 1):
        np.testing.assert_array_equal(res.sets[(0, h)], np.array(needles))
        s = res.scores[(0, h)]
        assert np.all(s[np.setdiff1d(np.arange(200), needles)] == 0.0)
        np.testing.assert_allclose(s[list(needles)], [40.0, 39.9, 39.8, 39.7], rtol=5e-3)
        idx = np.array(needles)
        want = _sdpa64(prob["q"][0, h], K[idx, 0], V[idx, 0], 1 / math.sqrt(d))
        np.testing.assert_allclose(res.out[(0, h)], want, rtol=1e-11, atol=1e-12)
    loc = np.array([0, 1, 195, 196, 197, 198, 199])       # sinks 0-1, window of 5
    for h in (2, 3):
        want = _sdpa64(prob["q"][0, h], K[loc, 1], V[loc, 1], 1 / math.sqrt(d))
        np.testing.assert_allclose(res.out[(0, h)], want, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- retained mass

def test_mass_retained_closed_forms():
    """Share of the full softmax mass on a kept set: the whole set gives 1, the
    empty set 0, and two tokens with logits l0, l1 give the logistic of their
    gap, 1 / (1 + e^(l1 - l0)) for keeping token 0 alone."""
    rng = np.random.default_rng(3)
    d = 16
    K = rng.standard_normal((40, d)).astype(np.float32)
    q = rng.standard_normal(d).astype(np.float32)
    assert O.mass_retained(q, K, np.arange(40), 0.25) == pytest.approx(1.0, abs=1e-15)
    assert O.mass_retained(q, K, np.zeros(0, np.int64), 0.25) == 0.0
    # two keys along q: logits are scale * <q, k> computed by hand
    q2 = np.zeros(d, np.float32)
    q2[0] = 2.0
    K2 = np.zeros((2, d), np.float32)
    K2[0, 0], K2[1, 0] = 3.0, -1.5                       # logits 0.5 * (6, -3) = (3, -1.5)
    want = 1.0 / (1.0 + math.exp(-1.5 - 3.0))
    assert O.mass_retained(q2, K2, [0], 0.5) == pytest.approx(want, rel=1e-14)
    assert O.mass_retained(q2, K2, [1], 0.5) == pytest.approx(1.0 - want, rel=1e-12)


@pytest.mark.parametrize("seed", range(6))
def test_mass_retained_is_the_exact_share_on_small_integer_logits(seed):
    """Logits that are small integers times ln 2 make every weight a power of
    two, so the share is an exact rational: sum_{j in S} 2^{a_j} / sum_j 2^{a_j}.
    Checked with Fraction arithmetic on every subset of a 7-token context (a
    dropped term, a wrong index or a missing normalisation fails one)."""
    rng = np.random.default_rng(100 + seed)
    a = rng.integers(-6, 7, size=7)
    d = 4
    K = np.zeros((7, d), np.float64)
    K[:, 0] = a * math.log(2.0)                          # logit_j = <q, k_j> = a_j ln 2
    q = np.zeros(d)
    q[0] = 1.0
    tot = sum(Fraction(2) ** int(x) for x in a)
    for mask in range(1 << 7):
        S = [j for j in range(7) if mask >> j & 1]
        want = sum((Fraction(2) ** int(a[j]) for j in S), Fraction(0)) / tot
        got = O.mass_retained(q, K, S, 1.0)
        assert got == pytest.approx(float(want), rel=1e-12, abs=1e-15)


def test_mass_retained_of_a_top_p_set_on_full_logits_reaches_p():
    """When the index scores are the attention logits themselves (identity
    projection, index scale = attention scale), the top-p set of the index
    holds at least p of the full softmax mass, and dropping its lowest-scored
    token leaves less than p: the defining property, read through the
    retained-mass diagnostic."""
    rng = np.random.default_rng(9)
    d = 16
    K = O.bf16_round(rng.standard_normal((300, d)) * 2.0)
    q = O.bf16_round(rng.standard_normal(d))
    s = O.index_scores(q, K, 0.25)
    for p in (0.5, 0.9, 0.99):
        S = O.select_top_p(s, p)
        m = O.mass_retained(q, K, S, 0.25)
        assert m >= p - 1e-12
        low = S[np.argmin(s[S])]
        assert O.mass_retained(q, K, np.setdiff1d(S, [low]), 0.25) < p


# ---------------------------------------------------------------- exact-score selection

def test_exact_scores_equal_index_scores_under_an_identity_index():
    """With r = d, P = I and c = attn_scale, the index of a key is the key
    itself (bf16 values round to themselves) and q~ = q, so index scoring and
    exact scoring coincide: the two selections must agree token for token."""
    rng = np.random.default_rng(21)
    d, n = 16, 400
    K = O.bf16_round(rng.standard_normal((n, d)))
    q = O.bf16_round(rng.standard_normal(d) * 2.0)
    P = np.eye(d)
    s_idx = O.index_scores(O.query_index(P, q), O.index_keys(P, K), 0.25)
    s_ex = O.exact_scores(q, K, 0.25)
    assert np.array_equal(s_idx, s_ex)
    for p in (0.5, 0.9):
        assert np.array_equal(O.select_top_p(s_idx, p), O.select_top_p(s_ex, p))
    assert np.array_equal(O.select_top_k(s_idx, 37), O.select_top_k(s_ex, 37))


@pytest.mark.parametrize("seed", range(8))
def test_exact_top_p_is_the_smallest_set_holding_p_of_the_attention_mass(seed):
    """Selecting by the exact logits, the top-p set is a minimum-size subset
    whose share of the full softmax (mass_retained) reaches p, and among those
    the one with the largest share: brute force over all subsets of a 10-token
    context."""
    rng = np.random.default_rng(300 + seed)
    d, n = 8, 10
    K = O.bf16_round(rng.standard_normal((n, d)) * 1.5)
    q = O.bf16_round(rng.standard_normal(d))
    p = float(rng.uniform(0.3, 0.95))
    S = O.select_top_p(O.exact_scores(q, K, 0.5), p)
    best = None
    for size in range(1, n + 1):
        cands = [c for c in itertools.combinations(range(n), size) if O.mass_retained(q, K, c, 0.5) >= p]
        if cands:
            best = (size, max(O.mass_retained(q, K, c, 0.5) for c in cands))
            break
    assert len(S) == best[0]
    assert O.mass_retained(q, K, S, 0.5) == pytest.approx(best[1], rel=1e-12)


def test_decode_step_with_exact_scores_selects_by_the_attention_logits():
    """A decode step in exact-score mode on planted keys: under a projection
    that hides the planted direction from the index, the index selection
    misses the planted tokens while the exact selection keeps exactly them
    (top-k = their number)."""
    rng = np.random.default_rng(5)
    d, n, G = 32, 64, 1
    K = rng.standard_normal((n, d)) * 0.1
    q = np.zeros(d)
    q[0] = 4.0
    planted = [5, 17, 40]
    for j in planted:
        K[j, 0] = 3.0                                    # large logits along q
    K = O.bf16_round(K)
    P = np.zeros((1, d, 16))
    P[0, 1:17, :] = np.eye(16)                           # the index never sees dimension 0
    kc = K.reshape(n // 16, 1, 16, d)
    pt = np.arange(n // 16)[None, :]
    base = dict(proj=P, q_pre=q[None, None, :], q=q[None, None, :], k_cache=kc, v_cache=kc,
                page_table=pt, seq_lens=np.array([n]))
    for score, want_all in (("exact", True), ("index", False)):
        cfg = O.OracleConfig(1, 1, d, 16, 16, [1], 0, 0, "top_k", top_k=3, score=score)
        S = O.decode_reference(cfg, **base).sets[(0, 0)]
        assert (set(S.tolist()) == set(planted)) == want_all
