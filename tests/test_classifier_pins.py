"""Pins of the data-free head classifier oracle ([AoH] Methodology §1-§4,
"Autonomy-of-Heads: Data-Free Sparse Attention from Frozen Query-Key
Geometry") against closed forms, weights with a known spectrum, and the two
routes to the spectrum (§1-2's SVD of M_h, §3's eigenvalues of C_h) against
each other.  CPU only."""

import math

import numpy as np
import pytest

import oracle as O


def _orthonormal_rows(rng, rows, cols):
    q, _ = np.linalg.qr(rng.normal(size=(cols, rows)))
    return q.T                                       # rows x cols, orthonormal rows


# ---------------------------------------------------------------- entropy closed forms

def test_effective_rank_closed_forms():
    assert O.effective_rank_of_spectrum([5.0]) == pytest.approx(1.0, abs=1e-15)
    for r in (2, 7, 64):
        assert O.effective_rank_of_spectrum([0.3] * r) == pytest.approx(r, rel=1e-13)
    want = math.exp(-(0.75 * math.log(0.75) + 0.25 * math.log(0.25)))
    assert O.effective_rank_of_spectrum([3.0, 1.0]) == pytest.approx(want, rel=1e-15)
    # scale-free: only the normalised spectrum matters
    assert O.effective_rank_of_spectrum([6.0, 2.0]) == pytest.approx(want, rel=1e-15)
    assert O.effective_rank_of_spectrum([]) == 1.0


# ---------------------------------------------------------------- known spectra

@pytest.mark.parametrize("route", ["direct", "sylvester"])
def test_equal_singular_values_give_er_equal_to_the_rank(route):
    """W_Q = c * V, W_K = V with V orthonormal rows: M_h = c V^T V is c times
    an orthogonal projector of rank d_head, all singular values c."""
    rng = np.random.default_rng(0)
    d_head, d_model = 16, 96
    v = _orthonormal_rows(rng, d_head, d_model)
    sv = O.singular_values_direct if route == "direct" else O.singular_values_sylvester
    s = sv(2.5 * v, v)
    assert s.size == d_head
    assert np.allclose(s, 2.5, rtol=1e-12)
    assert O.effective_rank_of_spectrum(s) == pytest.approx(d_head, rel=1e-12)


@pytest.mark.parametrize("route", ["direct", "sylvester"])
def test_rank_one_operator_has_er_one(route):
    rng = np.random.default_rng(1)
    d_head, d_model = 8, 64
    u = rng.normal(size=d_model)
    wq = np.outer(rng.normal(size=d_head), u)          # every row a multiple of u
    wk = rng.normal(size=(d_head, d_model))
    sv = O.singular_values_direct if route == "direct" else O.singular_values_sylvester
    s = sv(wq, wk)
    assert s.size == 1
    assert O.effective_rank_of_spectrum(s) == pytest.approx(1.0, abs=1e-12)


@pytest.mark.parametrize("route", ["direct", "sylvester"])
def test_prescribed_spectrum(route):
    """W_Q = diag(s) V, W_K = V: M_h = V^T diag(s) V has singular values s."""
    rng = np.random.default_rng(2)
    d_head, d_model = 12, 80
    v = _orthonormal_rows(rng, d_head, d_model)
    s = np.arange(1, d_head + 1, dtype=np.float64) ** -1.3
    sv = O.singular_values_direct if route == "direct" else O.singular_values_sylvester
    got = np.sort(sv(np.diag(s) @ v, v))[::-1]
    assert np.allclose(got, np.sort(s)[::-1], rtol=1e-10)
    p = s / s.sum()
    assert O.effective_rank_of_spectrum(got) == pytest.approx(math.exp(-np.sum(p * np.log(p))), rel=1e-12)


@pytest.mark.parametrize("seed", range(6))
def test_sylvester_route_equals_the_direct_svd(seed):
    """§3's d_head x d_head route against §1-2's d_model x d_model SVD on
    random weights: the same nonzero singular values, the same ER."""
    rng = np.random.default_rng(10 + seed)
    d_head, d_model = 32, 192
    wq = rng.normal(size=(d_head, d_model)) * rng.uniform(0.2, 3.0, size=(d_head, 1))
    wk = rng.normal(size=(d_head, d_model))
    a = np.sort(O.singular_values_direct(wq, wk))[::-1]
    b = np.sort(O.singular_values_sylvester(wq, wk))[::-1]
    assert a.size == b.size == d_head
    assert np.allclose(a, b, rtol=1e-9)
    assert O.effective_rank_of_spectrum(a) == pytest.approx(O.effective_rank_of_spectrum(b), rel=1e-11)


def test_concentrated_spectrum_has_lower_er_than_a_diffuse_one():
    """§1-2: a steep spectrum (few dominant matching directions) gives a lower
    ER than a flat one."""
    rng = np.random.default_rng(4)
    d_head, d_model = 16, 64
    v = _orthonormal_rows(rng, d_head, d_model)
    k = np.arange(1, d_head + 1, dtype=np.float64)
    steep = O.effective_rank_of_spectrum(O.singular_values_direct(np.diag(k ** -2.0) @ v, v))
    flat = O.effective_rank_of_spectrum(O.singular_values_direct(np.diag(k ** -0.1) @ v, v))
    assert steep < 4.0 < 15.0 < flat


# ---------------------------------------------------------------- layer and grouping

def test_layer_effective_ranks_picks_head_and_group_blocks():
    """Head h of the layer uses rows h*d_head.. of W_Q and the rows of KV head
    h // G of W_K: planting a known spectrum in one head's block moves only
    that head's ER."""
    rng = np.random.default_rng(5)
    Hq, Hkv, d_head, d_model = 4, 2, 8, 48
    w_q = rng.normal(size=(Hq * d_head, d_model))
    w_k = rng.normal(size=(Hkv * d_head, d_model))
    v = _orthonormal_rows(rng, d_head, d_model)
    w_k[d_head:2 * d_head] = v                          # KV head 1
    w_q[3 * d_head:4 * d_head] = 7.0 * v                 # head 3 (group 1): equal singular values
    er = O.layer_effective_ranks(w_q, w_k, Hq, Hkv, d_head)
    assert er[3] == pytest.approx(d_head, rel=1e-10)
    direct = O.layer_effective_ranks(w_q, w_k, Hq, Hkv, d_head, route="direct")
    assert np.allclose(er, direct, rtol=1e-10)


def test_classify_groups_hand_cases():
    er = [1.0, 3.0, 2.0, 2.0, 5.0, 0.5, 4.0, 4.0]      # group means 2, 2, 2.75, 4
    assert O.classify_groups(er, 4, 2).tolist() == [1, 1, 1, 1, 0, 0, 0, 0]
    assert O.classify_groups(er, 4, 1).tolist() == [1, 1, 0, 0, 0, 0, 0, 0]   # tie: lower group
    assert O.classify_groups(er, 4, 3).tolist() == [1, 1, 1, 1, 1, 1, 0, 0]
    assert O.classify_groups(er, 4, 0).tolist() == [0] * 8
    assert O.classify_groups(er, 8, 3).tolist() == [1, 0, 1, 0, 0, 1, 0, 0]   # MHA: per head, ties lower
