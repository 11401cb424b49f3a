"""Pins of the head-wise prefill oracle ([RTP] Methodology §1, [AoH]
Methodology §4): retrieval heads against torch's float64 causal
scaled-dot-product attention, local heads against the same routine with a
boolean band mask built by broadcasting, chunk invariance, and the one-token
chunk against the decode oracle.  CPU only."""

import math

import numpy as np
import pytest
import torch

import oracle as O


def _setup(N, Hq=4, Hkv=2, d=16, window=5, sinks=2, retr=(1, 0, 1, 0), seed=0, perm=False):
    rng = np.random.default_rng(seed)
    pages = math.ceil(N / 16)
    K = rng.normal(size=(pages, Hkv, 16, d))
    V = rng.normal(size=(pages, Hkv, 16, d))
    pt = np.arange(pages)
    if perm:
        pt = rng.permutation(pages)
    cfg = O.OracleConfig(num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, index_dim=16, page_size=16,
                         head_is_retrieval=list(retr), window=window, num_sinks=sinks, mode="top_p")
    return cfg, K, V, pt[None, :], rng


def _contiguous(cache, pt_row, n, g):
    return O.gather_rows(cache, pt_row, n, g, 16)


@pytest.mark.parametrize("N,window,sinks", [(1, 5, 2), (37, 5, 2), (40, 0, 3), (33, 64, 0), (50, 1, 0)])
def test_full_prefill_against_torch_sdpa(N, window, sinks):
    cfg, K, V, pt, rng = _setup(N, window=window, sinks=sinks, perm=True)
    q = rng.normal(size=(N, 4, 16))
    got = O.prefill_reference(cfg, q, K, V, pt, [N], [0, N])
    a = cfg.scales()[0]
    for h in range(4):
        g = h // 2
        Kc = torch.tensor(_contiguous(K, pt[0], N, g))
        Vc = torch.tensor(_contiguous(V, pt[0], N, g))
        qh = torch.tensor(q[:, h])
        if cfg.head_is_retrieval[h]:
            ref = torch.nn.functional.scaled_dot_product_attention(qh[None], Kc[None], Vc[None], is_causal=True,
                                                                   scale=a)[0]
        else:
            i = torch.arange(N)[:, None]
            j = torch.arange(N)[None, :]
            allowed = (j <= i) & ((j < sinks) | (j > i - window))
            ref = torch.nn.functional.scaled_dot_product_attention(qh[None], Kc[None], Vc[None],
                                                                   attn_mask=allowed[None], scale=a)[0]
        for r in range(N):
            assert np.allclose(got[(r, h)], ref[r].numpy(), rtol=1e-12, atol=1e-12), (h, r)


def test_chunked_prefill_equals_the_full_one():
    N = 45
    cfg, K, V, pt, rng = _setup(N, window=7, sinks=1)
    q = rng.normal(size=(N, 4, 16))
    full = O.prefill_reference(cfg, q, K, V, pt, [N], [0, N])
    for s in (0, 16, 44):
        part = O.prefill_reference(cfg, q[s:], K, V, pt, [N], [0, N - s])
        for (r, h), o in part.items():
            assert np.array_equal(o, full[(r + s, h)])


def test_one_token_chunk_equals_the_decode_output():
    """A chunk of one token is a decode step with every token selected for the
    retrieval heads (top-p 1) and the local set for the local heads."""
    N = 70
    cfg, K, V, pt, rng = _setup(N, window=9, sinks=3, seed=4)
    q = rng.normal(size=(1, 4, 16))
    got = O.prefill_reference(cfg, q, K, V, pt, [N], [0, 1])
    cfg.top_p = 1.0
    ref = O.decode_reference(cfg, np.zeros((2, 16, 16)), q, q, K, V, pt, [N])
    for h in range(4):
        assert np.allclose(got[(0, h)], ref.out[(0, h)], rtol=1e-13, atol=1e-13)


def test_two_sequences_packed():
    cfg, K, V, pt, rng = _setup(64, window=4, sinks=1, seed=6)
    pt2 = np.concatenate([pt, pt], axis=0)
    q = rng.normal(size=(10, 4, 16))
    got = O.prefill_reference(cfg, q, K, V, pt2, [30, 64], [0, 3, 10])
    one = O.prefill_reference(cfg, q[3:], K, V, pt2[1:], [64], [0, 7])
    for (r, h), o in one.items():
        assert np.array_equal(got[(r + 3, h)], o)
    # sequence 0's three queries sit at positions 27, 28, 29
    first = O.prefill_reference(cfg, q[:3], K, V, pt2[:1], [30], [0, 3])
    for (r, h), o in first.items():
        assert np.array_equal(got[(r, h)], o)
