"""GPU parity of the data-free head classifier (through the C ABI) against the
float64 oracle ([AoH] Methodology §1-§4).

Tolerances, from the arithmetic: the CUDA path is float64 throughout (Gram
sums of exact bf16 products, Cholesky, Jacobi converged to head_dim * eps), so
its ER agrees with the oracle's direct SVD of M_h to about 1e-12 relative;
1e-9 is asserted.  Against the oracle's eigenvalue route (C_h, used where the
d_model x d_model SVD is too slow), whose small singular values carry only
sqrt(eps) relative accuracy, 1e-7 is asserted.  Classifications (integers)
must match exactly; the synthetic groups are well separated.
"""

import numpy as np
import pytest
import torch

import oracle as O
from workloads import make_projections

pytestmark = pytest.mark.gpu

REL_DIRECT = 1e-9
REL_EIG = 1e-7


def _er(w_q, w_k, Hq, Hkv, D):
    from head_wise_sparse_02_b200 import sparse_decode as sd
    out = sd.sparse_decode_head_effective_rank(w_q, w_k, Hq, Hkv, D)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("L,d_model,Hq,Hkv,D", [
    (2, 256, 8, 2, 64),
    (1, 256, 4, 4, 128),
    (2, 192, 16, 2, 128),
    (1, 512, 8, 8, 64),
])
def test_effective_rank_against_the_direct_svd(L, d_model, Hq, Hkv, D):
    p = make_projections("cuda", seed=3, num_layers=L, d_model=d_model, num_q_heads=Hq, num_kv_heads=Hkv,
                         head_dim=D)
    got = _er(p.w_q, p.w_k, Hq, Hkv, D)
    for layer in range(L):
        want = O.layer_effective_ranks(_np(p.w_q[layer]), _np(p.w_k[layer]), Hq, Hkv, D, route="direct")
        assert np.allclose(got[layer], want, rtol=REL_DIRECT, atol=0), (layer, got[layer], want)


def _blocks(Hq, Hkv, D, d_model, wq_head, wk_head):
    w_q = torch.zeros((1, Hq * D, d_model), dtype=torch.bfloat16)
    w_k = torch.zeros((1, Hkv * D, d_model), dtype=torch.bfloat16)
    for h in range(Hq):
        w_q[0, h * D:(h + 1) * D] = wq_head(h)
    for g in range(Hkv):
        w_k[0, g * D:(g + 1) * D] = wk_head(g)
    return w_q.cuda(), w_k.cuda()


def test_structured_spectra():
    """Rank one (rows of W_Q are power-of-two multiples of one bf16 row, so
    the rank is exactly one after rounding), a zero block (no spectrum: ER 1),
    and blocks with nearly equal singular values, each against the direct SVD."""
    Hq, Hkv, D, d_model = 4, 2, 64, 128
    g = torch.Generator().manual_seed(5)
    u = torch.randn(d_model, generator=g).to(torch.bfloat16)
    scales = torch.tensor([2.0 ** (i % 7 - 3) for i in range(D)])
    dense = torch.randn((Hkv * D, d_model), generator=g).to(torch.bfloat16)
    eye = torch.zeros((D, d_model))
    eye[:, :D] = torch.eye(D)

    def wq_head(h):
        if h == 0:
            return (scales[:, None] * u[None, :].float()).to(torch.bfloat16)
        if h == 1:
            return torch.zeros((D, d_model), dtype=torch.bfloat16)
        if h == 2:
            return (3.0 * eye).to(torch.bfloat16)
        return torch.randn((D, d_model), generator=g).to(torch.bfloat16)

    def wk_head(gk):
        return eye.to(torch.bfloat16) if gk == 1 else dense[gk * D:(gk + 1) * D]

    w_q, w_k = _blocks(Hq, Hkv, D, d_model, wq_head, wk_head)
    got = _er(w_q, w_k, Hq, Hkv, D)[0]
    want = O.layer_effective_ranks(_np(w_q[0]), _np(w_k[0]), Hq, Hkv, D, route="direct")
    assert got[0] == pytest.approx(1.0, abs=1e-9) and want[0] == pytest.approx(1.0, abs=1e-9)
    assert got[1] == 1.0 and want[1] == 1.0
    assert got[3] == pytest.approx(want[3], rel=REL_DIRECT)
    assert got[2] == pytest.approx(want[2], rel=REL_DIRECT)


def test_llama3_8b_shapes_two_layers_and_classification():
    """Two layers at the full shape (d_model 4096, 32 / 8 heads of 128): every
    head against the eigenvalue route, one head against the direct SVD, and
    the group classification at half the groups retrieval (the AoH page's 50%
    setting) equal to the oracle's."""
    from head_wise_sparse_02_b200 import sparse_decode as sd
    p = make_projections("cuda", seed=8, num_layers=2)
    got = _er(p.w_q, p.w_k, 32, 8, 128)
    for layer in range(2):
        wq, wk = _np(p.w_q[layer]), _np(p.w_k[layer])
        want = O.layer_effective_ranks(wq, wk, 32, 8, 128, route="sylvester")
        assert np.allclose(got[layer], want, rtol=REL_EIG, atol=0), layer
        assert sd.sparse_decode_classify_heads(got[layer], 8, 4) == O.classify_groups(want, 8, 4).tolist()
    direct = O.effective_rank_of_spectrum(O.singular_values_direct(O.head_block(_np(p.w_q[1]), 5, 128),
                                                                   O.head_block(_np(p.w_k[1]), 1, 128)))
    assert got[1][5] == pytest.approx(direct, rel=REL_DIRECT)


def test_full_model_sampled_heads():
    """All 32 layers in one call (the launch the bench times), 24 sampled
    heads against the eigenvalue route."""
    p = make_projections("cuda", seed=9, num_layers=32)
    got = _er(p.w_q, p.w_k, 32, 8, 128)
    rng = np.random.default_rng(0)
    for _ in range(24):
        layer, h = int(rng.integers(32)), int(rng.integers(32))
        wq = O.head_block(_np(p.w_q[layer]), h, 128)
        wk = O.head_block(_np(p.w_k[layer]), h // 4, 128)
        want = O.effective_rank_of_spectrum(O.singular_values_sylvester(wq, wk))
        assert got[layer][h] == pytest.approx(want, rel=REL_EIG), (layer, h)
    del p
    torch.cuda.empty_cache()


def test_workspace_too_small_is_rejected_on_the_host():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    p = make_projections("cuda", seed=1, num_layers=1, d_model=256, num_q_heads=4, num_kv_heads=2, head_dim=64)
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(sd.SparseDecodeError) as e:
        sd.sparse_decode_head_effective_rank(p.w_q, p.w_k, 4, 2, 64, workspace=small)
    assert e.value.status == sd.SD_ERR_WORKSPACE
