"""Host side of the head classifier's C ABI, without a GPU: the group
ranking (sparse_decode_classify_heads) against the oracle on the same ER
arrays, bit for bit, and argument checks that return before any CUDA call."""

import math

import numpy as np
import pytest

import oracle as O


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (16, 2), (64, 8), (4, 1)])
@pytest.mark.parametrize("seed", range(4))
def test_classify_heads_matches_the_oracle(Hq, Hkv, seed):
    from head_wise_sparse_02_b200 import sparse_decode as sd
    rng = np.random.default_rng(seed)
    er = rng.uniform(1.0, 128.0, size=Hq)
    if seed % 2:                                     # exact ties between groups
        G = Hq // Hkv
        for g in range(1, Hkv, 2):
            er[g * G:(g + 1) * G] = er[(g - 1) * G:g * G]
    if seed == 3:
        er[0] = math.nan
    for n_ret in range(Hkv + 1):
        got = sd.sparse_decode_classify_heads(er.tolist(), Hkv, n_ret)
        want = O.classify_groups(er, Hkv, n_ret).tolist()
        assert got == want, (Hq, Hkv, n_ret)


def test_classify_heads_rejects_bad_arguments():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    with pytest.raises(sd.SparseDecodeError):
        sd.sparse_decode_classify_heads([1.0] * 8, 3, 1)             # Hkv does not divide Hq
    with pytest.raises(sd.SparseDecodeError):
        sd.sparse_decode_classify_heads([1.0] * 8, 4, 5)             # more groups than exist
    with pytest.raises(sd.SparseDecodeError):
        sd.sparse_decode_classify_heads([1.0] * 8, 4, -1)


def test_effective_rank_argument_checks_before_any_cuda_call():
    import ctypes
    from head_wise_sparse_02_b200 import sparse_decode as sd
    n = ctypes.c_size_t()
    assert sd.LIB.sparse_decode_head_er_workspace_size(2, 32, 8, 128, ctypes.byref(n)) == sd.SD_OK
    assert n.value == 2 * 40 * 128 * 128 * 8
    assert sd.LIB.sparse_decode_head_er_workspace_size(2, 32, 8, 96, ctypes.byref(n)) == sd.SD_ERR_UNSUPPORTED
    assert sd.LIB.sparse_decode_head_er_workspace_size(2, 30, 8, 128, ctypes.byref(n)) == sd.SD_ERR_INVALID_ARG
    f = sd.LIB.sparse_decode_head_effective_rank
    p = ctypes.c_void_p(16)
    assert f(p, p, 1, 4080, 32, 8, 128, p, p, 1 << 30, None) == sd.SD_ERR_UNSUPPORTED   # d_model % 32
    assert f(None, p, 1, 4096, 32, 8, 128, p, p, 1 << 30, None) == sd.SD_ERR_INVALID_ARG
    assert f(p, p, 1, 4096, 32, 8, 128, p, None, 0, None) == sd.SD_ERR_WORKSPACE
    assert f(ctypes.c_void_p(18), p, 1, 4096, 32, 8, 128, p, p, 1 << 30, None) == sd.SD_ERR_INVALID_ARG
    assert f(None, None, 0, 4096, 32, 8, 128, None, None, 0, None) == sd.SD_OK          # no layers: no-op
