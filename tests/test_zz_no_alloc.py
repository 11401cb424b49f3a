"""sparse_decode_attend_noalloc (attend on the library's built-in scratch)
against sparse_decode_attend with a caller workspace and against the float64
oracle, through the C ABI.  Collected last on purpose: it must also pass
after everything else ran in the same process."""

import numpy as np
import pytest
import torch

import oracle as O
from oracle.workload_inputs import oracle_config, oracle_inputs
from tests.helpers import assert_out_close, gpu_sets, make_step
from workloads import make_workload

pytestmark = pytest.mark.gpu


def test_noalloc_attend_matches_attend_twice_in_a_row():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    w = make_workload("llama3_8b_topp", "cuda", B=3, N=4000, window=300, permute=True)
    st = make_step(w)
    st.select(w.q_pre)
    ref = st.attend(w.q).clone()
    torch.cuda.synchronize()
    assert st.error_word() == 0
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        sd.sparse_decode_attend_noalloc(st.sd.handle, w.q, st.k_cache, st.v_cache, st.page_table,
                                        st.seq_lens, st.sel_idx, st.sel_count, out)
        torch.cuda.synchronize()
        assert st.error_word() == 0
        got, want = out.cpu().numpy(), ref.cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}: unwritten outputs"
        for b in range(w.batch):
            for h in range(w.num_q_heads):
                assert_out_close(got[b, h], want[b, h], f"call {call} b={b} h={h}")
    # and against the oracle: exact attention over the same selected sets
    # (retrieval heads) and over sinks + window (local heads)
    retr = [(b, h) for b in range(w.batch) for h in range(w.num_q_heads) if w.head_is_retrieval[h]]
    ref = O.decode_reference(oracle_config(w), **oracle_inputs(w), sets_override=gpu_sets(st, w, retr))
    for (b, h), o in ref.out.items():
        assert_out_close(got[b, h], o, f"oracle b={b} h={h}")
    st.close()


def test_noalloc_attend_rejects_bad_arguments_before_launching():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    w = make_workload("tiny_ref", "cuda")
    st = make_step(w)
    out = torch.empty((1, 4, 64), dtype=torch.float32, device="cuda")
    lib, h = sd.LIB, st.sd.handle
    args = [w.q.data_ptr(), st.k_cache.data_ptr(), st.v_cache.data_ptr(), st.page_table.data_ptr(),
            st.seq_lens.data_ptr()]
    sel = [st.sel_idx.data_ptr(), st.sel_count.data_ptr(), st.sel_idx.shape[-1], out.data_ptr(), None]
    assert lib.sparse_decode_attend_noalloc(h, *args, 2, *sel) == sd.SD_ERR_INVALID_ARG      # batch > max_batch
    assert lib.sparse_decode_attend_noalloc(h, *args, -1, *sel) == sd.SD_ERR_INVALID_ARG
    assert lib.sparse_decode_attend_noalloc(h, None, *args[1:], 1, *sel) == sd.SD_ERR_INVALID_ARG
    assert lib.sparse_decode_attend_noalloc(h, *args, 1, None, *sel[1:]) == sd.SD_ERR_INVALID_ARG
    assert lib.sparse_decode_attend_noalloc(h, *args, 0, *sel) == sd.SD_OK                    # empty batch
    st.close()


def test_noalloc_attend_rejects_a_batch_beyond_its_scratch():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    # 16 heads, all retrieval, 2^20 positions, 16 sequences: the union lists
    # alone take far more than the built-in scratch; nothing is launched
    proj = torch.zeros((2, 64, 16), dtype=torch.bfloat16, device="cuda")
    h = sd.sparse_decode_init(num_q_heads=16, num_kv_heads=2, head_dim=64, head_is_retrieval=[1] * 16,
                              num_pages=8, max_batch=16, max_pages_per_seq=65536, proj=proj)
    try:
        small = torch.zeros(16, dtype=torch.int32, device="cuda")
        q = torch.zeros((16, 16, 64), dtype=torch.bfloat16, device="cuda")
        kv = torch.zeros((8, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
        sel = torch.zeros((16, 16, 4), dtype=torch.int32, device="cuda")
        cnt = torch.zeros((16, 16), dtype=torch.int32, device="cuda")
        out = torch.zeros((16, 16, 64), dtype=torch.float32, device="cuda")
        with pytest.raises(sd.SparseDecodeError) as e:
            sd.sparse_decode_attend_noalloc(h, q, kv, kv, small.view(16, 1).expand(16, 1).contiguous(), small,
                                            sel, cnt, out)
        assert e.value.status == sd.SD_ERR_WORKSPACE
        assert "built-in scratch" in str(e.value)
    finally:
        sd.sparse_decode_destroy(h)
