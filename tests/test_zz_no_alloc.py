"""sparse_decode_attend_noalloc (attend on the library's built-in scratch)
against sparse_decode_attend with a caller workspace, through the C ABI.
Collected last on purpose: it must also pass after everything else ran in
the same process."""

import numpy as np
import pytest
import torch

from tests.helpers import assert_out_close, make_step
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
