"""Host-only checks of the C-ABI library: it loads without a GPU, exports
every function that include/*.h declares, and rejects bad arguments on the
host before touching CUDA."""

import ctypes
import glob
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"\b(sparse_decode_\w+)\s*\(", text))
    return names


def test_header_declares_the_boundary_calls():
    names = _declared()
    for n in ["sparse_decode_init", "sparse_decode_index_keys", "sparse_decode_select",
              "sparse_decode_attend", "sparse_decode_workspace_size", "sparse_decode_destroy",
              "sparse_decode_error_word", "sparse_decode_attend_noalloc"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    lib = ctypes.CDLL(sd.LIB_PATH)
    missing = [n for n in sorted(_declared()) if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    assert sd.status_string(sd.SD_OK) == "ok"
    assert "workspace" in sd.status_string(sd.SD_ERR_WORKSPACE)
    assert sd.status_string(sd.SD_ERR_HOST_MEMORY) == "host allocation failed"
    assert sd.status_string(99) == "unknown status"


def _cfg(sd, **over):
    retr = (ctypes.c_int32 * 4)(1, 1, 0, 0)
    base = dict(num_q_heads=4, num_kv_heads=2, head_dim=64, index_dim=16, page_size=16, num_pages=32,
                head_is_retrieval=ctypes.cast(retr, ctypes.POINTER(ctypes.c_int32)), window=64,
                num_sinks=4, mode=sd.SD_TOP_P, top_p=0.9, top_k=0, top_k_frac=0.0, attn_scale=0.0,
                index_scale=0.0, max_batch=1, max_pages_per_seq=32)
    base.update(over)
    return sd.SdConfig(**base), retr


@pytest.mark.parametrize("over,status", [
    (dict(head_dim=96), 2),
    (dict(index_dim=8), 2),
    (dict(page_size=32), 2),
    (dict(num_q_heads=5), 1),
    (dict(num_q_heads=64, num_kv_heads=2), 2),
    (dict(top_p=0.0), 1),
    (dict(top_p=1.5), 1),
    (dict(mode=1, top_k=0, top_k_frac=0.0), 1),
    (dict(mode=1, top_k=-3), 1),
    (dict(mode=7), 1),
    (dict(window=-1), 1),
    (dict(max_batch=0), 1),
    (dict(num_pages=0), 1),
])
def test_init_rejects_bad_configs_before_any_cuda_call(over, status):
    from head_wise_sparse_02_b200 import sparse_decode as sd
    cfg, keep = _cfg(sd, **over)
    out = ctypes.c_void_p(123)
    st = sd.LIB.sparse_decode_init(ctypes.byref(cfg), ctypes.c_void_p(1), ctypes.byref(out))
    assert st == status
    assert out.value is None


def test_null_arguments():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    out = ctypes.c_void_p()
    assert sd.LIB.sparse_decode_init(None, None, ctypes.byref(out)) == sd.SD_ERR_INVALID_ARG
    assert sd.LIB.sparse_decode_init(None, None, None) == sd.SD_ERR_INVALID_ARG
    n = ctypes.c_size_t()
    assert sd.LIB.sparse_decode_workspace_size(None, 1, ctypes.byref(n)) == sd.SD_ERR_INVALID_ARG
    assert sd.LIB.sparse_decode_select(None, None, None, None, None, 1, None, None, 1, None, 0, None) == sd.SD_ERR_INVALID_ARG
    assert sd.LIB.sparse_decode_attend_noalloc(None, None, None, None, None, None, 1, None, None, 1, None,
                                               None) == sd.SD_ERR_INVALID_ARG
    assert sd.LIB.sparse_decode_attend(None, None, None, None, None, None, 1, None, None, 1, None, None, 0,
                                       None) == sd.SD_ERR_INVALID_ARG
    assert sd.LIB.sparse_decode_index_keys(None, None, None, 1, None, None) == sd.SD_ERR_INVALID_ARG
    assert sd.LIB.sparse_decode_num_retrieval_heads(None) == 0
    assert sd.LIB.sparse_decode_last_error(None) == b""
    sd.LIB.sparse_decode_destroy(None)


def test_binding_fails_loudly_without_the_library(tmp_path):
    from head_wise_sparse_02_b200 import sparse_decode as sd
    with pytest.raises(ImportError):
        sd._load(str(tmp_path / "missing.so"))


def test_binding_checks_selection_shapes(monkeypatch):
    """The library addresses selection rows through raw pointers, so the binding
    checks their extents against the batch and the retrieval heads."""
    from head_wise_sparse_02_b200 import sparse_decode as sd
    monkeypatch.setattr(sd, "sparse_decode_num_retrieval_heads", lambda ctx: 4)
    ok_idx, ok_cnt = torch.zeros((3, 4, 10), dtype=torch.int32), torch.zeros((3, 4), dtype=torch.int32)
    sd._check_sets(1, ok_idx, ok_cnt, 3)
    sd._check_sets(1, ok_idx, ok_cnt, 2)            # rows beyond the batch are not read
    for idx, cnt in [(torch.zeros((3, 5, 10), dtype=torch.int32), ok_cnt),
                     (torch.zeros((2, 4, 10), dtype=torch.int32), ok_cnt),
                     (torch.zeros((3, 40), dtype=torch.int32), ok_cnt),
                     (ok_idx, torch.zeros((3, 3), dtype=torch.int32)),
                     (ok_idx, None)]:
        with pytest.raises(ValueError):
            sd._check_sets(1, idx, cnt, 3)
    monkeypatch.setattr(sd, "sparse_decode_num_retrieval_heads", lambda ctx: 0)
    sd._check_sets(1, None, None, 3)                 # no retrieval heads: nothing is read


def test_binding_rejects_an_unknown_mode():
    from head_wise_sparse_02_b200 import sparse_decode as sd
    with pytest.raises(ValueError):
        sd.sparse_decode_init(num_q_heads=4, num_kv_heads=2, head_dim=64, head_is_retrieval=[1] * 4,
                              num_pages=4, max_batch=1, max_pages_per_seq=4, proj=None, mode="topk")
