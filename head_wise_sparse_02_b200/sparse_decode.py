"""Thin ctypes binding of libsparsedecode.so (see include/sparse_decode.h).

Argument marshalling only: every step of the decode path runs in the CUDA
library.  Functions carry the C names and take torch tensors (for device
memory and streams); they check dtype, device and contiguity, pass raw
pointers and raise :class:`SparseDecodeError` on a non-zero status.  There is
no fallback: if the library is missing or fails to load, importing this
module raises.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_size_t, c_uint32, c_void_p
from typing import Optional, Sequence

import torch

LIB_PATH = os.environ.get("SPARSE_DECODE_LIB") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "lib", "libsparsedecode.so")

SD_OK, SD_ERR_INVALID_ARG, SD_ERR_UNSUPPORTED, SD_ERR_WORKSPACE, SD_ERR_CUDA, SD_ERR_TIMEOUT, \
    SD_ERR_DEVICE_DATA, SD_ERR_HOST_MEMORY = range(8)
SD_TOP_P, SD_TOP_K = 0, 1
SD_EBIT_PAGE, SD_EBIT_SEQLEN, SD_EBIT_SEL, SD_EBIT_SLOT, SD_EBIT_TIMEOUT = 1, 2, 4, 8, 16


class SparseDecodeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


class SdConfig(ctypes.Structure):
    _fields_ = [
        ("num_q_heads", c_int), ("num_kv_heads", c_int), ("head_dim", c_int), ("index_dim", c_int),
        ("page_size", c_int), ("num_pages", c_int), ("head_is_retrieval", POINTER(c_int32)),
        ("window", c_int), ("num_sinks", c_int), ("mode", c_int), ("top_p", c_float),
        ("top_k", c_int), ("top_k_frac", c_float), ("attn_scale", c_float),
        ("index_scale", c_float), ("max_batch", c_int), ("max_pages_per_seq", c_int),
    ]


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m head_wise_sparse_02_b200.build`")
    lib = ctypes.CDLL(path)
    P = c_void_p
    sig = {
        "sparse_decode_init": (c_int, [POINTER(SdConfig), P, POINTER(P)]),
        "sparse_decode_workspace_size": (c_int, [P, c_int, POINTER(c_size_t)]),
        "sparse_decode_index_keys": (c_int, [P, P, P, c_int, P, P]),
        "sparse_decode_select": (c_int, [P, P, P, P, P, c_int, P, P, c_int, P, c_size_t, P]),
        "sparse_decode_select_exact": (c_int, [P, P, P, P, P, c_int, P, P, c_int, P, c_size_t, P]),
        "sparse_decode_attend": (c_int, [P, P, P, P, P, P, c_int, P, P, c_int, P, P, c_size_t, P]),
        "sparse_decode_select_attend": (c_int, [P, P, P, P, P, P, P, P, c_int, P, P, c_int, P, P, c_size_t, P]),
        "sparse_decode_attend_noalloc": (c_int, [P, P, P, P, P, P, c_int, P, P, c_int, P, P]),
        "sparse_decode_error_word": (c_int, [P, P, POINTER(c_uint32)]),
        "sparse_decode_attend_split": (c_int, [P, P, P, P, P, P, P, P, c_int, P, P, c_int, P, P, c_size_t, P]),
        "sparse_decode_select_attend_split": (c_int, [P, P, P, P, P, P, P, P, P, P, c_int, P, P, c_int, P, P,
                                                      c_size_t, P]),
        "sparse_decode_local_append": (c_int, [P, P, P, P, P, c_int, P, P, P]),
        "sparse_decode_prefill": (c_int, [P, P, P, P, P, P, P, c_int, c_int, P, P]),
        "sparse_decode_num_retrieval_groups": (c_int, [P]),
        "sparse_decode_num_local_groups": (c_int, [P]),
        "sparse_decode_head_er_workspace_size": (c_int, [c_int, c_int, c_int, c_int, POINTER(c_size_t)]),
        "sparse_decode_head_effective_rank": (c_int, [P, P, c_int, c_int, c_int, c_int, c_int, P, P, c_size_t,
                                                      P]),
        "sparse_decode_classify_heads": (c_int, [P, c_int, c_int, c_int, P]),
        "sparse_decode_num_retrieval_heads": (c_int, [P]),
        "sparse_decode_testing_stall_prefill": (None, [c_int]),
        "sparse_decode_last_error": (c_char_p, [P]),
        "sparse_decode_status_string": (c_char_p, [c_int]),
        "sparse_decode_destroy": (None, [P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def status_string(status: int) -> str:
    return LIB.sparse_decode_status_string(status).decode()


def _check(status: int, ctx: Optional[int] = None) -> None:
    if status != SD_OK:
        msg = status_string(status)
        if ctx:
            detail = LIB.sparse_decode_last_error(ctx).decode()
            if detail:
                msg = f"{msg}: {detail}"
        raise SparseDecodeError(status, msg)


def _ptr(t: Optional[torch.Tensor], dtype: torch.dtype, name: str) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _check_sets(ctx: int, sel_idx, sel_count, batch: int) -> None:
    """With retrieval heads, sel_idx must be [>= B, H_ret, stride] and sel_count
    [>= B, H_ret]: the library addresses row (b, i) at (b * H_ret + i) * stride
    through raw pointers and cannot see the tensors' extents.  Without
    retrieval heads it reads neither."""
    h_ret = sparse_decode_num_retrieval_heads(ctx) if ctx else 0
    if h_ret == 0:
        return
    if sel_idx is None or sel_count is None:
        raise ValueError("sel_idx and sel_count are required with retrieval heads")
    if sel_idx.dim() != 3 or sel_idx.shape[0] < batch or sel_idx.shape[1] != h_ret:
        raise ValueError(f"sel_idx must be [B >= {batch}, H_ret = {h_ret}, stride], got {tuple(sel_idx.shape)}")
    if sel_count.dim() != 2 or sel_count.shape[0] < batch or sel_count.shape[1] != h_ret:
        raise ValueError(f"sel_count must be [B >= {batch}, H_ret = {h_ret}], got {tuple(sel_count.shape)}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ------------------------------------------------------------ C-named calls

def sparse_decode_init(*, num_q_heads: int, num_kv_heads: int, head_dim: int,
                       head_is_retrieval: Sequence[int], num_pages: int, max_batch: int,
                       max_pages_per_seq: int, proj: torch.Tensor, window: int = 0,
                       num_sinks: int = 0, mode: str = "top_p", top_p: float = 0.9,
                       top_k: int = 0, top_k_frac: float = 0.0, attn_scale: float = 0.0,
                       index_scale: float = 0.0, index_dim: int = 16, page_size: int = 16) -> int:
    """Create a context (returns the opaque handle)."""
    if mode not in ("top_p", "top_k"):
        raise ValueError(f"mode must be 'top_p' or 'top_k', got {mode!r}")
    retr = (c_int32 * num_q_heads)(*[int(x) for x in head_is_retrieval])
    cfg = SdConfig(num_q_heads, num_kv_heads, head_dim, index_dim, page_size, num_pages,
                   ctypes.cast(retr, POINTER(c_int32)), window, num_sinks,
                   SD_TOP_P if mode == "top_p" else SD_TOP_K, top_p, top_k, top_k_frac,
                   attn_scale, index_scale, max_batch, max_pages_per_seq)
    out = c_void_p()
    with torch.cuda.device(proj.device):
        _check(LIB.sparse_decode_init(ctypes.byref(cfg), _ptr(proj, torch.bfloat16, "proj"), ctypes.byref(out)))
    return out.value


def sparse_decode_workspace_size(ctx: int, batch: int) -> int:
    n = c_size_t()
    _check(LIB.sparse_decode_workspace_size(ctx, batch, ctypes.byref(n)), ctx)
    return n.value


def sparse_decode_index_keys(ctx: int, k_pre: torch.Tensor, slots: torch.Tensor,
                             index_cache: torch.Tensor, stream=None) -> None:
    _check(LIB.sparse_decode_index_keys(ctx, _ptr(k_pre, torch.bfloat16, "k_pre"),
                                        _ptr(slots, torch.int32, "slots"), int(slots.numel()),
                                        _ptr(index_cache, torch.bfloat16, "index_cache"),
                                        _stream(stream)), ctx)


def sparse_decode_select(ctx: int, q_pre, index_cache, page_table, seq_lens, sel_idx, sel_count,
                         workspace, stream=None) -> None:
    _check_sets(ctx, sel_idx, sel_count, int(seq_lens.numel()))
    _check(LIB.sparse_decode_select(
        ctx, _ptr(q_pre, torch.bfloat16, "q_pre"), _ptr(index_cache, torch.bfloat16, "index_cache"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        int(seq_lens.numel()), _ptr(sel_idx, torch.int32, "sel_idx"),
        _ptr(sel_count, torch.int32, "sel_count"), int(sel_idx.shape[-1]),
        _ptr(workspace, torch.uint8, "workspace"), int(workspace.numel()), _stream(stream)), ctx)


def sparse_decode_select_exact(ctx: int, q, k_cache, page_table, seq_lens, sel_idx, sel_count, workspace,
                               stream=None) -> None:
    """Sets chosen by the exact attention logits (post-RoPE q against the K cache)."""
    _check_sets(ctx, sel_idx, sel_count, int(seq_lens.numel()))
    _check(LIB.sparse_decode_select_exact(
        ctx, _ptr(q, torch.bfloat16, "q"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(page_table, torch.int32, "page_table"), _ptr(seq_lens, torch.int32, "seq_lens"),
        int(seq_lens.numel()), _ptr(sel_idx, torch.int32, "sel_idx"),
        _ptr(sel_count, torch.int32, "sel_count"), int(sel_idx.shape[-1]),
        _ptr(workspace, torch.uint8, "workspace"), int(workspace.numel()), _stream(stream)), ctx)


def sparse_decode_attend(ctx: int, q, k_cache, v_cache, page_table, seq_lens, sel_idx, sel_count,
                         out, workspace, stream=None) -> None:
    _check_sets(ctx, sel_idx, sel_count, int(seq_lens.numel()))
    stride = int(sel_idx.shape[-1]) if sel_idx is not None else 0
    _check(LIB.sparse_decode_attend(
        ctx, _ptr(q, torch.bfloat16, "q"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(seq_lens.numel()),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_count, torch.int32, "sel_count"), stride,
        _ptr(out, torch.float32, "out"), _ptr(workspace, torch.uint8, "workspace"),
        int(workspace.numel()), _stream(stream)), ctx)


def sparse_decode_select_attend(ctx: int, q_pre, q, index_cache, k_cache, v_cache, page_table, seq_lens,
                                sel_idx, sel_count, out, workspace, stream=None) -> None:
    """select followed by attend on the same sets, in one call."""
    _check_sets(ctx, sel_idx, sel_count, int(seq_lens.numel()))
    stride = int(sel_idx.shape[-1]) if sel_idx is not None else 0
    _check(LIB.sparse_decode_select_attend(
        ctx, _ptr(q_pre, torch.bfloat16, "q_pre"), _ptr(q, torch.bfloat16, "q"),
        _ptr(index_cache, torch.bfloat16, "index_cache"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(seq_lens.numel()),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_count, torch.int32, "sel_count"), stride,
        _ptr(out, torch.float32, "out"), _ptr(workspace, torch.uint8, "workspace"), int(workspace.numel()),
        _stream(stream)), ctx)


def _check_local(ctx: int, local_k, local_v, rows_needed: int) -> None:
    """The compacted local caches are addressed through raw pointers: check that
    both hold at least `rows_needed` sequences of [Lg, num_sinks + window, d]."""
    for name, t in (("local_k", local_k), ("local_v", local_v)):
        if t is None:
            continue
        if t.dim() != 4 or t.shape[0] < rows_needed or t.shape[1] != sparse_decode_num_local_groups(ctx):
            raise ValueError(f"{name} must be [>= {rows_needed}, Lg = {sparse_decode_num_local_groups(ctx)}, "
                             f"num_sinks + window, d], got {tuple(t.shape)}")


def sparse_decode_attend_split(ctx: int, q, k_ret, v_ret, local_k, local_v, page_table, seq_lens, sel_idx,
                               sel_count, out, workspace, stream=None) -> None:
    """attend on the split layout: paged caches of the retrieval groups only,
    compacted sink + window caches of the local groups."""
    _check_sets(ctx, sel_idx, sel_count, int(seq_lens.numel()))
    _check_local(ctx, local_k, local_v, int(seq_lens.numel()))
    stride = int(sel_idx.shape[-1]) if sel_idx is not None else 0
    _check(LIB.sparse_decode_attend_split(
        ctx, _ptr(q, torch.bfloat16, "q"), _ptr(k_ret, torch.bfloat16, "k_ret"),
        _ptr(v_ret, torch.bfloat16, "v_ret"), _ptr(local_k, torch.bfloat16, "local_k"),
        _ptr(local_v, torch.bfloat16, "local_v"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(seq_lens.numel()),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_count, torch.int32, "sel_count"), stride,
        _ptr(out, torch.float32, "out"), _ptr(workspace, torch.uint8, "workspace"),
        int(workspace.numel()), _stream(stream)), ctx)


def sparse_decode_select_attend_split(ctx: int, q_pre, q, index_cache, k_ret, v_ret, local_k, local_v,
                                      page_table, seq_lens, sel_idx, sel_count, out, workspace,
                                      stream=None) -> None:
    """select_attend on the split layout."""
    _check_sets(ctx, sel_idx, sel_count, int(seq_lens.numel()))
    _check_local(ctx, local_k, local_v, int(seq_lens.numel()))
    stride = int(sel_idx.shape[-1]) if sel_idx is not None else 0
    _check(LIB.sparse_decode_select_attend_split(
        ctx, _ptr(q_pre, torch.bfloat16, "q_pre"), _ptr(q, torch.bfloat16, "q"),
        _ptr(index_cache, torch.bfloat16, "index_cache"), _ptr(k_ret, torch.bfloat16, "k_ret"),
        _ptr(v_ret, torch.bfloat16, "v_ret"), _ptr(local_k, torch.bfloat16, "local_k"),
        _ptr(local_v, torch.bfloat16, "local_v"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(seq_lens.numel()),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_count, torch.int32, "sel_count"), stride,
        _ptr(out, torch.float32, "out"), _ptr(workspace, torch.uint8, "workspace"), int(workspace.numel()),
        _stream(stream)), ctx)


def sparse_decode_local_append(ctx: int, k_new, v_new, seq_ids, positions, local_k, local_v, max_batch: int,
                               stream=None) -> None:
    """Copy new tokens' keys and values ([T, Hkv, d]) of the local groups into
    the compacted caches ([max_batch, Lg, num_sinks + window, d])."""
    _check_local(ctx, local_k, local_v, max_batch)
    _check(LIB.sparse_decode_local_append(
        ctx, _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        _ptr(seq_ids, torch.int32, "seq_ids"), _ptr(positions, torch.int32, "positions"), int(seq_ids.numel()),
        _ptr(local_k, torch.bfloat16, "local_k"), _ptr(local_v, torch.bfloat16, "local_v"), _stream(stream)), ctx)


def sparse_decode_prefill(ctx: int, q, k_cache, v_cache, page_table, seq_lens, q_starts, out,
                          stream=None) -> None:
    """Head-wise prefill: q [total_q, Hq, d] packed by sequence (q_starts
    [B + 1], device int32), out float32 of q's shape."""
    B = int(seq_lens.numel())
    if q_starts.numel() != B + 1:
        raise ValueError(f"q_starts must hold batch + 1 = {B + 1} entries, got {q_starts.numel()}")
    if q.dim() != 3 or tuple(out.shape) != tuple(q.shape):
        raise ValueError(f"q must be [total_q, Hq, d] and out the same shape, got {tuple(q.shape)} / "
                         f"{tuple(out.shape)}")
    _check(LIB.sparse_decode_prefill(
        ctx, _ptr(q, torch.bfloat16, "q"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(q_starts, torch.int32, "q_starts"), B, int(q.shape[0]),
        _ptr(out, torch.float32, "out"), _stream(stream)), ctx)


def sparse_decode_num_retrieval_groups(ctx: int) -> int:
    return int(LIB.sparse_decode_num_retrieval_groups(ctx))


def sparse_decode_num_local_groups(ctx: int) -> int:
    return int(LIB.sparse_decode_num_local_groups(ctx))


def sparse_decode_head_effective_rank(w_q, w_k, num_q_heads: int, num_kv_heads: int, head_dim: int,
                                      eff_rank=None, workspace=None, stream=None) -> torch.Tensor:
    """ER of every query head from the frozen projections w_q [L, Hq*d_head,
    d_model] and w_k [L, Hkv*d_head, d_model] (bf16, CUDA); returns float64
    [L, Hq] on the device."""
    if w_q.dim() != 3 or w_k.dim() != 3 or w_q.shape[0] != w_k.shape[0] or w_q.shape[2] != w_k.shape[2]:
        raise ValueError(f"w_q / w_k must be [L, H*d_head, d_model], got {tuple(w_q.shape)} / {tuple(w_k.shape)}")
    L, d_model = int(w_q.shape[0]), int(w_q.shape[2])
    if w_q.shape[1] != num_q_heads * head_dim or w_k.shape[1] != num_kv_heads * head_dim:
        raise ValueError("w_q / w_k rows do not match the head counts")
    n = c_size_t()
    _check(LIB.sparse_decode_head_er_workspace_size(L, num_q_heads, num_kv_heads, head_dim, ctypes.byref(n)))
    if workspace is None:
        workspace = torch.empty(n.value, dtype=torch.uint8, device=w_q.device)
    if eff_rank is None:
        eff_rank = torch.empty((L, num_q_heads), dtype=torch.float64, device=w_q.device)
    if eff_rank.numel() < L * num_q_heads:
        raise ValueError("eff_rank too small")
    _check(LIB.sparse_decode_head_effective_rank(
        _ptr(w_q, torch.bfloat16, "w_q"), _ptr(w_k, torch.bfloat16, "w_k"), L, d_model, num_q_heads, num_kv_heads,
        head_dim, _ptr(eff_rank, torch.float64, "eff_rank"), _ptr(workspace, torch.uint8, "workspace"),
        int(workspace.numel()), _stream(stream)))
    return eff_rank


def sparse_decode_classify_heads(eff_rank, num_kv_heads: int, num_retrieval_groups: int) -> list:
    """head_is_retrieval of one layer from its heads' ER (host float64 [Hq])."""
    er = torch.as_tensor(eff_rank, dtype=torch.float64).detach().cpu().contiguous()
    out = torch.zeros(er.numel(), dtype=torch.int32)
    _check(LIB.sparse_decode_classify_heads(er.data_ptr(), int(er.numel()), num_kv_heads, num_retrieval_groups,
                                            out.data_ptr()))
    return out.tolist()


def sparse_decode_attend_noalloc(ctx: int, q, k_cache, v_cache, page_table, seq_lens, sel_idx, sel_count,
                                 out, stream=None) -> None:
    """attend on the library's built-in scratch (no workspace argument)."""
    _check_sets(ctx, sel_idx, sel_count, int(seq_lens.numel()))
    stride = int(sel_idx.shape[-1]) if sel_idx is not None else 0
    _check(LIB.sparse_decode_attend_noalloc(
        ctx, _ptr(q, torch.bfloat16, "q"), _ptr(k_cache, torch.bfloat16, "k_cache"),
        _ptr(v_cache, torch.bfloat16, "v_cache"), _ptr(page_table, torch.int32, "page_table"),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(seq_lens.numel()),
        _ptr(sel_idx, torch.int32, "sel_idx"), _ptr(sel_count, torch.int32, "sel_count"), stride,
        _ptr(out, torch.float32, "out"), _stream(stream)), ctx)


def sparse_decode_error_word(ctx: int, stream=None) -> int:
    """Wait for the stream, read and clear the device error word (0 = clean)."""
    w = c_uint32()
    st = LIB.sparse_decode_error_word(ctx, _stream(stream), ctypes.byref(w))
    if st not in (SD_OK, SD_ERR_DEVICE_DATA, SD_ERR_TIMEOUT):
        _check(st, ctx)
    return int(w.value)


def sparse_decode_testing_stall_prefill(on: bool) -> None:
    """Testing only: while on, the d = 128 prefill's device-side waits cannot
    end and run out after their bound (outputs zero, SD_EBIT_TIMEOUT)."""
    LIB.sparse_decode_testing_stall_prefill(1 if on else 0)


def sparse_decode_num_retrieval_heads(ctx: int) -> int:
    return int(LIB.sparse_decode_num_retrieval_heads(ctx))


def sparse_decode_destroy(ctx: int) -> None:
    LIB.sparse_decode_destroy(ctx)


# ------------------------------------------------------------ convenience

class SparseDecode:
    """Owns one context; methods forward to the C-named calls above."""

    def __init__(self, **cfg):
        self.cfg = dict(cfg)
        self.handle = sparse_decode_init(**cfg)
        self.num_retrieval_heads = sparse_decode_num_retrieval_heads(self.handle)
        self.device = cfg["proj"].device
        self.max_len = cfg["max_pages_per_seq"] * cfg.get("page_size", 16)

    def close(self):
        if self.handle:
            sparse_decode_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_size(self, batch: int) -> int:
        return sparse_decode_workspace_size(self.handle, batch)

    def sel_stride(self) -> int:
        if self.cfg.get("mode", "top_p") == "top_p":
            return self.max_len
        k = self.cfg.get("top_k", 0)
        if k > 0:
            return min(k, self.max_len)
        import math
        import numpy as np
        return min(self.max_len, max(1, math.floor(float(np.float32(self.cfg["top_k_frac"])) * self.max_len)))

    def alloc(self, batch: int):
        """Workspace, selection rows and counts for `batch` sequences."""
        ws = torch.empty(self.workspace_size(batch), dtype=torch.uint8, device=self.device)
        h = max(1, self.num_retrieval_heads)
        sel = torch.empty((batch, h, self.sel_stride()), dtype=torch.int32, device=self.device)
        cnt = torch.zeros((batch, h), dtype=torch.int32, device=self.device)
        return ws, sel, cnt

    def index_keys(self, k_pre, slots, index_cache, stream=None):
        sparse_decode_index_keys(self.handle, k_pre, slots, index_cache, stream)

    def select(self, q_pre, index_cache, page_table, seq_lens, sel_idx, sel_count, workspace, stream=None):
        sparse_decode_select(self.handle, q_pre, index_cache, page_table, seq_lens, sel_idx, sel_count,
                             workspace, stream)

    def select_exact(self, q, k_cache, page_table, seq_lens, sel_idx, sel_count, workspace, stream=None):
        sparse_decode_select_exact(self.handle, q, k_cache, page_table, seq_lens, sel_idx, sel_count,
                                   workspace, stream)

    def attend(self, q, k_cache, v_cache, page_table, seq_lens, sel_idx, sel_count, out, workspace,
               stream=None):
        sparse_decode_attend(self.handle, q, k_cache, v_cache, page_table, seq_lens, sel_idx, sel_count,
                             out, workspace, stream)

    def select_attend(self, q_pre, q, index_cache, k_cache, v_cache, page_table, seq_lens, sel_idx, sel_count,
                      out, workspace, stream=None):
        sparse_decode_select_attend(self.handle, q_pre, q, index_cache, k_cache, v_cache, page_table, seq_lens,
                                    sel_idx, sel_count, out, workspace, stream)

    def attend_split(self, q, k_ret, v_ret, local_k, local_v, page_table, seq_lens, sel_idx, sel_count, out,
                     workspace, stream=None):
        sparse_decode_attend_split(self.handle, q, k_ret, v_ret, local_k, local_v, page_table, seq_lens,
                                   sel_idx, sel_count, out, workspace, stream)

    def select_attend_split(self, q_pre, q, index_cache, k_ret, v_ret, local_k, local_v, page_table, seq_lens,
                            sel_idx, sel_count, out, workspace, stream=None):
        sparse_decode_select_attend_split(self.handle, q_pre, q, index_cache, k_ret, v_ret, local_k, local_v,
                                          page_table, seq_lens, sel_idx, sel_count, out, workspace, stream)

    def local_append(self, k_new, v_new, seq_ids, positions, local_k, local_v, stream=None):
        sparse_decode_local_append(self.handle, k_new, v_new, seq_ids, positions, local_k, local_v,
                                   self.cfg["max_batch"], stream)

    def prefill(self, q, k_cache, v_cache, page_table, seq_lens, q_starts, out, stream=None):
        sparse_decode_prefill(self.handle, q, k_cache, v_cache, page_table, seq_lens, q_starts, out, stream)

    def num_retrieval_groups(self) -> int:
        return sparse_decode_num_retrieval_groups(self.handle)

    def num_local_groups(self) -> int:
        return sparse_decode_num_local_groups(self.handle)

    def local_cache(self, max_batch: Optional[int] = None):
        """Zeroed compacted local caches (K, V) for `max_batch` sequences."""
        rows = self.cfg.get("window", 0) + self.cfg.get("num_sinks", 0)
        shape = (max_batch or self.cfg["max_batch"], self.num_local_groups(), rows, self.cfg["head_dim"])
        return (torch.zeros(shape, dtype=torch.bfloat16, device=self.device),
                torch.zeros(shape, dtype=torch.bfloat16, device=self.device))

    def error_word(self, stream=None) -> int:
        return sparse_decode_error_word(self.handle, stream)
