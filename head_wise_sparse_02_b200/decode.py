"""One decode step wired through the C ABI: index_keys for the appended
tokens, select, attend.  Torch is used only to hold device buffers."""

from __future__ import annotations

from typing import Optional, Sequence

import torch

from .sparse_decode import SparseDecode


class DecodeStep:
    """Holds a context, the index cache and the per-batch buffers of one layer.

    k_cache / v_cache: bf16 [num_pages, Hkv, 16, d]; page_table int32 [B, MAXP];
    seq_lens int32 [B]; proj bf16 [Hkv, d, 16].
    """

    def __init__(self, *, k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
                 seq_lens: torch.Tensor, proj: torch.Tensor, num_q_heads: int,
                 head_is_retrieval: Sequence[int], window: int, num_sinks: int, mode: str,
                 top_p: float = 0.9, top_k: int = 0, top_k_frac: float = 0.0,
                 attn_scale: float = 0.0, index_scale: float = 0.0,
                 index_cache: Optional[torch.Tensor] = None):
        num_pages, Hkv, page, d = k_cache.shape
        self.k_cache, self.v_cache = k_cache, v_cache
        self.page_table, self.seq_lens = page_table, seq_lens
        self.batch = int(seq_lens.shape[0])
        self.num_q_heads, self.head_dim = num_q_heads, d
        self.sd = SparseDecode(num_q_heads=num_q_heads, num_kv_heads=Hkv, head_dim=d,
                               head_is_retrieval=list(head_is_retrieval), num_pages=num_pages,
                               max_batch=self.batch, max_pages_per_seq=int(page_table.shape[1]),
                               proj=proj, window=window, num_sinks=num_sinks, mode=mode,
                               top_p=top_p, top_k=top_k, top_k_frac=top_k_frac,
                               attn_scale=attn_scale, index_scale=index_scale)
        dev = k_cache.device
        self.index_cache = index_cache if index_cache is not None else torch.zeros(
            (num_pages, Hkv, page, 16), dtype=torch.bfloat16, device=dev)
        self.workspace, self.sel_idx, self.sel_count = self.sd.alloc(self.batch)
        self.out = torch.empty((self.batch, num_q_heads, d), dtype=torch.float32, device=dev)

    def build_index(self, slots: torch.Tensor, keys: torch.Tensor, stream=None):
        """index_keys over the given slots (e.g. every cached position at setup)."""
        self.sd.index_keys(keys, slots, self.index_cache, stream)

    def select(self, q_pre: torch.Tensor, stream=None):
        self.sd.select(q_pre, self.index_cache, self.page_table, self.seq_lens, self.sel_idx,
                       self.sel_count, self.workspace, stream)

    def select_exact(self, q: torch.Tensor, stream=None):
        """Sets by the exact attention logits (post-RoPE q against the K cache)."""
        self.sd.select_exact(q, self.k_cache, self.page_table, self.seq_lens, self.sel_idx,
                             self.sel_count, self.workspace, stream)

    def attend(self, q: torch.Tensor, sel_idx=None, sel_count=None, stream=None):
        self.sd.attend(q, self.k_cache, self.v_cache, self.page_table, self.seq_lens,
                       self.sel_idx if sel_idx is None else sel_idx,
                       self.sel_count if sel_count is None else sel_count,
                       self.out, self.workspace, stream)
        return self.out

    def select_attend(self, q_pre: torch.Tensor, q: torch.Tensor, stream=None) -> torch.Tensor:
        """select then attend on the same sets, joined in one call."""
        self.sd.select_attend(q_pre, q, self.index_cache, self.k_cache, self.v_cache, self.page_table,
                              self.seq_lens, self.sel_idx, self.sel_count, self.out, self.workspace, stream)
        return self.out

    def step(self, q_pre: torch.Tensor, q: torch.Tensor, new_keys: Optional[torch.Tensor] = None,
             new_slots: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """One decode step: index the appended tokens, then select and attend."""
        if new_keys is not None:
            self.sd.index_keys(new_keys, new_slots, self.index_cache, stream)
        return self.select_attend(q_pre, q, stream)

    # ---- split layout: paged caches of the retrieval groups, compacted local caches

    def make_split(self, stream=None):
        """Build the split layout from the full caches: k_ret / v_ret keep the
        retrieval KV groups, and local_append copies every sequence's sinks
        and window (its local positions, in order) into compacted caches."""
        retr = self.sd.cfg["head_is_retrieval"]
        Hkv = self.k_cache.shape[1]
        G = self.num_q_heads // Hkv
        ret_g = [g for g in range(Hkv) if any(retr[g * G:(g + 1) * G])]
        if ret_g == list(range(Hkv)):                                  # every group retrieves
            self.k_ret, self.v_ret = self.k_cache, self.v_cache
        else:
            self.k_ret = self.k_cache[:, ret_g].contiguous()
            self.v_ret = self.v_cache[:, ret_g].contiguous()
        self.local_k, self.local_v = self.sd.local_cache()
        window, sinks = self.sd.cfg.get("window", 0), self.sd.cfg.get("num_sinks", 0)
        lens = self.seq_lens.tolist()
        seq, pos = [], []
        for b, n in enumerate(lens):
            keep = sorted(set(range(min(sinks, n))) | set(range(max(0, n - window), n)))
            seq += [b] * len(keep)
            pos += keep
        if pos:
            dev = self.k_cache.device
            seq_t = torch.tensor(seq, dtype=torch.int32, device=dev)
            pos_t = torch.tensor(pos, dtype=torch.int32, device=dev)
            page = self.page_table[seq_t.long(), (pos_t // 16).long()].long()
            off = (pos_t % 16).long()
            k_new = self.k_cache[page, :, off].contiguous()           # [T, Hkv, d]
            v_new = self.v_cache[page, :, off].contiguous()
            self.sd.local_append(k_new, v_new, seq_t, pos_t, self.local_k, self.local_v, stream)

    def attend_split(self, q: torch.Tensor, sel_idx=None, sel_count=None, stream=None):
        self.sd.attend_split(q, self.k_ret, self.v_ret, self.local_k, self.local_v, self.page_table,
                             self.seq_lens, self.sel_idx if sel_idx is None else sel_idx,
                             self.sel_count if sel_count is None else sel_count, self.out, self.workspace, stream)
        return self.out

    def select_attend_split(self, q_pre: torch.Tensor, q: torch.Tensor, stream=None) -> torch.Tensor:
        self.sd.select_attend_split(q_pre, q, self.index_cache, self.k_ret, self.v_ret, self.local_k,
                                    self.local_v, self.page_table, self.seq_lens, self.sel_idx, self.sel_count,
                                    self.out, self.workspace, stream)
        return self.out

    def error_word(self, stream=None) -> int:
        return self.sd.error_word(stream)

    def close(self):
        self.sd.close()
