"""Seeded synthetic decode workloads for head-wise sparse attention.

Input construction only: this module draws caches, queries, projections and
page tables with the shapes, distributions and planted structure of the five
workloads below.  It computes none of the method's results (no index, no
selection, no sparse attention) and imports neither the oracle nor the CUDA
library; both sides consume what it returns.

Random numbers come from torch generators seeded per tensor
(``seed * 1000 + stream``); the same seed gives the same values on the same
device type (CPU and CUDA streams differ).  Every tensor is drawn in float32
and rounded to bf16 (round to nearest even).

Workloads (sizes are the defaults; tests shrink them through keyword
overrides):
  tiny_ref        1 seq, Hq 4 / Hkv 2, d 64, N 512; heads 0-1 retrieval top-p
                  0.9, heads 2-3 local (window 64 + 4 sinks); 3 planted needles
                  per retrieval head.
  llama3_8b_topp  B 4, Hq 32 / Hkv 8, d 128, N 32768; heads 0-7 top-p 0.9,
                  8-31 local (window 1024 + 4 sinks); 1-16 needles per
                  retrieval head.
  topk_128k       B 16, Hq 32 / Hkv 8, d 128, N 131072; all heads top-k 2%;
                  query scale set per head so that the softmax of the full
                  logits has entropy U[0.2, 0.9] * ln N.
  long_zipf       B 1, Hq 64 / Hkv 8, d 128, N 262144; heads 0-15 top-p
                  (0.5 / 0.9 / 0.99), 16-63 local (window 4096 + 4 sinks);
                  index scores of the planted keys follow a Zipf(alpha) rank
                  profile.
  ragged_paged    B 64, N ~ U[4096, 131072], Hq 32 / Hkv 8, d 128; heads 0-7
                  top-p 0.9, 8-31 local (window 2048 + 4 sinks); randomly
                  permuted page table over one shared pool; 0-32 needles per
                  retrieval head.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

PAGE = 16
INDEX_DIM = 16

WORKLOAD_NAMES = ["tiny_ref", "llama3_8b_topp", "topk_128k", "long_zipf", "ragged_paged"]


@dataclass
class Workload:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    head_is_retrieval: List[int]
    window: int
    num_sinks: int
    mode: str                       # "top_p" | "top_k"
    top_p: float
    top_k: int
    top_k_frac: float
    seq_lens: torch.Tensor          # int32 [B]
    page_table: torch.Tensor        # int32 [B, max_pages]; -1 past the end
    k_cache: torch.Tensor           # bf16 [num_pages, Hkv, PAGE, d]
    v_cache: torch.Tensor           # bf16 [num_pages, Hkv, PAGE, d]
    q: torch.Tensor                 # bf16 [B, Hq, d] (post-RoPE query)
    q_pre: torch.Tensor             # bf16 [B, Hq, d] (pre-RoPE query)
    proj: torch.Tensor              # bf16 [Hkv, d, INDEX_DIM]
    index_dim: int = INDEX_DIM
    page_size: int = PAGE
    attn_scale: float = 0.0         # 0 = library default 1/sqrt(d)
    index_scale: float = 0.0        # 0 = library default sqrt(d)/r
    notes: Dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def num_pages(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def max_len(self) -> int:
        return self.max_pages * self.page_size

    def kv_positions(self, b: int):
        """(page ids, slots) of positions 0..N_b-1 of sequence b."""
        n = int(self.seq_lens[b])
        j = torch.arange(n, device=self.page_table.device)
        return self.page_table[b, j // self.page_size].long(), j % self.page_size


# ---------------------------------------------------------------- helpers

def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + stream)
    return g


def _randn_bf16(shape, gen, device, chunk_rows: int = 4096) -> torch.Tensor:
    """N(0,1) drawn in float32, rounded to bf16, generated in row chunks to
    bound temporary memory."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = shape[0]
    for a in range(0, rows, chunk_rows):
        b = min(rows, a + chunk_rows)
        out[a:b] = torch.randn((b - a,) + tuple(shape[1:]), generator=gen, device=device,
                               dtype=torch.float32).to(torch.bfloat16)
    return out


def _page_table(seq_lens: List[int], permute: bool, gen, device):
    pages_per = [math.ceil(n / PAGE) for n in seq_lens]
    total = sum(pages_per)
    if permute:
        ids = torch.randperm(total, generator=gen, device=device).to(torch.int32)
    else:
        ids = torch.arange(total, device=device, dtype=torch.int32)
    pt = torch.full((len(seq_lens), max(pages_per)), -1, dtype=torch.int32, device=device)
    c = 0
    for b, m in enumerate(pages_per):
        pt[b, :m] = ids[c:c + m]
        c += m
    return pt, total


def _plant_needles(w: Workload, counts: Dict[int, List[int]], gen, noise: float = 0.1):
    """For each (b, retrieval head h) plant counts[b][h_i] needle keys in the KV
    head of h at distinct positions (distinct across the heads of one group):
    k = 0.8 * sqrt(d) * q_h / |q_h| + N(0, noise^2)."""
    d = w.head_dim
    G = w.num_q_heads // w.num_kv_heads
    ret_heads = [h for h in range(w.num_q_heads) if w.head_is_retrieval[h]]
    dev = w.k_cache.device
    planted = {}
    for b in range(w.batch):
        n = int(w.seq_lens[b])
        by_group: Dict[int, List[int]] = {}
        for i, h in enumerate(ret_heads):
            by_group.setdefault(h // G, []).append(i)
        for g, idxs in by_group.items():
            need = sum(counts[b][i] for i in idxs)
            if need == 0:
                continue
            pos = torch.randperm(n, generator=gen, device=dev)[:need]
            c = 0
            for i in idxs:
                h = ret_heads[i]
                m = counts[b][i]
                if m == 0:
                    continue
                p = pos[c:c + m]              # fewer when the context is shorter than the needles
                c += m
                m = int(p.numel())
                if m == 0:
                    continue
                qh = w.q[b, h].float()
                key = 0.8 * math.sqrt(d) * qh / qh.norm()
                eps = noise * torch.randn((m, d), generator=gen, device=dev, dtype=torch.float32)
                page = w.page_table[b, p // PAGE].long()
                w.k_cache[page, g, p % PAGE] = (key[None, :] + eps).to(torch.bfloat16)
                planted[(b, h)] = sorted(p.tolist())
    w.notes["needles"] = planted


def _base(name, seed, device, seq_lens, Hq, Hkv, d, retr, window, sinks, mode,
          top_p=0.9, top_k=0, top_k_frac=0.0, permute=False) -> Workload:
    g_pt = _gen(device, seed, 1)
    pt, total = _page_table(seq_lens, permute, g_pt, device)
    kc = _randn_bf16((total, Hkv, PAGE, d), _gen(device, seed, 2), device)
    vc = _randn_bf16((total, Hkv, PAGE, d), _gen(device, seed, 3), device)
    B = len(seq_lens)
    q = _randn_bf16((B, Hq, d), _gen(device, seed, 4), device)
    proj = (torch.randn((Hkv, d, INDEX_DIM), generator=_gen(device, seed, 5), device=device,
                        dtype=torch.float32) / math.sqrt(d)).to(torch.bfloat16)
    return Workload(name=name, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d,
                    head_is_retrieval=list(retr), window=window, num_sinks=sinks, mode=mode,
                    top_p=top_p, top_k=top_k, top_k_frac=top_k_frac,
                    seq_lens=torch.tensor(seq_lens, dtype=torch.int32, device=device),
                    page_table=pt, k_cache=kc, v_cache=vc, q=q, q_pre=q, proj=proj)


# ---------------------------------------------------------------- workloads

def tiny_ref(device="cpu", seed=0, N=512, needles=3, permute=False) -> Workload:
    w = _base("tiny_ref", seed, device, [N], 4, 2, 64, [1, 1, 0, 0], 64, 4, "top_p",
              top_p=0.9, permute=permute)
    _plant_needles(w, {0: [needles, needles]}, _gen(device, seed, 6))
    return w


def llama3_8b_topp(device="cuda", seed=1, B=4, N=32768, max_needles=16, permute=False,
                   window=1024, sinks=4) -> Workload:
    retr = [1] * 8 + [0] * 24
    w = _base("llama3_8b_topp", seed, device, [N] * B, 32, 8, 128, retr, window, sinks, "top_p",
              top_p=0.9, permute=permute)
    g = _gen(device, seed, 6)
    counts = {b: torch.randint(1, max_needles + 1, (8,), generator=g, device=device).tolist()
              for b in range(B)}
    _plant_needles(w, counts, g)
    return w


def _entropy(beta, L):
    """Entropy of softmax(beta * L) along the last axis (beta broadcast)."""
    x = beta[..., None] * L
    lse = torch.logsumexp(x, dim=-1)
    p = torch.softmax(x, dim=-1)
    return lse - (p * x).sum(-1)


def topk_128k(device="cuda", seed=2, B=16, N=131072, top_k_frac=0.02, top_k=0,
              permute=False) -> Workload:
    retr = [1] * 32
    w = _base("topk_128k", seed, device, [N] * B, 32, 8, 128, retr, 0, 0, "top_k",
              top_k=top_k, top_k_frac=top_k_frac, permute=permute)
    d, G = 128, 4
    g = _gen(device, seed, 6)
    z = torch.randn((B, 32, d), generator=g, device=device, dtype=torch.float32)
    target = torch.empty((B, 32), device=device).uniform_(0.2, 0.9, generator=g) * math.log(N)
    q = torch.empty((B, 32, d), dtype=torch.bfloat16, device=device)
    realised = torch.empty((B, 32), device=device)
    for b in range(B):
        pages, slots = w.kv_positions(b)
        for kvh in range(8):
            K = w.k_cache[pages, kvh, slots].float()                  # [N, d]
            heads = slice(kvh * G, (kvh + 1) * G)
            L = (z[b, heads] @ K.T) / math.sqrt(d)                     # [G, N]
            lo = torch.zeros(G, device=device)
            hi = torch.ones(G, device=device)
            tgt = target[b, heads]
            for _ in range(60):                                        # bracket
                more = _entropy(hi, L) > tgt
                if not bool(more.any()):
                    break
                hi = torch.where(more, hi * 2, hi)
            for _ in range(50):                                        # bisect
                mid = 0.5 * (lo + hi)
                above = _entropy(mid, L) > tgt
                lo = torch.where(above, mid, lo)
                hi = torch.where(above, hi, mid)
            beta = 0.5 * (lo + hi)
            qb = (beta[:, None] * z[b, heads]).to(torch.bfloat16)
            q[b, heads] = qb
            realised[b, heads] = _entropy(torch.ones(G, device=device),
                                          (qb.float() @ K.T) / math.sqrt(d))
    w.q = q
    w.q_pre = q
    w.notes["target_entropy_over_lnN"] = (target / math.log(N)).cpu()
    w.notes["realised_entropy_over_lnN"] = (realised / math.log(N)).cpu()
    return w


def long_zipf(device="cuda", seed=3, N=262144, top_p=0.9, alpha=1.2, window=4096, sinks=4,
              query_spread=0.01, permute=False) -> Workload:
    """Index scores of the noiseless group query gamma*u_g against the planted
    keys are -alpha*ln(rank) (before bf16 rounding): each key of a retrieval
    KV head is xi_perp + a_j u_g with a_j solved from the group's projection."""
    Hq, Hkv, d = 64, 8, 128
    retr = [1] * 16 + [0] * 48
    w = _base("long_zipf", seed, device, [N], Hq, Hkv, d, retr, window, sinks, "top_p",
              top_p=top_p, permute=permute)
    G = Hq // Hkv
    g = _gen(device, seed, 6)
    gamma = math.sqrt(d)
    c = math.sqrt(d) / INDEX_DIM                     # the library's default index scale
    pages, slots = w.kv_positions(0)
    q = w.q.clone()
    for kvh in range(2):
        u = torch.randn(d, generator=g, device=device, dtype=torch.float32)
        u = u / u.norm()
        P = w.proj[kvh].float()                      # [d, r]
        Pu = P.T @ u                                 # [r]
        xi = w.k_cache[pages, kvh, slots].float()    # [N, d]
        xi_perp = xi - (xi @ u)[:, None] * u[None, :]
        rank = torch.randperm(N, generator=g, device=device).double() + 1.0
        target = (-alpha * torch.log(rank)).float()
        a = (target / (c * gamma) - (xi_perp @ P) @ Pu) / (Pu @ Pu)
        k = xi_perp + a[:, None] * u[None, :]
        w.k_cache[pages, kvh, slots] = k.to(torch.bfloat16)
        for h in range(kvh * G, (kvh + 1) * G):
            xh = torch.randn(d, generator=g, device=device, dtype=torch.float32)
            q[0, h] = (gamma * (u + query_spread * xh / math.sqrt(d))).to(torch.bfloat16)
        w.notes.setdefault("rank", {})[kvh] = rank.long().cpu()
    w.q = q
    w.q_pre = q
    w.notes["alpha"] = alpha
    return w


def ragged_paged(device="cuda", seed=4, B=64, N_min=4096, N_max=131072, max_needles=32,
                 window=2048, sinks=4) -> Workload:
    g = _gen(device, seed, 0)
    lens = torch.randint(N_min, N_max + 1, (B,), generator=g, device=device).tolist()
    retr = [1] * 8 + [0] * 24
    w = _base("ragged_paged", seed, device, lens, 32, 8, 128, retr, window, sinks, "top_p",
              top_p=0.9, permute=True)
    g6 = _gen(device, seed, 6)
    counts = {b: torch.randint(0, max_needles + 1, (8,), generator=g6, device=device).tolist()
              for b in range(B)}
    _plant_needles(w, counts, g6)
    return w


BUILDERS = {
    "tiny_ref": tiny_ref,
    "llama3_8b_topp": llama3_8b_topp,
    "topk_128k": topk_128k,
    "long_zipf": long_zipf,
    "ragged_paged": ragged_paged,
}


def prefill_inputs(w: Workload, chunk_lens, seed: int = 0, scale: float = 1.0):
    """Queries of a prefill chunk per sequence: the last chunk_lens[b] positions
    of sequence b (clamped to its length), packed by sequence.  Returns
    (q bf16 [total_q, Hq, d] drawn N(0, scale^2), q_starts int32 [B + 1])."""
    lens = w.seq_lens.tolist()
    t = [max(0, min(int(c), n)) for c, n in zip(chunk_lens, lens)]
    starts = [0]
    for x in t:
        starts.append(starts[-1] + x)
    dev = w.k_cache.device
    q = (_randn_bf16((max(1, starts[-1]), w.num_q_heads, w.head_dim), _gen(dev, seed, 7), dev).float()
         * scale).to(torch.bfloat16)[:starts[-1]].contiguous()
    return q, torch.tensor(starts, dtype=torch.int32, device=dev)


def make_workload(name: str, device="cuda", **overrides) -> Workload:
    return BUILDERS[name](device=device, **overrides)


def slots_of(w: Workload) -> torch.Tensor:
    """int32 slot ids (page * page_size + offset) of every cached position of
    every sequence, in sequence order: the argument that fills the whole index
    cache with one index-keys call."""
    out = []
    for b in range(w.batch):
        pages, s = w.kv_positions(b)
        out.append((pages * w.page_size + s).to(torch.int32))
    return torch.cat(out)


def keys_at(w: Workload, slots: torch.Tensor) -> torch.Tensor:
    """Pre-RoPE keys [T, Hkv, d] stored at the given slots (no RoPE in these
    workloads, so pre-RoPE keys are the cached keys)."""
    s = slots.long()
    return w.k_cache[s // w.page_size, :, s % w.page_size].contiguous()
