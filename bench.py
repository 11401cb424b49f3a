"""Decode-step benchmark of head-wise sparse attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload topk_128k]

A step is one pass of the whole decode path over one batch: index_keys for
the B appended tokens, select (index scoring + top-k / top-p) and attend
(gathered retrieval rows, sinks + window for local heads, split merge).  The
default workload is the 128K-context fixed-budget decode: 16 sequences of
131072 tokens, 32 q / 8 KV heads, d = 128, all heads retrieval with top-k 2%
(2621 tokens per head).  Inputs are synthetic and seeded; each rank runs its
own batch (weak scaling, no collective on the data path).

Rank 0 prints one JSON line.  `value` is whole-job head-steps/s (one
head-step = one (sequence, q head) output of one decode step), timed with
CUDA events over K steps after W warm-up steps, max over ranks.  The touched
bytes per step (~1.2 GB) exceed the 126 MB L2, so no flush is needed between
steps.  `--impl reference` times the float64 CPU oracle on the host cores on
a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse decode head-steps/s and achieved HBM GB/s vs 8 TB/s at 128K ctx"
UNIT = "head-steps/s"
CONTRACT_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------- rank plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling)."""
    return base + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and throttle-reason samples during the timed region, read
    through NVML every millisecond (the data nvidia-smi reports; nothing is
    set): the timed region of a default run lasts a few milliseconds.
    Falls back to `nvidia-smi -lms 200` when NVML is unavailable."""

    # NVML clocks-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.stop_evt = threading.Event()
        self.handle = None
        self.nvml = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        self.nvml = pynvml
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.cuda_index]) if vis and vis.split(",")[0].isdigit() else self.cuda_index
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        try:
            self.handle = self._handle()
            self.max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
        except Exception:
            self.handle = None
            return
        getr = getattr(self.nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(self.nvml, "nvmlDeviceGetCurrentClocksThrottleReasons")

        def loop():
            while not self.stop_evt.is_set():
                try:
                    self.samples.append((self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM),
                                         int(getr(self.handle))))
                except Exception:
                    pass
                time.sleep(0.001)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.handle is None:
            return None
        self.stop_evt.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return None
        sm = sorted(x for x, _ in self.samples)
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvml 1 ms"}


# ---------------------------------------------------------------- measurements

def load_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def code_only(text: bytes) -> bytes:
    """A C++/CUDA source without its comments (// and /* */ outside string and
    character literals) and with every run of whitespace made one space: the
    code the compiler sees, so that an edit of the comments alone keeps a
    capture taken on the source valid."""
    out, i, n = bytearray(), 0, len(text)
    while i < n:
        c = text[i:i + 1]
        if c in (b'"', b"'"):
            j = i + 1
            while j < n and text[j:j + 1] != c:
                j += 2 if text[j:j + 1] == b"\\" else 1
            out += text[i:j + 1]
            i = j + 1
        elif text.startswith(b"//", i):
            j = text.find(b"\n", i)
            i = n if j < 0 else j
        elif text.startswith(b"/*", i):
            j = text.find(b"*/", i + 2)
            i = n if j < 0 else j + 2
            out += b" "
        else:
            out += c
            i += 1
    return re.sub(rb"\s+", b" ", bytes(out)).strip()


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(code_only(fh.read()))
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "select": ["head_wise_sparse_02_b200/csrc/sd_select.cu", "head_wise_sparse_02_b200/csrc/sd_select_stream.cu",
               "head_wise_sparse_02_b200/csrc/sd_internal.cuh"],
    "attend": ["head_wise_sparse_02_b200/csrc/sd_attend.cu", "head_wise_sparse_02_b200/csrc/sd_internal.cuh"],
    "index_keys": ["head_wise_sparse_02_b200/csrc/sd_index.cu", "head_wise_sparse_02_b200/csrc/sd_internal.cuh"],
    # the joined call: the selection and attend kernels one step launches
    "select_attend": ["head_wise_sparse_02_b200/csrc/sd_select.cu", "head_wise_sparse_02_b200/csrc/sd_select_stream.cu",
                      "head_wise_sparse_02_b200/csrc/sd_attend.cu", "head_wise_sparse_02_b200/csrc/sd_internal.cuh"],
    # exact-score selection: the score kernel and the exact selector
    "select_exact": ["head_wise_sparse_02_b200/csrc/sd_exact.cu", "head_wise_sparse_02_b200/csrc/sd_select.cu",
                     "head_wise_sparse_02_b200/csrc/sd_internal.cuh"],
}
# the split layout's joined call runs the same kernels as the joined call
KERNEL_SOURCES["select_attend_split"] = KERNEL_SOURCES["select_attend"]
# ncu_traffic.json key of a call's dominant kernel, per score mode
TRAFFIC_KEY = {("exact", "select"): "select_exact"}


def ncu_traffic(kernel: str, workload: str, algorithmic_bytes: float):
    """DRAM bytes per call from a committed ncu summary of this call on this
    workload, if it was taken on the current kernel source (else None).  The
    summary stores DRAM bytes per algorithmic byte of the captured case (the
    bench's own size, or a smaller one that takes the same code path); both
    grow with the rows a call processes, so the ratio scales it to this call."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[f"{kernel}@{workload}"]
        if e.get("source_hash") != kernel_source_hash(KERNEL_SOURCES[kernel]):
            return None
        return round(float(e["dram_bytes_per_algorithmic_byte"]) * algorithmic_bytes)
    except Exception:
        return None


def kernels_per_step(w, score: str = "index", split: bool = False) -> int:
    """Kernels of this library one step launches: index_keys; select (top-k:
    window, stream, resolve; top-p: window, mass pass, cut pass, resolve;
    then the exact selector for flagged items; exact-score mode: the score
    kernel and the exact selector, no index_keys); attend (plan when there
    are retrieval heads, item layout, main); split layout: local_append of
    the new tokens when there are local heads."""
    ret = any(w.head_is_retrieval)
    loc = not all(w.head_is_retrieval)
    if score == "exact":
        return (2 if ret else 0) + (3 if ret else 2)
    n_sel = 0 if not ret else (4 if w.mode == "top_k" else 5)
    return 1 + (1 if split and loc else 0) + n_sel + (3 if ret else 2)


def kv_cache_bytes(w) -> dict:
    """K + V bytes the sequences of `w` occupy: every KV head keeps the whole
    context (full layout), or only the retrieval groups do and each local
    group keeps num_sinks + window rows (split layout)."""
    G = w.num_q_heads // w.num_kv_heads
    ret_groups = sum(1 for g in range(w.num_kv_heads) if any(w.head_is_retrieval[g * G:(g + 1) * G]))
    loc_groups = sum(1 for g in range(w.num_kv_heads) if not all(w.head_is_retrieval[g * G:(g + 1) * G]))
    row = 4 * w.head_dim
    tokens = sum(w.seq_lens.cpu().tolist())
    return {"full": tokens * w.num_kv_heads * row,
            "split": tokens * ret_groups * row + w.batch * loc_groups * (w.num_sinks + w.window) * row}


def union_rows(sel_idx, sel_count, w):
    """Distinct K/V rows each (sequence, KV group) reads: union over the
    group's retrieval heads plus the local set of its local heads."""
    import torch
    G = w.num_q_heads // w.num_kv_heads
    rows = {}
    r = 0
    ret_rows = {}
    for h in range(w.num_q_heads):
        if w.head_is_retrieval[h]:
            ret_rows[h] = r
            r += 1
    cnt = sel_count.cpu()
    lens = w.seq_lens.cpu().tolist()
    total = 0
    index_tokens = 0
    for b in range(w.batch):
        n = lens[b]
        for g in range(w.num_kv_heads):
            heads = range(g * G, (g + 1) * G)
            parts = []
            has_ret = False
            has_loc = False
            for h in heads:
                if w.head_is_retrieval[h]:
                    has_ret = True
                    k = int(cnt[b, ret_rows[h]])
                    parts.append(sel_idx[b, ret_rows[h], :k])
                else:
                    has_loc = True
            if has_loc:
                a = min(w.num_sinks, n)
                ws_ = max(a, n - w.window)
                parts.append(torch.arange(0, a, device=sel_idx.device, dtype=torch.int32))
                parts.append(torch.arange(ws_, n, device=sel_idx.device, dtype=torch.int32))
            if parts:
                total += int(torch.unique(torch.cat(parts)).numel())
            if has_ret:
                index_tokens += n
    return total, index_tokens


L2_BYTES = 126 * 2 ** 20
L2_FLUSH_BYTES = 512 * 2 ** 20
# a step that streams at least this many bytes (4x the L2, in the same order
# every step) leaves nothing useful in L2 for the next one: no flush is needed
NO_FLUSH_ABOVE = 4 * L2_BYTES


def streamed_bytes_lower_bound(w) -> int:
    """Bytes every step reads whatever the selection: the index of every
    retrieval (sequence, KV group) and the sink + window rows of every local
    one (selected rows come on top)."""
    G = w.num_q_heads // w.num_kv_heads
    ret_groups = sum(1 for g in range(w.num_kv_heads) if any(w.head_is_retrieval[g * G:(g + 1) * G]))
    loc_groups = sum(1 for g in range(w.num_kv_heads) if not all(w.head_is_retrieval[g * G:(g + 1) * G]))
    total = 0
    for n in w.seq_lens.cpu().tolist():
        local_rows = min(n, w.num_sinks) + max(0, n - max(min(n, w.num_sinks), n - w.window))
        total += ret_groups * 32 * n + loc_groups * local_rows * 4 * w.head_dim
    return total


def l2_flush_needed(mode: str, w) -> bool:
    if mode == "on":
        return True
    if mode == "off":
        return False
    return streamed_bytes_lower_bound(w) < NO_FLUSH_ABOVE


def workload_label(name: str, w) -> str:
    lens = w.seq_lens
    n = (f"N={int(lens.max())}" if int(lens.min()) == int(lens.max())
         else f"N={int(lens.min())}..{int(lens.max())}")
    mode = (f"top-k frac {w.top_k_frac}" if w.mode == "top_k" and not w.top_k
            else f"top-k {w.top_k}" if w.mode == "top_k" else f"top-p {w.top_p}")
    ret = sum(w.head_is_retrieval)
    heads = f"{ret} retrieval ({mode})"
    if ret < w.num_q_heads:
        heads += f" + {w.num_q_heads - ret} local (window {w.window} + {w.num_sinks} sinks)"
    return (f"{name}: B={w.batch}, Hq={w.num_q_heads}/Hkv={w.num_kv_heads}, d={w.head_dim}, {n}, "
            f"{heads}" + (f", {w.notes['profile']}" if "profile" in w.notes else ""))


def bench_config(args, w, ws: int, flush: bool):
    """The `config` object of the JSON line; both arms print the same one."""
    return {
        "workload": workload_label(args.workload, w) + (", exact-score selection" if args.score == "exact" else "")
        + (", split KV layout (compacted local caches)" if getattr(args, "kv_layout", "full") == "split" else ""),
        "batch_per_gpu": w.batch, "seq_len": int(w.seq_lens.max()),
        "parallelism": f"replicas x{ws} (sequences sharded, no collective)",
        "l2": ("flushed between steps (512 MiB write, untimed)" if flush
               else "no flush: every step streams more than 4x the 126 MB L2"),
    }


def selection_diagnostics(w, st, budget_s: float = 20.0, max_pairs: int = 16):
    """|S|/N of the retrieval heads and, on a sample of (sequence, retrieval
    head) pairs, the share of the full-attention softmax mass that the GPU's
    selected set holds (the oracle's mass_retained, float64 on the host).
    Diagnostics only: nothing here is timed or compared."""
    import numpy as np

    import oracle as O
    from oracle.workload_inputs import oracle_config, oracle_inputs
    retr = [h for h in range(w.num_q_heads) if w.head_is_retrieval[h]]
    if not retr:
        return {"retrieval_heads": 0}
    cnt = st.sel_count.cpu().numpy().astype(np.float64)
    lens = w.seq_lens.cpu().numpy().astype(np.float64)
    frac = cnt / np.maximum(lens[:, None], 1.0)
    cfg = oracle_config(w)
    attn_scale, _ = cfg.scales()
    G = w.num_q_heads // w.num_kv_heads
    rng = np.random.default_rng(0)
    pairs = [(int(b), int(retr[i])) for b, i in zip(rng.integers(0, w.batch, max_pairs),
                                                   rng.integers(0, len(retr), max_pairs))]
    masses = []
    t0 = time.perf_counter()
    for b, h in pairs:
        if time.perf_counter() - t0 > budget_s:
            break
        inp = oracle_inputs(w, [b])
        n = int(inp["seq_lens"][0])
        K = O.gather_rows(inp["k_cache"], inp["page_table"][0], n, h // G, cfg.page_size)
        r = retr.index(h)
        k = int(st.sel_count[b, r])
        S = st.sel_idx[b, r, :k].cpu().numpy().astype(np.int64)
        masses.append(O.mass_retained(inp["q"][0, h], K, S, attn_scale))
    out = {"selected_frac": {"mean": round(float(frac.mean()), 5), "min": round(float(frac.min()), 5),
                             "max": round(float(frac.max()), 5)}}
    if masses:
        out["mass_retained"] = {"mean": round(float(np.mean(masses)), 5), "min": round(float(np.min(masses)), 5),
                                "sample": f"{len(masses)} random (sequence, retrieval head) pairs; float64 "
                                          f"oracle on the host: share of the full softmax of q.k over all "
                                          f"N tokens that falls on the GPU-selected set"}
    return out


def size_overrides(args):
    """--batch / --seq-len shrink the workload (profiling cases); the JSON
    config reports the sizes actually run."""
    kw = {}
    if args.batch:
        kw["B"] = args.batch
    if args.seq_len and args.workload == "ragged_paged":
        kw["N_max"] = args.seq_len                  # lengths U[min(4096, N), N]
        kw["N_min"] = min(4096, args.seq_len)
    elif args.seq_len:
        kw["N"] = args.seq_len
    if args.top_p:
        kw["top_p"] = args.top_p
    if args.alpha:
        kw["alpha"] = args.alpha
    if args.top_k_frac:
        kw["top_k_frac"] = args.top_k_frac
    return kw


def workload_for_rank(args, device, rank: int):
    """The rank's own seeded batch: the workload's default seed (or --seed)
    offset per rank (weak scaling)."""
    from workloads import make_workload
    kw = size_overrides(args)
    if args.seed is not None or rank:
        import inspect
        from workloads.synthetic import BUILDERS
        base = args.seed if args.seed is not None else inspect.signature(BUILDERS[args.workload]).parameters["seed"].default
        kw["seed"] = rank_seed(base, rank)
    return make_workload(args.workload, device, **kw)


def run_ours(args):
    import torch
    import torch.distributed as dist

    from head_wise_sparse_02_b200.decode import DecodeStep
    from workloads import keys_at, make_workload, slots_of

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    w = workload_for_rank(args, dev, rank)
    B, Hq, d = w.batch, w.num_q_heads, w.head_dim
    st = DecodeStep(k_cache=w.k_cache, v_cache=w.v_cache, page_table=w.page_table, seq_lens=w.seq_lens,
                    proj=w.proj, num_q_heads=Hq, head_is_retrieval=w.head_is_retrieval, window=w.window,
                    num_sinks=w.num_sinks, mode=w.mode, top_p=w.top_p, top_k=w.top_k,
                    top_k_frac=w.top_k_frac)
    slots_all = slots_of(w)
    st.build_index(slots_all, keys_at(w, slots_all))          # prefill-time index (setup, untimed)
    # per step: the appended token of every sequence is position N_b - 1
    lens = w.seq_lens.long()
    new_slots = (w.page_table[torch.arange(B, device=dev), (lens - 1) // 16].long() * 16 + (lens - 1) % 16).to(torch.int32)
    new_keys = keys_at(w, new_slots)
    stream = torch.cuda.current_stream()

    exact = args.score == "exact"
    split = args.kv_layout == "split"
    # the decode step through the public API: index_keys for the appended
    # tokens, then the joined select + attend call (exact-score mode: the
    # exact-score select, then attend; no index is kept; split layout: the
    # appended tokens also go to the compacted local caches, and the joined
    # call reads the split caches)
    if split:
        st.make_split()                                   # setup, untimed
        pos_new = (lens - 1).to(torch.int32)
        seq_new = torch.arange(B, device=dev, dtype=torch.int32)
        page_new = w.page_table[seq_new.long(), (lens - 1) // 16].long()
        kn_new = w.k_cache[page_new, :, (lens - 1) % 16].contiguous()    # [B, Hkv, d] of the new tokens
        vn_new = w.v_cache[page_new, :, (lens - 1) % 16].contiguous()
    if exact:
        calls = ("index_keys", "select", "attend")
    elif split:
        calls = ("index_keys", "local_append", "select_attend_split")
    else:
        calls = ("index_keys", "select_attend")

    def step(ev=None):
        """One decode step; with `ev`, an event pair around each call."""
        if ev is not None:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
            e[0].record(stream)
        if exact:
            if ev is not None:
                e[1].record(stream)
            st.select_exact(w.q, stream)
            if ev is not None:
                e[2].record(stream)
            st.attend(w.q, stream=stream)
        elif split:
            st.sd.index_keys(new_keys, new_slots, st.index_cache, stream)
            if ev is not None:
                e[1].record(stream)
            st.sd.local_append(kn_new, vn_new, seq_new, pos_new, st.local_k, st.local_v, stream)
            if ev is not None:
                e[2].record(stream)
            st.select_attend_split(w.q_pre, w.q, stream)
        else:
            st.sd.index_keys(new_keys, new_slots, st.index_cache, stream)
            if ev is not None:
                e[1].record(stream)
            st.select_attend(w.q_pre, w.q, stream)
        if ev is not None:
            e[len(calls)].record(stream)
            for i, k in enumerate(calls):
                ev[k].append((e[i], e[i + 1]))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    word = st.error_word()
    if word:
        raise RuntimeError(f"device error word {word:#x} after warm-up")
    rows, index_tokens = union_rows(st.sel_idx, st.sel_count, w)
    sel_sizes = st.sel_count.float()
    row_bytes = 4 * d                                   # K + V row, bf16
    score_row = 2 * d if exact else 32                  # bytes scored per (token, retrieval group)
    step_bytes = score_row * index_tokens + row_bytes * rows
    flush = l2_flush_needed(args.l2_flush, w)
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None

    def timed(n_steps, with_calls):
        """Device time of n_steps steps (ms per step) and, with_calls, the
        per-call event pairs.  Without an L2 flush one event pair brackets
        all steps; with it, each step has its own pair and the flush (a
        write of a buffer larger than L2) runs between them, untimed."""
        ev = {k: [] for k in calls} if with_calls else None
        if not flush:
            a0 = torch.cuda.Event(enable_timing=True); a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(n_steps):
                step(ev)
            a1.record(stream)
            torch.cuda.synchronize()
            return a0.elapsed_time(a1) / n_steps, ev
        pairs = []
        for _ in range(n_steps):
            flush_buf.zero_()
            a0 = torch.cuda.Event(enable_timing=True); a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            step(ev)
            a1.record(stream)
            pairs.append((a0, a1))
        torch.cuda.synchronize()
        return sum(x.elapsed_time(y) for x, y in pairs) / n_steps, ev

    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    ms, _ = timed(args.steps, False)
    barrier()
    clk = clocks.stop()
    ms_max = max_over_ranks(ms, dev)
    # per-call device times: the same steps again, with an event pair around
    # each call (events between calls keep a call's first kernel from
    # overlapping the previous call's last one, so these sum to a little
    # more than the step time above)
    barrier()
    torch.cuda.synchronize()
    ms_calls, ev = timed(args.steps, True)
    barrier()
    per = {k: sum(a.elapsed_time(b) for a, b in v) / len(v) for k, v in ev.items()}

    # ---- end to end through the public API with host buffers ----
    q_h = w.q.cpu().pin_memory()
    qp_h = w.q_pre.cpu().pin_memory()
    nk_h = new_keys.cpu().pin_memory()
    ns_h = new_slots.cpu().pin_memory()
    out_h = torch.empty(st.out.shape, dtype=torch.float32).pin_memory()
    q_d, qp_d = torch.empty_like(w.q), torch.empty_like(w.q_pre)
    nk_d, ns_d = torch.empty_like(new_keys), torch.empty_like(new_slots)

    if split:
        kn_h, vn_h = kn_new.cpu().pin_memory(), vn_new.cpu().pin_memory()
        kn_d, vn_d = torch.empty_like(kn_new), torch.empty_like(vn_new)

    def e2e_step():
        q_d.copy_(q_h, non_blocking=True)
        if exact:
            st.select_exact(q_d, stream)
            st.attend(q_d, stream=stream)
        elif split:
            qp_d.copy_(qp_h, non_blocking=True)
            nk_d.copy_(nk_h, non_blocking=True); ns_d.copy_(ns_h, non_blocking=True)
            kn_d.copy_(kn_h, non_blocking=True); vn_d.copy_(vn_h, non_blocking=True)
            st.sd.index_keys(nk_d, ns_d, st.index_cache, stream)
            st.sd.local_append(kn_d, vn_d, seq_new, pos_new, st.local_k, st.local_v, stream)
            st.select_attend_split(qp_d, q_d, stream)
        else:
            qp_d.copy_(qp_h, non_blocking=True)
            nk_d.copy_(nk_h, non_blocking=True); ns_d.copy_(ns_h, non_blocking=True)
            st.sd.index_keys(nk_d, ns_d, st.index_cache, stream)
            st.select_attend(qp_d, q_d, stream)
        out_h.copy_(st.out, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    if not flush:
        a0 = torch.cuda.Event(enable_timing=True); a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        e2e_one = a0.elapsed_time(a1) / args.steps
    else:
        pairs = []
        for _ in range(args.steps):
            flush_buf.zero_()
            a0 = torch.cuda.Event(enable_timing=True); a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            e2e_step()
            a1.record(stream)
            pairs.append((a0, a1))
        torch.cuda.synchronize()
        e2e_one = sum(x.elapsed_time(y) for x, y in pairs) / args.steps
    barrier()
    e2e_ms = max_over_ranks(e2e_one, dev)
    word = st.error_word()
    if word:
        raise RuntimeError(f"device error word {word:#x} after timing")

    # ---- roofline of the dominant kernel ----
    index_bytes = score_row * index_tokens
    kv_bytes = row_bytes * rows
    if exact:
        kern_bytes = {"select": index_bytes, "attend": kv_bytes, "index_keys": 0}
    else:
        kern_bytes = {"select_attend": index_bytes + kv_bytes, "index_keys": B * w.num_kv_heads * (2 * d + 32)}
    if split:
        n_loc = sum(1 for g in range(w.num_kv_heads)
                    if not all(w.head_is_retrieval[g * (Hq // w.num_kv_heads):(g + 1) * (Hq // w.num_kv_heads)]))
        kern_bytes["select_attend_split"] = kern_bytes.pop("select_attend")
        kern_bytes["local_append"] = 2 * B * n_loc * 4 * d           # read and write K + V rows
        step_bytes += kern_bytes["local_append"]
    dominant = max(per, key=per.get)
    peak, peak_kind = load_peak()
    achieved = kern_bytes[dominant] / (per[dominant] * 1e-3) / 1e9
    head_steps = ws * B * Hq
    value = head_steps / (ms_max * 1e-3)
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "storage_dtype": "bf16",
        "data": "synthetic (seeded; no datasets or trained weights)",
        "config": bench_config(args, w, ws, flush),
        "tokens_per_s": round(ws * B / (ms_max * 1e-3), 1),
        "hbm_gbs_achieved_step": round(step_bytes / (ms * 1e-3) / 1e9, 1),
        "frac_of_8tbs_step": round(step_bytes / (ms * 1e-3) / 1e9 / CONTRACT_GBS, 4),
        "algorithmic_bytes_per_step": step_bytes,
        "ms_per_call": {k: round(v, 4) for k, v in per.items()},
        "ms_per_step_with_call_events": round(ms_calls, 4),
        "algorithmic_bytes_per_call": kern_bytes,
        "selected_per_head": {"mean": round(float(sel_sizes.mean()), 1), "min": int(sel_sizes.min()),
                              "max": int(sel_sizes.max())},
        "roofline": {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": f"{peak_kind} hbm_gbs (copy bandwidth)", "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "algorithmic_bytes_per_launch": kern_bytes[dominant],
                     "traffic": ncu_traffic(TRAFFIC_KEY.get((args.score, dominant), dominant), args.workload,
                                            kern_bytes[dominant])},
        "e2e": {"value": round(head_steps / (e2e_ms * 1e-3), 1), "unit": UNIT,
                "h2d_bytes_per_step": int(q_h.numel() * 2 + (0 if exact else
                                                             qp_h.numel() * 2 + nk_h.numel() * 2 + ns_h.numel() * 4)
                                          + (kn_h.numel() * 4 if split else 0)),
                "d2h_bytes_per_step": int(out_h.numel() * 4)},
        "gpu_launches": kernels_per_step(w, args.score, split) * args.steps,
        "kv_cache_bytes": dict(kv_cache_bytes(w), layout=args.kv_layout),
        "clocks": clk,
    }
    if rank == 0 and ws == 1 and not args.no_diagnostics:
        res["diagnostics"] = selection_diagnostics(w, st, budget_s=args.diag_budget)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget, score=args.score)
    st.close()
    if ws > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


# ---------------------------------------------------------------- oracle legs

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def oracle_slab_step(inp, cfg, b, g, index_g):
    """One decode step of the oracle for the heads of KV group g of sequence
    b, with the slab's index already built (as the GPU's index cache is)."""
    import numpy as np

    import oracle as O
    G = cfg.num_q_heads // cfg.num_kv_heads
    n = int(inp["seq_lens"][b])
    attn_scale, index_scale = cfg.scales()
    K = O.gather_rows(inp["k_cache"], inp["page_table"][b], n, g, cfg.page_size)
    V = O.gather_rows(inp["v_cache"], inp["page_table"][b], n, g, cfg.page_size)
    O.index_keys(inp["proj"][g], K[n - 1:n])                 # the appended token
    outs = []
    for h in range(g * G, (g + 1) * G):
        if cfg.head_is_retrieval[h]:
            s = (O.exact_scores(inp["q"][b, h], K, attn_scale) if cfg.score == "exact" else
                 O.index_scores(O.query_index(inp["proj"][g], inp["q_pre"][b, h]), index_g, index_scale))
            S = (O.select_top_p(s, O.stored_top_p(cfg.top_p)) if cfg.mode == "top_p"
                 else O.select_top_k(s, O.top_k_budget(n, cfg.top_k, cfg.top_k_frac)))
        else:
            S = O.local_positions(n, cfg.window, cfg.num_sinks)
        outs.append(O.attend_set(inp["q"][b, h], K, V, S, attn_scale))
    return np.stack(outs)


def cpu_baseline(w, budget_s=15.0, score="index"):
    """Time the oracle as it stands on (b, KV group) slabs of the workload
    until ~budget_s of CPU work; head-steps/s over the slabs processed."""
    import numpy as np

    import oracle as O
    from oracle.workload_inputs import oracle_config, oracle_inputs
    cfg = oracle_config(w)
    cfg.score = score
    G = w.num_q_heads // w.num_kv_heads
    done = 0
    elapsed = 0.0
    slabs = []
    b = 0
    while elapsed < budget_s and b < w.batch:
        inp = oracle_inputs(w, [b])
        n = int(inp["seq_lens"][0])
        for g in range(w.num_kv_heads):
            K = O.gather_rows(inp["k_cache"], inp["page_table"][0], n, g, cfg.page_size)
            index_g = O.index_keys(inp["proj"][g], K)          # setup (prefill), untimed
            t = time.perf_counter()
            oracle_slab_step(inp, cfg, 0, g, index_g)
            elapsed += time.perf_counter() - t
            done += G
            slabs.append((b, g))
            if elapsed >= budget_s:
                break
        b += 1
    return {"value": round(done / elapsed, 3), "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{len(slabs)} (sequence, KV group) slabs = {done} head-steps of the same workload, "
                      f"float64 numpy oracle, index prebuilt (untimed) as on the GPU; {elapsed:.1f} s"}


def run_reference(args):
    ws, rank, local = dist_env()
    if rank != 0:
        return
    import torch

    from oracle.workload_inputs import oracle_config, oracle_inputs
    from workloads import make_workload
    import oracle as O
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    w = workload_for_rank(args, dev, 0)
    cfg = oracle_config(w)
    cfg.score = args.score
    G = w.num_q_heads // w.num_kv_heads
    inp = oracle_inputs(w, [0])
    n = int(inp["seq_lens"][0])
    idx = {}
    for g in range(w.num_kv_heads):
        K = O.gather_rows(inp["k_cache"], inp["page_table"][0], n, g, cfg.page_size)
        idx[g] = O.index_keys(inp["proj"][g], K)
    # each step: one (sequence, KV group) slab = G head-steps
    for i in range(args.warmup):
        oracle_slab_step(inp, cfg, 0, i % w.num_kv_heads, idx[i % w.num_kv_heads])
    t = time.perf_counter()
    for i in range(args.steps):
        oracle_slab_step(inp, cfg, 0, i % w.num_kv_heads, idx[i % w.num_kv_heads])
    el = time.perf_counter() - t
    v = G * args.steps / el
    res = {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded; no datasets or trained weights)",
           "config": bench_config(args, w, ws, l2_flush_needed(args.l2_flush, w)),
           "cpu_baseline": {"kind": "oracle", "cores": _blas_threads(), "value": round(v, 3), "unit": UNIT,
                            "sample": f"each step: one (sequence, KV group) slab of the same workload = "
                                      f"{G} head-steps, float64 numpy oracle, index prebuilt (untimed); "
                                      f"{args.steps} slabs"},
           "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


# ---------------------------------------------------------------- head classifier

# float64 peak of the part: 148 SMs x 64 FP64 FMA per clock x 2 flops x 1965 MHz
# (the recipe's SM count and maximum clock; 64 FP64 lanes per SM)
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12
CLASSIFY_METRIC = "AoH data-free head classification: query heads classified/s (effective rank of W_K^T W_Q)"


def classifier_flops(L, Hq, Hkv, D, d_model) -> dict:
    """Algorithmic float64 flops of one call: the symmetric Gram matrices
    (D (D+1)/2 entries of d_model products each, query and key blocks), their
    Cholesky factors (D^3/3) and X = L_k^T L_q (triangular, D^3/3
    multiply-adds).  The Jacobi sweeps are iterative and not counted."""
    mats = L * (Hq + Hkv)
    return {"gram": 2.0 * mats * D * (D + 1) / 2 * d_model, "cholesky": mats * D ** 3 / 3.0,
            "x_product": L * Hq * 2.0 * D ** 3 / 3.0}


def run_classifier(args):
    import torch
    import torch.distributed as dist

    from head_wise_sparse_02_b200 import sparse_decode as sd
    from workloads import make_projections

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    L = args.layers
    p = make_projections(dev, seed=rank_seed(7 if args.seed is None else args.seed, rank), num_layers=L)
    Hq, Hkv, D, dm = p.num_q_heads, p.num_kv_heads, p.head_dim, p.d_model
    n = ctypes.c_size_t()
    sd._check(sd.LIB.sparse_decode_head_er_workspace_size(L, Hq, Hkv, D, ctypes.byref(n)))
    wsb = torch.empty(n.value, dtype=torch.uint8, device=dev)
    er = torch.empty((L, Hq), dtype=torch.float64, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        sd.sparse_decode_head_effective_rank(p.w_q, p.w_k, Hq, Hkv, D, eff_rank=er, workspace=wsb, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if not bool(torch.isfinite(er).all()):
        raise RuntimeError("a head's Jacobi sweeps did not converge")
    weight_bytes = (p.w_q.numel() + p.w_k.numel()) * 2
    flush = weight_bytes < NO_FLUSH_ABOVE
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    pairs = []
    for _ in range(args.steps):
        if flush:
            flush_buf.zero_()
        a0 = torch.cuda.Event(enable_timing=True); a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        step()
        a1.record(stream)
        pairs.append((a0, a1))
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in pairs) / args.steps
    ms_max = max_over_ranks(ms, dev)

    # end to end: the weights from pinned host memory, the call, the ERs back,
    # and the per-layer classification on the host
    wq_h, wk_h = p.w_q.cpu().pin_memory(), p.w_k.cpu().pin_memory()
    wq_d, wk_d = torch.empty_like(p.w_q), torch.empty_like(p.w_k)
    er_h = torch.empty((L, Hq), dtype=torch.float64).pin_memory()
    n_ret = Hkv // 2

    def e2e_step():
        wq_d.copy_(wq_h, non_blocking=True)
        wk_d.copy_(wk_h, non_blocking=True)
        sd.sparse_decode_head_effective_rank(wq_d, wk_d, Hq, Hkv, D, eff_rank=er, workspace=wsb, stream=stream)
        er_h.copy_(er, non_blocking=True)
        stream.synchronize()
        return [sd.sparse_decode_classify_heads(er_h[l], Hkv, n_ret) for l in range(L)]

    e2e_step()
    barrier()
    t0 = torch.cuda.Event(enable_timing=True); t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, dev)

    fl = classifier_flops(L, Hq, Hkv, D, dm)
    total_fl = sum(fl.values())
    achieved = total_fl / (ms * 1e-3) / 1e12
    heads = ws * L * Hq
    res = {
        "metric": CLASSIFY_METRIC, "value": round(heads / (ms_max * 1e-3), 1), "unit": "heads/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "storage_dtype": "bf16",
        "data": "synthetic (seeded bf16 projections with planted spectra; no trained weights)",
        "config": {"workload": f"aoh_llama3_8b: {L} layers, d_model {dm}, Hq {Hq} / Hkv {Hkv}, d_head {D} "
                               f"(Llama-3.1-8B attention shapes), {n_ret} of {Hkv} groups retrieval",
                   "parallelism": f"replicas x{ws}",
                   "l2": ("flushed between steps (512 MiB write, untimed)" if flush
                          else f"no flush: every step reads {weight_bytes / 1e9:.2f} GB of weights")},
        "roofline": {"kernel": "head_effective_rank (gram + cholesky + jacobi launches)", "bound": "alu",
                     "achieved": round(achieved, 3), "peak": round(FP64_PEAK_TFLOPS, 1),
                     "peak_kind": "derived fp64: 148 SMs x 64 FMA/clk x 2 x 1965 MHz", "unit": "TFLOP/s",
                     "frac": round(achieved / FP64_PEAK_TFLOPS, 4), "algorithmic_flops_per_launch": fl,
                     "traffic": None},
        "weights_hbm_gbs": round(weight_bytes / (ms * 1e-3) / 1e9, 1),
        "e2e": {"value": round(heads / (e2e_ms * 1e-3), 1), "unit": "heads/s",
                "h2d_bytes_per_step": int(weight_bytes), "d2h_bytes_per_step": int(L * Hq * 8)},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = classifier_cpu_baseline(p, budget_s=args.cpu_budget)
    if ws > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def classifier_cpu_baseline(p, budget_s: float = 15.0):
    """The oracle's eigenvalue route (C_h, float64 numpy), head by head over
    the layers in order, until the budget runs out: heads/s."""
    import numpy as np

    import oracle as O
    G = p.num_q_heads // p.num_kv_heads
    done, t0 = 0, time.perf_counter()
    for layer in range(p.num_layers):
        wq = p.w_q[layer].float().cpu().numpy().astype(np.float64)
        wk = p.w_k[layer].float().cpu().numpy().astype(np.float64)
        for h in range(p.num_q_heads):
            O.effective_rank_of_spectrum(O.singular_values_sylvester(
                O.head_block(wq, h, p.head_dim), O.head_block(wk, h // G, p.head_dim)))
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    return {"kind": "oracle", "value": round(done / el, 2), "unit": "heads/s", "cores": _blas_threads(),
            "sample": f"{done} heads of the same synthetic weights (layers in order), float64 numpy, "
                      "eigenvalues of C_h per head"}


# ---------------------------------------------------------------- head-wise prefill

PREFILL_METRIC = "head-wise prefill tokens/s (retrieval heads dense causal, local heads sinks + window)"


def load_bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def prefill_flops(w, chunk_lens) -> float:
    """Algorithmic flops of a prefill: 4 d per (query, head, key seen) (Q K^T
    and P V, two flops per multiply-add)."""
    import numpy as np
    total = 0.0
    n_ret = sum(1 for x in w.head_is_retrieval if x)
    n_loc = w.num_q_heads - n_ret
    for n, t in zip(w.seq_lens.cpu().tolist(), chunk_lens):
        pos = np.arange(n - t, n, dtype=np.float64)
        total += n_ret * float(np.sum(pos + 1))                           # keys 0 .. pos
        sinks = np.minimum(pos + 1, w.num_sinks)                           # keys [0, S) within [0, pos]
        win = np.maximum(0.0, pos - np.maximum(w.num_sinks, pos - w.window + 1) + 1)
        total += n_loc * float(np.sum(sinks + win))
    return 4.0 * w.head_dim * total


def prefill_workload(args, device, rank):
    from workloads import make_workload
    N = args.seq_len or 32768
    return make_workload("llama3_8b_topp", device, B=1, N=N, permute=True,
                         seed=rank_seed(1 if args.seed is None else args.seed, rank))


def run_prefill(args):
    import torch
    import torch.distributed as dist

    from head_wise_sparse_02_b200.sparse_decode import SparseDecode
    from workloads import prefill_inputs

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = prefill_workload(args, dev, rank)
    N = int(w.seq_lens[0])
    sd = SparseDecode(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                      head_is_retrieval=w.head_is_retrieval, num_pages=int(w.k_cache.shape[0]), max_batch=1,
                      max_pages_per_seq=int(w.page_table.shape[1]), proj=w.proj, window=w.window,
                      num_sinks=w.num_sinks, mode=w.mode, top_p=w.top_p)
    q, starts = prefill_inputs(w, [N], seed=5)
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        sd.prefill(q, w.k_cache, w.v_cache, w.page_table, w.seq_lens, starts, out, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if sd.error_word():
        raise RuntimeError("device error word set after warm-up")
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    pairs = []
    for _ in range(args.steps):
        flush_buf.zero_()
        a0 = torch.cuda.Event(enable_timing=True); a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        step()
        a1.record(stream)
        pairs.append((a0, a1))
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in pairs) / args.steps
    ms_max = max_over_ranks(ms, dev)

    # dense causal attention of every head over the same keys (torch SDPA,
    # bf16): the dense baseline the pages compare prefill against
    G = w.num_q_heads // w.num_kv_heads
    pages = w.page_table[0, :(N + 15) // 16].long()
    Kc = w.k_cache[pages].permute(1, 0, 2, 3).reshape(w.num_kv_heads, -1, w.head_dim)[:, :N]
    Vc = w.v_cache[pages].permute(1, 0, 2, 3).reshape(w.num_kv_heads, -1, w.head_dim)[:, :N]
    Kd = Kc.repeat_interleave(G, dim=0)[None].contiguous()
    Vd = Vc.repeat_interleave(G, dim=0)[None].contiguous()
    Qd = q.permute(1, 0, 2)[None].contiguous()
    dense = lambda: torch.nn.functional.scaled_dot_product_attention(Qd, Kd, Vd, is_causal=True)  # noqa: E731
    for _ in range(2):
        dense()
    torch.cuda.synchronize()
    d_pairs = []
    for _ in range(max(1, args.steps // 2)):
        flush_buf.zero_()
        a0 = torch.cuda.Event(enable_timing=True); a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        dense()
        a1.record(stream)
        d_pairs.append((a0, a1))
    torch.cuda.synchronize()
    dense_ms = sum(a.elapsed_time(b) for a, b in d_pairs) / len(d_pairs)
    del Kd, Vd, Qd
    # the same kernel with every head a retrieval head (dense causal): the
    # speed-up the head split itself buys, kernel quality aside
    sd_dense = SparseDecode(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                            head_is_retrieval=[1] * w.num_q_heads, num_pages=int(w.k_cache.shape[0]), max_batch=1,
                            max_pages_per_seq=int(w.page_table.shape[1]), proj=w.proj, window=w.window,
                            num_sinks=w.num_sinks, mode=w.mode, top_p=w.top_p)
    for _ in range(2):
        sd_dense.prefill(q, w.k_cache, w.v_cache, w.page_table, w.seq_lens, starts, out, stream)
    torch.cuda.synchronize()
    s_pairs = []
    for _ in range(max(1, args.steps // 2)):
        flush_buf.zero_()
        a0 = torch.cuda.Event(enable_timing=True); a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        sd_dense.prefill(q, w.k_cache, w.v_cache, w.page_table, w.seq_lens, starts, out, stream)
        a1.record(stream)
        s_pairs.append((a0, a1))
    torch.cuda.synchronize()
    same_ms = sum(a.elapsed_time(b) for a, b in s_pairs) / len(s_pairs)
    sd_dense.close()

    # end to end: queries from pinned host memory, the call, outputs back
    q_h = q.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    q_d = torch.empty_like(q)

    def e2e_step():
        q_d.copy_(q_h, non_blocking=True)
        sd.prefill(q_d, w.k_cache, w.v_cache, w.page_table, w.seq_lens, starts, out, stream)
        out_h.copy_(out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    t0 = torch.cuda.Event(enable_timing=True); t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, dev)

    fl = prefill_flops(w, [N])
    peak, kind = load_bf16_peak()
    achieved = fl / (ms * 1e-3) / 1e12
    tokens = ws * N
    n_ret = sum(w.head_is_retrieval)
    res = {
        "metric": PREFILL_METRIC, "value": round(tokens / (ms_max * 1e-3), 1), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "storage_dtype": "bf16",
        "data": "synthetic (seeded; no datasets or trained weights)",
        "config": {"workload": f"prefill_llama3_8b: B=1, N={N} full prefill, Hq={w.num_q_heads}/Hkv="
                               f"{w.num_kv_heads}, d={w.head_dim}, {n_ret} retrieval heads (dense causal) + "
                               f"{w.num_q_heads - n_ret} local (window {w.window} + {w.num_sinks} sinks)",
                   "parallelism": f"replicas x{ws}", "l2": "flushed between steps (512 MiB write, untimed)"},
        "roofline": {"kernel": ("prefill_tc_kernel (tcgen05, accumulators in tensor memory)" if w.head_dim == 128
                                else "prefill_kernel (mma.sync)"), "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": f"{kind} bf16_tflops (cuBLAS bf16 GEMM)", "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "algorithmic_flops_per_launch": fl, "traffic": None,
                     "note": "P V runs as two bf16 MMAs (P split hi + lo): 1.5x the algorithmic MMA work"},
        "dense_causal_sdpa_ms": round(dense_ms, 3),
        "speedup_vs_dense_sdpa": round(dense_ms / ms, 3),
        "dense_same_kernel_ms": round(same_ms, 3),
        "speedup_vs_dense_same_kernel": round(same_ms / ms, 3),
        "e2e": {"value": round(tokens / (e2e_ms * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(q_h.numel() * 2), "d2h_bytes_per_step": int(out_h.numel() * 4)},
        "gpu_launches": args.steps,
        "clocks": clk,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = prefill_cpu_baseline(w, q, starts, budget_s=args.cpu_budget)
    sd.close()
    if ws > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def prefill_cpu_baseline(w, q, starts, budget_s: float = 15.0):
    """The oracle on the host: query rows of the last positions (the longest
    key ranges) for every head, until the budget runs out; tokens/s."""
    import oracle as O
    from oracle.workload_inputs import oracle_config, oracle_inputs
    inp = oracle_inputs(w)
    cfg = oracle_config(w)
    qn = q.float().cpu().numpy()
    st = starts.cpu().numpy()
    total = int(st[-1])
    done, t0 = 0, time.perf_counter()
    r = total - 1
    while r >= 0 and time.perf_counter() - t0 < budget_s:
        O.prefill_reference(cfg, qn, inp["k_cache"], inp["v_cache"], inp["page_table"], inp["seq_lens"], st,
                            pairs=[(r, h) for h in range(w.num_q_heads)])
        done += 1
        r -= 1
    el = time.perf_counter() - t0
    return {"kind": "oracle", "value": round(done / el, 3), "unit": "tokens/s", "cores": _blas_threads(),
            "sample": f"the last {done} query positions (all heads) of the same prefill, float64 numpy "
                      "(the longest key ranges: a lower bound on the average rate)"}


def run_prefill_reference(args):
    """The oracle as the prefill's reference arm: each step one query position
    (all heads) of the same prefill, from the last position down."""
    ws, rank, local = dist_env()
    if rank != 0:
        return
    import torch

    from workloads import prefill_inputs
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    w = prefill_workload(args, dev, 0)
    N = int(w.seq_lens[0])
    q, starts = prefill_inputs(w, [N], seed=5)
    t = time.perf_counter()
    base = prefill_cpu_baseline(w, q, starts, budget_s=args.cpu_budget)
    el = time.perf_counter() - t
    v = base["value"]
    n_ret = sum(w.head_is_retrieval)
    res = {"impl": "reference", "metric": PREFILL_METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 / v, 3) if v else None,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded; no datasets or trained weights)",
           "config": {"workload": f"prefill_llama3_8b: B=1, N={N} full prefill, Hq={w.num_q_heads}/Hkv="
                                  f"{w.num_kv_heads}, d={w.head_dim}, {n_ret} retrieval heads (dense causal) + "
                                  f"{w.num_q_heads - n_ret} local (window {w.window} + {w.num_sinks} sinks)",
                      "parallelism": f"replicas x{ws}", "l2": "flushed between steps (512 MiB write, untimed)"},
           "cpu_baseline": dict(base, sample=base["sample"] + f"; {el:.1f} s"),
           "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def run_classifier_reference(args):
    """The oracle as the classifier's reference arm: each step one query head
    of the same synthetic weights by the eigenvalue route, on the host."""
    ws, rank, local = dist_env()
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle as O
    from workloads import make_projections
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    L = args.layers
    p = make_projections(dev, seed=7 if args.seed is None else args.seed, num_layers=L)
    G = p.num_q_heads // p.num_kv_heads
    wq = p.w_q[0].float().cpu().numpy().astype(np.float64)
    wk = p.w_k[0].float().cpu().numpy().astype(np.float64)

    def one(i):
        h = i % p.num_q_heads
        O.effective_rank_of_spectrum(O.singular_values_sylvester(O.head_block(wq, h, p.head_dim),
                                                                 O.head_block(wk, h // G, p.head_dim)))

    for i in range(args.warmup):
        one(i)
    t = time.perf_counter()
    for i in range(args.steps):
        one(i)
    el = time.perf_counter() - t
    v = args.steps / el
    flush = (p.w_q.numel() + p.w_k.numel()) * 2 < NO_FLUSH_ABOVE
    res = {"impl": "reference", "metric": CLASSIFY_METRIC, "value": round(v, 3), "unit": "heads/s", "n_gpus": ws,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded bf16 projections with planted spectra; no trained weights)",
           "config": {"workload": f"aoh_llama3_8b: {L} layers, d_model {p.d_model}, Hq {p.num_q_heads} / Hkv "
                                  f"{p.num_kv_heads}, d_head {p.head_dim} (Llama-3.1-8B attention shapes), "
                                  f"{p.num_kv_heads // 2} of {p.num_kv_heads} groups retrieval",
                      "parallelism": f"replicas x{ws}",
                      "l2": ("flushed between steps (512 MiB write, untimed)" if flush
                             else f"no flush: every step reads {(p.w_q.numel() + p.w_k.numel()) * 2 / 1e9:.2f} "
                                  "GB of weights")},
           "cpu_baseline": {"kind": "oracle", "cores": _blas_threads(), "value": round(v, 3), "unit": "heads/s",
                            "sample": f"each step: one query head of layer 0 (eigenvalues of C_h, float64 "
                                      f"numpy); {args.steps} heads"},
           "e2e": {"value": round(v, 3), "unit": "heads/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="topk_128k")
    ap.add_argument("--seed", type=int, default=None, help="base seed (default: the workload's own)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling)")
    ap.add_argument("--seq-len", type=int, default=0, help="override the workload's context length")
    ap.add_argument("--top-p", type=float, default=0.0, help="override the workload's top-p")
    ap.add_argument("--alpha", type=float, default=0.0, help="long_zipf: Zipf exponent of the score profile")
    ap.add_argument("--top-k-frac", type=float, default=0.0, help="override the workload's top-k fraction")
    ap.add_argument("--score", choices=["index", "exact"], default="index",
                    help="select by the r = 16 index (the method) or by the exact logits (reference selector)")
    ap.add_argument("--l2-flush", choices=["auto", "on", "off"], default="auto",
                    help="flush L2 between timed steps (auto: when a step touches < 8x the L2)")
    ap.add_argument("--kv-layout", choices=["full", "split"], default="full",
                    help="split: paged caches of the retrieval groups only, compacted local caches")
    ap.add_argument("--no-diagnostics", action="store_true")
    ap.add_argument("--diag-budget", type=float, default=20.0)
    ap.add_argument("--layers", type=int, default=32, help="aoh_llama3_8b: layers classified per step")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)          # timing rule: at least 3 warm-up steps
    if args.workload == "prefill_llama3_8b":
        if args.impl == "reference":
            run_prefill_reference(args)
        else:
            run_prefill(args)
    elif args.workload == "aoh_llama3_8b":
        if args.impl == "reference":
            run_classifier_reference(args)
        else:
            run_classifier(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
