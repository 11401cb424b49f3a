"""Host-side logic of bench.py: rank plumbing over gloo (world size 2) and
the oracle leg of the CPU baseline / reference arm."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle as O
from tests.helpers import oracle_config, oracle_inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        m = bench.max_over_ranks(1.5 + r, device="cpu")
        bench.barrier()
        q.put((r, ws, m, bench.rank_seed(2, r)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_seeds_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[2] for g in got] == [2.5, 2.5]           # max over ranks reaches every rank
    assert got[0][1] == got[1][1] == 2
    assert got[0][3] != got[1][3]                      # each rank draws its own batch


def test_single_process_max_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_oracle_slab_step_matches_decode_reference():
    from workloads import make_workload
    w = make_workload("llama3_8b_topp", "cpu", B=1, N=900, window=100)
    cfg = oracle_config(w)
    inp = oracle_inputs.__wrapped__(w) if hasattr(oracle_inputs, "__wrapped__") else None
    # oracle_inputs moves tensors with .cpu(); the workload is already on the CPU
    inp = oracle_inputs(w, [0])
    G = w.num_q_heads // w.num_kv_heads
    ref = O.decode_reference(cfg, **inp)
    for g in (0, 1, 5):
        K = O.gather_rows(inp["k_cache"], inp["page_table"][0], 900, g, 16)
        out = bench.oracle_slab_step(inp, cfg, 0, g, O.index_keys(inp["proj"][g], K))
        for i, h in enumerate(range(g * G, (g + 1) * G)):
            np.testing.assert_array_equal(out[i], ref.out[(0, h)])


def test_reference_arm_prints_one_contract_line(capsys):
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the keys the harness reads, on a shrunken workload."""
    import json
    bench.main(["--impl", "reference", "--workload", "tiny_ref", "--seq-len", "300", "--steps", "2",
                "--warmup", "1"])
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3   # warm-up raised to 3
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_kernel_hash_ignores_comments_only():
    """roofline.traffic stays tied to the code it was captured on: the hash
    leaves comments and whitespace out, and changes with any code token."""
    src = (b'// header\n#include <x.h>\n/* block\n comment */ int f(int a) {  // why\n'
           b'  const char *s = "a // not a comment /* nor this */";\n  return a + \'/\';\n}\n')
    edited = (b'// a new header, longer\n\n#include <x.h>\n/* other */ int f(int a) {\n'
              b'  const char *s = "a // not a comment /* nor this */";   // note\n  return a + \'/\';\n}\n')
    changed = src.replace(b"a + '/'", b"a - '/'")
    assert bench.code_only(src) == bench.code_only(edited)
    assert bench.code_only(src) != bench.code_only(changed)
    assert b'"a // not a comment /* nor this */"' in bench.code_only(src)
    assert b"header" not in bench.code_only(src) and b"why" not in bench.code_only(src)
