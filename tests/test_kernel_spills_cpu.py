"""Register spills of the decode step's kernels (CPU only: nvcc cross-compiles for sm_100a).

A kernel that spills at its launch configuration moves the spilled registers
through local memory.  On the 1024-thread fused union resolve, 16 register-held
buffer entries per thread spilled, and the spill stores mostly missed L1 at its
shared-memory footprint: about 22 MB of local-memory traffic per launch,
against about 6 MB of bytes the kernel needs.  These tests compile the decode
sources with `ptxas -v` and require no spill stores or loads in the kernels
that the d_head 128 decode workloads launch (query heads per KV head 1, 2, 4
or 8).  The d_head 64 attend instantiations are left out: ptxas keeps them at
128 registers with a few dozen bytes of spills, and the workload that runs
them is bound by launch latency.
"""

import os
import re
import subprocess
import tempfile

import pytest

from head_wise_sparse_02_b200 import build as B


def _spills(src: str) -> dict:
    """{mangled kernel name: (stack frame, spill stores, spill loads)} of one source."""
    try:
        cc = B.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not found")
    with tempfile.TemporaryDirectory(prefix="sd_spill_") as tmp:
        r = subprocess.run([cc, *B.ARCH, *B.FLAGS, "-Xptxas", "-v", "-c", os.path.join(B.CSRC, src),
                            "-o", os.path.join(tmp, "x.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    out, name = {}, None
    for line in (r.stdout + r.stderr).splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            name = m.group(1)
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and name:
            out[name] = tuple(int(x) for x in m.groups())
            name = None
    return out


def _check(report: dict, patterns) -> None:
    for pat in patterns:
        hits = {k: v for k, v in report.items() if re.search(pat, k)}
        assert hits, f"no kernel matches {pat}"
        spilling = {k: v for k, v in hits.items() if v[1] or v[2]}
        assert not spilling, f"spills (stack, stores, loads): {spilling}"


@pytest.mark.timeout(300)
def test_selection_kernels_do_not_spill():
    _check(_spills("sd_select_stream.cu"), [
        r"resolve_union_kernelILb[01]ELi[124]E",        # fused union resolve, top-k and top-p
        r"topk_resolve_kernel",
        r"topp_resolve_kernel",
        r"stream_kernelILi[1248]ELi[012]E",             # index stream passes
        r"window_kernelILi[1248]ELb[01]E",              # sample window
    ])


@pytest.mark.timeout(300)
def test_attend_kernels_do_not_spill_at_d128():
    _check(_spills("sd_attend.cu"), [
        r"attend_main_kernelILi128ELi[1248]E",
        r"attend_plan_kernelILi128ELi[1248]E",
        r"attend_prefix_kernelILi128E",
    ])
