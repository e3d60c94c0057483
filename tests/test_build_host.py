"""Register budgets of the kernels, checked at compile time (no GPU).

Every source is compiled for sm_100a with the library's flags and
`-Xptxas -v`. The tensor-core loops (prefill, CTA-pair prefill, the bf16
split-K decode, the 32-row multi-token kernel) must not spill: a spill there
puts local-memory traffic on every key tile. The two instances that already
spill a little stay within their measured budgets (the 64-row multi-token
kernel's running state at 255 registers, the int8 head_dim-256 decode's
prologue at its 128-register launch bound), so an edit that grows them is
caught here before it costs GPU time."""
from __future__ import annotations

import concurrent.futures as cf
import os
import re
import shutil
import subprocess
import tempfile

import pytest

from hybrid_local_global_b200 import build

ENTRY = re.compile(r"Compiling entry function '([^']+)' for 'sm_100a'")
SPILL = re.compile(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads")
REGS = re.compile(r"Used (\d+) registers")

# (pattern in the mangled name, largest spill store bytes, largest spill load
# bytes); the two nonzero budgets sit a little above what they compile to
# today (64-row multi-token: 56-68 / 68-80; int8 head_dim 256: 76 / 116)
BUDGETS = [
    (r"k_prefill_tcILi\d+ELb[01]E", 0, 0),
    (r"k_prefill_pairILi\d+E", 0, 0),
    (r"k_decode_splitILi\d+ELi\d+ELb[01]E", 0, 0),
    (r"k_verify_tcILi\d+ELi32ELb[01]E", 0, 0),
    (r"k_verify_tcILi\d+ELi64ELb[01]E", 80, 96),
    (r"k_decode_split_q8ILi512ELb[01]E", 0, 0),
    (r"k_decode_split_q8ILi256ELb[01]E", 96, 128),
    (r"k_prefill_ropeILi\d+ELb[01]E", 0, 0),
    (r"k_decode_rope_appendILi\d+E", 0, 0),
    (r"k_decode_combineILi\d+E", 0, 0),
]


def _ptxas_report(src, out_dir):
    cmd = [build.NVCC, *build.ARCH, *build.FLAGS, "-Xptxas", "-v", "-c", src,
           "-o", os.path.join(out_dir, os.path.basename(src) + ".o")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    kernels, name = {}, None
    for line in r.stderr.splitlines():
        m = ENTRY.search(line)
        if m:
            name = m.group(1)
            continue
        m = SPILL.search(line)
        if m and name:
            kernels.setdefault(name, {}).update(stack=int(m.group(1)), st=int(m.group(2)), ld=int(m.group(3)))
        m = REGS.search(line)
        if m and name:
            kernels.setdefault(name, {})["regs"] = int(m.group(1))
    return kernels


@pytest.fixture(scope="module")
def report():
    if not os.path.exists(build.NVCC):
        pytest.skip("nvcc not found")
    out = tempfile.mkdtemp(prefix="ptxas_")
    try:
        with cf.ThreadPoolExecutor(max_workers=8) as ex:
            parts = list(ex.map(lambda s: _ptxas_report(s, out), build.sources()))
    finally:
        shutil.rmtree(out, ignore_errors=True)
    merged = {}
    for p in parts:
        merged.update(p)
    return merged


def test_every_budgeted_kernel_is_compiled(report):
    for pat, _, _ in BUDGETS:
        assert any(re.search(pat, k) for k in report), "no kernel matches %s" % pat


def test_spills_within_budget(report):
    for pat, st_max, ld_max in BUDGETS:
        for name, r in report.items():
            if re.search(pat, name):
                assert r["st"] <= st_max and r["ld"] <= ld_max, \
                    "%s: %d / %d bytes of spill stores / loads (budget %d / %d)" % (name, r["st"], r["ld"], st_max, ld_max)


# register ceilings that give the residency the kernels are tuned for (65,536
# registers per SM): four 128-thread decode CTAs per SM at head_dim 256, two
# 192-thread local multi-token CTAs per SM
RESIDENCY = [
    (r"k_decode_splitILi256ELi4ELb[01]E", 128),
    (r"k_decode_split_q8ILi256ELb[01]E", 128),
    (r"k_verify_tcILi256ELi32ELb1E", 65536 // (2 * 192)),
]


def test_registers_give_the_intended_residency(report):
    for pat, cap in RESIDENCY:
        hits = [(n, r["regs"]) for n, r in report.items() if re.search(pat, n)]
        assert hits, pat
        for n, regs in hits:
            assert regs <= cap, "%s: %d registers, at most %d for its residency" % (n, regs, cap)
