"""Profiling helpers: a small driver to put under ``ncu``, and summaries of
what ``ncu`` writes.

    python -m hybrid_local_global_b200.profiling run --workload NAME [--reps R] [--layers 0,4]
    python -m hybrid_local_global_b200.profiling launches LAUNCHES.csv
    python -m hybrid_local_global_b200.profiling raw RAW.csv [--per-launch-units U]

``run`` builds one workload of ``workloads.WORKLOADS`` (synthetic, seeded
inputs, as in bench.py) and runs its prefill or decode block R times, with
nothing else launched, so that ``ncu -k ... -c ...`` captures a known launch.
``--layers`` restricts the pass to some layers (a global-only capture).

``launches`` folds an ``ncu --metrics gpu__time_duration.sum --csv`` launch
list into one row per kernel: launches, total time and share of the total.

``raw`` reads ``ncu -i REP --page raw --csv`` and prints, per captured launch,
the DRAM bytes, duration, and the throughput, tensor-pipe, occupancy and
warp-stall counters the roofline uses.

``digest`` prints the source digest of a kernel (its .cu file and the
headers it includes): summaries under profiles/ carry one in their
``traffic-record:`` line, and bench.py reports a recorded DRAM traffic only
while the kernel's sources still have that digest.
"""
from __future__ import annotations

import argparse
import collections
import csv
import hashlib
import os
import re
import sys

CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc")

# the sources each recorded kernel is built from
KERNEL_SOURCES = {
    "k_prefill_tc": ("prefill_tc.cu", "tc.cuh", "common.cuh", "tmap.cu", "tmap.h"),
    "k_prefill_pair": ("prefill_pair.cu", "pair.cuh", "tc.cuh", "common.cuh", "tmap.cu", "tmap.h"),
    "k_decode_split": ("decode.cu", "mma_sync.cuh", "common.cuh"),
    "k_decode_split_q8": ("decode_q8.cu", "mma_sync.cuh", "tc.cuh", "common.cuh", "tmap.cu", "tmap.h"),
    "k_verify_tc": ("verify_tc.cu", "tc.cuh", "common.cuh", "tmap.cu", "tmap.h"),
}


def _code_only(text: str) -> str:
    """Source text without comments and blank lines (string literals in
    these sources hold no comment markers), so that a record outlives an
    edit of comments only."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_digest(kernel: str) -> str:
    """First 16 hex digits of sha256 over the code (comments and blank lines
    removed) of the kernel's source files, in order."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_records(profiles_dir: str) -> list[dict]:
    """``traffic-record: key=value ...`` lines of the summaries in profiles_dir."""
    out = []
    if not os.path.isdir(profiles_dir):
        return out
    for name in sorted(os.listdir(profiles_dir)):
        if not name.endswith((".md", ".txt")):
            continue
        for line in open(os.path.join(profiles_dir, name)):
            line = line.strip().strip("`")
            if line.startswith("traffic-record:"):
                rec = dict(kv.split("=", 1) for kv in line[len("traffic-record:"):].split())
                rec["file"] = name
                out.append(rec)
    return out


def _kernel_short(name: str) -> str:
    for pre in ("void ", "hlg::", "(anonymous namespace)::", "<unnamed>::", "unnamed>::"):
        name = name.replace(pre, "")
    return name.split("(")[0].strip()


def _rows(path):
    rows = list(csv.reader(open(path, newline="")))
    hdr_i = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    return rows[hdr_i], rows[hdr_i + 1:]


def summarize_launches(path: str) -> str:
    hdr, data = _rows(path)
    ki, mi, vi = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    ui = hdr.index("Metric Unit") if "Metric Unit" in hdr else None
    agg = collections.OrderedDict()
    for r in data:
        if len(r) <= vi or r[mi] != "gpu__time_duration.sum":
            continue
        v = float(r[vi].replace(",", ""))
        unit = r[ui] if ui is not None else "ns"
        v_us = v / 1e3 if unit in ("ns", "nsecond") else (v if unit in ("us", "usecond") else v * 1e3)
        k = _kernel_short(r[ki])
        n, t = agg.get(k, (0, 0.0))
        agg[k] = (n + 1, t + v_us)
    tot = sum(t for _, t in agg.values()) or 1.0
    out = ["%-44s %9s %13s %12s %8s" % ("kernel", "launches", "total (us)", "avg (us)", "share")]
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        out.append("%-44s %9d %13.1f %12.2f %7.2f%%" % (k[:44], n, t, t / n, 100.0 * t / tot))
    out.append("%-44s %9d %13.1f" % ("all", sum(n for n, _ in agg.values()), tot))
    return "\n".join(out)


RAW_KEYS = [
    ("gpu__time_duration.sum", "duration"),
    ("dram__bytes_read.sum", "DRAM read"),
    ("dram__bytes_write.sum", "DRAM write"),
    ("gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed", "DRAM throughput % of peak"),
    ("dram__cycles_active.avg.pct_of_peak_sustained_elapsed", "DRAM active %"),
    ("sm__throughput.avg.pct_of_peak_sustained_elapsed", "SM throughput %"),
    ("lts__t_bytes.sum", "L2 bytes"),
    ("launch__registers_per_thread", "registers / thread"),
    ("launch__grid_size", "grid"),
    ("launch__block_size", "block"),
    ("sm__warps_active.avg.pct_of_peak_sustained_active", "warps active %"),
]


def summarize_raw(path: str, units: float | None = None) -> str:
    hdr, data = _rows(path)
    # the raw page is wide: one row per launch, one column per metric
    name_i = hdr.index("Kernel Name")
    units_row = data[0] if data and not data[0][name_i] else None
    launches = [r for r in data if len(r) > name_i and r[name_i]]
    out = []
    for r in launches:
        get = {h: r[i] for i, h in enumerate(hdr) if i < len(r)}
        unit_of = {h: units_row[i] for i, h in enumerate(hdr)} if units_row else {}
        out.append("launch: %s" % _kernel_short(get["Kernel Name"]))
        for key, label in RAW_KEYS:
            if key in get:
                out.append("  %-34s %s %s  (%s)" % (label, get[key], unit_of.get(key, ""), key))
        tensor = [h for h in hdr if re.match(r"sm__pipe_tensor.*cycles_active.*pct", h) or
                  re.match(r"sm__inst_executed_pipe_tensor.*pct", h)]
        for h in sorted(tensor):
            out.append("  %-34s %s  (%s)" % ("tensor pipe", get.get(h, ""), h))
        stalls = []
        for h in hdr:
            m = re.match(r"smsp__average_warps_issue_stalled_(\w+)_per_issue_active\.ratio$", h)
            if m and get.get(h):
                try:
                    stalls.append((float(get[h].replace(",", "")), m.group(1)))
                except ValueError:
                    pass
        if stalls:
            stalls.sort(reverse=True)
            out.append("  top warp stalls (cycles per issued instruction): " +
                       ", ".join("%s %.2f" % (n, v) for v, n in stalls[:6]))
        if units and "dram__bytes_read.sum" in get:
            def _b(key):
                v = float(get[key].replace(",", ""))
                u = unit_of.get(key, "byte")
                scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6,
                         "GB": 1e9}.get(u, 1)
                return v * scale
            tot = _b("dram__bytes_read.sum") + _b("dram__bytes_write.sum")
            out.append("  DRAM bytes per unit: %.1f (units %g)" % (tot / units, units))
    return "\n".join(out)


def run(workload: str, reps: int, layers: list[int] | None) -> None:
    import torch

    from . import native, synth
    from .stack import AttentionStack
    from .workloads import WORKLOADS

    w = WORKLOADS[workload]
    dev = torch.device("cuda", 0)
    st = AttentionStack(w, dev)
    g = synth.generator(w.seed, dev)
    todo = layers if layers else list(range(st.n_layers))
    if w.kind == "prefill":
        ws = torch.empty(st.prefill_workspace_bytes(), dtype=torch.uint8, device=dev)
        lens = torch.full((w.batch,), w.prior, dtype=torch.int32, device=dev) if w.prior else None
        bufs = {}
        for l in todo:
            t = st.layer_type(l)
            q = synth.randn_bf16((w.batch, w.seq, w.n_q_heads, t.head_dim), g, dev)
            k = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, dev, scale=w.k_scale)
            v = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, dev)
            if w.prior and not st.is_shared(l):
                synth.fill_randn_bf16_(st.k_cache[l][:, :, :w.prior], g)
                synth.fill_randn_bf16_(st.v_cache[l][:, :, :w.prior], g)
            bufs[l] = (q, k, v, torch.empty_like(q))
        for _ in range(reps):
            for l in todo:
                q, k, v, out = bufs[l]
                st.prefill_layer(l, q, k, v, out, workspace=ws, seq_lens_before=lens)
    else:
        if w.len_lo == w.len_hi:
            lens_cpu = torch.full((w.batch,), w.len_hi, dtype=torch.int32)
        else:
            lens_cpu = synth.decode_lengths(w.batch, w.len_lo, w.len_hi, seed=w.seed)
        lens = lens_cpu.to(dev)
        max_len = int(lens_cpu.max())
        for l in todo:
            if not st.is_shared(l):
                synth.fill_cache_(st.k_cache[l], g)
                if st.v_cache[l] is not st.k_cache[l]:
                    synth.fill_cache_(st.v_cache[l], g)
        T = w.tokens  # > 1: multi-token decode
        ws_bytes = st.decode_multi_workspace_bytes(T, max_len) if T > 1 else st.decode_workspace_bytes(max_len)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        tok = (T,) if T > 1 else ()
        bufs = {}
        for l in todo:
            t = st.layer_type(l)
            q = synth.randn_bf16((w.batch,) + tok + (w.n_q_heads, t.head_dim), g, dev)
            k = synth.randn_bf16((w.batch,) + tok + (t.n_kv_heads, t.head_dim), g, dev)
            v = synth.randn_bf16((w.batch,) + tok + (t.n_kv_heads, t.head_dim), g, dev)
            bufs[l] = (q, k, v, torch.empty_like(q))
        layer_call = st.decode_multi_layer if T > 1 else st.decode_layer
        for _ in range(reps):
            for l in todo:
                q, k, v, out = bufs[l]
                layer_call(l, q, k, v, out, seq_lens=lens, max_seq_len=max_len, workspace=ws)
    torch.cuda.synchronize()
    rc = native.gemma_attn_sync_status()
    if rc != 0:
        raise SystemExit("device status %d: %s" % (rc, native.gemma_last_error()))
    print("ran %s x%d, layers %s" % (workload, reps, todo))


def main(argv=None):
    ap = argparse.ArgumentParser(prog="python -m hybrid_local_global_b200.profiling")
    sub = ap.add_subparsers(dest="cmd", required=True)
    r = sub.add_parser("run")
    r.add_argument("--workload", required=True)
    r.add_argument("--reps", type=int, default=2)
    r.add_argument("--layers", default="")
    la = sub.add_parser("launches")
    la.add_argument("csv")
    rw = sub.add_parser("raw")
    rw.add_argument("csv")
    rw.add_argument("--per-launch-units", type=float, default=None)
    dg = sub.add_parser("digest")
    dg.add_argument("kernel", choices=sorted(KERNEL_SOURCES))
    a = ap.parse_args(argv)
    if a.cmd == "run":
        layers = [int(x) for x in a.layers.split(",") if x.strip()] or None
        run(a.workload, a.reps, layers)
    elif a.cmd == "launches":
        print(summarize_launches(a.csv))
    elif a.cmd == "digest":
        print(kernel_digest(a.kernel))
    else:
        print(summarize_raw(a.csv, a.per_launch_units))


if __name__ == "__main__":
    sys.exit(main())
