#!/usr/bin/env python
"""Benchmark of the interleaved local/global attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--decode-workload NAME|none]
                    [--decode-int8-workload NAME|none]

One JSON line on rank 0. A step is one pass of the prefill block named by
--workload (default: the E2B-shaped 5-layer block, B1 S8192: layer schedule,
RoPE + cache write, attention for every layer) over resident synthetic
inputs; `value` is its algorithmic TFLOP/s (4*B*Hq*D per visible query-key
pair, masked pairs not counted) over all ranks. The `decode` object measures
the batched decode block named by --decode-workload (default: 31B-shaped,
6 layers, B64, KV lengths U[4096,131072], last two layers shared) in KV GB/s;
`decode_int8` the same block on int8 KV caches (GB/s of the int8 rows read,
and `bf16_equivalent_gbs`: the bf16 bytes the same keys would take, per
second).

Each part runs two timed passes of the same steps, both bracketed by a
barrier and a synchronize and timed with CUDA events on the stream: the step
time comes from an uninstrumented pass; the per-kernel device times of the
roofline (`kernels`, `roofline.achieved`) come from the second pass, where
the library records events around every launch.

--impl reference times the fp64 CPU oracle (the path's reference
implementation here) on the host cores, each step a bounded sample of rows
of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hybrid_local_global_b200 import synth  # noqa: E402
from hybrid_local_global_b200.workloads import WORKLOADS, prefill_flops, visible_pairs_prefill  # noqa: E402

METRIC = "attention prefill TFLOP/s and decode KV GB/s on 1 B200, as % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every 2 ms."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._h = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception as e:  # pragma: no cover - depends on the box
            self.error = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM))
                r = self._nvml.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "note": getattr(self, "error", "no samples")}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- distributed
RANKS = None  # hybrid_local_global_b200.dist.Ranks of this process


def dist_setup(n_gpus):
    global RANKS
    from hybrid_local_global_b200 import dist as hdist
    RANKS = hdist.setup("nccl")
    return RANKS.world, RANKS.rank, RANKS.local


def barrier(world):
    RANKS.barrier()


def max_over_ranks(x: float, world: int) -> float:
    return RANKS.max_over_ranks(x)


# --------------------------------------------------------------------------- prefill (ours)
def make_prefill(w, dev):
    from hybrid_local_global_b200.stack import AttentionStack
    st = AttentionStack(w, dev)
    g = synth.generator(w.seed, dev)
    layers = []
    for l in range(st.n_layers):
        t = st.layer_type(l)
        q = synth.randn_bf16((w.batch, w.seq, w.n_q_heads, t.head_dim), g, dev)
        k = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, dev, scale=w.k_scale)
        v = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, dev)
        out = torch.empty((w.batch, w.seq, w.n_q_heads, t.head_dim), dtype=torch.bfloat16, device=dev)
        if w.prior and not st.is_shared(l):
            synth.fill_randn_bf16_(st.k_cache[l][:, :, :w.prior], g)
            synth.fill_randn_bf16_(st.v_cache[l][:, :, :w.prior], g)
        layers.append((q, k, v, out))
    ws = torch.empty(st.prefill_workspace_bytes(), dtype=torch.uint8, device=dev)
    lens = torch.full((w.batch,), w.prior, dtype=torch.int32, device=dev) if w.prior else None
    return st, layers, ws, lens


def recorded_traffic(kernel, workload=None):
    """DRAM bytes per launch recorded by an ncu capture under profiles/
    (``traffic-record:`` lines), keyed by layer type; only records whose
    kernel-source digest matches the sources built now count."""
    from hybrid_local_global_b200.profiling import kernel_digest, traffic_records
    digest = kernel_digest(kernel)
    out = {}
    for r in traffic_records(os.path.join(ROOT, "profiles")):
        if r.get("kernel") != kernel or r.get("digest") != digest:
            continue
        if workload is not None and r.get("workload") != workload:
            continue
        out[r.get("layer", "")] = r
    return out


def kernel_totals(native):
    res = {}
    for k, name in native.KERNEL_NAMES.items():
        ms, n = native.gemma_attn_profile_read(k)
        if n:
            res[name] = {"ms": round(ms, 4), "launches": n}
    return res


def timed_passes(native, step, args, world, dev, before_step=None):
    """Two timed passes of args.steps steps each, bracketed by a barrier and a
    synchronize: the first, uninstrumented, gives the step time (`value`);
    the second records the library's CUDA events around each launch
    (gemma_attn_profile) for the per-kernel device times of the roofline.
    The events cost a few microseconds of serialisation per launch, so they
    stay out of the step time. -> (step ms summed over steps, max over ranks;
    wall seconds of the first pass; per-kernel totals; clock record)."""
    def run(evs):
        barrier(world)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for a, b in evs:
            if before_step is not None:
                before_step()
            a.record()
            step()
            b.record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        barrier(world)
        return wall

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    evs2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    with ClockSampler(dev.index or 0) as clk:
        wall = run(evs)
        native.gemma_attn_profile(True)
        run(evs2)
    rc = native.gemma_attn_sync_status()
    assert rc == 0, native.gemma_last_error()
    dev_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world)
    kern = kernel_totals(native)
    native.gemma_attn_profile(False)
    return dev_ms, wall, kern, clk


def bench_prefill(args, w, dev, world, peaks):
    from hybrid_local_global_b200 import native
    st, layers, ws, lens = make_prefill(w, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        for l, (q, k, v, out) in enumerate(layers):
            st.prefill_layer(l, q, k, v, out, workspace=ws, seq_lens_before=lens)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    dev_ms_max, wall, kern, clk = timed_passes(native, step, args, world, dev, before_step=flush.zero_)
    flops = prefill_flops(w, st.is_global)
    value = world * flops * args.steps / (dev_ms_max / 1e3) / 1e12
    attn = kern.get("prefill_attn", {"ms": float("nan"), "launches": 0})
    achieved = flops * args.steps / (attn["ms"] / 1e3) / 1e12
    peak = peaks[0]["bf16_tflops"]
    roof = {"bound": "tensor", "kernel": "prefill attention", "achieved": round(achieved, 2),
            "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "peak_source": "%s bf16 burst (MEASURED_PEAKS.json)" % peaks[1] if peaks[1] == "measured"
            else "fallback 1.59 PF/s", "traffic": None,
            "per_launch": "algorithmic FLOPs of all attention launches / their summed device time "
                          "(%d launches, %d per step; CUDA events around each launch, in a second timed "
                          "pass of the same steps)" % (attn["launches"], st.n_layers)}
    # the kernel that runs each layer type: CTA pairs on head_dim 512 (both
    # model shapes have an even number of q heads per KV head), one CTA per
    # query tile on head_dim 256
    rec = {}
    for kind, lt in (("local", w.local), ("global", w.global_)):
        r = recorded_traffic("k_prefill_pair" if lt.head_dim == 512 else "k_prefill_tc", w.name)
        if kind in r:
            rec[kind] = r[kind]
    kinds = ["global" if g else "local" for g in st.is_global]
    if all(k in rec for k in kinds):
        roof["traffic"] = round(sum(float(rec[k]["bytes"]) for k in kinds) / len(kinds))
        roof["traffic_note"] = ("DRAM read+write bytes per attention launch, mean over the step's layers, "
                                "from ncu captures in %s" % ", ".join(sorted({rec[k]["file"] for k in kinds})))
    else:
        roof["traffic_note"] = "no ncu capture of the current kernel sources for this workload"
    launches = sum(v["launches"] for v in kern.values())
    res = dict(value=value, ms_per_step=dev_ms_max / args.steps, roofline=roof, kernels=kern,
               gpu_launches=launches, clocks=clk.summary(), wall_s=wall, flops_per_step=flops)
    if not args.no_e2e:
        res["e2e"] = e2e_prefill(args, st, layers, ws, lens, flops, world)
    return res, st, layers


def e2e_prefill(args, st, layers, ws, lens, flops, world):
    """Same step through the public API with host-resident inputs:
    AttentionStack.prefill_from_host copies every layer's q/k/v from pinned
    host memory and every output back inside the timed region, overlapping
    the two copy directions with the attention on separate streams."""
    host_in = [tuple(x.cpu().pin_memory() for x in (q, k, v)) for (q, k, v, _) in layers]
    host_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for (_, _, _, out) in layers]
    h2d = sum(x.numel() * x.element_size() for t in host_in for x in t)
    d2h = sum(x.numel() * x.element_size() for x in host_out)

    def step():
        st.prefill_from_host(host_in, host_out, layers, workspace=ws, seq_lens_before=lens)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world)
    for a, b in evs:
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world)
    return {"value": round(world * flops * args.steps / (ms / 1e3) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / args.steps, 4)}


# --------------------------------------------------------------------------- decode (ours)
def decode_bytes(w, st, lens_cpu):
    """Algorithmic bytes of one decode step: visible K and V rows read once per
    KV head (every layer, shared ones included: they attend over their
    source's cache; K only on a K = V layer), plus q, the new k/v and the
    output."""
    total = 0
    for l in range(st.n_layers):
        t = st.layer_type(l)
        kv = 1 if st.keqv(l) else 2
        total += visible_kv_bytes(st, l, lens_cpu)
        total += w.batch * w.n_q_heads * t.head_dim * 2 * 2
        if not st.is_shared(l):
            total += w.batch * t.n_kv_heads * t.head_dim * 2 * kv
    return total


def visible_kv_bytes(st, l, lens_cpu, bf16_equivalent=False):
    """Cached K (and V unless K = V) bytes layer l's decode reads: head_dim
    bf16 per key, or on int8 caches head_dim codes plus an 8-byte (min,
    step) pair (bf16_equivalent: the bf16 bytes of the same keys)."""
    t = st.layer_type(l)
    L = lens_cpu.to(torch.int64)
    vis = torch.clamp(L, max=t.window) if t.window else L
    row = t.head_dim + 8 if (st.w.kv_int8 and not bf16_equivalent) else t.head_dim * 2
    return int(vis.sum()) * t.n_kv_heads * row * (1 if st.keqv(l) else 2)


def bench_decode(args, w, dev, world, peaks):
    from hybrid_local_global_b200 import native
    from hybrid_local_global_b200.stack import AttentionStack
    st = AttentionStack(w, dev)
    if w.len_lo == w.len_hi:
        lens_cpu = torch.full((w.batch,), w.len_hi, dtype=torch.int32)
    else:
        lens_cpu = synth.decode_lengths(w.batch, w.len_lo, w.len_hi, seed=w.seed)
    lens = lens_cpu.to(dev)
    max_len = int(lens_cpu.max())
    g = synth.generator(w.seed, dev)
    seen = set()
    for l in range(st.n_layers):
        kc = st.k_cache[l]
        if kc.data_ptr() in seen:
            continue
        seen.add(kc.data_ptr())
        synth.fill_cache_(kc, g)
        if st.v_cache[l] is not kc:
            synth.fill_cache_(st.v_cache[l], g)
    layers = []
    for l in range(st.n_layers):
        t = st.layer_type(l)
        q = synth.randn_bf16((w.batch, w.n_q_heads, t.head_dim), g, dev)
        k = synth.randn_bf16((w.batch, t.n_kv_heads, t.head_dim), g, dev)
        v = synth.randn_bf16((w.batch, t.n_kv_heads, t.head_dim), g, dev)
        out = torch.empty_like(q)
        layers.append((q, k, v, out))
    ws = torch.empty(st.decode_workspace_bytes(max_len), dtype=torch.uint8, device=dev)

    def step():
        for l, (q, k, v, out) in enumerate(layers):
            st.decode_layer(l, q, k, v, out, seq_lens=lens, max_seq_len=max_len, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    dev_ms, _, kern, clk = timed_passes(native, step, args, world, dev)
    nbytes = decode_bytes(w, st, lens_cpu)
    kv_bytes = sum(visible_kv_bytes(st, l, lens_cpu) for l in range(st.n_layers))
    value = world * nbytes * args.steps / (dev_ms / 1e3) / 1e9
    sp = kern.get("decode_split", {"ms": float("nan"), "launches": 0})
    achieved = kv_bytes * args.steps / (sp["ms"] / 1e3) / 1e9
    peak = peaks[0]["hbm_gbs"]
    roof = {"bound": "hbm", "kernel": "split-K decode attention", "achieved": round(achieved, 1),
            "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
            "peak_source": "%s HBM copy (MEASURED_PEAKS.json)" % peaks[1], "traffic": None,
            "per_launch": "visible K (and V unless K = V) bytes of all split launches / their summed device time "
                          "(%d launches, %d per step; CUDA events around each launch, in a second timed pass "
                          "of the same steps)" % (sp["launches"], st.n_layers)}
    rec = recorded_traffic("k_decode_split_q8" if w.kv_int8 else "k_decode_split")
    if rec:
        # each layer takes the traffic/algorithmic ratio captured for its layer
        # type (or the other type's, when only one was captured)
        ratio = {k: float(r["bytes"]) / float(r["units"]) for k, r in rec.items()}
        any_ratio = next(iter(ratio.values()))
        per_layer = [ratio.get("global" if st.layer_type(l).window == 0 else "local", any_ratio)
                     * visible_kv_bytes(st, l, lens_cpu) for l in range(st.n_layers)]
        roof["traffic"] = round(sum(per_layer) / st.n_layers)
        roof["traffic_note"] = ("DRAM bytes per split launch: each layer's visible K+V bytes x the "
                                "traffic/algorithmic ratio of the ncu capture for its layer type (%s), mean "
                                "over the block's launches; this block is too large to capture"
                                % ", ".join("%s %.4f: %s in %s" % (k, ratio[k], rec[k]["workload"], rec[k]["file"])
                                            for k in sorted(rec)))
    else:
        roof["traffic_note"] = "no ncu capture of the current kernel sources"
    res = {"metric": "decode KV GB/s", "value": round(value, 1), "unit": "GB/s",
            "workload": w.name, "description": w.description, "ms_per_step": round(dev_ms / args.steps, 4),
            "bytes_per_step": nbytes, "kv_bytes_per_step": kv_bytes,
            "kv_lengths": {"min": int(lens_cpu.min()), "max": max_len, "sum": int(lens_cpu.sum())},
            "shared_layers": [l for l in range(st.n_layers) if st.is_shared(l)],
            "cache_bytes_owned": st.owned_cache_bytes(),
            "roofline": roof, "kernels": kern, "clocks": clk.summary(),
            "gpu_launches": sum(v["launches"] for v in kern.values())}
    if w.kv_int8:
        eq = sum(visible_kv_bytes(st, l, lens_cpu, bf16_equivalent=True) for l in range(st.n_layers))
        res["bf16_equivalent_gbs"] = round(world * eq * args.steps / (dev_ms / 1e3) / 1e9, 1)
        res["bf16_equivalent_note"] = ("bf16 bytes of the same visible keys per second of the whole step: "
                                       "the bandwidth a bf16 cache would need to match this step time")
    return res


# --------------------------------------------------------------------------- oracle (CPU)
def oracle_sample_rows(w, is_global, rows_per_layer, seed):
    """A bounded, seeded sample of attention rows for each layer."""
    rng = np.random.default_rng(seed)
    sample = []
    for l, g in enumerate(is_global):
        n = rows_per_layer[1] if g else rows_per_layer[0]
        r = np.stack([rng.integers(0, w.batch, n), rng.integers(0, w.n_q_heads, n),
                      rng.integers(0, w.seq, n)], axis=1).astype(np.int32)
        sample.append(r)
    return sample


def time_oracle(w, layers_bits, is_global, sample):
    """Runs the oracle on the sampled rows; returns (seconds, algorithmic FLOPs)."""
    import oracle
    secs, flops = 0.0, 0
    for l, g in enumerate(is_global):
        t = w.global_ if g else w.local
        q, k, v = layers_bits[l]
        rows = sample[l]
        t0 = time.perf_counter()
        oracle.attention(q, k, v, q_pos0=w.prior, n_keys=w.prior + w.seq, rot_from=w.prior,
                         window=t.window, rope_frac=t.rope_frac, theta=t.rope_theta, scale=t.scale,
                         rows=rows)
        secs += time.perf_counter() - t0
        pos = w.prior + rows[:, 2].astype(np.int64)
        vis = np.minimum(pos + 1, t.window) if t.window else pos + 1
        flops += int(4 * t.head_dim * vis.sum())
    return secs, flops


def host_layers_bits(w, layers):
    return [(synth.bits(q), synth.bits(k), synth.bits(v)) for (q, k, v, _) in layers]


def cpu_layers_bits(w, is_global):
    """Workload inputs drawn on the CPU (for the reference arm, no GPU needed)."""
    g = synth.generator(w.seed)
    out = []
    for gl in is_global:
        t = w.global_ if gl else w.local
        q = synth.randn_bf16((w.batch, w.seq, w.n_q_heads, t.head_dim), g)
        k = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, scale=w.k_scale)
        v = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g)
        out.append((synth.bits(q), synth.bits(k), synth.bits(v)))
    return out


def schedule_of(w):
    if w.fixed_kinds:
        return [k == "global" for k in w.fixed_kinds]
    from hybrid_local_global_b200 import native
    return native.gemma_layer_schedule(w.n_layers, w.ratio, w.n_shared)[0]


def run_reference(args, world, rank):
    import oracle
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    if w.kind != "prefill" or w.prior:
        print(json.dumps({"impl": "reference", "unavailable": "reference arm implemented for "
                          "prefill workloads without a cached prefix"}))
        return
    is_global = schedule_of(w)
    layers = cpu_layers_bits(w, is_global)
    cores = oracle.default_threads()
    per = (args.ref_rows_local, args.ref_rows_global)
    for i in range(args.warmup):
        time_oracle(w, layers, is_global, oracle_sample_rows(w, is_global, per, seed=i))
    secs, flops = 0.0, 0
    for i in range(args.steps):
        s, f = time_oracle(w, layers, is_global, oracle_sample_rows(w, is_global, per, seed=1000 + i))
        secs += s
        flops += f
    value = flops / secs / 1e12
    sample = "%d rows per local layer + %d rows of the global layer per step, seeded uniform over (b, h, i)" % per
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: bf16 ~N(0,1), seeded",
            "config": {"workload": w.name, "description": w.description, "batch": w.batch, "seq_len": w.seq,
                       "n_layers": len(is_global), "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="e2b_block_s8192", choices=sorted(WORKLOADS))
    ap.add_argument("--decode-workload", default="31b_decode_b64")
    ap.add_argument("--decode-int8-workload", default="31b_decode_b64_int8")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-rows-local", type=int, default=256)
    ap.add_argument("--ref-rows-global", type=int, default=256)
    ap.add_argument("--cpu-rows-local", type=int, default=16384)
    ap.add_argument("--cpu-rows-global", type=int, default=49152)
    args = ap.parse_args()

    if args.impl == "reference":
        # the oracle on the host cores: rank 0 alone runs it, no process group
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args.gpus)

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    w = WORKLOADS[args.workload]
    pre, st, layers = bench_prefill(args, w, dev, world, peaks)
    line = {"metric": METRIC, "value": round(pre["value"], 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(pre["ms_per_step"], 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: bf16 ~N(0,1) Q/K/V, seeded per workload (no dataset)",
            "config": {"workload": w.name, "description": w.description, "batch": w.batch,
                       "seq_len": w.seq, "n_q_heads": w.n_q_heads,
                       "layers": ["global" if g else "local" for g in st.is_global],
                       "parallelism": "independent replica per GPU (dp%d)" % world,
                       "l2": "flushed between timed steps (256 MiB write, outside the step events)"},
            "roofline": pre["roofline"], "gpu_launches": pre["gpu_launches"], "clocks": pre["clocks"],
            "kernels": pre["kernels"], "flops_per_step": pre["flops_per_step"]}
    if "e2e" in pre:
        line["e2e"] = pre["e2e"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        is_global = st.is_global
        bits_layers = host_layers_bits(w, layers)
        sample = oracle_sample_rows(w, is_global, (args.cpu_rows_local, args.cpu_rows_global), seed=77)
        secs, flops = time_oracle(w, bits_layers, is_global, sample)
        line["cpu_baseline"] = {
            "value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.default_threads(),
            "kind": "oracle", "seconds": round(secs, 2),
            "sample": "%d seeded random rows per local layer and %d of the global layer of the same "
                      "workload (rows are independent, so the rate is the workload's)" % (
                          args.cpu_rows_local, args.cpu_rows_global)}
        del bits_layers
    del layers, st
    torch.cuda.empty_cache()
    if args.decode_workload != "none":
        dw = WORKLOADS[args.decode_workload]
        line["decode"] = bench_decode(args, dw, dev, world, peaks)
        line["gpu_launches"] += line["decode"]["gpu_launches"]
    if args.decode_int8_workload != "none":
        dw = WORKLOADS[args.decode_int8_workload]
        line["decode_int8"] = bench_decode(args, dw, dev, world, peaks)
        line["gpu_launches"] += line["decode_int8"]["gpu_launches"]
    if rank == 0:
        print(json.dumps(line))
    RANKS.close()


if __name__ == "__main__":
    main()
