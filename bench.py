#!/usr/bin/env python
"""Benchmark of the interleaved local/global attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--extra-prefill A,B|none]
                    [--decode-workload NAME|none] [--decode-int8-workload NAME|none]
                    [--extra-decode A,B|none]

One JSON line on rank 0. A step is one pass of the prefill block named by
--workload (default: the 31B-shaped 6-layer block, B2 S32768, 5 local + 1
global: layer schedule, RoPE + cache write, attention for every layer) over
resident synthetic inputs; `value` is its algorithmic TFLOP/s (4*B*Hq*D per
visible query-key pair, masked pairs not counted) over all ranks.

Every other workload shape gets an object of its own, with its step time,
roofline and oracle baseline:
  configs.<name>  the prefill workloads of --extra-prefill (default: the
                  single local layer B1 S1024, the E2B-shaped block B1 S8192,
                  the 4096-query chunk against a 256K global cache) and the
                  decode workloads of --extra-decode (default: single-token
                  decode at 256K), in TFLOP/s or KV GB/s;
  decode          the 31B-shaped batched decode block (B64, KV lengths
                  U[4096,131072], 6 layers, last two shared) in KV GB/s;
  decode_int8     the same block on int8 KV caches (GB/s of the int8 rows
                  read, and `bf16_equivalent_gbs`).

Each part runs two timed passes of the same steps, both bracketed by a
barrier and a synchronize and timed with CUDA events on the stream: the step
time comes from an uninstrumented pass; the per-kernel device times of the
roofline (`kernels`, `roofline.achieved`) come from the second pass, where
the library records events around every launch.

`cpu_baseline` objects time the fp64 CPU oracle on the host cores over a
bounded, seeded sample of rows (prefill) or sequences (decode) of the same
workload and inputs, and report in `parity` how far the GPU's outputs of the
last timed step sit from the oracle's on that sample. --impl reference times the oracle alone, on the
headline workload, each step a bounded sample of its rows.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
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
from hybrid_local_global_b200.workloads import (WORKLOADS, layer_shape_tag, prefill_attn_bytes,  # noqa: E402
                                                prefill_flops, visible_pairs_prefill)

METRIC = "attention prefill TFLOP/s and decode KV GB/s on 1 B200, as % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HEADLINE = "31b_block_s32768"
EXTRA_PREFILL = "local_s1024,e2b_block_s8192,global_chunk_256k"
EXTRA_DECODE = "global_decode_256k"
# nominal per-GPU figures, for the second fraction each roofline object reports
NOMINAL_BF16_TFLOPS = 2250.0   # dense bf16 (the 2:4-sparse figure halved)
NOMINAL_HBM_GBS = 7700.0       # HBM3e, HGX B200


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# A timed pass this long runs the tensor cores under the 1 kW power cap, as
# the sustained GEMM loop of the measured peaks did; shorter passes compare
# with the burst figure.
SUSTAINED_AFTER_S = 1.0


def tensor_peak(peaks, timed_s):
    d, src = peaks
    if timed_s >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in d:
        return d["bf16_tflops_sustained"], "%s bf16 sustained (MEASURED_PEAKS.json; timed pass %.1f s)" % (src, timed_s)
    return d["bf16_tflops"], "%s bf16 burst (MEASURED_PEAKS.json; timed pass %.2f s)" % (src, timed_s)


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
            out = {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                   "note": getattr(self, "error", "no samples")}
        else:
            out = {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                   "reasons": sorted(self.reasons), "samples": len(self.samples)}
        if getattr(self, "rejected_first", None) is not None:
            out["rejected_first_attempt"] = self.rejected_first
        return out


SLOWDOWNS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def clock_rejected(summary) -> bool:
    """A timed region whose clock record disqualifies it: a hardware or
    thermal slowdown was active, or the median SM clock sat well below its
    maximum (under 80 %) with no reason reported (a clock left locked).
    sw_power_cap alone is kept: a dense kernel on a 1 kW part runs under it."""
    reasons = set(summary.get("reasons") or [])
    if reasons & SLOWDOWNS:
        return True
    mhz, top = summary.get("sm_mhz"), summary.get("sm_max_mhz")
    return bool(mhz and top and mhz < 0.8 * top and not (reasons - {"applications_clocks"}))


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


# --------------------------------------------------------------------------- inputs
def draw_prefill_layer(w, t, g, dev):
    """One layer's q, k, v (k scaled by the workload's k_scale), drawn in the
    workload's order: q, then k, then v."""
    q = synth.randn_bf16((w.batch, w.seq, w.n_q_heads, t.head_dim), g, dev)
    k = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, dev, scale=w.k_scale)
    v = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, dev)
    return q, k, v


def make_prefill(w, dev):
    from hybrid_local_global_b200.stack import AttentionStack
    st = AttentionStack(w, dev)
    g = synth.generator(w.seed, dev)
    layers = []
    for l in range(st.n_layers):
        q, k, v = draw_prefill_layer(w, st.layer_type(l), g, dev)
        out = torch.empty_like(q)
        if w.prior and not st.is_shared(l):
            synth.fill_randn_bf16_(st.k_cache[l][:, :, :w.prior], g)
            synth.fill_randn_bf16_(st.v_cache[l][:, :, :w.prior], g)
        layers.append((q, k, v, out))
    ws = torch.empty(st.prefill_workspace_bytes(), dtype=torch.uint8, device=dev)
    lens = torch.full((w.batch,), w.prior, dtype=torch.int32, device=dev) if w.prior else None
    return st, layers, ws, lens


def current_records(kernel):
    """DRAM bytes per launch recorded by ncu captures under profiles/
    (``traffic-record:`` lines) for a kernel whose sources still have the
    digest recorded with them."""
    from hybrid_local_global_b200.profiling import kernel_digest, traffic_records
    digest = kernel_digest(kernel)
    return [r for r in traffic_records(os.path.join(ROOT, "profiles"))
            if r.get("kernel") == kernel and r.get("digest") == digest]


def no_traffic_note(kernel, what="no ncu capture of the current kernel sources"):
    """Why traffic is null: no capture at all, or captures of an earlier
    version of the kernel (their digest differs from the built sources')."""
    from hybrid_local_global_b200.profiling import kernel_digest, traffic_records
    digest = kernel_digest(kernel)
    old = sorted({r.get("file", "?") for r in traffic_records(os.path.join(ROOT, "profiles"))
                  if r.get("kernel") == kernel and r.get("digest") != digest})
    if not old:
        return what
    return "%s: %s holds a capture of an earlier version of %s (the sources have changed since), " \
           "so its DRAM bytes are not reported for this one" % (what, ", ".join(old), kernel)


def recorded_traffic(kernel, workload=None):
    """current_records of one workload (or of any, the last per layer type),
    keyed by layer type."""
    out = {}
    for r in current_records(kernel):
        if workload is None or r.get("workload") == workload:
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
    """timed_passes_once, taken again once when its clock record disqualifies
    it on any rank (clock_rejected); the decision is reduced over the ranks,
    so all of them take the same collective steps. The clock record of a
    repeated measurement carries the rejected one's summary."""
    res = timed_passes_once(native, step, args, world, dev, before_step)
    first = res[3].summary()
    if max_over_ranks(1.0 if clock_rejected(first) else 0.0, world) > 0:
        res = timed_passes_once(native, step, args, world, dev, before_step)
        res[3].rejected_first = first
    return res


def timed_passes_once(native, step, args, world, dev, before_step=None):
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


# --------------------------------------------------------------------------- prefill (ours)
def bench_prefill(args, w, dev, world, peaks, e2e=False, cpu=False):
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
    peak, peak_source = tensor_peak(peaks, dev_ms_max / 1e3)
    burst = peaks[0]["bf16_tflops"]
    roof = {"bound": "tensor", "kernel": "prefill attention", "achieved": round(achieved, 2),
            "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "peak_source": peak_source,
            "frac_of_nominal": round(achieved / NOMINAL_BF16_TFLOPS, 4),
            "frac_of_burst": round(achieved / burst, 4), "traffic": None,
            "per_launch": "algorithmic FLOPs of all attention launches / their summed device time "
                          "(%d launches, %d per step; CUDA events around each launch, in a second timed "
                          "pass of the same steps)" % (attn["launches"], st.n_layers)}
    # DRAM traffic of each layer type's launch: a capture of this workload, or
    # of a smaller one of the same per-head shape scaled by the bytes moved
    # (traffic / algorithmic bytes of the captured launch x this launch's)
    per_kind, files = {}, set()
    for kind, lt in (("local", w.local), ("global", w.global_)):
        kname = "k_prefill_pair" if lt.head_dim == 512 else "k_prefill_tc"
        exact = recorded_traffic(kname, w.name)
        if kind in exact:
            per_kind[kind] = (float(exact[kind]["bytes"]), "%s (this workload)" % exact[kind]["file"])
            continue
        for r in current_records(kname):
            if r.get("shape") == layer_shape_tag(w, lt) and "units" in r and r.get("layer") == kind:
                ratio = float(r["bytes"]) / float(r["units"])
                per_kind[kind] = (ratio * prefill_attn_bytes(w, lt),
                                  "%s (%s, %.3f x the algorithmic bytes)" % (r["file"], r["workload"], ratio))
                break
    kinds = ["global" if g else "local" for g in st.is_global]
    if all(k in per_kind for k in kinds):
        roof["traffic"] = round(sum(per_kind[k][0] for k in kinds) / len(kinds))
        roof["traffic_note"] = ("DRAM read+write bytes per attention launch, mean over the step's layers, from "
                                "ncu captures: %s" % "; ".join(sorted({per_kind[k][1] for k in kinds})))
    else:
        roof["traffic_note"] = "; ".join(sorted({no_traffic_note(
            "k_prefill_pair" if (w.global_ if g else w.local).head_dim == 512 else "k_prefill_tc",
            "no ncu capture of the current kernel sources for this layer shape") for g in st.is_global}))
    launches = sum(v["launches"] for v in kern.values())
    res = {"metric": "prefill attention TFLOP/s", "value": round(value, 3), "unit": "TFLOP/s",
           "workload": w.name, "description": w.description,
           "ms_per_step": round(dev_ms_max / args.steps, 4), "flops_per_step": flops,
           "layers": ["global" if g else "local" for g in st.is_global],
           "roofline": roof, "kernels": kern, "gpu_launches": launches, "clocks": clk.summary(),
           "wall_s": round(wall, 3)}
    if e2e:
        res["e2e"] = e2e_prefill(args, st, layers, ws, lens, flops, world)
    if cpu:
        res["cpu_baseline"] = prefill_cpu_baseline(w, st.is_global, layers, st, args.cpu_flops)
    del layers, st, ws, flush
    torch.cuda.empty_cache()
    return res


def e2e_prefill(args, st, layers, ws, lens, flops, world):
    """Same step through the public API with host-resident inputs:
    AttentionStack.prefill_from_host copies every layer's q/k/v from pinned
    host memory and every output back inside the timed region, overlapping
    the two copy directions with the attention on separate streams."""
    host_in, host_out = [], []
    for (q, k, v, out) in layers:
        hs = []
        for x in (q, k, v):
            h = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
            h.copy_(x)
            hs.append(h)
        host_in.append(tuple(hs))
        host_out.append(torch.empty(out.shape, dtype=out.dtype, pin_memory=True))
    h2d = sum(x.numel() * x.element_size() for t in host_in for x in t)
    d2h = sum(x.numel() * x.element_size() for x in host_out)

    def step():
        st.prefill_from_host(host_in, host_out, layers, workspace=ws, seq_lens_before=lens)

    for _ in range(max(1, min(args.warmup, 2))):
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
    del host_in, host_out
    return {"value": round(world * flops * args.steps / (ms / 1e3) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / args.steps, 4)}


# --------------------------------------------------------------------------- oracle on prefill rows
def rows_for_budget(w, is_global, flops_budget):
    """Sampled rows per layer so that the oracle's work is about flops_budget
    (split evenly over the layers), capped at every row of the layer."""
    per_layer = flops_budget / max(1, len(is_global))
    total_rows = w.batch * w.n_q_heads * w.seq
    out = []
    for g in is_global:
        t = w.global_ if g else w.local
        per_row = 4 * t.head_dim * visible_pairs_prefill(w.seq, w.prior, t.window) / w.seq
        out.append(int(min(total_rows, max(64, per_layer // per_row))))
    return out


def sample_rows(w, n, seed):
    """n seeded rows (b, h, i), uniform over the layer's rows; every row when
    n covers them all."""
    total = w.batch * w.n_q_heads * w.seq
    if n >= total:
        bb, hh, ii = np.meshgrid(np.arange(w.batch), np.arange(w.n_q_heads), np.arange(w.seq), indexing="ij")
        return np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1).astype(np.int32)
    rng = np.random.default_rng(seed)
    return np.stack([rng.integers(0, w.batch, n), rng.integers(0, w.n_q_heads, n),
                     rng.integers(0, w.seq, n)], axis=1).astype(np.int32)


class Parity:
    """Largest and mean |GPU - oracle| over the outputs a CPU baseline
    computed anyway, against the parity tolerance of the tests (max 2e-2,
    mean 2e-3 for bf16 outputs)."""

    def __init__(self):
        self.mx, self.sum, self.n, self.rows = 0.0, 0.0, 0, 0

    def add(self, gpu, ref):
        gpu, ref = np.asarray(gpu, dtype=np.float64), np.asarray(ref, dtype=np.float64)
        err = np.abs(gpu - ref)
        if not np.isfinite(gpu).all():
            err = np.full_like(err, np.inf)
        self.mx = max(self.mx, float(err.max()) if err.size else 0.0)
        self.sum += float(err.sum())
        self.n += err.size
        self.rows += err.size // ref.shape[-1] if err.size else 0

    def summary(self, what):
        mean = self.sum / max(self.n, 1)
        return {"max_abs": float("%.4g" % self.mx), "mean_abs": float("%.4g" % mean), "rows": self.rows,
                "within_tolerance": bool(self.mx <= 2e-2 and mean <= 2e-3), "compared": what}


def oracle_prefill_rows(w, t, q, k, v, rows):
    """Times the oracle on `rows` of one layer (q [B,S,Hq,D], k/v [B,T,Hkv,D]
    bf16 bits in position order, the first w.prior keys already rotated);
    returns (seconds, algorithmic FLOPs of those rows, the rows' outputs
    [n, D])."""
    import oracle
    t0 = time.perf_counter()
    out, _ = oracle.attention(q, k, v, q_pos0=w.prior, n_keys=w.prior + w.seq, rot_from=w.prior,
                              window=t.window, rope_frac=t.rope_frac, theta=t.rope_theta, scale=t.scale,
                              rows=rows)
    secs = time.perf_counter() - t0
    pos = w.prior + rows[:, 2].astype(np.int64)
    vis = np.minimum(pos + 1, t.window) if t.window else pos + 1
    return secs, int(4 * t.head_dim * vis.sum()), out


def layer_bits_for_oracle(w, st, l, q, k, v):
    """Host bf16 bits of one layer's inputs as the oracle takes them: keys and
    values in position order, a cached prefix (already rotated) first."""
    if w.prior:
        kc, vc = st.k_cache[l], st.v_cache[l]
        k = torch.cat([kc[:, :, :w.prior].transpose(1, 2), k], dim=1)
        v = torch.cat([vc[:, :, :w.prior].transpose(1, 2), v], dim=1)
    return synth.bits(q), synth.bits(k), synth.bits(v)


def prefill_cpu_baseline(w, is_global, layers, st, flops_budget):
    """The oracle on a bounded, seeded sample of each layer's rows, on the
    inputs the GPU steps used (rows are independent, so the sample's rate is
    the workload's)."""
    import oracle
    n_rows = rows_for_budget(w, is_global, flops_budget)
    secs, flops = 0.0, 0
    par = Parity()
    for l, g in enumerate(is_global):
        t = w.global_ if g else w.local
        q, k, v, out = layers[l]
        qb, kb, vb = layer_bits_for_oracle(w, st, l, q, k, v)
        rows = sample_rows(w, n_rows[l], seed=77 + l)
        s, f, ref = oracle_prefill_rows(w, t, qb, kb, vb, rows)
        secs += s
        flops += f
        idx = torch.as_tensor(rows.astype(np.int64), device=out.device)
        par.add(out[idx[:, 0], idx[:, 2], idx[:, 1]].double().cpu().numpy(), ref)
    n_all = w.batch * w.n_q_heads * w.seq
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.default_threads(),
            "kind": "oracle", "seconds": round(secs, 2),
            "parity": par.summary("the sampled rows, against the GPU output of the last timed step"),
            "sample": ("every row of every layer" if all(n >= n_all for n in n_rows) else
                       "%s seeded random rows (b, h, i) of the layers [%s] of the same workload and inputs "
                       "(rows are independent, so the rate is the workload's)"
                       % ("/".join(str(n) for n in n_rows), ",".join("G" if g else "L" for g in is_global)))}


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


def visible_kv_bytes(st, l, lens_cpu, bf16_equivalent=False, seqs=None):
    """Cached K (and V unless K = V) bytes layer l's decode reads: head_dim
    bf16 per key, or on int8 caches head_dim codes plus an 8-byte (min,
    step) pair (bf16_equivalent: the bf16 bytes of the same keys); `seqs`
    restricts the count to those sequences."""
    t = st.layer_type(l)
    L = lens_cpu.to(torch.int64)
    if seqs is not None:
        L = L[list(seqs)]
    vis = torch.clamp(L, max=t.window) if t.window else L
    row = t.head_dim + 8 if (st.w.kv_int8 and not bf16_equivalent) else t.head_dim * 2
    return int(vis.sum()) * t.n_kv_heads * row * (1 if st.keqv(l) else 2)


def decode_cpu_baseline(w, st, layers, lens_cpu, n_random=2):
    """The oracle on a seeded sample of sequences (the shortest, the longest
    and n_random others) of every layer, after the GPU steps: each sampled
    sequence's q rotated by the oracle at its position, attending over the
    sequence's visible cached rows (the new token included), dequantized by
    the oracle on int8 caches. Rate = the sample's visible K+V bytes per
    second of oracle time."""
    import oracle
    from hybrid_local_global_b200 import native
    lens = [int(x) for x in lens_cpu]
    rng = np.random.default_rng(99)
    pick = {int(np.argmin(lens)), int(np.argmax(lens))}
    others = [b for b in range(len(lens)) if b not in pick]
    pick |= set(int(x) for x in rng.choice(others, size=min(n_random, len(others)), replace=False)) if others else set()
    seqs = sorted(pick)
    threads = oracle.default_threads()
    secs, nbytes = 0.0, 0
    par = Parity()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        for l in range(st.n_layers):
            t = st.layer_type(l)
            q, out = layers[l][0], layers[l][3]
            kc, vc = st.k_cache[l], st.v_cache[l]
            keqv = st.keqv(l)
            G = w.n_q_heads // t.n_kv_heads
            for b in seqs:
                L = lens[b]
                first = max(0, L - t.window) if t.window else 0
                slots = [(p % t.window) if t.window else p for p in range(first, L)]
                qbits = synth.bits(q[b])
                qrot = np.stack([oracle.rope_bf16(qbits[h], L - 1, t.rope_frac, t.rope_theta)
                                 for h in range(w.n_q_heads)])
                idx = torch.as_tensor(slots, dtype=torch.long, device=q.device)
                t0 = time.perf_counter()
                if isinstance(kc, native.Int8KVCache):
                    def rows_of(c):
                        codes = c.codes[b].index_select(1, idx).cpu().numpy()
                        prm = c.params[b].index_select(1, idx).cpu().numpy()
                        return codes, prm
                    kcod, kprm = rows_of(kc)
                    vcod, vprm = (kcod, kprm) if keqv else rows_of(vc)
                    t0 = time.perf_counter()
                    kf = oracle.dequantize_rows_u8(kcod, kprm[..., 0], kprm[..., 1])
                    vf = kf if keqv else oracle.dequantize_rows_u8(vcod, vprm[..., 0], vprm[..., 1])
                    deq = time.perf_counter() - t0
                else:
                    kf = kc[b].index_select(1, idx).double().cpu().numpy()
                    vf = kf if keqv else vc[b].index_select(1, idx).double().cpu().numpy()
                    deq = 0.0
                n = len(slots)
                t0 = time.perf_counter()
                futs = [ex.submit(oracle.attend_rows, qrot[h:h + 1], kf[h // G], vf[h // G], 0, n, t.scale)
                        for h in range(w.n_q_heads)]
                ref = np.concatenate([f.result()[0] for f in futs])
                secs += time.perf_counter() - t0 + deq
                par.add(out[b].double().cpu().numpy(), ref)
                del kf, vf
            nbytes += visible_kv_bytes(st, l, lens_cpu, seqs=seqs)
    return {"value": round(nbytes / secs / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "seconds": round(secs, 2),
            "parity": par.summary("every q head of the sampled sequences, against the GPU output of the last "
                                  "timed step"),
            "sample": "sequences %s (%s) of every layer, all q heads; bytes = their visible K+V cache bytes"
                      % (seqs, "the only one" if len(lens) == 1 else
                         "shortest, longest and %d seeded others" % (len(seqs) - 2))}


def make_decode_stack(w, dev):
    """A decode workload's stack with every owned cache filled from the
    workload's seed, and its per-sequence lengths (CPU and device)."""
    from hybrid_local_global_b200.stack import AttentionStack
    st = AttentionStack(w, dev)
    if w.len_lo == w.len_hi:
        lens_cpu = torch.full((w.batch,), w.len_hi, dtype=torch.int32)
    else:
        lens_cpu = synth.decode_lengths(w.batch, w.len_lo, w.len_hi, seed=w.seed)
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
    return st, lens_cpu, lens_cpu.to(dev), int(lens_cpu.max()), g


def bench_decode(args, w, dev, world, peaks, cpu=False):
    from hybrid_local_global_b200 import native
    st, lens_cpu, lens, max_len, g = make_decode_stack(w, dev)
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
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
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
                                "over the block's launches" % ", ".join(
                                    "%s %.4f: %s in %s" % (k, ratio[k], rec[k]["workload"], rec[k]["file"])
                                    for k in sorted(rec)))
    else:
        roof["traffic_note"] = no_traffic_note("k_decode_split_q8" if w.kv_int8 else "k_decode_split")
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
    if cpu:
        res["cpu_baseline"] = decode_cpu_baseline(w, st, layers, lens_cpu)
    del layers, st, ws
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- multi-token decode (ours)
def verify_kv_bytes(st, l, lens_cpu, T, seqs=None):
    """Algorithmic K (and V unless K = V) bytes of one multi-token decode of
    layer l: the keys at least one of the T new tokens sees, once per KV
    head. A global layer: every position of the sequence; a local layer:
    the last window + T - 1 positions (the oldest slot of a full ring is
    older than every new token's window)."""
    t = st.layer_type(l)
    L = lens_cpu.to(torch.int64)
    if seqs is not None:
        L = L[list(seqs)]
    keys = torch.clamp(L, max=t.window + T - 1) if t.window else L
    return int(keys.sum()) * t.n_kv_heads * t.head_dim * 2 * (1 if st.keqv(l) else 2)


def verify_cpu_baseline(w, st, layers, lens_cpu, n_random=1):
    """The oracle on a seeded sample of sequences (the shortest, the longest
    and n_random others) of every layer, after the GPU steps: each of the T
    new tokens' q rows rotated by the oracle at its position, attending over
    its visible positions among the rows cached after the step (on a local
    layer the ring then holds the last `window` positions, so an early token
    sees up to T - 1 fewer keys than on the GPU). Rate = the sample's K+V
    bytes as counted for the GPU per second of oracle time."""
    import oracle
    T = w.tokens
    lens = [int(x) for x in lens_cpu]
    rng = np.random.default_rng(99)
    pick = {int(np.argmin(lens)), int(np.argmax(lens))}
    others = [b for b in range(len(lens)) if b not in pick]
    pick |= set(int(x) for x in rng.choice(others, size=min(n_random, len(others)), replace=False)) if others else set()
    seqs = sorted(pick)
    threads = oracle.default_threads()
    secs, nbytes = 0.0, 0
    par = Parity()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        for l in range(st.n_layers):
            t = st.layer_type(l)
            q, out = layers[l][0], layers[l][3]
            kc, vc = st.k_cache[l], st.v_cache[l]
            keqv = st.keqv(l)
            G = w.n_q_heads // t.n_kv_heads
            for b in seqs:
                L = lens[b]
                first = max(0, L - t.window) if t.window else 0
                slots = [(p % t.window) if t.window else p for p in range(first, L)]
                idx = torch.as_tensor(slots, dtype=torch.long, device=q.device)
                kf = kc[b].index_select(1, idx).double().cpu().numpy()
                vf = kf if keqv else vc[b].index_select(1, idx).double().cpu().numpy()
                qbits = synth.bits(q[b])  # [T, Hq, D]
                t0 = time.perf_counter()
                qr = np.stack([np.stack([oracle.rope_bf16(qbits[tok, h], L - T + tok, t.rope_frac, t.rope_theta)
                                         for h in range(w.n_q_heads)]) for tok in range(T)])  # [T, Hq, D]
                lo = np.array([max(0, L - T + tok - t.window + 1 - first) if t.window else 0 for tok in range(T)])
                hi = np.array([L - T + tok + 1 - first for tok in range(T)])
                order = [(hk, tok) for hk in range(t.n_kv_heads) for tok in range(T)]
                futs = [ex.submit(oracle.attend_rows, qr[tok, hk * G:(hk + 1) * G], kf[hk], vf[hk], lo[tok],
                                  hi[tok] - lo[tok], t.scale)
                        for hk, tok in order]
                refs = [f.result()[0] for f in futs]
                secs += time.perf_counter() - t0
                gpu_b = out[b].double().cpu().numpy()  # [T, Hq, D]
                for (hk, tok), ref in zip(order, refs):
                    # on a local ring an earlier token's oldest keys are overwritten by the step's own tokens
                    if t.window == 0 or tok == T - 1:
                        par.add(gpu_b[tok, hk * G:(hk + 1) * G], ref)
                del kf, vf
            nbytes += verify_kv_bytes(st, l, lens_cpu, T, seqs=seqs)
    return {"value": round(nbytes / secs / 1e9, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "seconds": round(secs, 2),
            "parity": par.summary("the sampled sequences' outputs whose keys all stay cached after the step "
                                  "(every token on global layers, the last on local rings), against the GPU "
                                  "output of the last timed step"),
            "sample": "sequences %s (shortest, longest and %d seeded other) of every layer, all q heads and "
                      "all %d new tokens; bytes = their K+V bytes as counted for the GPU"
                      % (seqs, len(seqs) - 2, T)}


def bench_verify(args, w, dev, world, peaks, cpu=False):
    """Multi-token decode (w.tokens new tokens per sequence) through every
    layer of the stack, and a single-token decode step of the same stack
    for the ratio."""
    from hybrid_local_global_b200 import native
    st, lens_cpu, lens, max_len, g = make_decode_stack(w, dev)
    T = w.tokens
    layers, dlayers = [], []
    for l in range(st.n_layers):
        t = st.layer_type(l)
        q = synth.randn_bf16((w.batch, T, w.n_q_heads, t.head_dim), g, dev)
        k = synth.randn_bf16((w.batch, T, t.n_kv_heads, t.head_dim), g, dev)
        v = synth.randn_bf16((w.batch, T, t.n_kv_heads, t.head_dim), g, dev)
        layers.append((q, k, v, torch.empty_like(q)))
        dlayers.append(tuple(x[:, 0].contiguous() for x in (q, k, v)) + (torch.empty_like(q[:, 0]),))
    ws = torch.empty(max(st.decode_multi_workspace_bytes(T, max_len), st.decode_workspace_bytes(max_len)),
                     dtype=torch.uint8, device=dev)

    def step():
        for l, (q, k, v, out) in enumerate(layers):
            st.decode_multi_layer(l, q, k, v, out, seq_lens=lens, max_seq_len=max_len, workspace=ws)

    def dstep():
        for l, (q, k, v, out) in enumerate(dlayers):
            st.decode_layer(l, q, k, v, out, seq_lens=lens, max_seq_len=max_len, workspace=ws)

    for fn in (dstep, step):
        for _ in range(args.warmup):
            fn()
    torch.cuda.synchronize()
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    d_ms, _, dkern, _ = timed_passes(native, dstep, args, world, dev)
    dev_ms, _, kern, clk = timed_passes(native, step, args, world, dev)
    kv_bytes = sum(verify_kv_bytes(st, l, lens_cpu, T) for l in range(st.n_layers))
    io_bytes = sum(w.batch * T * (w.n_q_heads * st.layer_type(l).head_dim * 2 * 2 +
                                  st.layer_type(l).n_kv_heads * st.layer_type(l).head_dim * 2 * 2)
                   for l in range(st.n_layers))
    nbytes = kv_bytes + io_bytes
    value = world * nbytes * args.steps / (dev_ms / 1e3) / 1e9
    sp = kern.get("decode_split", {"ms": float("nan"), "launches": 0})
    achieved = kv_bytes * args.steps / (sp["ms"] / 1e3) / 1e9
    peak = peaks[0]["hbm_gbs"]
    roof = {"bound": "hbm", "kernel": "multi-token decode attention (transposed tensor-core kernel)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "peak_source": "%s HBM copy (MEASURED_PEAKS.json)" % peaks[1], "traffic": None,
            "per_launch": "K (and V unless K = V) bytes of all attention launches / their summed device time "
                          "(%d launches, %d per step; CUDA events around each launch, in a second timed pass "
                          "of the same steps)" % (sp["launches"], st.n_layers)}
    rec = recorded_traffic("k_verify_tc")
    if rec:
        ratio = {k: float(r["bytes"]) / float(r["units"]) for k, r in rec.items()}
        any_ratio = next(iter(ratio.values()))
        per_layer = [ratio.get("global" if st.layer_type(l).window == 0 else "local", any_ratio)
                     * verify_kv_bytes(st, l, lens_cpu, T) for l in range(st.n_layers)]
        roof["traffic"] = round(sum(per_layer) / st.n_layers)
        roof["traffic_note"] = ("DRAM bytes per attention launch: each layer's K+V bytes x the traffic/algorithmic "
                                "ratio of the ncu capture for its layer type (%s), mean over the block's launches"
                                % ", ".join("%s %.4f: %s in %s" % (k, ratio[k], rec[k]["workload"], rec[k]["file"])
                                            for k in sorted(rec)))
    else:
        roof["traffic_note"] = no_traffic_note("k_verify_tc")
    res = {"metric": "multi-token decode KV GB/s", "value": round(value, 1), "unit": "GB/s",
           "workload": w.name, "description": w.description, "tokens": T,
           "ms_per_step": round(dev_ms / args.steps, 4),
           "decode_ms_per_step": round(d_ms / args.steps, 4),
           "ratio_to_decode_step": round(dev_ms / d_ms, 4),
           "ratio_note": "one multi-token step (T tokens per sequence) / one single-token decode step of the "
                         "same stack, lengths and inputs (the first of the T tokens)",
           "bytes_per_step": nbytes, "kv_bytes_per_step": kv_bytes,
           "kv_lengths": {"min": int(lens_cpu.min()), "max": max_len, "sum": int(lens_cpu.sum())},
           "roofline": roof, "kernels": kern, "decode_kernels": dkern, "clocks": clk.summary(),
           "gpu_launches": sum(v["launches"] for v in kern.values()) +
                           sum(v["launches"] for v in dkern.values())}
    if cpu:
        res["cpu_baseline"] = verify_cpu_baseline(w, st, layers, lens_cpu)
    del layers, dlayers, st, ws
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- reference arm (the oracle)
def schedule_of(w):
    """The oracle's layer schedule (the reference arm takes nothing from the
    product library)."""
    if w.fixed_kinds:
        return [k == "global" for k in w.fixed_kinds]
    import oracle
    return oracle.layer_schedule(w.n_layers, w.ratio)


def run_reference(args, world, rank):
    """Times the oracle on the headline workload: every step a seeded sample
    of rows of every layer. The inputs are the workload's own (drawn on the
    GPU with the workload's seed when one is present, else on the CPU), copied
    to the host one layer at a time; only the oracle's time is counted."""
    import oracle
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    if w.kind != "prefill" or w.prior:
        print(json.dumps({"impl": "reference", "unavailable": "reference arm implemented for "
                          "prefill workloads without a cached prefix"}))
        return
    is_global = schedule_of(w)
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    g = synth.generator(w.seed, dev)
    cores = oracle.default_threads()
    per = (args.ref_rows_local, args.ref_rows_global)
    secs = [0.0] * args.steps
    flops = [0] * args.steps
    for l, gl in enumerate(is_global):
        t = w.global_ if gl else w.local
        q, k, v = draw_prefill_layer(w, t, g, dev)
        qb, kb, vb = synth.bits(q), synth.bits(k), synth.bits(v)
        del q, k, v
        n = per[1] if gl else per[0]
        for i in range(args.warmup):
            oracle_prefill_rows(w, t, qb, kb, vb, sample_rows(w, n, seed=100 * l + i))
        for i in range(args.steps):
            s, f, _ = oracle_prefill_rows(w, t, qb, kb, vb, sample_rows(w, n, seed=100000 + 100 * l + i))
            secs[i] += s
            flops[i] += f
        del qb, kb, vb
    value = sum(flops) / sum(secs) / 1e12
    sample = ("%d rows per local layer + %d rows of each global layer per step, seeded uniform over "
              "(b, h, i)" % per)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sum(secs) * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: bf16 ~N(0,1), seeded",
            "config": {"workload": w.name, "description": w.description, "batch": w.batch, "seq_len": w.seq,
                       "n_layers": len(is_global), "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# --------------------------------------------------------------------------- main
def names(arg):
    return [] if arg in ("", "none") else [x for x in arg.split(",") if x]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--extra-prefill", default=EXTRA_PREFILL)
    ap.add_argument("--decode-workload", default="31b_decode_b64")
    ap.add_argument("--decode-int8-workload", default="31b_decode_b64_int8")
    ap.add_argument("--extra-decode", default=EXTRA_DECODE)
    ap.add_argument("--verify-workload", default="31b_verify_b64_k4")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-flops", type=float, default=4e11,
                    help="oracle work per prefill cpu_baseline (FLOPs of the sampled rows)")
    ap.add_argument("--ref-rows-local", type=int, default=256)
    ap.add_argument("--ref-rows-global", type=int, default=256)
    args = ap.parse_args()

    if args.impl == "reference":
        # the oracle on the host cores: rank 0 alone runs it, no process group
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args.gpus)

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    w = WORKLOADS[args.workload]
    pre = bench_prefill(args, w, dev, world, peaks, e2e=not args.no_e2e, cpu=cpu)
    line = {"metric": METRIC, "value": pre["value"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": pre["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: bf16 ~N(0,1) Q/K/V, seeded per workload (no dataset)",
            "config": {"workload": w.name, "description": w.description, "batch": w.batch,
                       "seq_len": w.seq, "n_q_heads": w.n_q_heads, "layers": pre["layers"],
                       "parallelism": "independent replica per GPU (dp%d)" % world,
                       "l2": "flushed between timed steps (256 MiB write, outside the step events)"},
            "roofline": pre["roofline"], "gpu_launches": pre["gpu_launches"], "clocks": pre["clocks"],
            "kernels": pre["kernels"], "flops_per_step": pre["flops_per_step"]}
    for key in ("e2e", "cpu_baseline"):
        if key in pre:
            line[key] = pre[key]
    configs = {}
    for name in names(args.extra_prefill):
        if name == w.name:
            continue
        configs[name] = bench_prefill(args, WORKLOADS[name], dev, world, peaks, cpu=cpu)
    if args.decode_workload != "none":
        line["decode"] = bench_decode(args, WORKLOADS[args.decode_workload], dev, world, peaks, cpu=cpu)
    if args.decode_int8_workload != "none":
        line["decode_int8"] = bench_decode(args, WORKLOADS[args.decode_int8_workload], dev, world, peaks, cpu=cpu)
    for name in names(args.extra_decode):
        configs[name] = bench_decode(args, WORKLOADS[name], dev, world, peaks, cpu=cpu)
    if args.verify_workload != "none":
        vw = WORKLOADS[args.verify_workload]
        line["verify_k%d" % vw.tokens] = bench_verify(args, vw, dev, world, peaks, cpu=cpu)
    if configs:
        line["configs"] = configs
    for obj in list(configs.values()) + [line.get("decode"), line.get("decode_int8")] + \
            [v for k, v in line.items() if k.startswith("verify_k")]:
        if obj:
            line["gpu_launches"] += obj["gpu_launches"]
    if rank == 0:
        print(json.dumps(line))
    RANKS.close()


if __name__ == "__main__":
    main()
