"""Workload shapes of the interleaved local/global attention path.

Layer types follow "Gemma 4 Architecture Reference" ("Attention
Architecture": window 512 on the small models, 1024 on the large ones; GQA
2:1 local, 8:1 global with doubled key dimension; "Positional Encoding":
p-RoPE with p = 0.25, theta = 1e6 on global layers) and "Gemma 4: End-to-End
Architecture Walkthrough", 3a (4:1 / 5:1 interleave, last layer global).
Local layers use full RoPE with theta = 1e4 (the pages give no value). The
logit scale is 1/sqrt(head_dim) (the pages give none; no soft-capping).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field


@dataclass(frozen=True)
class LayerType:
    window: int          # 0 = global
    n_kv_heads: int
    head_dim: int
    rope_frac: float
    rope_theta: float

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" | "decode"
    batch: int
    n_q_heads: int
    n_layers: int
    ratio: int           # local layers per global layer
    local: LayerType
    global_: LayerType
    seq: int = 0                 # prefill: new tokens per sequence
    prior: int = 0               # prefill: tokens already cached (chunked prefill)
    len_lo: int = 0              # decode: KV length range (incl. the new token)
    len_hi: int = 0
    n_shared: int = 0            # last-N-layer KV sharing
    k_scale: float = 1.0         # K drawn as N(0, k_scale^2)
    seed: int = 0
    fixed_kinds: tuple = ()      # overrides the schedule: e.g. ("local",) for one local layer
    k_eq_v: bool = False         # global layers use K = V (values are the cached keys)
    kv_int8: bool = False        # int8 KV caches (codes + (min, step) per row)
    tokens: int = 1              # decode: new tokens per sequence (> 1: multi-token decode)
    description: str = field(default="", compare=False)


E2B_LOCAL = LayerType(window=512, n_kv_heads=4, head_dim=256, rope_frac=1.0, rope_theta=1e4)
E2B_GLOBAL = LayerType(window=0, n_kv_heads=1, head_dim=512, rope_frac=0.25, rope_theta=1e6)
L31B_LOCAL = LayerType(window=1024, n_kv_heads=16, head_dim=256, rope_frac=1.0, rope_theta=1e4)
L31B_GLOBAL = LayerType(window=0, n_kv_heads=4, head_dim=512, rope_frac=0.25, rope_theta=1e6)

WORKLOADS = {
    "local_s1024": Workload(
        "local_s1024", "prefill", batch=1, n_q_heads=8, n_layers=1, ratio=1,
        local=E2B_LOCAL, global_=E2B_GLOBAL, seq=1024, seed=0, fixed_kinds=("local",),
        description="single local layer prefill: B1 S1024 W512 Hq8 Hkv4 D256, RoPE 1e4"),
    "e2b_block_s8192": Workload(
        "e2b_block_s8192", "prefill", batch=1, n_q_heads=8, n_layers=5, ratio=4,
        local=E2B_LOCAL, global_=E2B_GLOBAL, seq=8192, seed=1,
        description="E2B-shaped 5-layer prefill (4 local + global): B1 S8192 Hq8"),
    "31b_block_s32768": Workload(
        "31b_block_s32768", "prefill", batch=2, n_q_heads=32, n_layers=6, ratio=5,
        local=L31B_LOCAL, global_=L31B_GLOBAL, seq=32768, k_scale=0.5, seed=2,
        description="31B-shaped 6-layer prefill (5 local + global): B2 S32768 Hq32, K x0.5"),
    "31b_decode_b64": Workload(
        "31b_decode_b64", "decode", batch=64, n_q_heads=32, n_layers=6, ratio=5,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=4096, len_hi=131072, n_shared=2, seed=3,
        description="31B-shaped 6-layer decode: B64, KV length U[4096,131072], ring 1024, "
                    "last 2 layers shared"),
    "31b_verify_b64_k4": Workload(
        "31b_verify_b64_k4", "decode", batch=64, n_q_heads=32, n_layers=6, ratio=5,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=4096, len_hi=131072, seed=3, tokens=4,
        description="31B-shaped 6-layer multi-token decode (checking k = 4 drafted tokens): B64, "
                    "KV length U[4096,131072] including the 4 new tokens, ring 1024, no shared layers"),
    "31b_verify_b8_k4": Workload(
        "31b_verify_b8_k4", "decode", batch=8, n_q_heads=32, n_layers=6, ratio=5,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=16384, len_hi=32768, seed=5, tokens=4,
        description="31B-shaped 6-layer multi-token decode, k = 4, B8, KV length U[16384,32768] "
                    "(a capture-sized case: every layer's K+V above the L2 size)"),
    "31b_decode_b64_int8": Workload(
        "31b_decode_b64_int8", "decode", batch=64, n_q_heads=32, n_layers=6, ratio=5,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=4096, len_hi=131072, n_shared=2, seed=3,
        kv_int8=True,
        description="31B-shaped 6-layer decode on int8 KV caches: B64, KV length U[4096,131072], "
                    "ring 1024, last 2 layers shared"),
    "31b_decode_b16_12l_shared": Workload(
        "31b_decode_b16_12l_shared", "decode", batch=16, n_q_heads=32, n_layers=12, ratio=5,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=4096, len_hi=131072, n_shared=2, seed=7,
        description="31B-shaped 12-layer decode (two 5:1 patterns), last 2 layers shared: "
                    "10 -> 9 (local), 11 -> 5 (global); B16, KV length U[4096,131072]"),
    "global_chunk_256k": Workload(
        "global_chunk_256k", "prefill", batch=1, n_q_heads=32, n_layers=1, ratio=0,
        local=L31B_LOCAL, global_=L31B_GLOBAL, seq=4096, prior=262144 - 4096, seed=4,
        fixed_kinds=("global",),
        description="chunked prefill of 4096 queries at 258048.. against a 256K global cache"),
    "31b_local_s8192": Workload(
        "31b_local_s8192", "prefill", batch=1, n_q_heads=32, n_layers=1, ratio=0,
        local=L31B_LOCAL, global_=L31B_GLOBAL, seq=8192, k_scale=0.5, seed=2, fixed_kinds=("local",),
        description="one 31B-shaped local layer, B1 S8192 Hq32 Hkv16 D256 W1024 (a kernel-profiling case)"),
    "global_chunk_64k": Workload(
        "global_chunk_64k", "prefill", batch=1, n_q_heads=32, n_layers=1, ratio=0,
        local=L31B_LOCAL, global_=L31B_GLOBAL, seq=1024, prior=65536 - 1024, seed=4,
        fixed_kinds=("global",),
        description="chunked prefill of 1024 queries at 64512.. against a 64K global cache "
                    "(a kernel-profiling case)"),
    "global_s16384": Workload(
        "global_s16384", "prefill", batch=1, n_q_heads=32, n_layers=1, ratio=0,
        local=L31B_LOCAL, global_=L31B_GLOBAL, seq=16384, seed=5, fixed_kinds=("global",),
        description="one 31B-shaped global layer, B1 S16384 Hq32 Hkv4 D512 (a kernel-profiling case)"),
    "global_decode_256k_keqv": Workload(
        "global_decode_256k_keqv", "decode", batch=1, n_q_heads=32, n_layers=1, ratio=0,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=262144, len_hi=262144, seed=6,
        fixed_kinds=("global",), k_eq_v=True,
        description="single-token decode at KV length 262144, one global layer with K = V"),
    "global_decode_256k": Workload(
        "global_decode_256k", "decode", batch=1, n_q_heads=32, n_layers=1, ratio=0,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=262144, len_hi=262144, seed=4,
        fixed_kinds=("global",),
        description="single-token decode at KV length 262144, one global layer"),
    "local_decode_b64_int8": Workload(
        "local_decode_b64_int8", "decode", batch=64, n_q_heads=32, n_layers=1, ratio=0,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=4096, len_hi=131072, seed=3,
        fixed_kinds=("local",), kv_int8=True,
        description="one 31B-shaped local layer's decode on an int8 ring: B64, ring 1024"),
    "global_decode_256k_int8": Workload(
        "global_decode_256k_int8", "decode", batch=1, n_q_heads=32, n_layers=1, ratio=0,
        local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=262144, len_hi=262144, seed=4,
        fixed_kinds=("global",), kv_int8=True,
        description="single-token decode at KV length 262144 on an int8 KV cache, one global layer"),
}


def visible_pairs_prefill(seq: int, prior: int, window: int) -> int:
    """Number of (query, key) pairs a causal (window-limited) chunk attends."""
    total = 0
    if window == 0:
        # query at position p sees p + 1 keys
        first, last = prior, prior + seq - 1
        return (first + 1 + last + 1) * seq // 2
    for i in range(seq):
        p = prior + i
        total += min(p + 1, window)
    return total


def prefill_flops(w: Workload, is_global: list[bool]) -> int:
    """Algorithmic FLOPs of a prefill workload: 4 * B * Hq * D * visible pairs
    per layer (QK^T and PV, 2 FLOPs per multiply-add); masked or skipped
    pairs are not counted. `is_global` is the layer schedule."""
    total = 0
    for g in is_global:
        t = w.global_ if g else w.local
        total += 4 * w.batch * w.n_q_heads * t.head_dim * visible_pairs_prefill(w.seq, w.prior, t.window)
    return total


def prefill_attn_bytes(w: Workload, t: LayerType) -> int:
    """Algorithmic DRAM bytes of one prefill attention launch of layer type t:
    the queries read and the outputs written, the chunk's keys and values
    read (rotated keys from the cache or the workspace, values from the
    caller), and on a chunk after cached tokens the cached prefix's keys and
    values, each element once (bf16)."""
    q = w.batch * w.seq * w.n_q_heads * t.head_dim * 2
    kv = w.batch * w.seq * t.n_kv_heads * t.head_dim * 2
    if w.prior:
        vis_prior = min(w.prior, t.window) if t.window else w.prior
        kv += w.batch * vis_prior * t.n_kv_heads * t.head_dim * 2
    return 2 * q + (1 if w.k_eq_v else 2) * kv


def layer_shape_tag(w: Workload, t: LayerType) -> str:
    """Per-(batch, head) shape of a layer's attention: q heads, KV heads, head
    dim, window, and whether the chunk follows cached tokens (c) or not (f).
    Traffic records of one shape scale with the bytes moved."""
    return "%d-%d-%d-%d-%s" % (w.n_q_heads, t.n_kv_heads, t.head_dim, t.window, "c" if w.prior else "f")
