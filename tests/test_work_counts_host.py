"""The algorithmic work behind every reported rate, checked without a GPU.

bench.py divides FLOPs (prefill) or bytes (decode, multi-token decode) by
device time. Those counts come from `workloads.py` and bench.py's byte
counters; here they are held to brute-force sums over the oracle's own
visibility rule (a query at position p sees keys p - W < j <= p, all j <= p
on a global layer: "Gemma 4: End-to-End Architecture Walkthrough", 3a) and
to closed forms at the benchmarked sizes."""
from __future__ import annotations

import pytest
import torch

import bench
import oracle
from hybrid_local_global_b200 import synth
from hybrid_local_global_b200.workloads import WORKLOADS, prefill_flops, visible_pairs_prefill


def brute_pairs(seq, prior, window):
    n_keys = prior + seq
    return sum(oracle.visible_range(prior + i, window, n_keys)[2] for i in range(seq))


def keys_some_token_sees(L, T, window):
    """Size of the union of the oracle's visible ranges (inclusive [lo, hi])
    of the queries at positions L-T..L-1 among L keys."""
    total, covered_to = 0, -1
    for p in range(L - T, L):
        lo, hi, cnt = oracle.visible_range(p, window, L)
        if cnt:
            total += hi - max(lo, covered_to + 1) + 1 if hi > covered_to else 0
            covered_to = max(covered_to, hi)
    return total


@pytest.mark.parametrize("seq,prior,window", [
    (1, 0, 0), (1, 0, 4), (7, 0, 0), (7, 0, 3), (7, 0, 7), (7, 0, 9), (40, 0, 16), (40, 5, 16),
    (40, 100, 16), (3, 100, 16), (40, 100, 0), (129, 300, 128), (16, 0, 1)])
def test_visible_pairs_equal_brute_force(seq, prior, window):
    assert visible_pairs_prefill(seq, prior, window) == brute_pairs(seq, prior, window)


def test_visible_pairs_closed_forms_at_benchmarked_sizes():
    """A window W over S >= W queries from position 0: the first W queries
    see 1..W keys, the rest W each. A global layer: S(S+1)/2. A chunk at
    positions P..P+S-1 on a global layer: the sum of p + 1."""
    def local(S, W):
        return W * (W + 1) // 2 + (S - W) * W

    assert visible_pairs_prefill(1024, 0, 512) == local(1024, 512) == 393_472
    assert visible_pairs_prefill(8192, 0, 512) == local(8192, 512) == 4_063_488
    assert visible_pairs_prefill(32768, 0, 1024) == local(32768, 1024) == 33_030_656
    assert visible_pairs_prefill(8192, 0, 0) == 8192 * 8193 // 2 == 33_558_528
    assert visible_pairs_prefill(32768, 0, 0) == 32768 * 32769 // 2 == 536_887_296
    P, S = 262144 - 4096, 4096
    assert visible_pairs_prefill(S, P, 0) == S * P + S * (S + 1) // 2 == 1_065_355_264


@pytest.mark.parametrize("name", ["local_s1024", "e2b_block_s8192", "31b_block_s32768", "global_chunk_256k"])
def test_prefill_flops_of_benchmarked_workloads(name):
    """4 FLOPs per head dimension per visible (query, key) pair and q head:
    one multiply-add each for Q K^T and for P V."""
    w = WORKLOADS[name]
    sched = bench.schedule_of(w)
    want = 0
    for g in sched:
        t = w.global_ if g else w.local
        pairs = brute_pairs(w.seq, w.prior, t.window) if w.seq <= 2048 else \
            visible_pairs_prefill(w.seq, w.prior, t.window)  # pinned by the closed forms above
        want += 2 * 2 * w.batch * w.n_q_heads * t.head_dim * pairs
    assert prefill_flops(w, sched) == want


def test_headline_prefill_flops_value():
    """The 31B-shaped block: 5 local layers of 2.16e12 FLOPs and one global
    layer of 7.04e13 (B2, Hq32; local D256 W1024, global D512)."""
    w = WORKLOADS["31b_block_s32768"]
    sched = bench.schedule_of(w)
    assert sched == [False] * 5 + [True]
    local = 4 * 2 * 32 * 256 * 33_030_656
    glob = 4 * 2 * 32 * 512 * 536_887_296
    assert prefill_flops(w, sched) == 5 * local + glob
    assert abs(prefill_flops(w, sched) - 8.12e13) / 8.12e13 < 2e-3


class _Stack:
    """The parts of AttentionStack that bench.py's byte counters read, built
    from the oracle's schedule and share rule."""

    def __init__(self, w):
        self.w = w
        self.n_layers = w.n_layers
        self.sched = bench.schedule_of(w)
        self.src = [oracle.share_source(w.n_layers, w.ratio, w.n_shared, l) if w.n_shared else l
                    for l in range(w.n_layers)]

    def layer_type(self, l):
        return self.w.global_ if self.sched[l] else self.w.local

    def keqv(self, l):
        return bool(self.w.k_eq_v and self.sched[l])

    def is_shared(self, l):
        return self.src[l] not in (l, -1)


def lengths_of(w):
    if w.len_lo == w.len_hi:
        return torch.full((w.batch,), w.len_hi, dtype=torch.int32)
    return synth.decode_lengths(w.batch, w.len_lo, w.len_hi, seed=w.seed)


@pytest.mark.parametrize("name", ["31b_decode_b64", "31b_decode_b64_int8", "31b_decode_b16_12l_shared",
                                  "global_decode_256k", "global_decode_256k_keqv", "local_decode_b64_int8"])
def test_decode_kv_bytes_equal_visible_keys(name):
    """Decode reads every visible key's K and V row once per KV head (K only
    on a K = V layer): D bf16 elements a row, or D codes and one fp32
    (min, step) pair on an int8 cache. A shared layer reads its source's
    cache, so it counts too."""
    w = WORKLOADS[name]
    st = _Stack(w)
    lens = lengths_of(w)
    for l in range(w.n_layers):
        t = st.layer_type(l)
        row = t.head_dim + 8 if w.kv_int8 else 2 * t.head_dim
        keys = sum(oracle.visible_range(int(L) - 1, t.window, int(L))[2] for L in lens)
        want = keys * t.n_kv_heads * row * (1 if st.keqv(l) else 2)
        assert bench.visible_kv_bytes(st, l, lens) == want


@pytest.mark.parametrize("name", ["31b_verify_b64_k4", "31b_verify_b8_k4"])
def test_multi_token_kv_bytes_equal_keys_some_token_sees(name):
    """T new tokens at positions L-T..L-1: the keys counted are those at
    least one of them sees (the union of their visible ranges), once per KV
    head, K and V."""
    w = WORKLOADS[name]
    st = _Stack(w)
    lens = lengths_of(w)
    T = w.tokens
    for l in range(w.n_layers):
        t = st.layer_type(l)
        keys = sum(keys_some_token_sees(L, T, t.window) for L in lens.tolist())
        want = keys * t.n_kv_heads * 2 * t.head_dim * (1 if st.keqv(l) else 2)
        assert bench.verify_kv_bytes(st, l, lens, T) == want


def test_multi_token_kv_bytes_short_sequences():
    """Rings not yet full and sequences no longer than the new tokens."""
    w = WORKLOADS["31b_verify_b8_k4"]
    st = _Stack(w)
    T = 4
    lens = torch.tensor([4, 5, 700, 1027, 1028, 1029, 5000], dtype=torch.int32)
    for l in range(w.n_layers):
        t = st.layer_type(l)
        keys = 0
        for L in lens.tolist():
            seen = set()  # brute force: every visible key of every new token
            for p in range(L - T, L):
                lo, hi, cnt = oracle.visible_range(p, t.window, L)
                seen.update(range(lo, hi + 1) if cnt else ())
            assert len(seen) == keys_some_token_sees(L, T, t.window)
            keys += len(seen)
        assert bench.verify_kv_bytes(st, l, lens, T) == keys * t.n_kv_heads * 4 * t.head_dim


@pytest.mark.parametrize("name", ["31b_decode_b64", "31b_decode_b16_12l_shared", "global_decode_256k_keqv"])
def test_decode_step_bytes(name):
    """A decode step's bytes: each layer's visible K/V rows, its queries read
    and outputs written (bf16), and, on a layer that owns its cache, the new
    token's K (and V unless K = V) row written; a shared layer writes none."""
    w = WORKLOADS[name]
    st = _Stack(w)
    lens = lengths_of(w)
    want = 0
    for l in range(w.n_layers):
        t = st.layer_type(l)
        kv = 1 if st.keqv(l) else 2
        keys = sum(oracle.visible_range(int(L) - 1, t.window, int(L))[2] for L in lens)
        want += keys * t.n_kv_heads * 2 * t.head_dim * kv
        want += w.batch * w.n_q_heads * t.head_dim * 2 * 2
        if oracle.share_source(w.n_layers, w.ratio, w.n_shared, l) in (l, -1):
            want += w.batch * t.n_kv_heads * t.head_dim * 2 * kv
    assert bench.decode_bytes(w, st, lens) == want
    if name == "31b_decode_b16_12l_shared":
        assert [st.is_shared(l) for l in range(w.n_layers)] == [False] * 10 + [True, True]


def test_prefill_attention_bytes_match_the_capture_records():
    """The algorithmic bytes a prefill traffic record is scaled by: queries
    read and outputs written once, the chunk's K and V read once (plus the
    visible cached prefix on a chunk after cached tokens), bf16. They equal
    the units each committed capture record states for its workload."""
    import os
    from hybrid_local_global_b200.profiling import traffic_records
    from hybrid_local_global_b200.workloads import prefill_attn_bytes
    recs = [r for r in traffic_records(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                                                    "profiles"))
            if r["kernel"] in ("k_prefill_tc", "k_prefill_pair") and "units" in r]
    assert recs
    for r in recs:
        w = WORKLOADS[r["workload"]]
        t = w.global_ if r["layer"] == "global" else w.local
        assert prefill_attn_bytes(w, t) == int(r["units"]), r
    w = WORKLOADS["31b_local_s8192"]
    q = 8192 * 32 * 256 * 2
    kv = 8192 * 16 * 256 * 2
    assert prefill_attn_bytes(w, w.local) == 2 * q + 2 * kv == 402_653_184


def test_decode_bytes_match_the_capture_records():
    """Each committed decode and multi-token capture record's algorithmic
    units equal what bench.py's counters give for its workload and layer."""
    import os
    from hybrid_local_global_b200.profiling import traffic_records
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    seen = 0
    for r in traffic_records(os.path.join(root, "profiles")):
        if r["kernel"] not in ("k_decode_split", "k_decode_split_q8", "k_verify_tc") or "units" not in r:
            continue
        w = WORKLOADS[r["workload"]]
        st = _Stack(w)
        lens = lengths_of(w)
        layers = [l for l in range(w.n_layers) if (st.layer_type(l).window == 0) == (r["layer"] == "global")]
        l = layers[0]
        if r["kernel"] == "k_verify_tc":
            got = bench.verify_kv_bytes(st, l, lens, w.tokens)
        else:
            got = bench.visible_kv_bytes(st, l, lens)
        assert got == int(r["units"]), (r, got)
        seen += 1
    assert seen >= 5
