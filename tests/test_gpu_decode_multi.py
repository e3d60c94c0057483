"""GPU parity of multi-token decode (several new tokens per sequence, as when
the target model checks a drafter's proposals in speculative decoding)
against the fp64 oracle, through the C ABI. Covered: the tensor-core path of
bf16 layers (global: q heads x tokens packed in one tile, split over the
cached keys, combined; unshared local: the ring as it was plus the new rows),
the per-token decode route of int8 global layers, and the chunked-prefill
route of the rest (int8 local, shared local, more than 128 rows per KV head);
cache slots written, KV sharing, K = V, paged caches, bounded-wait timeouts
and the device range check on every route."""
import math

import numpy as np
import pytest
import torch

from hybrid_local_global_b200 import native, synth
from hybrid_local_global_b200.stack import AttentionStack
from hybrid_local_global_b200.workloads import L31B_GLOBAL, L31B_LOCAL, Workload

from gpu_util import assert_close, assert_rotated_bf16, to_bits

pytestmark = pytest.mark.gpu


def run_multi_case(oracle, *, lens, T, Hq, Hkv, D, W, frac, theta, seed, shared=False, keqv=False,
                   cap_extra=16, expect_status=False):
    """expect_status: the call is expected to report GEMMA_ERR_DEVICE_TIMEOUT
    (a test hook dropped a copy); only that is checked."""
    dev = torch.device("cuda")
    B = len(lens)
    g = synth.generator(seed)
    max_len = max(lens)
    cap = W if W else max_len + cap_extra
    kc = torch.full((B, Hkv, cap, D), float("nan"), dtype=torch.bfloat16)
    vc = kc.clone()
    k_log = torch.zeros((B, max_len, Hkv, D), dtype=torch.bfloat16)
    v_log = torch.zeros_like(k_log)
    for b in range(B):
        n = lens[b] - T
        first = max(0, n - W) if W else 0
        kr = synth.randn_bf16((Hkv, n - first, D), g)
        vr = synth.randn_bf16((Hkv, n - first, D), g)
        for i, p in enumerate(range(first, n)):
            slot = p % W if W else p
            kc[b, :, slot], vc[b, :, slot] = kr[:, i], vr[:, i]
        k_log[b, first:n] = kr.transpose(0, 1)
        v_log[b, first:n] = vr.transpose(0, 1)
    q = synth.randn_bf16((B, T, Hq, D), g)
    kn = synth.randn_bf16((B, T, Hkv, D), g)
    vn = synth.randn_bf16((B, T, Hkv, D), g)
    for b in range(B):
        n = lens[b] - T
        k_log[b, n:lens[b]] = kn[b]
        v_log[b, n:lens[b]] = vn[b]
        if shared:
            # the new tokens' K/V are in the (source layer's) cache already, rotated
            for t in range(T):
                slot = (n + t) % W if W else n + t
                kc[b, :, slot], vc[b, :, slot] = kn[b, t], vn[b, t]
    if keqv:
        vc, vn, v_log = kc, kn, None
    kcd = kc.to(dev)
    vcd = kcd if keqv else vc.to(dev)
    out = torch.full((B, T, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    flags = (native.GEMMA_F_SHARED if shared else 0) | (native.GEMMA_F_KEQV if keqv else 0)
    native.gemma_attn_decode_multi(q.to(dev), None if shared else kn.to(dev),
                                   None if (shared or keqv) else vn.to(dev), kcd, None if keqv else vcd,
                                   seq_lens=sl, max_seq_len=max_len, window=W, rope_frac=frac,
                                   rope_theta=theta, scale=scale, out=out, flags=flags)
    if expect_status:
        assert native.gemma_attn_sync_status() == native.GEMMA_ERR_DEVICE_TIMEOUT
        return out
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    before = [L - T for L in lens]
    ref, _ = oracle.attention(to_bits(q), to_bits(k_log), None if keqv else to_bits(v_log), q_pos0=before,
                              n_keys=lens, rot_from=lens if shared else before, window=W,
                              rope_frac=frac, theta=theta, scale=scale)
    got = out.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
    assert_close(got, ref, what="multi-token decode T=%d" % T)
    kc1, vc1 = kcd.cpu(), vcd.cpu()
    for b in range(B):
        written = torch.zeros(cap, dtype=torch.bool)
        for t in range(T):
            p = before[b] + t
            slot = p % W if W else p
            if W and p < lens[b] - W:
                continue  # overwritten later in the same call by a newer token
            written[slot] = True
            if shared:
                continue
            if not keqv:
                assert torch.equal(vc1[b, :, slot], vn[b, t]), "V slot %d" % slot
            for h in range(Hkv):
                exp = torch.from_numpy(oracle.rope_bf16(to_bits(kn[b, t, h]), p, frac, theta)).to(torch.bfloat16)
                assert_rotated_bf16(kc1[b, h, slot], exp, kn[b, t, h], "K slot %d" % slot)
        keep = ~written if not shared else torch.ones(cap, dtype=torch.bool)
        # unwritten slots keep their bytes (NaN included)
        assert torch.equal(kc1[b][:, keep].view(torch.int16), kc[b][:, keep].view(torch.int16))
        assert torch.equal(vc1[b][:, keep].view(torch.int16), vc[b][:, keep].view(torch.int16))
    return out


GLOBAL_CASES = [
    dict(lens=[3000, 700], T=4, Hq=32, Hkv=4, D=512, seed=301),            # 31B global shape, 3 splits
    dict(lens=[4], T=4, Hq=32, Hkv=4, D=512, seed=302),                    # the tokens are the sequence
    dict(lens=[1, 2000], T=1, Hq=8, Hkv=1, D=512, seed=303),               # one token (= decode)
    dict(lens=[2500, 130, 9], T=2, Hq=8, Hkv=1, D=512, seed=304),          # E2B global shape
    dict(lens=[5000, 1031], T=8, Hq=32, Hkv=4, D=512, seed=305),           # 64 rows a tile
    dict(lens=[1500, 16], T=16, Hq=32, Hkv=4, D=512, seed=306),            # 128 rows: the full tile
    dict(lens=[2049, 300], T=3, Hq=8, Hkv=4, D=256, seed=307, frac=1.0, theta=1e4),  # head_dim 256
    dict(lens=[1024, 1025], T=5, Hq=12, Hkv=2, D=512, seed=308),           # split edges, G = 6
]


@pytest.mark.parametrize("case", GLOBAL_CASES,
                         ids=["31b", "LeqT", "T1", "e2b", "T8", "T16", "D256", "edges"])
def test_multi_global_tensor_core(oracle, case):
    case = dict(case)
    run_multi_case(oracle, W=0, frac=case.pop("frac", 0.25), theta=case.pop("theta", 1e6), **case)


def test_multi_global_shared(oracle):
    run_multi_case(oracle, lens=[2100, 77], T=4, Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6, seed=311,
                   shared=True)


def test_multi_global_keqv(oracle):
    run_multi_case(oracle, lens=[1800, 5], T=4, Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6, seed=312,
                   keqv=True)


def test_multi_global_exact_capacity(oracle):
    """The last key sits in the last cache row (no padding past the sequence)."""
    run_multi_case(oracle, lens=[1280, 1000], T=4, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=313,
                   cap_extra=0)


@pytest.mark.parametrize("case", [
    dict(lens=[3000, 700, 4], T=4, Hq=32, Hkv=16, D=256, W=1024, seed=321),    # 31B local shape, 4 ring splits
    dict(lens=[3000], T=4, Hq=32, Hkv=16, D=256, W=1024, seed=325),            # one sequence: 8 ring splits
    dict(lens=[1028, 1027, 1029, 5], T=4, Hq=32, Hkv=16, D=256, W=1024, seed=326),  # ring just full / not
    dict(lens=[600, 65], T=3, Hq=8, Hkv=4, D=256, W=64, seed=322),             # ring wraps inside the call
    dict(lens=[900, 8], T=8, Hq=32, Hkv=4, D=256, W=512, seed=327),            # 64 query rows
    dict(lens=[300, 17], T=16, Hq=8, Hkv=4, D=512, W=16, seed=328, frac=0.25, theta=1e6),  # T = window
])
def test_multi_local_tensor_core(oracle, case):
    """Local layers: the ring as it was, plus a tail tile of the new tokens;
    the ring is written after the attention."""
    case = dict(case)
    run_multi_case(oracle, frac=case.pop("frac", 1.0), theta=case.pop("theta", 1e4), **case)


@pytest.mark.parametrize("case", [
    dict(lens=[40], T=40, Hq=4, Hkv=2, D=256, W=16, seed=323),                 # more tokens than the window
    dict(lens=[700, 90], T=40, Hq=4, Hkv=2, D=256, W=64, seed=329),            # 80 query rows
    dict(lens=[3000, 700], T=17, Hq=32, Hkv=4, D=512, W=0, seed=324, frac=0.25, theta=1e6),  # 136 rows: route
], ids=["T_gt_W", "local_rows80", "global_route"])
def test_multi_routed_layers(oracle, case):
    case = dict(case)
    run_multi_case(oracle, frac=case.pop("frac", 1.0), theta=case.pop("theta", 1e4), **case)


@pytest.mark.parametrize("keqv", [False, True])
def test_multi_int8_global_equals_consecutive_decodes(oracle, keqv):
    """An int8 global layer takes the tokens one at a time through
    single-token decode: bit-identical to T gemma_attn_decode calls at
    lengths seq_lens - T + 1 .. seq_lens on a copy of the cache (which the
    int8 decode tests hold to the oracle), with the same codes written."""
    dev = torch.device("cuda")
    B, T, Hq, Hkv, D, lens = 2, 4, 32, 4, 512, [1500, 300]
    cap = 1600
    g = synth.generator(331 + keqv, "cuda")

    def fresh():
        return synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, cap, D, dev), g)

    kc = fresh()
    vc = kc if keqv else fresh()
    kc2 = native.Int8KVCache(B, Hkv, cap, D, dev)
    kc2.buf.copy_(kc.buf)
    vc2 = kc2
    if not keqv:
        vc2 = native.Int8KVCache(B, Hkv, cap, D, dev)
        vc2.buf.copy_(vc.buf)
    q = synth.randn_bf16((B, T, Hq, D), g, "cuda")
    kn = synth.randn_bf16((B, T, Hkv, D), g, "cuda")
    vn = None if keqv else synth.randn_bf16((B, T, Hkv, D), g, "cuda")
    flags = native.GEMMA_F_KEQV if keqv else 0
    kw = dict(window=0, rope_frac=0.25, rope_theta=1e6, scale=1.0 / math.sqrt(D), flags=flags)
    o1 = torch.empty((B, T, Hq, D), dtype=torch.bfloat16, device=dev)
    native.gemma_attn_decode_multi(q, kn, vn, kc, None if keqv else vc, max_seq_len=max(lens), out=o1,
                                   seq_lens=torch.tensor(lens, dtype=torch.int32, device=dev), **kw)
    o2 = torch.empty_like(o1)
    for t in range(T):
        ot = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
        native.gemma_attn_decode(q[:, t].contiguous(), kn[:, t].contiguous(),
                                 None if keqv else vn[:, t].contiguous(), kc2, None if keqv else vc2,
                                 seq_lens=torch.tensor([L - T + t + 1 for L in lens], dtype=torch.int32, device=dev),
                                 max_seq_len=max(lens), out=ot, **kw)
        o2[:, t] = ot
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(kc.buf, kc2.buf) and torch.equal(vc.buf, vc2.buf)


def test_multi_int8_local_matches_prefill_route(oracle):
    """An int8 local layer goes through the chunked prefill: bit-identical
    to gemma_attn_prefill after seq_lens - T cached tokens."""
    dev = torch.device("cuda")
    B, T, Hq, Hkv, D, W, lens = 2, 4, 32, 16, 256, 1024, [1500, 300]
    g = synth.generator(333, "cuda")
    kc = synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, W, D, dev), g)
    vc = synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, W, D, dev), g)
    kc2, vc2 = native.Int8KVCache(B, Hkv, W, D, dev), native.Int8KVCache(B, Hkv, W, D, dev)
    kc2.buf.copy_(kc.buf)
    vc2.buf.copy_(vc.buf)
    q = synth.randn_bf16((B, T, Hq, D), g, "cuda")
    kn = synth.randn_bf16((B, T, Hkv, D), g, "cuda")
    vn = synth.randn_bf16((B, T, Hkv, D), g, "cuda")
    kw = dict(window=W, rope_frac=1.0, rope_theta=1e4, scale=1.0 / math.sqrt(D))
    o1 = torch.empty((B, T, Hq, D), dtype=torch.bfloat16, device=dev)
    o2 = torch.empty_like(o1)
    native.gemma_attn_decode_multi(q, kn, vn, kc, vc, max_seq_len=max(lens), out=o1,
                                   seq_lens=torch.tensor(lens, dtype=torch.int32, device=dev), **kw)
    native.gemma_attn_prefill(q, kn, vn, kc2, vc2, out=o2,
                              seq_lens_before=torch.tensor([L - T for L in lens], dtype=torch.int32, device=dev), **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(kc.buf, kc2.buf) and torch.equal(vc.buf, vc2.buf)


def test_multi_equals_consecutive_decodes(oracle):
    """T tokens in one call against T single-token decode calls on a copy of
    the cache: the same rows within the parity tolerance (the two paths
    round the query scaling differently), and the same cache bytes."""
    dev = torch.device("cuda")
    B, T, Hq, Hkv, D, lens = 3, 4, 32, 4, 512, [2000, 37, 4100]
    cap = max(lens) + 8
    g = synth.generator(341)
    kc = synth.randn_bf16((B, Hkv, cap, D), g).to(dev)
    vc = synth.randn_bf16((B, Hkv, cap, D), g).to(dev)
    kc2, vc2 = kc.clone(), vc.clone()
    q = synth.randn_bf16((B, T, Hq, D), g).to(dev)
    kn = synth.randn_bf16((B, T, Hkv, D), g).to(dev)
    vn = synth.randn_bf16((B, T, Hkv, D), g).to(dev)
    kw = dict(window=0, rope_frac=0.25, rope_theta=1e6, scale=1.0 / math.sqrt(D))
    o1 = torch.empty((B, T, Hq, D), dtype=torch.bfloat16, device=dev)
    native.gemma_attn_decode_multi(q, kn, vn, kc, vc, seq_lens=torch.tensor(lens, dtype=torch.int32, device=dev),
                                   max_seq_len=max(lens), out=o1, **kw)
    o2 = torch.empty_like(o1)
    for t in range(T):
        sl = torch.tensor([L - T + t + 1 for L in lens], dtype=torch.int32, device=dev)
        ot = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
        native.gemma_attn_decode(q[:, t].contiguous(), kn[:, t].contiguous(), vn[:, t].contiguous(), kc2, vc2,
                                 seq_lens=sl, max_seq_len=max(lens), out=ot, **kw)
        o2[:, t] = ot
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(kc.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vc2.view(torch.int16))
    assert_close(o1.float().cpu().numpy(), o2.float().cpu().numpy(), what="one call vs T decode calls")


def test_multi_range_check_reports(oracle):
    """seq_lens below the token count: the device check reports
    GEMMA_ERR_DEVICE_RANGE, writes zeros for that sequence, and the other
    sequences are unaffected."""
    dev = torch.device("cuda")
    B, T, Hq, Hkv, D = 2, 4, 8, 1, 512
    cap = 512
    g = synth.generator(351)
    kc = synth.randn_bf16((B, Hkv, cap, D), g).to(dev)
    vc = synth.randn_bf16((B, Hkv, cap, D), g).to(dev)
    q = synth.randn_bf16((B, T, Hq, D), g).to(dev)
    kn = synth.randn_bf16((B, T, Hkv, D), g).to(dev)
    vn = synth.randn_bf16((B, T, Hkv, D), g).to(dev)
    out = torch.full((B, T, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    sl = torch.tensor([300, 3], dtype=torch.int32, device=dev)
    native.gemma_attn_decode_multi(q, kn, vn, kc, vc, seq_lens=sl, max_seq_len=300, window=0, rope_frac=0.25,
                                   rope_theta=1e6, scale=1.0 / math.sqrt(D), out=out)
    assert native.gemma_attn_sync_status() == native.GEMMA_ERR_DEVICE_RANGE
    assert torch.count_nonzero(out[1].float()) == 0
    assert torch.isfinite(out[0].float()).all()
    assert native.gemma_attn_sync_status() == 0  # reading the status clears it


@pytest.mark.parametrize("route", ["int8_global", "chunked_prefill"])
def test_multi_range_check_other_routes(route):
    """seq_lens below the token count on the two routes that do not run the
    tensor-core multi-token kernel: the int8 global layer's per-token
    decodes and the chunked prefill (q heads per KV head x tokens above
    128). The device check reports GEMMA_ERR_DEVICE_RANGE, and the valid
    sequence's output is bit-identical to a call where every length is
    valid."""
    dev = torch.device("cuda")
    B, Hq, Hkv, D, cap = 2, 32, 4, 512, 512
    T = 4 if route == "int8_global" else 17
    g = synth.generator(353, "cuda")
    if route == "int8_global":
        kc = synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, cap, D, dev), g)
        vc = synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, cap, D, dev), g)
    else:
        kc = synth.randn_bf16((B, Hkv, cap, D), g, "cuda")
        vc = synth.randn_bf16((B, Hkv, cap, D), g, "cuda")
    q = synth.randn_bf16((B, T, Hq, D), g, "cuda")
    kn = synth.randn_bf16((B, T, Hkv, D), g, "cuda")
    vn = synth.randn_bf16((B, T, Hkv, D), g, "cuda")
    kw = dict(max_seq_len=300, window=0, rope_frac=0.25, rope_theta=1e6, scale=1.0 / math.sqrt(D))
    bad = torch.full((B, T, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    native.gemma_attn_decode_multi(q, kn, vn, kc, vc, out=bad,
                                   seq_lens=torch.tensor([300, T - 1], dtype=torch.int32, device=dev), **kw)
    assert native.gemma_attn_sync_status() == native.GEMMA_ERR_DEVICE_RANGE
    good = torch.empty_like(bad)
    native.gemma_attn_decode_multi(q, kn, vn, kc, vc, out=good,
                                   seq_lens=torch.tensor([300, 300], dtype=torch.int32, device=dev), **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.isfinite(good.float()).all()
    assert torch.equal(bad[0].view(torch.int16), good[0].view(torch.int16))


def test_multi_stack_31b_block(oracle):
    """k = 4 tokens per sequence through every layer of a 31B-shaped
    6-layer stack (5 local with ring caches, 1 global) with the stack's
    multi-token decode call."""
    prior, kq = [3000, 700], 4
    w = Workload("verify_k4", "decode", batch=2, n_q_heads=32, n_layers=6, ratio=5,
                 local=L31B_LOCAL, global_=L31B_GLOBAL, len_lo=1, len_hi=max(prior) + kq, seed=17)
    dev = torch.device("cuda")
    st = AttentionStack(w, dev)
    g = synth.generator(17)
    lens_l = [p + kq for p in prior]
    ws = torch.empty(st.decode_multi_workspace_bytes(kq, max(lens_l)), dtype=torch.uint8, device=dev)
    lens = torch.tensor(lens_l, dtype=torch.int32, device=dev)
    T = max(lens_l)
    for l in range(st.n_layers):
        t = st.layer_type(l)
        Hkv, D, W = t.n_kv_heads, t.head_dim, t.window
        k_log = torch.zeros((w.batch, T, Hkv, D), dtype=torch.bfloat16)
        v_log = torch.zeros_like(k_log)
        kc = torch.full(tuple(st.k_cache[l].shape), float("nan"), dtype=torch.bfloat16)
        vc = kc.clone()
        for b in range(w.batch):
            first = max(0, prior[b] - W) if W else 0
            kr = synth.randn_bf16((Hkv, prior[b] - first, D), g)
            vr = synth.randn_bf16((Hkv, prior[b] - first, D), g)
            for i, p in enumerate(range(first, prior[b])):
                slot = p % W if W else p
                kc[b, :, slot], vc[b, :, slot] = kr[:, i], vr[:, i]
            k_log[b, first:prior[b]] = kr.transpose(0, 1)
            v_log[b, first:prior[b]] = vr.transpose(0, 1)
        st.k_cache[l].copy_(kc)
        st.v_cache[l].copy_(vc)
        q = synth.randn_bf16((w.batch, kq, w.n_q_heads, D), g)
        k = synth.randn_bf16((w.batch, kq, Hkv, D), g)
        v = synth.randn_bf16((w.batch, kq, Hkv, D), g)
        for b in range(w.batch):
            k_log[b, prior[b]:prior[b] + kq] = k[b]
            v_log[b, prior[b]:prior[b] + kq] = v[b]
        out = torch.full((w.batch, kq, w.n_q_heads, D), float("nan"), dtype=torch.bfloat16, device=dev)
        st.decode_multi_layer(l, q.to(dev), k.to(dev), v.to(dev), out, seq_lens=lens, max_seq_len=T, workspace=ws)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        ref, _ = oracle.attention(to_bits(q), to_bits(k_log), to_bits(v_log), q_pos0=prior,
                                  n_keys=lens_l, rot_from=prior, window=W,
                                  rope_frac=t.rope_frac, theta=t.rope_theta, scale=t.scale)
        got = out.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
        assert_close(got, ref, what="verify layer %d (%s)" % (l, "global" if W == 0 else "local"))


SENTINEL = -7.5  # bf16-exact fill of pool rows no sequence owns


@pytest.mark.parametrize("T,keqv", [(4, False), (8, False), (16, False), (4, True)],
                         ids=["rows32", "rows64", "rows128", "keqv"])
def test_multi_paged_equals_contiguous(T, keqv):
    """A paged global cache (random page order, spare pages) gives the
    contiguous path's outputs bit for bit, holds the same rows at the same
    positions, and leaves pages no sequence owns untouched."""
    dev = torch.device("cuda")
    B, Hq, Hkv, D, ps, lens = 3, 32, 4, 512, 256, [2000, 37, 4100]
    g = synth.generator(360 + T + keqv)
    pps = (max(lens) + ps - 1) // ps + 1
    n_pages, cap = B * pps + 3, pps * ps
    kc = synth.randn_bf16((B, Hkv, cap, D), g)
    vc = kc if keqv else synth.randn_bf16((B, Hkv, cap, D), g)
    table = torch.tensor(np.random.default_rng(T).permutation(n_pages)[:B * pps].reshape(B, pps), dtype=torch.int32)

    def to_pool(c):
        pool = torch.full((n_pages, Hkv, ps, D), SENTINEL, dtype=torch.bfloat16)
        for b in range(B):
            for p in range(pps):
                pool[int(table[b, p])] = c[b, :, p * ps:(p + 1) * ps]
        return pool

    kp = to_pool(kc).to(dev)
    vp = kp if keqv else to_pool(vc).to(dev)
    kcd = kc.to(dev)
    vcd = kcd if keqv else vc.to(dev)
    q = synth.randn_bf16((B, T, Hq, D), g).to(dev)
    kn = synth.randn_bf16((B, T, Hkv, D), g).to(dev)
    vn = None if keqv else synth.randn_bf16((B, T, Hkv, D), g).to(dev)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    kw = dict(seq_lens=sl, max_seq_len=max(lens), rope_frac=0.25, rope_theta=1e6, scale=1.0 / math.sqrt(D),
              flags=native.GEMMA_F_KEQV if keqv else 0)
    o1 = torch.empty((B, T, Hq, D), dtype=torch.bfloat16, device=dev)
    o2 = torch.empty_like(o1)
    native.gemma_attn_decode_multi(q, kn, vn, kcd, None if keqv else vcd, window=0, out=o1, **kw)
    native.gemma_attn_decode_multi_paged(q, kn, vn, kp, None if keqv else vp, table.to(dev), out=o2, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    kp1, vp1 = kp.cpu(), vp.cpu()
    kc1, vc1 = kcd.cpu(), vcd.cpu()
    owned = torch.zeros(n_pages, dtype=torch.bool)
    owned[table.flatten().long()] = True
    for b in range(B):
        for p in range(pps):
            pg = int(table[b, p])
            assert torch.equal(kp1[pg].view(torch.int16), kc1[b, :, p * ps:(p + 1) * ps].view(torch.int16))
            assert torch.equal(vp1[pg].view(torch.int16), vc1[b, :, p * ps:(p + 1) * ps].view(torch.int16))
    assert (kp1[~owned] == SENTINEL).all() and (vp1[~owned] == SENTINEL).all()


@pytest.mark.parametrize("W", [0, 64], ids=["global", "local"])
def test_multi_bounded_wait_times_out_and_context_survives(oracle, W):
    """The tensor-core kernel's first copy is not issued (test hook): the
    MMA warp's bounded wait gives up, the softmax warps leave together, the
    status says GEMMA_ERR_DEVICE_TIMEOUT, and the next call on the same
    context is correct."""
    native.gemma_attn_set_wait_limit(20_000_000)  # 20 ms
    try:
        native.gemma_attn_debug_drop_next_copy(True)
        run_multi_case(oracle, lens=[700, 300], T=4, Hq=8, Hkv=1 if W == 0 else 4, D=512 if W == 0 else 256, W=W,
                       frac=0.25 if W == 0 else 1.0, theta=1e6 if W == 0 else 1e4, seed=371, expect_status=True)
    finally:
        native.gemma_attn_set_wait_limit(0)
    run_multi_case(oracle, lens=[700, 300], T=4, Hq=8, Hkv=1 if W == 0 else 4, D=512 if W == 0 else 256, W=W,
                   frac=0.25 if W == 0 else 1.0, theta=1e6 if W == 0 else 1e4, seed=372)


def test_multi_31b_b64_k4_sampled(oracle):
    """The benchmarked multi-token block at full size (B64, KV lengths
    U[4096,131072], 4 new tokens, 5 local + 1 global layer), as bench.py
    runs it: sampled sequences (the shortest, the longest and two seeded
    others; rows are independent) of every layer against the oracle over the
    cache as it was plus the new tokens."""
    from hybrid_local_global_b200.workloads import WORKLOADS
    w = WORKLOADS["31b_verify_b64_k4"]
    T = w.tokens
    dev = torch.device("cuda")
    st = AttentionStack(w, dev)
    lens_cpu = synth.decode_lengths(w.batch, w.len_lo, w.len_hi, seed=w.seed)
    lens = lens_cpu.to(dev)
    max_len = int(lens_cpu.max())
    g = synth.generator(w.seed, "cuda")
    for l in range(st.n_layers):
        synth.fill_randn_bf16_(st.k_cache[l], g)
        synth.fill_randn_bf16_(st.v_cache[l], g)
    ws = torch.empty(st.decode_multi_workspace_bytes(T, max_len), dtype=torch.uint8, device=dev)
    rng = np.random.default_rng(w.seed)
    pick = set(rng.choice(w.batch, size=2, replace=False).tolist())
    pick |= {int(lens_cpu.argmin()), int(lens_cpu.argmax())}
    for l in range(st.n_layers):
        t = st.layer_type(l)
        D, Hkv, W = t.head_dim, t.n_kv_heads, t.window
        q = synth.randn_bf16((w.batch, T, w.n_q_heads, D), g, "cuda")
        kn = synth.randn_bf16((w.batch, T, Hkv, D), g, "cuda")
        vn = synth.randn_bf16((w.batch, T, Hkv, D), g, "cuda")
        snaps = {}
        for b in pick:
            n = int(lens_cpu[b]) - T  # cached positions before the new tokens
            if W:
                first = max(0, n - W)
                slots = torch.tensor([p % W for p in range(first, n)], dtype=torch.long, device=dev)
                snaps[b] = (first, st.k_cache[l][b].index_select(1, slots).cpu(),
                            st.v_cache[l][b].index_select(1, slots).cpu())
            else:
                snaps[b] = (0, st.k_cache[l][b, :, :n].cpu(), st.v_cache[l][b, :, :n].cpu())
        out = torch.empty_like(q)
        st.decode_multi_layer(l, q, kn, vn, out, seq_lens=lens, max_seq_len=max_len, workspace=ws)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        for b in sorted(pick):
            L = int(lens_cpu[b])
            first, kc_b, vc_b = snaps[b]
            k_log = torch.zeros((1, L, Hkv, D), dtype=torch.bfloat16)
            v_log = torch.zeros_like(k_log)
            k_log[0, first:L - T] = kc_b.transpose(0, 1)
            v_log[0, first:L - T] = vc_b.transpose(0, 1)
            k_log[0, L - T:] = kn[b].cpu()
            v_log[0, L - T:] = vn[b].cpu()
            ref, _ = oracle.attention(to_bits(q[b:b + 1].cpu()), to_bits(k_log), to_bits(v_log), q_pos0=L - T,
                                      n_keys=L, rot_from=L - T, window=W, rope_frac=t.rope_frac,
                                      theta=t.rope_theta, scale=t.scale)
            got = out[b:b + 1].float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
            assert_close(got, ref, what="31b_verify_b64_k4 layer %d b=%d L=%d" % (l, b, L))
        del snaps
