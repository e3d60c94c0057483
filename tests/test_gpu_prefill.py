"""GPU parity of the prefill path (RoPE + cache write + attention) against the
fp64 oracle, through the C ABI. Small cases compare every row; the
full-size workloads compare sampled rows (every attention row is
independent, so sampled rows are exact)."""
import math

import numpy as np
import pytest
import torch

from hybrid_local_global_b200 import native, synth
from hybrid_local_global_b200.stack import AttentionStack
from hybrid_local_global_b200.workloads import WORKLOADS

from gpu_util import (assert_close, assert_close_to_model, assert_rotated_bf16, gather_rows,
                      prefill_query_multiplier, rotate_round, sample_rows, to_bits)

pytestmark = pytest.mark.gpu


def _expected_rotated_bf16(oracle, k_bits_row, pos, frac, theta):
    y = oracle.rope_bf16(k_bits_row, pos, frac, theta)
    return torch.from_numpy(y).to(torch.bfloat16)


def run_prefill_case(oracle, *, B, S, Hq, Hkv, D, W, frac, theta, seed, prior=None, q_scale=1.0,
                     k_scale=1.0, tol=(2e-2, 2e-3), check_cache=True, check_lse=True, cache_fill=0.0,
                     keqv=False):
    dev = torch.device("cuda")
    g = synth.generator(seed)
    q = synth.randn_bf16((B, S, Hq, D), g, scale=q_scale)
    k = synth.randn_bf16((B, S, Hkv, D), g, scale=k_scale)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    prior = list(prior) if prior else [0] * B
    T = max(prior) + S
    cap = W if W else T + 16
    # slots past the sequence hold whatever the caller left there: cache_fill
    # = nan checks that no such value reaches an output
    kc = torch.full((B, Hkv, cap, D), cache_fill, dtype=torch.bfloat16)
    vc = torch.full((B, Hkv, cap, D), cache_fill, dtype=torch.bfloat16)
    for b in range(B):
        if prior[b]:
            kc[b, :, :prior[b]] = synth.randn_bf16((Hkv, prior[b], D), g)
            vc[b, :, :prior[b]] = synth.randn_bf16((Hkv, prior[b], D), g)
    if keqv:
        vc = kc  # K = V: one cache, and the values are the cached (rotated) keys
    kc0, vc0 = kc.clone(), vc.clone()
    qd, kd, vd, kcd = (x.to(dev) for x in (q, k, v, kc))
    vcd = kcd if keqv else vc.to(dev)
    out = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev)
    lens = torch.tensor(prior, dtype=torch.int32, device=dev) if any(prior) else None
    scale = 1.0 / math.sqrt(D)
    native.gemma_attn_prefill(qd, kd, None if keqv else vd, kcd, None if keqv else vcd, window=W,
                              rope_frac=frac, rope_theta=theta, scale=scale, out=out,
                              seq_lens_before=lens, lse=lse,
                              flags=native.GEMMA_F_KEQV if keqv else 0)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()

    # oracle on logical K/V: cached prefix (already rotated) + the new keys
    k_log = torch.zeros((B, T, Hkv, D), dtype=torch.bfloat16)
    v_log = torch.zeros((B, T, Hkv, D), dtype=torch.bfloat16)
    for b in range(B):
        k_log[b, :prior[b]] = kc0[b, :, :prior[b]].transpose(0, 1)
        v_log[b, :prior[b]] = vc0[b, :, :prior[b]].transpose(0, 1)
        k_log[b, prior[b]:prior[b] + S] = k[b]
        v_log[b, prior[b]:prior[b] + S] = v[b]
    ref, ref_lse = oracle.attention(to_bits(q), to_bits(k_log), None if keqv else to_bits(v_log), q_pos0=prior,
                                    n_keys=[p + S for p in prior], rot_from=prior, window=W,
                                    rope_frac=frac, theta=theta, scale=scale)
    got = out.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)  # (b, h, i) rows
    if tol is not None:
        assert_close(got, ref, *tol, what="prefill out")
    if check_lse:
        gl = lse.cpu().double().numpy().reshape(-1)
        assert np.abs(gl - ref_lse).max() < 2e-2 * max(1.0, q_scale)

    if check_cache:
        kc1, vc1 = kcd.cpu(), vcd.cpu()
        n_same = n_all = 0
        for b in range(B):
            for s in range(S):
                pos = prior[b] + s
                if W and s < S - W:
                    continue
                slot = pos % W if W else pos
                if not keqv:
                    assert torch.equal(vc1[b, :, slot], v[b, s]), "V slot %d" % slot
                for h in range(Hkv):
                    exp = _expected_rotated_bf16(oracle, to_bits(k[b, s, h]), pos, frac, theta)
                    got_k = kc1[b, h, slot]
                    if frac == 0.0:
                        assert torch.equal(got_k, k[b, s, h])
                    else:
                        assert_rotated_bf16(got_k, exp, k[b, s, h], "K slot %d" % slot)
                        n_same += int((got_k == exp).sum())
                        n_all += exp.numel()
        if n_all:
            assert n_same >= 0.98 * n_all, "only %d of %d rotated K values bit-identical" % (n_same, n_all)
        if W == 0:
            # untouched slots keep their bytes
            bits = lambda t: t.view(torch.int16)
            for b in range(B):
                for c1, c0 in ((kc1, kc0), (vc1, vc0)):
                    assert torch.equal(bits(c1[b, :, :prior[b]]), bits(c0[b, :, :prior[b]]))
                    assert torch.equal(bits(c1[b, :, prior[b] + S:]), bits(c0[b, :, prior[b] + S:]))
    return out


CASES = [
    dict(B=2, S=1, Hq=8, Hkv=4, D=256, W=512, frac=1.0, theta=1e4, seed=101),
    dict(B=2, S=200, Hq=4, Hkv=2, D=256, W=48, frac=1.0, theta=1e4, seed=102),
    dict(B=1, S=300, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=103),
    dict(B=2, S=130, Hq=2, Hkv=2, D=256, W=0, frac=0.25, theta=1e6, seed=104),
    dict(B=1, S=257, Hq=8, Hkv=4, D=512, W=64, frac=1.0, theta=1e4, seed=105),
    dict(B=1, S=96, Hq=4, Hkv=4, D=256, W=16, frac=0.0, theta=1e4, seed=106),
    dict(B=2, S=100, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=107, prior=[37, 250]),
    dict(B=1, S=64, Hq=16, Hkv=2, D=256, W=0, frac=1.0, theta=1e4, seed=108, prior=[1000]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dS%dH%d-%dD%dW%d%s" % (
    c["B"], c["S"], c["Hq"], c["Hkv"], c["D"], c["W"], "P" if c.get("prior") else ""))
def test_prefill_small(oracle, case):
    run_prefill_case(oracle, **case)


PAIR_CASES = [
    dict(B=1, S=300, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=111, cache_fill=float("nan")),
    dict(B=2, S=100, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=112, prior=[37, 250],
         cache_fill=float("nan")),
    dict(B=1, S=257, Hq=8, Hkv=4, D=512, W=64, frac=1.0, theta=1e4, seed=113),
    dict(B=2, S=383, Hq=4, Hkv=2, D=256, W=0, frac=0.25, theta=1e6, seed=114, cache_fill=float("nan")),
    dict(B=1, S=520, Hq=8, Hkv=4, D=256, W=128, frac=1.0, theta=1e4, seed=115),
    dict(B=1, S=1, Hq=8, Hkv=4, D=256, W=512, frac=1.0, theta=1e4, seed=116),
]


@pytest.mark.parametrize("kernel", ["single", "pair", "hpair"])
@pytest.mark.parametrize("case", PAIR_CASES, ids=lambda c: "B%dS%dH%d-%dD%dW%d%s%s" % (
    c["B"], c["S"], c["Hq"], c["Hkv"], c["D"], c["W"], "P" if c.get("prior") else "",
    "nan" if c.get("cache_fill") else ""))
def test_prefill_each_kernel(oracle, monkeypatch, kernel, case):
    """Every attention kernel (one query tile per CTA; two query tiles, or two
    q heads of one KV head, per CTA pair on cta_group::2 MMAs) on ragged
    lengths, odd tile counts, a cached prefix, and caches whose unused slots
    hold nan (the key tile that crosses the sequence end must not let them
    reach an output)."""
    monkeypatch.setenv("GEMMA_PREFILL_KERNEL", kernel)
    run_prefill_case(oracle, **case)


WAVE_CASES = [
    # more work items than SMs: several waves of CTAs or clusters
    dict(B=2, S=1200, Hq=8, Hkv=4, D=256, W=128, frac=1.0, theta=1e4, seed=141),
    dict(B=1, S=600, Hq=32, Hkv=4, D=256, W=0, frac=0.25, theta=1e6, seed=142, cache_fill=float("nan")),
    dict(B=3, S=300, Hq=24, Hkv=12, D=256, W=0, frac=1.0, theta=1e4, seed=143, prior=[0, 129, 700]),
]


@pytest.mark.parametrize("kernel", ["single", "hpair"])
@pytest.mark.parametrize("case", WAVE_CASES, ids=["W128", "global", "prior"])
def test_prefill_more_tiles_than_sms(oracle, monkeypatch, kernel, case):
    """More (query tile, head) items than SMs, so CTAs and CTA pairs run in
    several waves with unequal key ranges."""
    monkeypatch.setenv("GEMMA_PREFILL_KERNEL", kernel)
    run_prefill_case(oracle, **case)


KEQV_CASES = [
    dict(B=1, S=300, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=121, cache_fill=float("nan")),
    dict(B=2, S=100, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=122, prior=[37, 250]),
    dict(B=1, S=200, Hq=4, Hkv=2, D=256, W=0, frac=1.0, theta=1e4, seed=123, cache_fill=float("nan")),
]


@pytest.mark.parametrize("kernel", ["single", "pair", "hpair"])
@pytest.mark.parametrize("case", KEQV_CASES, ids=["D512", "D512P", "D256"])
def test_prefill_k_equals_v(oracle, monkeypatch, kernel, case):
    """K = V (GEMMA_F_KEQV) on global layers: only the rotated keys are written
    and they serve as values; the oracle takes its values from the keys."""
    monkeypatch.setenv("GEMMA_PREFILL_KERNEL", kernel)
    run_prefill_case(oracle, keqv=True, **case)


def test_prefill_local_s1024_full(oracle):
    """Single local layer, B1 S1024 W512 Hq8 Hkv4 D256, full RoPE 1e4, every row."""
    run_prefill_case(oracle, B=1, S=1024, Hq=8, Hkv=4, D=256, W=512, frac=1.0, theta=1e4, seed=0)


@pytest.mark.parametrize("kernel", ["single", "pair", "hpair"])
@pytest.mark.parametrize("D,W,Hkv,frac,theta", [(256, 512, 4, 1.0, 1e4), (512, 0, 1, 0.25, 1e6)])
def test_prefill_peaky(oracle, monkeypatch, kernel, D, W, Hkv, frac, theta):
    """Queries x8: near one-hot attention, so a wrong mask boundary or a
    missing key cannot hide behind near-uniform weights (such a bug moves an
    output by O(1)).

    The logits grow 8x, and with them the effect of rounding the rotated
    operands to bf16, which the GPU path does by design (q times scale *
    log2 e, and k, each rounded once). So the GPU is held to the exact
    attention of those rounded operands (the oracle on operands it rotated,
    rounded the same way, with RoPE off) within the bound its own bf16
    roundings of P and of the output allow, and to the exact oracle within
    that model's error plus the same bound (the triangle inequality): no
    fixed multiple of the parity tolerance."""
    monkeypatch.setenv("GEMMA_PREFILL_KERNEL", kernel)
    B, S, Hq, seed = 1, 640, 8, 7
    out = run_prefill_case(oracle, B=B, S=S, Hq=Hq, Hkv=Hkv, D=D, W=W, frac=frac, theta=theta, seed=seed,
                           q_scale=8.0, tol=None, check_cache=False, check_lse=False)
    g = synth.generator(seed)  # the inputs run_prefill_case drew
    q = synth.randn_bf16((B, S, Hq, D), g, scale=8.0)
    k = synth.randn_bf16((B, S, Hkv, D), g)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    assert_matches_rounded_model(oracle, out, q, k, v, W, frac, theta, "prefill peaky")


def assert_matches_rounded_model(oracle, out, q, k, v, W, frac, theta, what):
    """GPU output against the exact attention of the operands rounded as the
    prefill kernels round them (parity tolerance), and against the exact
    oracle within that model's error plus the tolerance."""
    B, S, Hq, D = q.shape
    scale = 1.0 / math.sqrt(D)
    c = prefill_query_multiplier(scale)
    qr = rotate_round(oracle, q, [0] * B, frac, theta, mult=c)
    kr = rotate_round(oracle, k, [0] * B, frac, theta)
    model, _ = oracle.attention(to_bits(qr), to_bits(kr), to_bits(v), q_pos0=0, n_keys=S, rot_from=S, window=W,
                                rope_frac=0.0, theta=theta, scale=scale / c)
    exact, _ = oracle.attention(to_bits(q), to_bits(k), to_bits(v), q_pos0=0, n_keys=S, rot_from=0, window=W,
                                rope_frac=frac, theta=theta, scale=scale)
    got = out.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
    assert_close_to_model(got, model, exact, float(v.float().abs().max()), what)


@pytest.mark.parametrize("kernel", ["single", "hpair"])
def test_prefill_growing_logits(oracle, monkeypatch, kernel):
    """Keys scaled up along the sequence (x1 at the start to x3 at the end)
    and queries x3: every later key tile holds larger logits, so the running
    row maximum keeps moving and O is rescaled in TMEM several times per
    row."""
    monkeypatch.setenv("GEMMA_PREFILL_KERNEL", kernel)
    B, S, Hq, Hkv, D, frac, theta = 2, 1000, 8, 1, 512, 0.25, 1e6
    dev = torch.device("cuda")
    g = synth.generator(151)
    q = synth.randn_bf16((B, S, Hq, D), g, scale=3.0)
    k0 = synth.randn_bf16((B, S, Hkv, D), g)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    ramp = (1.0 + 2.0 * torch.arange(S, dtype=torch.float32) / S).view(1, S, 1, 1)
    k = (k0.float() * ramp).to(torch.bfloat16)
    kc = torch.zeros((B, Hkv, S, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    out = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    native.gemma_attn_prefill(q.to(dev), k.to(dev), v.to(dev), kc, vc, window=0, rope_frac=frac, rope_theta=theta,
                              scale=1.0 / math.sqrt(D), out=out)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert_matches_rounded_model(oracle, out, q, k, v, 0, frac, theta, "growing logits")


def test_visible_ranges_bit_exact(oracle):
    dev = torch.device("cuda")
    for B, S, W, prior in ((1, 1024, 512, None), (2, 333, 48, None), (2, 100, 0, [0, 4095]),
                           (1, 4096, 1024, None), (1, 37, 16, None)):
        r = torch.full((B, S, 3), -7, dtype=torch.int32, device=dev)
        lens = torch.tensor(prior, dtype=torch.int32, device=dev) if prior else None
        native.gemma_attn_visible_ranges(B, S, W, r, seq_lens_before=lens)
        assert native.gemma_attn_sync_status() == 0
        r = r.cpu().numpy()
        for b in range(B):
            p0 = prior[b] if prior else 0
            for i in range(S):
                lo, hi, cnt = oracle.visible_range(p0 + i, W, p0 + S)
                assert tuple(r[b, i]) == (lo, hi, cnt), (b, i)


def test_lse_counts_with_zero_queries(oracle):
    """Q = 0: every visible key weighs the same, so exp(lse) is the visible
    count; checks the kernel's per-row key set exactly."""
    dev = torch.device("cuda")
    for D, W, S, Hkv in ((256, 48, 300, 2), (512, 0, 257, 1)):
        B, Hq = 1, 8
        q = torch.zeros((B, S, Hq, D), dtype=torch.bfloat16, device=dev)
        g = synth.generator(5, "cuda")
        k = synth.randn_bf16((B, S, Hkv, D), g, "cuda")
        v = synth.randn_bf16((B, S, Hkv, D), g, "cuda")
        cap = W if W else S
        kc = torch.zeros((B, Hkv, cap, D), dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
        out = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
        native.gemma_attn_prefill(q, k, v, kc, vc, window=W, rope_frac=1.0, rope_theta=1e4,
                                  scale=0.1, out=out, lse=lse)
        assert native.gemma_attn_sync_status() == 0
        cnt = torch.exp(lse.double()).cpu().numpy()
        for i in range(S):
            want = oracle.visible_range(i, W, S)[2]
            assert np.all(np.rint(cnt[0, :, i]) == want) and np.abs(cnt[0, :, i] - want).max() < 1e-3 * want


def test_shared_global_layer_reads_source_and_writes_nothing(oracle):
    """A shared layer (GEMMA_F_SHARED, no k/v) attends over its source's cache
    and leaves every cache byte as it was."""
    dev = torch.device("cuda")
    B, S, Hq, Hkv, D = 1, 200, 8, 1, 512
    g = synth.generator(9)
    q0 = synth.randn_bf16((B, S, Hq, D), g)
    q1 = synth.randn_bf16((B, S, Hq, D), g)
    k = synth.randn_bf16((B, S, Hkv, D), g)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    kc = torch.zeros((B, Hkv, S, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    out0 = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=dev)
    out1 = torch.empty_like(out0)
    kw = dict(window=0, rope_frac=0.25, rope_theta=1e6, scale=1 / math.sqrt(D))
    native.gemma_attn_prefill(q0.to(dev), k.to(dev), v.to(dev), kc, vc, out=out0, **kw)
    assert native.gemma_attn_sync_status() == 0
    before = (kc.clone(), vc.clone())
    native.gemma_attn_prefill(q1.to(dev), None, None, kc, vc, out=out1, flags=native.GEMMA_F_SHARED, **kw)
    assert native.gemma_attn_sync_status() == 0
    assert torch.equal(kc, before[0]) and torch.equal(vc, before[1])
    ref, _ = oracle.attention(to_bits(q1), to_bits(k), to_bits(v), q_pos0=0, n_keys=S, rot_from=0,
                              window=0, rope_frac=0.25, theta=1e6, scale=1 / math.sqrt(D))
    got = out1.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
    assert_close(got, ref, what="shared layer")


# --------------------------------------------------------------------------- full-size workloads
def _run_block(oracle, name, n_random=256):
    w = WORKLOADS[name]
    dev = torch.device("cuda")
    st = AttentionStack(w, dev)
    g = synth.generator(w.seed, "cuda")
    ws = torch.empty(st.prefill_workspace_bytes(), dtype=torch.uint8, device=dev)
    lens = None
    if w.prior:
        lens = torch.full((w.batch,), w.prior, dtype=torch.int32, device=dev)
    results = []
    for l in range(st.n_layers):
        t = st.layer_type(l)
        q = synth.randn_bf16((w.batch, w.seq, w.n_q_heads, t.head_dim), g, "cuda")
        k = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, "cuda", scale=w.k_scale)
        v = synth.randn_bf16((w.batch, w.seq, t.n_kv_heads, t.head_dim), g, "cuda")
        prior_k = prior_v = None
        if w.prior:
            # cached context before the chunk: already-rotated keys
            synth.fill_randn_bf16_(st.k_cache[l][:, :, :w.prior], g)
            synth.fill_randn_bf16_(st.v_cache[l][:, :, :w.prior], g)
            prior_k = st.k_cache[l][:, :, :w.prior].clone()
            prior_v = st.v_cache[l][:, :, :w.prior].clone()
        out = torch.empty((w.batch, w.seq, w.n_q_heads, t.head_dim), dtype=torch.bfloat16, device=dev)
        st.prefill_layer(l, q, k, v, out, workspace=ws, seq_lens_before=lens)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        rows = sample_rows(w.batch, w.n_q_heads, w.seq, n_random, seed=1000 + l, window=t.window,
                           prior=w.prior)
        if w.prior:
            k_log = torch.cat([prior_k.transpose(1, 2), k], dim=1)
            v_log = torch.cat([prior_v.transpose(1, 2), v], dim=1)
            del prior_k, prior_v
        else:
            k_log, v_log = k, v
        ref, _ = oracle.attention(to_bits(q), to_bits(k_log), to_bits(v_log), q_pos0=w.prior,
                                  n_keys=w.prior + w.seq, rot_from=w.prior, window=t.window,
                                  rope_frac=t.rope_frac, theta=t.rope_theta, scale=t.scale, rows=rows)
        got = gather_rows(out, rows)
        results.append(assert_close(got, ref, what="%s layer %d" % (name, l)))
        del q, k, v, out, k_log, v_log
    return results


def test_prefill_e2b_block_s8192(oracle):
    _run_block(oracle, "e2b_block_s8192")


def test_prefill_31b_block_s32768(oracle):
    _run_block(oracle, "31b_block_s32768", n_random=128)


def test_prefill_global_chunk_256k(oracle):
    _run_block(oracle, "global_chunk_256k", n_random=48)


def test_prefill_from_host_matches_layer_by_layer():
    """AttentionStack.prefill_from_host (copies on their own streams,
    overlapped with the attention) gives bit-identical outputs to copying
    everything first and running the layers one by one."""
    from hybrid_local_global_b200.workloads import E2B_GLOBAL, E2B_LOCAL, Workload
    w = Workload("tiny_block", "prefill", batch=1, n_q_heads=8, n_layers=5, ratio=4,
                 local=E2B_LOCAL, global_=E2B_GLOBAL, seq=700, seed=9)
    dev = torch.device("cuda")
    st = AttentionStack(w, dev)
    g = synth.generator(9)
    host_in, host_out, bufs = [], [], []
    for l in range(st.n_layers):
        t = st.layer_type(l)
        shp_q = (w.batch, w.seq, w.n_q_heads, t.head_dim)
        shp_k = (w.batch, w.seq, t.n_kv_heads, t.head_dim)
        hin = tuple(synth.randn_bf16(s, g).pin_memory() for s in (shp_q, shp_k, shp_k))
        host_in.append(hin)
        host_out.append(torch.empty(shp_q, dtype=torch.bfloat16).pin_memory())
        bufs.append(tuple(torch.empty(x.shape, dtype=x.dtype, device=dev) for x in hin) +
                    (torch.empty(shp_q, dtype=torch.bfloat16, device=dev),))
    ws = torch.empty(st.prefill_workspace_bytes(), dtype=torch.uint8, device=dev)
    for _ in range(2):  # the second pass reuses the buffers of the first
        st.prefill_from_host(host_in, host_out, bufs, workspace=ws)
    torch.cuda.current_stream().synchronize()
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    ref = []
    for l, (hq, hk, hv) in enumerate(host_in):
        q, k, v = (x.to(dev) for x in (hq, hk, hv))
        out = torch.empty_like(q)
        st.prefill_layer(l, q, k, v, out, workspace=ws)
        ref.append(out.cpu())
    for l in range(st.n_layers):
        assert torch.equal(host_out[l].view(torch.int16), ref[l].view(torch.int16)), "layer %d" % l


def run_local_chunk_case(oracle, *, B, S, Hq, Hkv, D, W, prior, seed, frac=1.0, theta=1e4,
                         tol=(2e-2, 2e-3)):
    """A chunk of S tokens on a local layer after prior[b] cached tokens: the
    ring holds (rotated) keys and values of the last W cached positions; the
    chunk's queries attend to those and to the chunk, and the ring ends up
    holding the last W positions of cache + chunk."""
    dev = torch.device("cuda")
    g = synth.generator(seed)
    q = synth.randn_bf16((B, S, Hq, D), g)
    k = synth.randn_bf16((B, S, Hkv, D), g)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    kc = torch.full((B, Hkv, W, D), float("nan"), dtype=torch.bfloat16)
    vc = torch.full((B, Hkv, W, D), float("nan"), dtype=torch.bfloat16)
    T = max(prior) + S
    k_log = torch.zeros((B, T, Hkv, D), dtype=torch.bfloat16)
    v_log = torch.zeros((B, T, Hkv, D), dtype=torch.bfloat16)
    for b in range(B):
        for p in range(max(0, prior[b] - W), prior[b]):  # what the ring holds
            kr = synth.randn_bf16((Hkv, D), g)
            vr = synth.randn_bf16((Hkv, D), g)
            kc[b, :, p % W], vc[b, :, p % W] = kr, vr
            k_log[b, p], v_log[b, p] = kr, vr
        k_log[b, prior[b]:prior[b] + S] = k[b]
        v_log[b, prior[b]:prior[b] + S] = v[b]
    kcd, vcd = kc.to(dev), vc.to(dev)
    out = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lens = torch.tensor(prior, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    native.gemma_attn_prefill(q.to(dev), k.to(dev), v.to(dev), kcd, vcd, window=W, rope_frac=frac,
                              rope_theta=theta, scale=scale, out=out, seq_lens_before=lens)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    ref, _ = oracle.attention(to_bits(q), to_bits(k_log), to_bits(v_log), q_pos0=prior,
                              n_keys=[p + S for p in prior], rot_from=prior, window=W,
                              rope_frac=frac, theta=theta, scale=scale)
    got = out.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
    assert_close(got, ref, *tol, what="chunked local prefill")
    kc1, vc1 = kcd.cpu(), vcd.cpu()
    for b in range(B):
        end = prior[b] + S
        for p in range(max(0, end - W), end):
            slot = p % W
            if p >= prior[b]:
                s_ = p - prior[b]
                assert torch.equal(vc1[b, :, slot], v[b, s_]), "V slot %d" % slot
                for h in range(Hkv):
                    exp = torch.from_numpy(oracle.rope_bf16(to_bits(k[b, s_, h]), p, frac, theta)).to(torch.bfloat16)
                    assert_rotated_bf16(kc1[b, h, slot], exp, k[b, s_, h], "K slot %d" % slot)
            else:
                assert torch.equal(kc1[b, :, slot], kc[b, :, slot]) and torch.equal(vc1[b, :, slot], vc[b, :, slot])


@pytest.mark.parametrize("case", [
    dict(B=2, S=200, Hq=8, Hkv=4, D=256, W=512, prior=[700, 3], seed=131),
    dict(B=1, S=700, Hq=8, Hkv=4, D=256, W=512, prior=[1000], seed=132),   # chunk longer than the window
    dict(B=2, S=1, Hq=4, Hkv=2, D=256, W=64, prior=[64, 129], seed=133),   # one-token chunks
    dict(B=1, S=130, Hq=8, Hkv=4, D=512, W=128, prior=[257], seed=134, frac=0.25, theta=1e6),
    dict(B=2, S=400, Hq=24, Hkv=12, D=256, W=512, prior=[1000, 5], seed=135),  # more tiles than SMs
], ids=["S200", "S700", "S1", "D512", "H24"])
@pytest.mark.parametrize("kernel", ["single", "hpair"])
def test_prefill_local_chunk_after_cached_tokens(oracle, monkeypatch, kernel, case):
    monkeypatch.setenv("GEMMA_PREFILL_KERNEL", kernel)
    run_local_chunk_case(oracle, **case)


def test_multi_query_verify_chunk_across_layer_types(oracle):
    """Speculative verify / multi-query decode: k = 4 new tokens per sequence
    after a long cached context, through every layer of a 31B-shaped 6-layer
    stack (5 local with ring caches, 1 global). It is a small chunked
    prefill: each new token sees the cached context (window-limited on local
    layers) and the earlier new tokens (causal tail)."""
    from hybrid_local_global_b200.workloads import L31B_GLOBAL, L31B_LOCAL, Workload
    prior, kq = [3000, 700], 4
    w = Workload("verify_k4", "prefill", batch=2, n_q_heads=32, n_layers=6, ratio=5,
                 local=L31B_LOCAL, global_=L31B_GLOBAL, seq=kq, seed=17)
    dev = torch.device("cuda")
    st = AttentionStack(w, dev, global_capacity=max(prior) + kq)
    g = synth.generator(17)
    ws = torch.empty(st.prefill_workspace_bytes(), dtype=torch.uint8, device=dev)
    lens = torch.tensor(prior, dtype=torch.int32, device=dev)
    T = max(prior) + kq
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
        st.prefill_layer(l, q.to(dev), k.to(dev), v.to(dev), out, workspace=ws, seq_lens_before=lens)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        ref, _ = oracle.attention(to_bits(q), to_bits(k_log), to_bits(v_log), q_pos0=prior,
                                  n_keys=[p + kq for p in prior], rot_from=prior, window=W,
                                  rope_frac=t.rope_frac, theta=t.rope_theta, scale=t.scale)
        got = out.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
        assert_close(got, ref, what="verify layer %d (%s)" % (l, "global" if W == 0 else "local"))
