"""GPU parity of the batched decode path (append + split-K attention + combine)
against the fp64 oracle, through the C ABI; ring-buffer slots, KV sharing,
the device range check and the bounded-wait timeout path."""
import math

import numpy as np
import pytest
import torch

from hybrid_local_global_b200 import native, synth
from hybrid_local_global_b200.stack import AttentionStack
from hybrid_local_global_b200.workloads import WORKLOADS

from gpu_util import assert_close, assert_close_to_model, assert_rotated_bf16, rotate_round, to_bits

pytestmark = pytest.mark.gpu


def logical_kv(kc, vc, length, window, k_new=None, v_new=None):
    """Cache [Hkv, cap, D] of one sequence -> keys/values in position order
    0..length-1 ([T, Hkv, D]); positions the ring no longer holds are zero
    (they are outside the window). The new token goes at position length-1."""
    Hkv, cap, D = kc.shape
    k = torch.zeros((length, Hkv, D), dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    first = max(0, length - window) if window else 0
    for p in range(first, length - 1):
        slot = p % window if window else p
        k[p] = kc[:, slot]
        v[p] = vc[:, slot]
    if k_new is not None:
        k[length - 1] = k_new
        v[length - 1] = v_new
    return k, v


def fill_cache_for_lengths(kc, vc, lens, window, g):
    """Random already-rotated K/V for positions < len-1 at their slots."""
    B = kc.shape[0]
    for b in range(B):
        n = lens[b] - 1
        if n <= 0:
            continue
        if window:
            first = max(0, n - window)
            for p in range(first, n):
                kc[b, :, p % window] = synth.randn_bf16((kc.shape[1], kc.shape[3]), g)
                vc[b, :, p % window] = synth.randn_bf16((kc.shape[1], kc.shape[3]), g)
        else:
            kc[b, :, :n] = synth.randn_bf16((kc.shape[1], n, kc.shape[3]), g)
            vc[b, :, :n] = synth.randn_bf16((kc.shape[1], n, kc.shape[3]), g)


def run_decode_case(oracle, *, lens, Hq, Hkv, D, W, frac, theta, seed, q_scale=1.0,
                    tol=(2e-2, 2e-3), shared=False, keqv=False):
    dev = torch.device("cuda")
    B = len(lens)
    g = synth.generator(seed)
    max_len = max(lens)
    cap = W if W else max_len + 16
    kc = torch.zeros((B, Hkv, cap, D), dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    fill_cache_for_lengths(kc, vc, lens, W, g)
    q = synth.randn_bf16((B, Hq, D), g, scale=q_scale)
    kn = synth.randn_bf16((B, Hkv, D), g)
    vn = synth.randn_bf16((B, Hkv, D), g)
    if shared:
        # the new token's K/V are already in the (source layer's) cache, rotated
        for b in range(B):
            p = lens[b] - 1
            slot = p % W if W else p
            kc[b, :, slot] = kn[b]
            vc[b, :, slot] = vn[b]
    if keqv:
        vc, vn = kc, kn  # K = V: one cache; the oracle takes the values from the keys
    kcd = kc.to(dev)
    vcd = kcd if keqv else vc.to(dev)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    flags = (native.GEMMA_F_SHARED if shared else 0) | (native.GEMMA_F_KEQV if keqv else 0)
    native.gemma_attn_decode(q.to(dev), None if shared else kn.to(dev),
                             None if (shared or keqv) else vn.to(dev), kcd, None if keqv else vcd,
                             seq_lens=sl, max_seq_len=max_len, window=W, rope_frac=frac,
                             rope_theta=theta, scale=scale, out=out, flags=flags)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    kc1, vc1 = kcd.cpu(), vcd.cpu()
    for b in range(B):
        L = lens[b]
        kl, vl = logical_kv(kc[b], vc[b], L, W, kn[b], vn[b])
        ref, _ = oracle.attention(to_bits(q[b].reshape(1, 1, Hq, D)), to_bits(kl[None]),
                                  None if keqv else to_bits(vl[None]),
                                  q_pos0=L - 1, n_keys=L, rot_from=L if shared else L - 1, window=W,
                                  rope_frac=frac, theta=theta, scale=scale)
        got = out[b].float().cpu().double().numpy()
        if tol is not None:
            assert_close(got, ref, *tol, what="decode b=%d len=%d" % (b, L))
        slot = (L - 1) % W if W else L - 1
        if shared:
            assert torch.equal(kc1[b], kc[b]) and torch.equal(vc1[b], vc[b])
        else:
            if not keqv:
                assert torch.equal(vc1[b, :, slot], vn[b])
            for h in range(Hkv):
                exp = torch.from_numpy(oracle.rope_bf16(to_bits(kn[b, h]), L - 1, frac, theta)).to(torch.bfloat16)
                assert_rotated_bf16(kc1[b, h, slot], exp, kn[b, h], "new K slot")
            other = torch.ones(cap, dtype=torch.bool)
            other[slot] = False
            assert torch.equal(kc1[b][:, other], kc[b][:, other])
    return out, q, kn, vn, kc, vc


CASES = [
    dict(lens=[1, 37, 300], Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=201),
    dict(lens=[1, 5, 64, 65, 1000], Hq=8, Hkv=4, D=256, W=64, frac=1.0, theta=1e4, seed=202),
    dict(lens=[4097, 2], Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6, seed=203),
    dict(lens=[3000], Hq=32, Hkv=16, D=256, W=1024, frac=1.0, theta=1e4, seed=204),
    dict(lens=[17, 16, 15], Hq=2, Hkv=2, D=256, W=16, frac=1.0, theta=1e4, seed=205),
    dict(lens=[7777, 123], Hq=16, Hkv=2, D=512, W=0, frac=0.25, theta=1e6, seed=206),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "L%s-H%d-%dD%dW%d" % (
    "_".join(map(str, c["lens"])), c["Hq"], c["Hkv"], c["D"], c["W"]))
def test_decode_small(oracle, case):
    run_decode_case(oracle, **case)


def test_decode_shared_layer(oracle):
    run_decode_case(oracle, lens=[900, 33], Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=207,
                    shared=True)
    run_decode_case(oracle, lens=[900, 33], Hq=8, Hkv=4, D=256, W=64, frac=1.0, theta=1e4, seed=208,
                    shared=True)


@pytest.mark.parametrize("case", [
    dict(lens=[1, 37, 300, 2049], Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=211),
    dict(lens=[4097, 2], Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6, seed=212),
    dict(lens=[130, 17], Hq=4, Hkv=2, D=256, W=0, frac=1.0, theta=1e4, seed=213),
], ids=["Hq8", "Hq32", "D256"])
def test_decode_k_equals_v(oracle, case):
    """K = V (GEMMA_F_KEQV): only the key is appended and the rotated keys in
    the cache serve as values; the oracle takes its values from the keys."""
    run_decode_case(oracle, keqv=True, **case)
    run_decode_case(oracle, keqv=True, shared=True, **dict(case, seed=case["seed"] + 100))


def test_decode_peaky(oracle):
    """Queries x8 (near one-hot attention). As in the prefill peaky test, the
    GPU is held to the exact attention of its rounded operands (decode
    rounds the rotated q and the new k to bf16) within the bound of its own
    bf16 roundings, and to the exact oracle within that model's error plus
    the same bound."""
    lens, Hq, Hkv, D, frac, theta, seed = [5000, 700], 8, 1, 512, 0.25, 1e6, 209
    res = run_decode_case(oracle, lens=lens, Hq=Hq, Hkv=Hkv, D=D, W=0, frac=frac, theta=theta, seed=seed,
                          q_scale=8.0, tol=None)
    out, q, kn, vn, kc, vc = res
    scale = 1.0 / math.sqrt(D)
    for b, L in enumerate(lens):
        kl, vl = logical_kv(kc[b], vc[b], L, 0, kn[b], vn[b])
        qb = q[b].reshape(1, 1, Hq, D)
        exact, _ = oracle.attention(to_bits(qb), to_bits(kl[None]), to_bits(vl[None]), q_pos0=L - 1, n_keys=L,
                                    rot_from=L - 1, window=0, rope_frac=frac, theta=theta, scale=scale)
        qr = rotate_round(oracle, qb, [L - 1], frac, theta)
        klr = kl.clone()
        klr[L - 1] = rotate_round(oracle, kn[b].reshape(1, 1, Hkv, D), [L - 1], frac, theta)[0, 0]
        model, _ = oracle.attention(to_bits(qr), to_bits(klr[None]), to_bits(vl[None]), q_pos0=L - 1, n_keys=L,
                                    rot_from=L, window=0, rope_frac=0.0, theta=theta, scale=scale)
        got = out[b].float().cpu().double().numpy()
        assert_close_to_model(got, model, exact, float(vl.float().abs().max()), "decode peaky b=%d" % b)


def test_decode_range_check_reports_status():
    dev = torch.device("cuda")
    B, Hq, Hkv, D = 2, 8, 1, 512
    kc = torch.zeros((B, Hkv, 64, D), dtype=torch.bfloat16, device=dev)
    q = torch.zeros((B, Hq, D), dtype=torch.bfloat16, device=dev)
    kn = torch.zeros((B, Hkv, D), dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(q)
    sl = torch.tensor([10, 99], dtype=torch.int32, device=dev)  # 99 > max_seq_len
    native.gemma_attn_decode(q, kn, kn.clone(), kc, kc.clone(), seq_lens=sl, max_seq_len=64, window=0,
                             rope_frac=0.25, rope_theta=1e6, scale=0.05, out=out)
    assert native.gemma_attn_sync_status() == native.GEMMA_ERR_DEVICE_RANGE
    assert native.gemma_attn_sync_status() == 0  # read clears it


def test_decode_bounded_wait_times_out_and_context_survives(oracle):
    """A barrier nothing completes (the first copy is not issued): the bounded
    wait gives up after its deadline, the status says so, and the next call
    on the same context is correct."""
    native.gemma_attn_set_wait_limit(20_000_000)  # 20 ms
    try:
        native.gemma_attn_debug_drop_next_copy(True)
        dev = torch.device("cuda")
        B, Hq, Hkv, D, L = 1, 8, 1, 512, 2000
        g = synth.generator(11, "cuda")
        kc = synth.randn_bf16((B, Hkv, L, D), g, "cuda")
        vc = synth.randn_bf16((B, Hkv, L, D), g, "cuda")
        q = synth.randn_bf16((B, Hq, D), g, "cuda")
        kn = synth.randn_bf16((B, Hkv, D), g, "cuda")
        vn = synth.randn_bf16((B, Hkv, D), g, "cuda")
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
        sl = torch.tensor([L], dtype=torch.int32, device=dev)
        kw = dict(seq_lens=sl, max_seq_len=L, window=0, rope_frac=0.25, rope_theta=1e6, scale=0.05, out=out)
        native.gemma_attn_decode(q, kn, vn, kc, vc, **kw)
        assert native.gemma_attn_sync_status() == native.GEMMA_ERR_DEVICE_TIMEOUT
    finally:
        native.gemma_attn_set_wait_limit(0)
    native.gemma_attn_decode(q, kn, vn, kc, vc, **kw)
    assert native.gemma_attn_sync_status() == 0
    kl = kc[0].transpose(0, 1).cpu()
    vl = vc[0].transpose(0, 1).cpu()
    ref, _ = oracle.attention(to_bits(q.cpu().reshape(1, 1, Hq, D)), to_bits(kl[None]), to_bits(vl[None]),
                              q_pos0=L - 1, n_keys=L, rot_from=L, window=0, rope_frac=0.25, theta=1e6,
                              scale=0.05)
    assert_close(out[0].float().cpu().double().numpy(), ref, what="after timeout")


# --------------------------------------------------------------------------- full-size workloads
def _decode_workload(oracle, name, n_sample):
    w = WORKLOADS[name]
    dev = torch.device("cuda")
    st = AttentionStack(w, dev)
    if w.len_lo == w.len_hi:
        lens_cpu = torch.full((w.batch,), w.len_hi, dtype=torch.int32)
    else:
        lens_cpu = synth.decode_lengths(w.batch, w.len_lo, w.len_hi, seed=w.seed)
    lens = lens_cpu.to(dev)
    max_len = int(lens_cpu.max())
    g = synth.generator(w.seed, "cuda")
    owned = set()
    for l in range(st.n_layers):
        if not st.is_shared(l) and st.k_cache[l].data_ptr() not in owned:
            owned.add(st.k_cache[l].data_ptr())
            synth.fill_randn_bf16_(st.k_cache[l], g)
            synth.fill_randn_bf16_(st.v_cache[l], g)
    ws = torch.empty(st.decode_workspace_bytes(max_len), dtype=torch.uint8, device=dev)
    rng = np.random.default_rng(w.seed)
    pick = set(rng.choice(w.batch, size=min(n_sample, w.batch), replace=False).tolist())
    pick |= {int(lens_cpu.argmin()), int(lens_cpu.argmax())}
    for l in range(st.n_layers):
        t = st.layer_type(l)
        D, Hkv = t.head_dim, t.n_kv_heads
        q = synth.randn_bf16((w.batch, w.n_q_heads, D), g, "cuda")
        kn = synth.randn_bf16((w.batch, Hkv, D), g, "cuda")
        vn = synth.randn_bf16((w.batch, Hkv, D), g, "cuda")
        shared = st.is_shared(l)
        # snapshot of the picked sequences' caches as the kernel will see them
        n_keep = {b: min(st.k_cache[l].shape[2], int(lens_cpu[b])) for b in pick}
        snaps = {b: (st.k_cache[l][b, :, :n_keep[b]].cpu(), st.v_cache[l][b, :, :n_keep[b]].cpu())
                 for b in pick}
        out = torch.empty((w.batch, w.n_q_heads, D), dtype=torch.bfloat16, device=dev)
        st.decode_layer(l, q, kn, vn, out, seq_lens=lens, max_seq_len=max_len, workspace=ws)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        for b in sorted(pick):
            L = int(lens_cpu[b])
            kc_b, vc_b = snaps[b]
            if shared:
                # the source layer already appended this step's token
                kl, vl = logical_kv(kc_b, vc_b, L, t.window)
                slot = (L - 1) % t.window if t.window else L - 1
                kl[L - 1] = kc_b[:, slot]
                vl[L - 1] = vc_b[:, slot]
                rot_from = L
            else:
                kl, vl = logical_kv(kc_b, vc_b, L, t.window, kn[b].cpu(), vn[b].cpu())
                rot_from = L - 1
            ref, _ = oracle.attention(to_bits(q[b].cpu().reshape(1, 1, w.n_q_heads, D)), to_bits(kl[None]),
                                      None if st.keqv(l) else to_bits(vl[None]),
                                      q_pos0=L - 1, n_keys=L, rot_from=rot_from,
                                      window=t.window, rope_frac=t.rope_frac, theta=t.rope_theta,
                                      scale=t.scale)
            assert_close(out[b].float().cpu().double().numpy(), ref, what="%s layer %d b=%d" % (name, l, b))
        del snaps


def test_decode_31b_b64(oracle):
    _decode_workload(oracle, "31b_decode_b64", n_sample=8)


def test_decode_31b_12_layers_two_shared(oracle):
    """The 12-layer form of the 31B-shaped decode block: layer 10 reads layer
    9's ring and layer 11 reads layer 5's global cache (latest earlier layer
    of the same type), and the owned cache bytes match the oracle's byte
    counter for that stack."""
    w = WORKLOADS["31b_decode_b16_12l_shared"]
    is_global, src = native.gemma_layer_schedule(w.n_layers, w.ratio, w.n_shared)
    assert [src[l] for l in (10, 11)] == [9, 5]
    assert [is_global[l] for l in (5, 9, 10, 11)] == [True, False, False, True]
    st = AttentionStack(w, torch.device("cuda"))
    expect = oracle.stack_cache_bytes(w.n_layers, w.ratio, w.n_shared, w.batch, local_kv_heads=16,
                                      local_head_dim=256, local_capacity=1024, global_kv_heads=4,
                                      global_head_dim=512, global_capacity=w.len_hi, which="all")
    assert st.owned_cache_bytes() == expect
    del st
    torch.cuda.empty_cache()
    _decode_workload(oracle, "31b_decode_b16_12l_shared", n_sample=3)


def test_decode_global_256k_k_equals_v(oracle):
    _decode_workload(oracle, "global_decode_256k_keqv", n_sample=1)


def test_decode_global_256k(oracle):
    _decode_workload(oracle, "global_decode_256k", n_sample=1)
