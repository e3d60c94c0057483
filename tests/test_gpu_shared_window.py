"""GPU parity of KV-shared local layers after cached tokens
(GEMMA_F_SOURCE_WINDOW): the source layer's chunk has replaced ring slots
that the chunk's earlier queries still see, so a sharing layer attends to
the K/V window its source's call left in the workspace. Through the C ABI
(bf16 and int8 rings, one and two sharers) and through the layer stack
(chunked prefill and multi-token decode of a 31B-shaped stack whose last
local layer shares), against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from hybrid_local_global_b200 import native, synth
from hybrid_local_global_b200.stack import AttentionStack
from hybrid_local_global_b200.workloads import L31B_GLOBAL, L31B_LOCAL, Workload

from gpu_util import assert_close, to_bits

pytestmark = pytest.mark.gpu


def ring_with_history(B, Hkv, W, D, prior, g):
    """A ring holding rotated keys / values of positions prior-W .. prior-1
    (NaN elsewhere) and the same rows in position order."""
    T = max(prior)
    kc = torch.full((B, Hkv, W, D), float("nan"), dtype=torch.bfloat16)
    vc = kc.clone()
    k_log = torch.zeros((B, T, Hkv, D), dtype=torch.bfloat16)
    v_log = torch.zeros_like(k_log)
    for b in range(B):
        for p in range(max(0, prior[b] - W), prior[b]):
            kr, vr = synth.randn_bf16((Hkv, D), g), synth.randn_bf16((Hkv, D), g)
            kc[b, :, p % W], vc[b, :, p % W] = kr, vr
            k_log[b, p], v_log[b, p] = kr, vr
    return kc, vc, k_log, v_log


@pytest.mark.parametrize("case", [
    dict(B=2, S=200, Hq=8, Hkv=4, D=256, W=512, prior=[700, 3], seed=401),
    dict(B=1, S=512, Hq=32, Hkv=16, D=256, W=512, prior=[2000], seed=402),    # chunk = window
    dict(B=3, S=4, Hq=32, Hkv=16, D=256, W=1024, prior=[5000, 1024, 0], seed=403),  # a 4-token chunk
    dict(B=1, S=100, Hq=8, Hkv=4, D=512, W=128, prior=[130], seed=404, frac=0.25, theta=1e6),
], ids=["S200", "SeqW", "S4", "D512"])
@pytest.mark.parametrize("source_flag", [False, True])
def test_shared_local_after_cached_tokens(oracle, case, source_flag):
    case = dict(case)
    B, S, Hq, Hkv, D, W, prior = (case[k] for k in ("B", "S", "Hq", "Hkv", "D", "W", "prior"))
    frac, theta = case.get("frac", 1.0), case.get("theta", 1e4)
    dev = torch.device("cuda")
    g = synth.generator(case["seed"])
    kc, vc, k_log, v_log = ring_with_history(B, Hkv, W, D, prior, g)
    q_src = synth.randn_bf16((B, S, Hq, D), g)
    k = synth.randn_bf16((B, S, Hkv, D), g)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    q_sh = [synth.randn_bf16((B, S, Hq, D), g) for _ in range(2)]
    T = max(prior) + S
    k_full = torch.zeros((B, T, Hkv, D), dtype=torch.bfloat16)
    v_full = torch.zeros_like(k_full)
    k_full[:, :k_log.shape[1]], v_full[:, :v_log.shape[1]] = k_log, v_log
    for b in range(B):
        k_full[b, prior[b]:prior[b] + S], v_full[b, prior[b]:prior[b] + S] = k[b], v[b]
    kcd, vcd = kc.to(dev), vc.to(dev)
    lens = torch.tensor(prior, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    kw = dict(window=W, rope_frac=frac, rope_theta=theta, scale=scale, seq_lens_before=lens)
    ws = torch.empty(native.gemma_attn_prefill_workspace_size_cached(B, S, Hq, Hkv, D, W, W, 0),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=dev)
    native.gemma_attn_prefill(q_src.to(dev), k.to(dev), v.to(dev), kcd, vcd, out=out, workspace=ws,
                              flags=native.GEMMA_F_SOURCE_WINDOW if source_flag else 0, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    after_src = (kcd.clone(), vcd.clone())
    for i, qs in enumerate(q_sh):  # two sharers of one source
        o = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
        native.gemma_attn_prefill(qs.to(dev), None, None, kcd, vcd, out=o, workspace=ws,
                                  flags=native.GEMMA_F_SHARED | native.GEMMA_F_SOURCE_WINDOW, **kw)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        ref, _ = oracle.attention(to_bits(qs), to_bits(k_full), to_bits(v_full), q_pos0=prior,
                                  n_keys=[p + S for p in prior], rot_from=prior, window=W,
                                  rope_frac=frac, theta=theta, scale=scale)
        got = o.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
        assert_close(got, ref, what="sharer %d" % i)
        assert torch.equal(kcd.view(torch.int16), after_src[0].view(torch.int16)), "a sharer writes nothing"
        assert torch.equal(vcd.view(torch.int16), after_src[1].view(torch.int16))


def test_shared_local_without_flag_is_unsupported():
    dev = torch.device("cuda")
    B, S, Hq, Hkv, D, W = 1, 8, 8, 4, 256, 64
    kc = torch.zeros((B, Hkv, W, D), dtype=torch.bfloat16, device=dev)
    q = torch.zeros((B, S, Hq, D), dtype=torch.bfloat16, device=dev)
    with pytest.raises(native.GemmaError) as e:
        native.gemma_attn_prefill(q, None, None, kc, kc, window=W, rope_frac=1.0, rope_theta=1e4, scale=0.0625,
                                  out=torch.empty_like(q), seq_lens_before=torch.tensor([100], dtype=torch.int32,
                                                                                        device=dev),
                                  flags=native.GEMMA_F_SHARED)
    assert e.value.code == native.GEMMA_ERR_UNSUPPORTED


def quantize(oracle, rows: torch.Tensor):
    """bf16 rows [..., D] -> (codes, params [..., 2]) from the oracle."""
    c, lo, st = oracle.quantize_rows_u8(to_bits(rows.contiguous()))
    return torch.from_numpy(c), torch.from_numpy(np.stack([lo, st], axis=-1))


def dequant(oracle, codes: torch.Tensor, params: torch.Tensor) -> np.ndarray:
    p = params.numpy()
    return oracle.dequantize_rows_u8(codes.numpy(), p[..., 0], p[..., 1])


@pytest.mark.parametrize("case", [
    dict(B=2, S=200, Hq=8, Hkv=4, D=256, W=512, prior=[700, 3], seed=411),
    dict(B=1, S=64, Hq=32, Hkv=16, D=256, W=1024, prior=[1500], seed=412),
])
def test_shared_local_after_cached_tokens_int8(oracle, case):
    """Int8 ring: the sharer attends to its source's window of dequantized
    cached rows and reads the chunk's rows back from the codes the source
    wrote, as a shared layer reads every row. The reference quantizes the
    oracle's rotated chunk keys and the values itself."""
    B, S, Hq, Hkv, D, W, prior = (case[k] for k in ("B", "S", "Hq", "Hkv", "D", "W", "prior"))
    dev = torch.device("cuda")
    g = synth.generator(case["seed"])
    old_k = synth.randn_bf16((B, Hkv, W, D), g)
    old_v = synth.randn_bf16((B, Hkv, W, D), g)
    ck, pk = quantize(oracle, old_k)
    cv, pv = quantize(oracle, old_v)
    kc = native.Int8KVCache(B, Hkv, W, D, dev)
    vc = native.Int8KVCache(B, Hkv, W, D, dev)
    kc.codes.copy_(ck)
    kc.params.copy_(pk)
    vc.codes.copy_(cv)
    vc.params.copy_(pv)
    q_src = synth.randn_bf16((B, S, Hq, D), g)
    k = synth.randn_bf16((B, S, Hkv, D), g)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    q_sh = synth.randn_bf16((B, S, Hq, D), g)
    lens = torch.tensor(prior, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    kw = dict(window=W, rope_frac=1.0, rope_theta=1e4, scale=scale, seq_lens_before=lens)
    ws = torch.empty(native.gemma_attn_prefill_workspace_size_cached(B, S, Hq, Hkv, D, W, W,
                                                                     native.GEMMA_F_KV_INT8),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=dev)
    native.gemma_attn_prefill(q_src.to(dev), k.to(dev), v.to(dev), kc, vc, out=out, workspace=ws, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    o = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    native.gemma_attn_prefill(q_sh.to(dev), None, None, kc, vc, out=o, workspace=ws,
                              flags=native.GEMMA_F_SHARED | native.GEMMA_F_SOURCE_WINDOW, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    G = Hq // Hkv
    got = o.float().cpu().double().numpy()
    for b in range(B):
        P0 = prior[b]
        lo = max(0, P0 - W)
        n = P0 + S - lo
        keys = np.zeros((Hkv, n, D))
        vals = np.zeros((Hkv, n, D))
        for idx, p in enumerate(range(lo, P0)):
            keys[:, idx] = dequant(oracle, ck[b, :, p % W], pk[b, :, p % W])
            vals[:, idx] = dequant(oracle, cv[b, :, p % W], pv[b, :, p % W])
        for s in range(S):
            rot = np.stack([oracle.rope_bf16(to_bits(k[b, s, h]), P0 + s, 1.0, 1e4) for h in range(Hkv)])
            rot_bf16 = torch.from_numpy(rot).to(torch.bfloat16)
            c_k, p_k = quantize(oracle, rot_bf16)
            c_v, p_v = quantize(oracle, v[b, s])
            keys[:, P0 - lo + s] = dequant(oracle, c_k, p_k)
            vals[:, P0 - lo + s] = dequant(oracle, c_v, p_v)
        rows_q, begin, count = [], [], []
        for i in range(S):
            P = P0 + i
            vis_lo = max(lo, P - W + 1)
            for h in range(Hq):
                rows_q.append(oracle.rope_bf16(to_bits(q_sh[b, i, h]), P, 1.0, 1e4))
                begin.append((h // G) * n + (vis_lo - lo))
                count.append(P - vis_lo + 1)
        ref, _ = oracle.attend_rows(np.array(rows_q), keys.reshape(Hkv * n, D), vals.reshape(Hkv * n, D),
                                    begin, count, scale)
        assert_close(got[b].reshape(S * Hq, D), ref, 2e-2, 2e-3, what="int8 sharer b=%d" % b)


def fill_layer(st, l, prior, g):
    """Random rotated history in layer l's cache; its rows in position order."""
    t = st.layer_type(l)
    Hkv, D, W = t.n_kv_heads, t.head_dim, t.window
    B = len(prior)
    T = max(prior)
    k_log = torch.zeros((B, T, Hkv, D), dtype=torch.bfloat16)
    v_log = torch.zeros_like(k_log)
    kc = torch.full(tuple(st.k_cache[l].shape), float("nan"), dtype=torch.bfloat16)
    vc = kc.clone()
    for b in range(B):
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
    return k_log, v_log


@pytest.mark.parametrize("mode", ["prefill", "decode_multi"])
def test_stack_with_shared_local_layer(oracle, mode):
    """A 31B-shaped 6-layer stack whose last local layer (4) shares layer
    3's K/V: a chunk (prefill) or 4 new tokens (multi-token decode) after
    cached tokens through every layer, each held to the oracle; layer 4
    attends to layer 3's keys and values with its own queries."""
    prior, S = [3000, 700], (48 if mode == "prefill" else 4)
    w = Workload("shared_stack", "prefill" if mode == "prefill" else "decode", batch=2, n_q_heads=32,
                 n_layers=6, ratio=5, local=L31B_LOCAL, global_=L31B_GLOBAL, seq=S, prior=max(prior),
                 len_lo=1, len_hi=max(prior) + S, n_shared=2, seed=421, tokens=S)
    dev = torch.device("cuda")
    st = AttentionStack(w, dev, global_capacity=max(prior) + S)
    assert st.is_shared(4) and st.descs[4].shared_from == 3 and not st.is_shared(5)
    g = synth.generator(421)
    lens_before = torch.tensor(prior, dtype=torch.int32, device=dev)
    lens_after = torch.tensor([p + S for p in prior], dtype=torch.int32, device=dev)
    T = max(prior) + S
    ws = torch.empty(max(st.prefill_workspace_bytes(after_cached=True),
                         st.decode_multi_workspace_bytes(S, T)), dtype=torch.uint8, device=dev)
    logs = {}
    for l in range(st.n_layers):
        t = st.layer_type(l)
        Hkv, D, W = t.n_kv_heads, t.head_dim, t.window
        q = synth.randn_bf16((w.batch, S, w.n_q_heads, D), g)
        if st.is_shared(l):
            k_full, v_full = logs[st.descs[l].shared_from]
            k = v = None
        else:
            k_log, v_log = fill_layer(st, l, prior, g)
            k = synth.randn_bf16((w.batch, S, Hkv, D), g)
            v = synth.randn_bf16((w.batch, S, Hkv, D), g)
            k_full = torch.zeros((w.batch, T, Hkv, D), dtype=torch.bfloat16)
            v_full = torch.zeros_like(k_full)
            k_full[:, :max(prior)], v_full[:, :max(prior)] = k_log, v_log
            for b in range(w.batch):
                k_full[b, prior[b]:prior[b] + S], v_full[b, prior[b]:prior[b] + S] = k[b], v[b]
            logs[l] = (k_full, v_full)
        out = torch.full((w.batch, S, w.n_q_heads, D), float("nan"), dtype=torch.bfloat16, device=dev)
        kd = None if k is None else k.to(dev)
        vd = None if v is None else v.to(dev)
        if mode == "prefill":
            st.prefill_layer(l, q.to(dev), kd, vd, out, workspace=ws, seq_lens_before=lens_before)
        else:
            st.decode_multi_layer(l, q.to(dev), kd, vd, out, seq_lens=lens_after, max_seq_len=T, workspace=ws)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        ref, _ = oracle.attention(to_bits(q), to_bits(k_full), to_bits(v_full), q_pos0=prior,
                                  n_keys=[p + S for p in prior], rot_from=prior, window=W,
                                  rope_frac=t.rope_frac, theta=t.rope_theta, scale=t.scale)
        got = out.float().cpu().double().numpy().transpose(0, 2, 1, 3).reshape(-1, D)
        assert_close(got, ref, what="%s layer %d (%s%s)" % (mode, l, "global" if W == 0 else "local",
                                                           ", shared" if st.is_shared(l) else ""))
