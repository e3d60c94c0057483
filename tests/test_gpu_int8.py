"""GPU parity of the int8 KV cache (GEMMA_F_KV_INT8) against the oracle,
through the C ABI: the codes and (min, step) rows that prefill and decode
write, and decode attention over an int8 cache.

Cached rows are quantized by the oracle (oracle.quantize_rows_u8) from seeded
bf16 rows; the expected attention is the oracle's over the dequantized rows
(oracle.attend_rows). Where the GPU's input to a code decision is exactly the
oracle's (values, and keys without RoPE) codes and rows must be bit-exact;
rotated keys come from fp32 (GPU) and fp64 (oracle) rotations that agree up
to a bf16 rounding, so their rows are compared within one code step.
"""
import math

import numpy as np
import pytest
import torch

from hybrid_local_global_b200 import native, synth

from gpu_util import assert_close, to_bits

pytestmark = pytest.mark.gpu

SENTINEL = 0xAB


def f64_to_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16)


def quantize(oracle, rows: torch.Tensor):
    """bf16 rows [..., D] -> (codes uint8 tensor, params float32 [..., 2]) from the oracle."""
    c, lo, st = oracle.quantize_rows_u8(to_bits(rows.contiguous()))
    return torch.from_numpy(c), torch.from_numpy(np.stack([lo, st], axis=-1))


def dequant(oracle, codes: torch.Tensor, params: torch.Tensor) -> np.ndarray:
    p = params.numpy()
    return oracle.dequantize_rows_u8(codes.numpy(), p[..., 0], p[..., 1])


def rotated_bf16(oracle, x: torch.Tensor, pos, frac, theta) -> torch.Tensor:
    """[..., D] bf16 -> the oracle's (p-)RoPE at `pos`, rounded to bf16."""
    flat = x.reshape(-1, x.shape[-1])
    rows = [f64_to_bf16(oracle.rope_bf16(to_bits(r), pos, frac, theta)) for r in flat]
    return torch.stack(rows).reshape(x.shape)


def assert_rows_within_step(oracle, codes, params, exp_codes, exp_params, what):
    """Rotated keys: the dequantized rows agree within one code step (the bf16
    rotated inputs of the two sides may differ in a last bit)."""
    got = dequant(oracle, codes, params)
    exp = dequant(oracle, exp_codes, exp_params)
    step = np.maximum(params[..., 1].numpy(), exp_params[..., 1].numpy())[..., None].astype(np.float64)
    tol = 1.01 * step + 2.0 ** -7 * np.abs(exp)
    assert (np.abs(got - exp) <= tol).all(), what
    same = (codes == exp_codes).reshape(-1, codes.shape[-1]).all(dim=1).float().mean().item()
    assert same >= 0.5, "%s: only %.0f%% of rows bit-identical" % (what, 100 * same)


# ---------------------------------------------------------------------- prefill
PREFILL_CASES = [
    dict(B=2, S=200, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=301),
    dict(B=1, S=300, Hq=8, Hkv=4, D=256, W=128, frac=1.0, theta=1e4, seed=302),
    dict(B=2, S=96, Hq=4, Hkv=2, D=256, W=0, frac=0.0, theta=1e4, seed=303),      # NoPE: K codes exact
    dict(B=1, S=130, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=304, keqv=True),
    dict(B=1, S=40, Hq=8, Hkv=4, D=256, W=64, frac=0.0, theta=1e4, seed=305),      # chunk shorter than the ring
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=["global", "local", "nope", "keqv", "short"])
def test_prefill_writes_int8_rows(oracle, case):
    case = dict(case)
    keqv = case.pop("keqv", False)
    B, S, Hq, Hkv, D, W = (case[k] for k in ("B", "S", "Hq", "Hkv", "D", "W"))
    frac, theta = case["frac"], case["theta"]
    dev = torch.device("cuda")
    g = synth.generator(case["seed"])
    q = synth.randn_bf16((B, S, Hq, D), g)
    k = synth.randn_bf16((B, S, Hkv, D), g)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    cap = W if W else S + 16
    kc = native.Int8KVCache(B, Hkv, cap, D, dev, fill=SENTINEL)
    vc = kc if keqv else native.Int8KVCache(B, Hkv, cap, D, dev, fill=SENTINEL)
    out8 = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    scale = 1.0 / math.sqrt(D)
    flags = native.GEMMA_F_KEQV if keqv else 0
    kw = dict(window=W, rope_frac=frac, rope_theta=theta, scale=scale, flags=flags)
    native.gemma_attn_prefill(q.to(dev), k.to(dev), None if keqv else v.to(dev), kc, None if keqv else vc,
                              out=out8, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    # the attention itself is the bf16 path's: same kernels, same rotated chunk
    kb = torch.zeros((B, Hkv, cap, D), dtype=torch.bfloat16, device=dev)
    vb = kb if keqv else torch.zeros_like(kb)
    outb = torch.full_like(out8, float("nan"))
    native.gemma_attn_prefill(q.to(dev), k.to(dev), None if keqv else v.to(dev), kb, None if keqv else vb,
                              out=outb, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(out8.view(torch.int16), outb.view(torch.int16))
    codes_k, par_k = kc.codes.cpu(), kc.params.cpu()
    codes_v, par_v = vc.codes.cpu(), vc.params.cpu()
    written = torch.zeros((B, cap), dtype=torch.bool)
    first = max(0, S - W) if W else 0
    for b in range(B):
        for p in range(first, S):
            slot = p % W if W else p
            written[b, slot] = True
            if not keqv:
                ec, ep = quantize(oracle, v[b, p])
                assert torch.equal(codes_v[b, :, slot], ec), "V codes b=%d p=%d" % (b, p)
                assert torch.equal(par_v[b, :, slot], ep), "V (min, step) b=%d p=%d" % (b, p)
            ec, ep = quantize(oracle, rotated_bf16(oracle, k[b, p], p, frac, theta))
            if frac == 0.0:
                assert torch.equal(codes_k[b, :, slot], ec), "K codes b=%d p=%d" % (b, p)
                assert torch.equal(par_k[b, :, slot], ep), "K (min, step) b=%d p=%d" % (b, p)
            else:
                assert_rows_within_step(oracle, codes_k[b, :, slot], par_k[b, :, slot], ec, ep,
                                        "K rows b=%d p=%d" % (b, p))
    untouched = ~written
    for c in (codes_k, codes_v):
        assert (c.permute(0, 2, 1, 3)[untouched] == SENTINEL).all()
    for par in (par_k, par_v):
        raw = par.view(torch.int32).permute(0, 2, 1, 3)[untouched]
        assert (raw == int(np.uint32(0xABABABAB).view(np.int32))).all()


# ----------------------------------------------------------------------- decode
def run_decode_int8(oracle, *, lens, Hq, Hkv, D, W, frac, theta, seed, keqv=False, shared=False,
                    v_scale=1.0, tol=(2e-2, 2e-3)):
    dev = torch.device("cuda")
    B = len(lens)
    g = synth.generator(seed)
    max_len = max(lens)
    cap = W if W else max_len + 16 + (max_len % 2)
    # cached rows (already rotated), quantized by the oracle, at their slots
    k_rows = synth.randn_bf16((B, Hkv, cap, D), g)
    v_rows = synth.randn_bf16((B, Hkv, cap, D), g, scale=v_scale)
    q = synth.randn_bf16((B, Hq, D), g)
    kn = synth.randn_bf16((B, Hkv, D), g)
    vn = synth.randn_bf16((B, Hkv, D), g, scale=v_scale)
    if keqv:
        v_rows, vn = k_rows, kn
    ck, pk = quantize(oracle, k_rows)
    cv, pv = (ck, pk) if keqv else quantize(oracle, v_rows)
    if shared:
        # the new token's rows are already in the (source layer's) cache
        for b in range(B):
            slot = (lens[b] - 1) % W if W else lens[b] - 1
            ck[b, :, slot], pk[b, :, slot] = quantize(oracle, kn[b])
            if not keqv:
                cv[b, :, slot], pv[b, :, slot] = quantize(oracle, vn[b])
            else:
                cv, pv = ck, pk
    kc = native.Int8KVCache(B, Hkv, cap, D, dev)
    kc.codes.copy_(ck)
    kc.params.copy_(pk)
    vc = kc
    if not keqv:
        vc = native.Int8KVCache(B, Hkv, cap, D, dev)
        vc.codes.copy_(cv)
        vc.params.copy_(pv)
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    flags = (native.GEMMA_F_SHARED if shared else 0) | (native.GEMMA_F_KEQV if keqv else 0)
    native.gemma_attn_decode(q.to(dev), None if shared else kn.to(dev),
                             None if (shared or keqv) else vn.to(dev), kc, None if keqv else vc,
                             seq_lens=sl, max_seq_len=max_len, window=W, rope_frac=frac, rope_theta=theta,
                             scale=scale, out=out, flags=flags)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    ck1, pk1, cv1, pv1 = kc.codes.cpu(), kc.params.cpu(), vc.codes.cpu(), vc.params.cpu()
    G = Hq // Hkv
    for b in range(B):
        L = lens[b]
        slot_new = (L - 1) % W if W else L - 1
        # the new token's rows as the oracle writes them
        if shared:
            nk_c, nk_p = ck[b, :, slot_new], pk[b, :, slot_new]
            nv_c, nv_p = cv[b, :, slot_new], pv[b, :, slot_new]
        else:
            nk_c, nk_p = quantize(oracle, rotated_bf16(oracle, kn[b], L - 1, frac, theta))
            nv_c, nv_p = (nk_c, nk_p) if keqv else quantize(oracle, vn[b])
            if not keqv:
                assert torch.equal(cv1[b, :, slot_new], nv_c) and torch.equal(pv1[b, :, slot_new], nv_p)
            if frac == 0.0:
                assert torch.equal(ck1[b, :, slot_new], nk_c) and torch.equal(pk1[b, :, slot_new], nk_p)
            else:
                assert_rows_within_step(oracle, ck1[b, :, slot_new], pk1[b, :, slot_new], nk_c, nk_p,
                                        "new K row b=%d" % b)
            other = torch.ones(cap, dtype=torch.bool)
            other[slot_new] = False
            assert torch.equal(ck1[b][:, other], ck[b][:, other])
        first = max(0, L - W) if W else 0
        positions = list(range(first, L))
        keys = np.zeros((Hkv, len(positions), D))
        vals = np.zeros((Hkv, len(positions), D))
        for i, p in enumerate(positions):
            if p == L - 1:
                keys[:, i] = dequant(oracle, nk_c, nk_p)
                vals[:, i] = dequant(oracle, nv_c, nv_p)
            else:
                s = p % W if W else p
                keys[:, i] = dequant(oracle, ck[b, :, s], pk[b, :, s])
                vals[:, i] = dequant(oracle, cv[b, :, s], pv[b, :, s])
        n = len(positions)
        qrot = np.stack([oracle.rope_bf16(to_bits(q[b, h]), L - 1, frac, theta) for h in range(Hq)])
        ref, _ = oracle.attend_rows(qrot, keys.reshape(Hkv * n, D), vals.reshape(Hkv * n, D),
                                    [(h // G) * n for h in range(Hq)], [n] * Hq, scale)
        assert_close(out[b].float().cpu().double().numpy(), ref, *tol, what="int8 decode b=%d len=%d" % (b, L))


DECODE_CASES = [
    dict(lens=[1, 37, 300, 4097], Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=311),
    dict(lens=[1, 5, 64, 65, 1000], Hq=8, Hkv=4, D=256, W=64, frac=1.0, theta=1e4, seed=312),
    dict(lens=[17, 16, 15, 33], Hq=32, Hkv=16, D=256, W=16, frac=0.0, theta=1e4, seed=313),
    dict(lens=[7777, 123], Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6, seed=314),
    dict(lens=[3000, 900], Hq=32, Hkv=16, D=256, W=1024, frac=1.0, theta=1e4, seed=315),
    dict(lens=[2, 129], Hq=8, Hkv=4, D=256, W=0, frac=0.0, theta=1e4, seed=316),   # NoPE: new K row exact
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "L%s_H%d-%dD%dW%d" % (
    "_".join(map(str, c["lens"])), c["Hq"], c["Hkv"], c["D"], c["W"]))
def test_decode_int8(oracle, case):
    run_decode_int8(oracle, **case)


def test_decode_int8_k_equals_v(oracle):
    run_decode_int8(oracle, lens=[1, 37, 300, 2049], Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=321,
                    keqv=True)


@pytest.mark.parametrize("W,D,Hkv", [(0, 512, 1), (64, 256, 4)])
def test_decode_int8_shared_layer(oracle, W, D, Hkv):
    run_decode_int8(oracle, lens=[900, 33], Hq=8, Hkv=Hkv, D=D, W=W, frac=0.25 if W == 0 else 1.0,
                    theta=1e6 if W == 0 else 1e4, seed=322, shared=True)


@pytest.mark.parametrize("v_scale", [1e-3, 40.0])
def test_decode_int8_value_ranges(oracle, v_scale):
    """Rows whose steps are far from 1: the fp16 weights of the codes are
    scaled by a power of two that keeps them in range."""
    run_decode_int8(oracle, lens=[300, 1500], Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=323,
                    v_scale=v_scale, tol=(2e-2 * v_scale, 2e-3 * v_scale))


# ------------------------------------------------- prefill after cached tokens
def run_prefill_int8_chunk(oracle, *, before, S, Hq, Hkv, D, W, frac, theta, seed, keqv=False):
    """A chunk of S tokens after `before[b]` cached tokens on an int8 cache.

    The cached rows are the oracle's quantization of seeded (already rotated)
    rows; the chunk attends to them dequantized (min + code * step) and to
    its own keys and values; its rows are then quantized into the cache."""
    dev = torch.device("cuda")
    B = len(before)
    g = synth.generator(seed)
    cap = W if W else max(before) + S + 16 + (max(before) + S) % 2
    k_rows = synth.randn_bf16((B, Hkv, cap, D), g)
    v_rows = k_rows if keqv else synth.randn_bf16((B, Hkv, cap, D), g)
    q = synth.randn_bf16((B, S, Hq, D), g)
    kn = synth.randn_bf16((B, S, Hkv, D), g)
    vn = kn if keqv else synth.randn_bf16((B, S, Hkv, D), g)
    ck, pk = quantize(oracle, k_rows)
    cv, pv = (ck, pk) if keqv else quantize(oracle, v_rows)
    kc = native.Int8KVCache(B, Hkv, cap, D, dev)
    kc.codes.copy_(ck)
    kc.params.copy_(pk)
    vc = kc
    if not keqv:
        vc = native.Int8KVCache(B, Hkv, cap, D, dev)
        vc.codes.copy_(cv)
        vc.params.copy_(pv)
    out = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(D)
    native.gemma_attn_prefill(q.to(dev), kn.to(dev), None if keqv else vn.to(dev), kc, None if keqv else vc,
                              window=W, rope_frac=frac, rope_theta=theta, scale=scale, out=out, lse=lse,
                              seq_lens_before=torch.tensor(before, dtype=torch.int32, device=dev),
                              flags=native.GEMMA_F_KEQV if keqv else 0)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    ck1, pk1, cv1, pv1 = kc.codes.cpu(), kc.params.cpu(), vc.codes.cpu(), vc.params.cpu()
    G = Hq // Hkv
    out_c, lse_c = out.float().cpu().double().numpy(), lse.cpu().double().numpy()
    for b in range(B):
        P0 = before[b]
        lo = max(0, P0 - W) if W else 0
        positions = list(range(lo, P0 + S))
        n = len(positions)
        keys = np.zeros((Hkv, n, D))
        vals = np.zeros((Hkv, n, D))
        written = torch.zeros(cap, dtype=torch.bool)
        for idx, p in enumerate(positions):
            if p < P0:  # cached: the rows the cache held before the call
                s = p % W if W else p
                keys[:, idx] = dequant(oracle, ck[b, :, s], pk[b, :, s])
                vals[:, idx] = dequant(oracle, cv[b, :, s], pv[b, :, s])
            else:       # the chunk's own rotated key and value
                i = p - P0
                keys[:, idx] = np.stack([oracle.rope_bf16(to_bits(kn[b, i, h]), p, frac, theta)
                                         for h in range(Hkv)])
                # K = V: the values are the rotated keys
                vals[:, idx] = keys[:, idx] if keqv else vn[b, i].double().numpy()
                if W and i < S - W:
                    continue  # overwritten later in the same chunk: never reaches the ring
                s = p % W if W else p
                written[s] = True
                ec, ep = quantize(oracle, rotated_bf16(oracle, kn[b, i], p, frac, theta))
                if frac == 0.0:
                    assert torch.equal(ck1[b, :, s], ec) and torch.equal(pk1[b, :, s], ep)
                else:
                    assert_rows_within_step(oracle, ck1[b, :, s], pk1[b, :, s], ec, ep, "K b=%d p=%d" % (b, p))
                if not keqv:
                    ec, ep = quantize(oracle, vn[b, i])
                    assert torch.equal(cv1[b, :, s], ec) and torch.equal(pv1[b, :, s], ep), "V b=%d p=%d" % (b, p)
        # rows the chunk does not write keep their codes
        assert torch.equal(ck1[b][:, ~written], ck[b][:, ~written])
        assert torch.equal(pk1[b][:, ~written], pk[b][:, ~written])
        rows_q, begin, count = [], [], []
        for i in range(S):
            P = P0 + i
            vis_lo = max(lo, P - W + 1) if W else 0
            for h in range(Hq):
                rows_q.append(oracle.rope_bf16(to_bits(q[b, i, h]), P, frac, theta))
                begin.append((h // G) * n + (vis_lo - lo))
                count.append(P - vis_lo + 1)
        ref, ref_lse = oracle.attend_rows(np.array(rows_q), keys.reshape(Hkv * n, D), vals.reshape(Hkv * n, D),
                                          begin, count, scale)
        assert_close(out_c[b].reshape(S * Hq, D), ref, 2e-2, 2e-3, what="int8 chunk b=%d before=%d" % (b, P0))
        got_lse = lse_c[b].transpose(1, 0).reshape(S * Hq)
        assert np.abs(got_lse - ref_lse).max() < 2e-2, "lse b=%d" % b


CHUNK_CASES = [
    dict(before=[300, 0, 1000], S=200, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=331),
    dict(before=[4096], S=256, Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6, seed=332),
    dict(before=[77, 200], S=96, Hq=4, Hkv=2, D=256, W=0, frac=0.0, theta=1e4, seed=333),
    dict(before=[50, 300, 0], S=100, Hq=8, Hkv=4, D=256, W=128, frac=1.0, theta=1e4, seed=334),
    dict(before=[500, 3], S=300, Hq=8, Hkv=4, D=256, W=128, frac=1.0, theta=1e4, seed=335),
    dict(before=[64, 65], S=4, Hq=32, Hkv=16, D=256, W=64, frac=0.0, theta=1e4, seed=336),
]


@pytest.mark.parametrize("case", CHUNK_CASES, ids=["global", "global_h32", "global_d256_nope", "local",
                                                   "local_long_chunk", "local_verify4"])
def test_prefill_int8_after_cached_tokens(oracle, case):
    run_prefill_int8_chunk(oracle, **case)


def test_prefill_int8_after_cached_tokens_k_equals_v(oracle):
    run_prefill_int8_chunk(oracle, before=[129, 700], S=130, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6,
                           seed=337, keqv=True)


# ------------------------------------------------------- shared layer's prefill
def run_prefill_int8_shared(oracle, *, before, S, Hq, Hkv, D, W, frac, theta, seed, keqv=False):
    """A KV-shared layer's prefill on an int8 cache: its source has already
    quantized every row, the chunk's included; the layer attends to all of
    them dequantized and writes nothing."""
    dev = torch.device("cuda")
    B = len(before)
    g = synth.generator(seed)
    cap = W if W else max(before) + S + 16 + (max(before) + S) % 2
    k_rows = synth.randn_bf16((B, Hkv, cap, D), g)
    v_rows = k_rows if keqv else synth.randn_bf16((B, Hkv, cap, D), g)
    q = synth.randn_bf16((B, S, Hq, D), g)
    ck, pk = quantize(oracle, k_rows)
    cv, pv = (ck, pk) if keqv else quantize(oracle, v_rows)
    kc = native.Int8KVCache(B, Hkv, cap, D, dev)
    kc.codes.copy_(ck)
    kc.params.copy_(pk)
    vc = kc
    if not keqv:
        vc = native.Int8KVCache(B, Hkv, cap, D, dev)
        vc.codes.copy_(cv)
        vc.params.copy_(pv)
    out = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    scale = 1.0 / math.sqrt(D)
    lens = torch.tensor(before, dtype=torch.int32, device=dev) if any(before) else None
    native.gemma_attn_prefill(q.to(dev), None, None, kc, None if keqv else vc, window=W, rope_frac=frac,
                              rope_theta=theta, scale=scale, out=out, seq_lens_before=lens,
                              flags=native.GEMMA_F_SHARED | (native.GEMMA_F_KEQV if keqv else 0))
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(kc.codes.cpu(), ck) and torch.equal(kc.params.cpu(), pk), "a shared layer writes nothing"
    if not keqv:
        assert torch.equal(vc.codes.cpu(), cv) and torch.equal(vc.params.cpu(), pv)
    G = Hq // Hkv
    out_c = out.float().cpu().double().numpy()
    for b in range(B):
        P0 = before[b]
        lo = max(0, P0 - W) if W else 0
        positions = list(range(lo, P0 + S))
        n = len(positions)
        keys = np.zeros((Hkv, n, D))
        vals = np.zeros((Hkv, n, D))
        for idx, p in enumerate(positions):
            s = p % W if W else p
            keys[:, idx] = dequant(oracle, ck[b, :, s], pk[b, :, s])
            vals[:, idx] = dequant(oracle, cv[b, :, s], pv[b, :, s])
        rows_q, begin, count = [], [], []
        for i in range(S):
            P = P0 + i
            vis_lo = max(lo, P - W + 1) if W else 0
            for h in range(Hq):
                rows_q.append(oracle.rope_bf16(to_bits(q[b, i, h]), P, frac, theta))
                begin.append((h // G) * n + (vis_lo - lo))
                count.append(P - vis_lo + 1)
        ref, _ = oracle.attend_rows(np.array(rows_q), keys.reshape(Hkv * n, D), vals.reshape(Hkv * n, D),
                                    begin, count, scale)
        assert_close(out_c[b].reshape(S * Hq, D), ref, 2e-2, 2e-3, what="int8 shared b=%d before=%d" % (b, P0))


SHARED_CASES = [
    dict(before=[300, 0], S=200, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=341),
    dict(before=[0], S=300, Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6, seed=342),
    dict(before=[0, 0], S=100, Hq=8, Hkv=4, D=256, W=128, frac=1.0, theta=1e4, seed=343),
    dict(before=[0], S=64, Hq=32, Hkv=16, D=256, W=64, frac=1.0, theta=1e4, seed=344),
]


@pytest.mark.parametrize("case", SHARED_CASES, ids=["global_prior", "global", "local", "local_full_ring"])
def test_prefill_int8_shared_layer(oracle, case):
    run_prefill_int8_shared(oracle, **case)


def test_prefill_int8_shared_layer_k_equals_v(oracle):
    run_prefill_int8_shared(oracle, before=[129], S=130, Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6,
                            seed=345, keqv=True)


# ------------------------------------------------- the benchmarked int8 block
def test_decode_31b_b64_int8_sampled(oracle):
    """The 31B-shaped decode block on int8 caches, as bench.py times it (B64,
    KV lengths U[4096,131072], 5 local + 1 global layer, layer 4 sharing
    layer 3), with seeded synthetic codes and (min, step) rows. Sampled
    sequences (rows are independent) are held to the oracle over the
    dequantized rows; global-layer samples are kept to at most 40000 keys so
    that the fp64 key arrays stay small."""
    from hybrid_local_global_b200.stack import AttentionStack
    from hybrid_local_global_b200.workloads import WORKLOADS
    w = WORKLOADS["31b_decode_b64_int8"]
    dev = torch.device("cuda")
    st = AttentionStack(w, dev)
    lens_cpu = synth.decode_lengths(w.batch, w.len_lo, w.len_hi, seed=w.seed)
    lens = lens_cpu.to(dev)
    max_len = int(lens_cpu.max())
    g = synth.generator(w.seed, "cuda")
    owned = set()
    for l in range(st.n_layers):
        if not st.is_shared(l) and st.k_cache[l].data_ptr() not in owned:
            owned.add(st.k_cache[l].data_ptr())
            synth.fill_int8_cache_(st.k_cache[l], g)
            if st.v_cache[l] is not st.k_cache[l]:
                synth.fill_int8_cache_(st.v_cache[l], g)
    ws = torch.empty(st.decode_workspace_bytes(max_len), dtype=torch.uint8, device=dev)
    rng = np.random.default_rng(w.seed)
    pick = set(rng.choice(w.batch, size=4, replace=False).tolist()) | {int(lens_cpu.argmin())}
    for l in range(st.n_layers):
        t = st.layer_type(l)
        D, Hkv, W = t.head_dim, t.n_kv_heads, t.window
        G = w.n_q_heads // Hkv
        q = synth.randn_bf16((w.batch, w.n_q_heads, D), g, "cuda")
        kn = synth.randn_bf16((w.batch, Hkv, D), g, "cuda")
        vn = synth.randn_bf16((w.batch, Hkv, D), g, "cuda")
        shared = st.is_shared(l)
        checked = [b for b in sorted(pick) if W or int(lens_cpu[b]) <= 40000]
        kc, vc = st.k_cache[l], st.v_cache[l]
        snaps = {}
        for b in checked:
            n = min(kc.shape[2], int(lens_cpu[b]))
            snaps[b] = (kc.codes[b, :, :n].cpu(), kc.params[b, :, :n].cpu(),
                        vc.codes[b, :, :n].cpu(), vc.params[b, :, :n].cpu())
        out = torch.empty((w.batch, w.n_q_heads, D), dtype=torch.bfloat16, device=dev)
        st.decode_layer(l, q, kn, vn, out, seq_lens=lens, max_seq_len=max_len, workspace=ws)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        for b in checked:
            L = int(lens_cpu[b])
            ck, pk, cv, pv = snaps[b]
            slot_new = (L - 1) % W if W else L - 1
            if shared:  # the source layer has appended this step's rows already
                nk_c, nk_p, nv_c, nv_p = ck[:, slot_new], pk[:, slot_new], cv[:, slot_new], pv[:, slot_new]
            else:
                nk_c, nk_p = quantize(oracle, rotated_bf16(oracle, kn[b].cpu(), L - 1, t.rope_frac, t.rope_theta))
                nv_c, nv_p = quantize(oracle, vn[b].cpu())
            positions = np.arange(max(0, L - W) if W else 0, L)
            n = len(positions)
            slots = torch.from_numpy(positions % W if W else positions)
            keys = dequant(oracle, ck[:, slots], pk[:, slots])  # [Hkv, n, D]
            vals = dequant(oracle, cv[:, slots], pv[:, slots])
            keys[:, n - 1] = dequant(oracle, nk_c, nk_p)          # position L - 1: this step's rows
            vals[:, n - 1] = dequant(oracle, nv_c, nv_p)
            qrot = np.stack([oracle.rope_bf16(to_bits(q[b, h].cpu()), L - 1, t.rope_frac, t.rope_theta)
                             for h in range(w.n_q_heads)])
            ref, _ = oracle.attend_rows(qrot, keys.reshape(Hkv * n, D), vals.reshape(Hkv * n, D),
                                        [(h // G) * n for h in range(w.n_q_heads)], [n] * w.n_q_heads, t.scale)
            assert_close(out[b].float().cpu().double().numpy(), ref,
                         what="31b int8 layer %d b=%d len=%d" % (l, b, L))
        del snaps


def test_decode_int8_bounded_wait_times_out_and_context_survives(oracle):
    """The int8 decode's first copy is not issued, so a barrier is never
    completed: the bounded wait gives up after its deadline, the status says
    so, and the next calls on the same context are correct."""
    native.gemma_attn_set_wait_limit(20_000_000)  # 20 ms
    try:
        native.gemma_attn_debug_drop_next_copy(True)
        dev = torch.device("cuda")
        B, Hq, Hkv, D, L = 1, 8, 1, 512, 2000
        g = synth.generator(350, "cuda")
        kc = synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, L + 16, D, dev), g)
        vc = synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, L + 16, D, dev), g)
        q = synth.randn_bf16((B, Hq, D), g, "cuda")
        kn = synth.randn_bf16((B, Hkv, D), g, "cuda")
        vn = synth.randn_bf16((B, Hkv, D), g, "cuda")
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
        sl = torch.tensor([L], dtype=torch.int32, device=dev)
        native.gemma_attn_decode(q, kn, vn, kc, vc, seq_lens=sl, max_seq_len=L, window=0, rope_frac=0.25,
                                 rope_theta=1e6, scale=0.05, out=out)
        assert native.gemma_attn_sync_status() == native.GEMMA_ERR_DEVICE_TIMEOUT
    finally:
        native.gemma_attn_set_wait_limit(0)
    run_decode_int8(oracle, lens=[2000, 37], Hq=8, Hkv=1, D=512, W=0, frac=0.25, theta=1e6, seed=351)
