"""GPU parity of the paged global cache (gemma_attn_prefill_paged /
gemma_attn_decode_paged), through the C ABI.

The paged path reads and writes the same rows as the contiguous one, only
at other addresses, so its outputs must be bit-identical to the contiguous
path's on the same inputs (which the other GPU tests hold to the oracle);
one case per entry point is also checked against the oracle directly. The
pages must hold exactly the rows the contiguous cache holds at the same
positions, pages no sequence owns stay untouched, and a page table entry
outside the pool is reported (GEMMA_ERR_DEVICE_RANGE) without a fault.
"""
import math

import numpy as np
import pytest
import torch

from hybrid_local_global_b200 import native, synth

from gpu_util import assert_close, to_bits

pytestmark = pytest.mark.gpu

SENTINEL = -7.5  # bf16-exact fill of every pool row before a call


def make_table(B, pps, n_pages, seed):
    """A random assignment of distinct pool pages to every (sequence, page)."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_pages)[:B * pps].reshape(B, pps)
    return torch.tensor(perm, dtype=torch.int32)


def to_pool(cache, table, ps, n_pages):
    """Contiguous [B, Hkv, cap, D] -> pool [n_pages, Hkv, ps, D] (cap = pps * ps)."""
    B, Hkv, cap, D = cache.shape
    pool = torch.full((n_pages, Hkv, ps, D), SENTINEL, dtype=cache.dtype)
    for b in range(B):
        for p in range(table.shape[1]):
            pool[int(table[b, p])] = cache[b, :, p * ps:(p + 1) * ps]
    return pool


def from_pool(pool, table, ps):
    B, pps = table.shape
    n_pages, Hkv, _, D = pool.shape
    out = torch.empty((B, Hkv, pps * ps, D), dtype=pool.dtype)
    for b in range(B):
        for p in range(pps):
            out[b, :, p * ps:(p + 1) * ps] = pool[int(table[b, p])]
    return out


def owned_mask(table, n_pages):
    m = torch.zeros(n_pages, dtype=torch.bool)
    m[table.flatten().long()] = True
    return m


def bits(t):
    return t.view(torch.int16)


# ---------------------------------------------------------------------- decode
DECODE_CASES = [
    dict(lens=[1, 130, 300, 1025], Hq=8, Hkv=1, D=512, ps=128, seed=401),
    dict(lens=[4097, 2], Hq=32, Hkv=4, D=512, ps=256, seed=402),
    dict(lens=[640, 129, 17], Hq=8, Hkv=4, D=256, ps=128, seed=403),
]


def run_decode_paged(oracle, *, lens, Hq, Hkv, D, ps, seed, keqv=False, shared=False, check_oracle=False):
    dev = torch.device("cuda")
    B = len(lens)
    g = synth.generator(seed)
    max_len = max(lens)
    pps = (max_len + ps - 1) // ps + 1
    n_pages = B * pps + 3                        # pages no sequence owns stay untouched
    cap = pps * ps
    kc = synth.randn_bf16((B, Hkv, cap, D), g)   # already-rotated keys/values at every position
    vc = kc if keqv else synth.randn_bf16((B, Hkv, cap, D), g)
    q = synth.randn_bf16((B, Hq, D), g)
    kn = synth.randn_bf16((B, Hkv, D), g)
    vn = kn if keqv else synth.randn_bf16((B, Hkv, D), g)
    table = make_table(B, pps, n_pages, seed)
    kp, vp = to_pool(kc, table, ps, n_pages), None
    vp = kp if keqv else to_pool(vc, table, ps, n_pages)
    kcd, kpd = kc.to(dev), kp.to(dev)
    vcd = kcd if keqv else vc.to(dev)
    vpd = kpd if keqv else vp.to(dev)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    td = table.to(dev)
    scale = 1.0 / math.sqrt(D)
    flags = (native.GEMMA_F_SHARED if shared else 0) | (native.GEMMA_F_KEQV if keqv else 0)
    kw = dict(seq_lens=sl, max_seq_len=max_len, rope_frac=0.25, rope_theta=1e6, scale=scale, flags=flags)
    kn_d = None if shared else kn.to(dev)
    vn_d = None if (shared or keqv) else vn.to(dev)
    out_c = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    native.gemma_attn_decode(q.to(dev), kn_d, vn_d, kcd, None if keqv else vcd, window=0, out=out_c, **kw)
    out_p = torch.full_like(out_c, float("nan"))
    native.gemma_attn_decode_paged(q.to(dev), kn_d, vn_d, kpd, None if keqv else vpd, td, out=out_p, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(bits(out_p), bits(out_c))
    # the pages hold what the contiguous cache holds; unowned pages are untouched
    kp1, kc1 = kpd.cpu(), kcd.cpu()
    assert torch.equal(bits(from_pool(kp1, table, ps)), bits(kc1))
    if not keqv:
        assert torch.equal(bits(from_pool(vpd.cpu(), table, ps)), bits(vcd.cpu()))
    free = ~owned_mask(table, n_pages)
    assert (kp1[free] == SENTINEL).all()
    if check_oracle:
        for b in range(B):
            L = lens[b]
            kl = kc1[b, :, :L].permute(1, 0, 2).contiguous()
            vl = kl if keqv else vcd.cpu()[b, :, :L].permute(1, 0, 2).contiguous()
            ref, _ = oracle.attention(to_bits(q[b].reshape(1, 1, Hq, D)), to_bits(kl[None]),
                                      None if keqv else to_bits(vl[None]), q_pos0=L - 1, n_keys=L, rot_from=L,
                                      window=0, rope_frac=0.25, theta=1e6, scale=scale)
            assert_close(out_p[b].float().cpu().double().numpy(), ref, what="paged decode b=%d" % b)


@pytest.mark.parametrize("case", DECODE_CASES, ids=["ps128", "ps256", "D256"])
def test_decode_paged_matches_contiguous(oracle, case):
    run_decode_paged(oracle, check_oracle=case["seed"] == 401, **case)


def test_decode_paged_k_equals_v(oracle):
    run_decode_paged(oracle, lens=[1, 300, 1500], Hq=8, Hkv=1, D=512, ps=128, seed=404, keqv=True)


def test_decode_paged_shared_layer(oracle):
    run_decode_paged(oracle, lens=[900, 33], Hq=8, Hkv=1, D=512, ps=256, seed=405, shared=True)


# --------------------------------------------------------------------- prefill
PREFILL_CASES = [
    dict(B=2, S=300, Hq=8, Hkv=1, D=512, ps=128, prior=None, seed=411),
    dict(B=2, S=200, Hq=8, Hkv=1, D=512, ps=256, prior=[37, 300], seed=412),
    dict(B=1, S=520, Hq=16, Hkv=2, D=256, ps=128, prior=[1000], seed=413),
]


@pytest.mark.parametrize("kernel", ["single", "pair", "hpair"])
@pytest.mark.parametrize("case", PREFILL_CASES, ids=["chunk", "prior", "D256"])
def test_prefill_paged_matches_contiguous(oracle, monkeypatch, kernel, case):
    monkeypatch.setenv("GEMMA_PREFILL_KERNEL", kernel)
    dev = torch.device("cuda")
    B, S, Hq, Hkv, D, ps = (case[k] for k in ("B", "S", "Hq", "Hkv", "D", "ps"))
    prior = case["prior"] or [0] * B
    g = synth.generator(case["seed"])
    q = synth.randn_bf16((B, S, Hq, D), g)
    k = synth.randn_bf16((B, S, Hkv, D), g)
    v = synth.randn_bf16((B, S, Hkv, D), g)
    pps = (max(prior) + S + ps - 1) // ps + 1
    cap = pps * ps
    n_pages = B * pps + 2
    kc = torch.full((B, Hkv, cap, D), SENTINEL, dtype=torch.bfloat16)
    vc = torch.full_like(kc, SENTINEL)
    for b in range(B):
        if prior[b]:
            kc[b, :, :prior[b]] = synth.randn_bf16((Hkv, prior[b], D), g)
            vc[b, :, :prior[b]] = synth.randn_bf16((Hkv, prior[b], D), g)
    table = make_table(B, pps, n_pages, case["seed"])
    kp, vp = to_pool(kc, table, ps, n_pages), to_pool(vc, table, ps, n_pages)
    kcd, vcd, kpd, vpd = kc.to(dev), vc.to(dev), kp.to(dev), vp.to(dev)
    lens = torch.tensor(prior, dtype=torch.int32, device=dev) if case["prior"] else None
    scale = 1.0 / math.sqrt(D)
    kw = dict(rope_frac=0.25, rope_theta=1e6, scale=scale, seq_lens_before=lens)
    out_c = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    out_p = torch.full_like(out_c, float("nan"))
    lse_c = torch.full((B, Hq, S), float("nan"), dtype=torch.float32, device=dev)
    lse_p = torch.full_like(lse_c, float("nan"))
    native.gemma_attn_prefill(q.to(dev), k.to(dev), v.to(dev), kcd, vcd, window=0, out=out_c, lse=lse_c, **kw)
    native.gemma_attn_prefill_paged(q.to(dev), k.to(dev), v.to(dev), kpd, vpd, table.to(dev), out=out_p, lse=lse_p,
                                    **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(bits(out_p), bits(out_c))
    assert torch.equal(lse_p.view(torch.int32), lse_c.view(torch.int32))
    assert torch.equal(bits(from_pool(kpd.cpu(), table, ps)), bits(kcd.cpu()))
    assert torch.equal(bits(from_pool(vpd.cpu(), table, ps)), bits(vcd.cpu()))
    free = ~owned_mask(table, n_pages)
    assert (kpd.cpu()[free] == SENTINEL).all() and (vpd.cpu()[free] == SENTINEL).all()
    if kernel == "single" and case["seed"] == 412:
        rows = np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in (0, 1, S // 2, S - 1)],
                        dtype=np.int32)
        kl = torch.zeros((B, max(prior) + S, Hkv, D), dtype=torch.bfloat16)
        vl = torch.zeros_like(kl)
        for b in range(B):
            kl[b, :prior[b]] = kc[b, :, :prior[b]].permute(1, 0, 2)
            vl[b, :prior[b]] = vc[b, :, :prior[b]].permute(1, 0, 2)
            kl[b, prior[b]:prior[b] + S] = k[b]
            vl[b, prior[b]:prior[b] + S] = v[b]
        ref, _ = oracle.attention(to_bits(q), to_bits(kl), to_bits(vl), q_pos0=prior,
                                  n_keys=[p + S for p in prior], rot_from=prior, window=0, rope_frac=0.25,
                                  theta=1e6, scale=scale, rows=rows)
        got = out_p[rows[:, 0], rows[:, 2], rows[:, 1]].float().cpu().double().numpy()
        assert_close(got, ref, what="paged prefill")


def test_page_outside_the_pool_is_reported():
    """A table entry naming no page of the pool: the call reports
    GEMMA_ERR_DEVICE_RANGE, writes nothing there, and the context stays usable."""
    dev = torch.device("cuda")
    B, Hq, Hkv, D, ps = 1, 8, 1, 512, 128
    g = synth.generator(421)
    pps, n_pages = 4, 6
    pool = torch.full((n_pages, Hkv, ps, D), SENTINEL, dtype=torch.bfloat16, device=dev)
    vpool = pool.clone()
    table = torch.tensor([[0, 1, 7, 2]], dtype=torch.int32, device=dev)  # page 7 is outside the pool
    q = synth.randn_bf16((B, Hq, D), g).to(dev)
    kn = synth.randn_bf16((B, Hkv, D), g).to(dev)
    vn = synth.randn_bf16((B, Hkv, D), g).to(dev)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
    sl = torch.tensor([300], dtype=torch.int32, device=dev)  # position 299 is in table entry 2
    native.gemma_attn_decode_paged(q, kn, vn, pool, vpool, table, seq_lens=sl, max_seq_len=300, rope_frac=0.25,
                                   rope_theta=1e6, scale=0.044, out=out)
    assert native.gemma_attn_sync_status() == native.GEMMA_ERR_DEVICE_RANGE
    assert (pool.cpu() == SENTINEL).all()
    # the context still works
    table[0, 2] = 3
    native.gemma_attn_decode_paged(q, kn, vn, pool, vpool, table, seq_lens=sl, max_seq_len=300, rope_frac=0.25,
                                   rope_theta=1e6, scale=0.044, out=out)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.isfinite(out.float()).all()


# ------------------------------------------------------------- int8 pools
def int8_pool_from(cache, table, ps, n_pages, dev):
    """An Int8KVCache pool (n_pages "sequences" of ps rows) holding, page by
    page, the rows of a contiguous Int8KVCache; other pages hold 0xAB."""
    B, Hkv, cap, D = cache.shape
    pool = native.Int8KVCache(n_pages, Hkv, ps, D, dev, fill=0xAB)
    codes, params = cache.codes.cpu(), cache.params.cpu()
    pc, pp = pool.codes.cpu(), pool.params.cpu()
    for b in range(B):
        for p in range(table.shape[1]):
            pc[int(table[b, p])] = codes[b, :, p * ps:(p + 1) * ps]
            pp[int(table[b, p])] = params[b, :, p * ps:(p + 1) * ps]
    pool.codes.copy_(pc)
    pool.params.copy_(pp)
    return pool


def assert_int8_pool_matches(pool, cache, table, ps, n_pages):
    pc, pp = pool.codes.cpu(), pool.params.cpu()
    assert torch.equal(from_pool(pc, table, ps), cache.codes.cpu())
    assert torch.equal(from_pool(pp, table, ps).view(torch.int32), cache.params.cpu().view(torch.int32))
    free = ~owned_mask(table, n_pages)
    assert (pc[free] == 0xAB).all()


def seeded_int8_cache(oracle, B, Hkv, cap, D, g, dev):
    """A contiguous int8 cache holding the oracle's quantization of seeded rows."""
    c = native.Int8KVCache(B, Hkv, cap, D, dev)
    codes, lo, step = oracle.quantize_rows_u8(to_bits(synth.randn_bf16((B, Hkv, cap, D), g)))
    c.codes.copy_(torch.from_numpy(codes))
    c.params.copy_(torch.from_numpy(np.stack([lo, step], axis=-1)))
    return c


@pytest.mark.parametrize("keqv", [False, True], ids=["kv", "keqv"])
def test_decode_paged_int8_matches_contiguous(oracle, keqv):
    dev = torch.device("cuda")
    lens, Hq, Hkv, D, ps = [1, 300, 4097, 129], 32, 4, 512, 256
    B = len(lens)
    g = synth.generator(421)
    pps = (max(lens) + ps - 1) // ps + 1
    cap, n_pages = pps * ps, B * pps + 3
    kc = seeded_int8_cache(oracle, B, Hkv, cap, D, g, dev)
    vc = kc if keqv else seeded_int8_cache(oracle, B, Hkv, cap, D, g, dev)
    table = make_table(B, pps, n_pages, 421)
    kp = int8_pool_from(kc, table, ps, n_pages, dev)
    vp = kp if keqv else int8_pool_from(vc, table, ps, n_pages, dev)
    q = synth.randn_bf16((B, Hq, D), g).to(dev)
    kn = synth.randn_bf16((B, Hkv, D), g).to(dev)
    vn = None if keqv else synth.randn_bf16((B, Hkv, D), g).to(dev)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    kw = dict(seq_lens=sl, max_seq_len=max(lens), rope_frac=0.25, rope_theta=1e6, scale=1 / math.sqrt(D),
              flags=native.GEMMA_F_KEQV if keqv else 0)
    out_c = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    out_p = torch.full_like(out_c, float("nan"))
    native.gemma_attn_decode(q, kn, vn, kc, None if keqv else vc, window=0, out=out_c, **kw)
    native.gemma_attn_decode_paged(q, kn, vn, kp, None if keqv else vp, table.to(dev), out=out_p, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(bits(out_p), bits(out_c))
    assert_int8_pool_matches(kp, kc, table, ps, n_pages)
    if not keqv:
        assert_int8_pool_matches(vp, vc, table, ps, n_pages)


@pytest.mark.parametrize("prior", [None, [700, 0, 129]], ids=["fresh", "after_cached"])
def test_prefill_paged_int8_matches_contiguous(oracle, prior):
    dev = torch.device("cuda")
    B, S, Hq, Hkv, D, ps = 3, 200, 8, 1, 512, 128
    before = prior or [0] * B
    g = synth.generator(422)
    pps = (max(before) + S + ps - 1) // ps + 1
    cap, n_pages = pps * ps, B * pps + 2
    kc = seeded_int8_cache(oracle, B, Hkv, cap, D, g, dev)
    vc = seeded_int8_cache(oracle, B, Hkv, cap, D, g, dev)
    table = make_table(B, pps, n_pages, 422)
    kp = int8_pool_from(kc, table, ps, n_pages, dev)
    vp = int8_pool_from(vc, table, ps, n_pages, dev)
    q = synth.randn_bf16((B, S, Hq, D), g).to(dev)
    k = synth.randn_bf16((B, S, Hkv, D), g).to(dev)
    v = synth.randn_bf16((B, S, Hkv, D), g).to(dev)
    lens = torch.tensor(prior, dtype=torch.int32, device=dev) if prior else None
    kw = dict(rope_frac=0.25, rope_theta=1e6, scale=1 / math.sqrt(D), seq_lens_before=lens)
    out_c = torch.full((B, S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    out_p = torch.full_like(out_c, float("nan"))
    native.gemma_attn_prefill(q, k, v, kc, vc, window=0, out=out_c, **kw)
    native.gemma_attn_prefill_paged(q, k, v, kp, vp, table.to(dev), out=out_p, **kw)
    assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
    assert torch.equal(bits(out_p), bits(out_c))
    assert_int8_pool_matches(kp, kc, table, ps, n_pages)
    assert_int8_pool_matches(vp, vc, table, ps, n_pages)
