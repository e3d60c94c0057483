"""gemma_attn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (a plugin inside a runtime that owns all device
memory and gives it no allocator, or a latency-critical loop that cannot
afford cudaMalloc). Its split-K scratch is the library's fixed 32 MiB array.

The test calls it through the C ABI twice in a row, with different inputs,
and checks each result against gemma_attn_decode given a caller-allocated
workspace. Both calls run the same kernels with the same split plan (the plan
does not depend on the workspace size), so the outputs must be bit-identical;
the second call would expose scratch left over from the first. The int8 case
goes through the Python binding's cache-kind detection. The file is named to
be collected last, and it passes both alone in a fresh process and after the
other tests.
"""
import math

import pytest
import torch

from hybrid_local_global_b200 import native, synth

pytestmark = pytest.mark.gpu


def _case(seed, lens, Hq, Hkv, D, W, frac, theta, int8=False):
    dev = torch.device("cuda")
    g = synth.generator(seed, "cuda")
    B = len(lens)
    max_len = max(lens)
    cap = W if W else max_len
    if int8:
        kc = synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, cap, D, dev), g)
        vc = synth.fill_int8_cache_(native.Int8KVCache(B, Hkv, cap, D, dev), g)
    else:
        kc = synth.randn_bf16((B, Hkv, cap, D), g, "cuda")
        vc = synth.randn_bf16((B, Hkv, cap, D), g, "cuda")
    q = synth.randn_bf16((B, Hq, D), g, "cuda")
    kn = synth.randn_bf16((B, Hkv, D), g, "cuda")
    vn = synth.randn_bf16((B, Hkv, D), g, "cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    kw = dict(seq_lens=sl, max_seq_len=max_len, window=W, rope_frac=frac, rope_theta=theta,
              scale=1.0 / math.sqrt(D))
    return (q, kn, vn, kc, vc), kw


def _bits(t):
    return t.view(torch.int16)


def _clone_cache(c):
    if isinstance(c, native.Int8KVCache):
        d = native.Int8KVCache(*c.shape, c.device)
        d.buf.copy_(c.buf)
        return d
    return c.clone()


def _cache_bytes(c):
    return c.buf if isinstance(c, native.Int8KVCache) else _bits(c)


@pytest.mark.parametrize("shape", [
    dict(lens=[3000, 9001, 17, 12000], Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6),
    dict(lens=[5000, 700, 1024], Hq=32, Hkv=16, D=256, W=1024, frac=1.0, theta=1e4),
    dict(lens=[4000, 33, 2049], Hq=32, Hkv=4, D=512, W=0, frac=0.25, theta=1e6, int8=True),
], ids=["global", "local", "global_int8"])
def test_noalloc_decode_matches_workspace_decode_twice(shape):
    for call, seed in enumerate((301, 302)):
        (q, kn, vn, kc, vc), kw = _case(seed, **shape)
        need = native.gemma_attn_decode_workspace_size(q.shape[0], q.shape[1], kc.shape[1], q.shape[2],
                                                       kw["window"], kw["max_seq_len"])
        assert 0 < need <= native.NOALLOC_SCRATCH_BYTES
        ref = torch.empty_like(q)
        kc_ref, vc_ref = _clone_cache(kc), _clone_cache(vc)
        native.gemma_attn_decode(q, kn, vn, kc_ref, vc_ref, out=ref, **kw)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        out = torch.full_like(q, float("nan"))
        native.gemma_attn_decode_noalloc(q, kn, vn, kc, vc, out=out, **kw)
        assert native.gemma_attn_sync_status() == 0, native.gemma_last_error()
        # same kernels, same split plan: bit-identical outputs
        assert torch.equal(_bits(out), _bits(ref)), "no-alloc decode differs, call %d" % (call + 1)
        # the cache append is the same operation
        assert torch.equal(_cache_bytes(kc), _cache_bytes(kc_ref))
        assert torch.equal(_cache_bytes(vc), _cache_bytes(vc_ref))


def test_noalloc_decode_rejects_more_scratch_than_it_has():
    dev = torch.device("cuda")
    B, Hq, Hkv, D, L = 64, 32, 4, 512, 131072
    need = native.gemma_attn_decode_workspace_size(B, Hq, Hkv, D, 0, L)
    assert need > native.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, Hq, D), dtype=torch.bfloat16, device=dev)
    kn = torch.zeros((B, Hkv, D), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((1, 1, 1, D), dtype=torch.bfloat16, device=dev)  # never touched
    sl = torch.full((B,), L, dtype=torch.int32, device=dev)
    rc = native._decode_noalloc(native._ptr(q), native._ptr(kn), native._ptr(kn), native._ptr(kc),
                                native._ptr(kc), L, native._ptr(sl), L, B, 0, Hq, Hkv, D, 0.25, 1e6,
                                0.05, native._ptr(q), 0, None)
    assert rc == native.GEMMA_ERR_CAPACITY
    assert "scratch" in native.gemma_last_error()
    assert native.gemma_attn_sync_status() == 0
