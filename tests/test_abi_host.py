"""Host-side checks of libgemma_attn.so that need no GPU: the library loads
and exports every entry point include/gemma_attn.h declares; the layer
schedule and share map match the oracle; share binding and argument
validation return the documented codes before touching any pointer."""
import ctypes
import os
import re

import pytest

from hybrid_local_global_b200 import native

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "gemma_attn.h")
FAKE = 0x10000  # never dereferenced: validation fails before any device work


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(gemma_\w+)\s*\(", src, flags=re.M)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 11, names
    lib = ctypes.CDLL(native.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(native.EXPORTED) == names


@pytest.mark.parametrize("n,r,ns", [(5, 4, 0), (6, 5, 2), (12, 5, 2), (35, 4, 0), (42, 5, 3),
                                    (60, 5, 10), (42, 4, 0), (8, 0, 3), (1, 5, 0), (1, 0, 1)])
def test_schedule_matches_oracle(oracle, n, r, ns):
    g, s = native.gemma_layer_schedule(n, r, ns)
    assert g == oracle.layer_schedule(n, r)
    assert s == [oracle.share_source(n, r, ns, l) for l in range(n)]


def test_schedule_rejects_bad_arguments():
    for args in ((0, 4, 0), (5, -1, 0), (5, 4, 6), (5, 4, -1)):
        with pytest.raises(native.GemmaError) as e:
            native.gemma_layer_schedule(*args)
        assert e.value.code == native.GEMMA_ERR_INVALID_ARG


def _desc(layer, window, cap, hkv=4, d=512, frac=0.25, theta=1e6, k=FAKE, v=FAKE + 0x1000, keqv=0):
    x = native.gemma_kv_desc()
    x.k_cache, x.v_cache, x.layer, x.cache_cap, x.window = k, v, layer, cap, window
    x.n_kv_heads, x.head_dim, x.rope_frac, x.rope_theta, x.shared_from = hkv, d, frac, theta, -1
    x.k_eq_v = keqv
    return x


def test_share_bind_aliases_and_resolves_chains():
    src = _desc(5, 0, 4096)
    dst = _desc(11, 0, 4096, k=None, v=None)
    native.gemma_kv_share_bind(dst, src)
    assert dst.k_cache == src.k_cache and dst.v_cache == src.v_cache and dst.shared_from == 5
    dst2 = _desc(13, 0, 4096, k=None, v=None)
    native.gemma_kv_share_bind(dst2, dst)           # chain resolves to the root
    assert dst2.shared_from == 5 and dst2.k_cache == src.k_cache


def test_share_bind_k_equals_v():
    """A K = V source has no value cache; its sharer aliases the key cache,
    and a K = V layer only aliases a K = V layer."""
    src = _desc(5, 0, 4096, v=None, keqv=1)
    dst = _desc(11, 0, 4096, k=None, v=None, keqv=1)
    native.gemma_kv_share_bind(dst, src)
    assert dst.k_cache == src.k_cache and not dst.v_cache and dst.shared_from == 5
    for a, b in ((_desc(5, 0, 4096), _desc(11, 0, 4096, k=None, v=None, keqv=1)),
                 (_desc(5, 0, 4096, v=None, keqv=1), _desc(11, 0, 4096, k=None, v=None))):
        with pytest.raises(native.GemmaError) as e:
            native.gemma_kv_share_bind(b, a)
        assert e.value.code in (native.GEMMA_ERR_SHARE_MISMATCH, native.GEMMA_ERR_INVALID_ARG)


@pytest.mark.parametrize("change", ["type", "window", "heads", "dim", "frac", "theta", "order", "cap", "int8"])
def test_share_bind_rejects_mismatch(change):
    src = _desc(3, 1024, 1024, hkv=16, d=256, frac=1.0, theta=1e4)
    kw = dict(layer=4, window=1024, cap=1024, hkv=16, d=256, frac=1.0, theta=1e4, k=None, v=None)
    if change == "type":
        kw.update(window=0, cap=4096)
    elif change == "window":
        kw.update(window=512, cap=512)
    elif change == "heads":
        kw.update(hkv=8)
    elif change == "dim":
        kw.update(d=512)
    elif change == "frac":
        kw.update(frac=0.25)
    elif change == "theta":
        kw.update(theta=1e6)
    elif change == "order":
        kw.update(layer=2)
    elif change == "cap":
        kw.update(cap=2048)
    dst = _desc(**kw)
    if change == "int8":
        dst.kv_int8 = 1
    with pytest.raises(native.GemmaError) as e:
        native.gemma_kv_share_bind(dst, src)
    assert e.value.code == native.GEMMA_ERR_SHARE_MISMATCH
    assert not dst.k_cache and dst.shared_from == -1  # unchanged


def _prefill_raw(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, cap=512, lens=None, B=1, S=16, W=512,
             Hq=8, Hkv=4, D=256, frac=1.0, theta=1e4, scale=0.0625, out=FAKE, lse=None,
             ws=FAKE, wsb=1 << 30, flags=0)
    a.update(over)
    return native._prefill(a["q"], a["k"], a["v"], a["kc"], a["vc"], a["cap"], a["lens"], a["B"],
                           a["S"], a["W"], a["Hq"], a["Hkv"], a["D"], a["frac"], a["theta"],
                           a["scale"], a["out"], a["lse"], a["ws"], a["wsb"], a["flags"], None)


def _decode_raw(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, cap=4096, lens=FAKE, maxlen=4096, B=2, W=0,
             Hq=32, Hkv=4, D=512, frac=0.25, theta=1e6, scale=0.044, out=FAKE, ws=FAKE,
             wsb=1 << 30, flags=0)
    a.update(over)
    return native._decode(a["q"], a["k"], a["v"], a["kc"], a["vc"], a["cap"], a["lens"], a["maxlen"],
                          a["B"], a["W"], a["Hq"], a["Hkv"], a["D"], a["frac"], a["theta"],
                          a["scale"], a["out"], a["ws"], a["wsb"], a["flags"], None)


E = native
# the plain workspace of the prefill harness's shapes on a global layer
PLAIN_WS_GLOBAL = native.gemma_attn_prefill_workspace_size(1, 16, 8, 4, 256, 0)


@pytest.mark.parametrize("over,code", [
    (dict(Hq=6), E.GEMMA_ERR_INVALID_ARG),            # Hq not a multiple of Hkv
    (dict(Hq=64, Hkv=4), E.GEMMA_ERR_UNSUPPORTED),   # 16 q heads per KV head
    (dict(D=128), E.GEMMA_ERR_UNSUPPORTED),
    (dict(frac=1.5), E.GEMMA_ERR_INVALID_ARG),
    (dict(frac=-0.1), E.GEMMA_ERR_INVALID_ARG),
    (dict(theta=0.0), E.GEMMA_ERR_INVALID_ARG),
    (dict(W=500, cap=500), E.GEMMA_ERR_INVALID_ARG),  # window not a multiple of 16
    (dict(cap=1024), E.GEMMA_ERR_INVALID_ARG),        # local ring must hold exactly the window
    (dict(lens=FAKE, wsb=16), E.GEMMA_ERR_CAPACITY),   # chunked local prefill is accepted
    (dict(lens=FAKE, flags=1, k=None, v=None), E.GEMMA_ERR_UNSUPPORTED),  # ... but not on a shared layer
    (dict(lens=FAKE, flags=9, k=None, v=None, wsb=16), E.GEMMA_ERR_CAPACITY),  # ... unless on its source's window
    (dict(lens=FAKE, flags=8, wsb=16), E.GEMMA_ERR_CAPACITY),          # the source's own call may pass the flag
    (dict(flags=9, k=None, v=None), E.GEMMA_ERR_INVALID_ARG),          # the flag needs cached tokens
    (dict(W=0, cap=4096, lens=FAKE, flags=9, k=None, v=None), E.GEMMA_ERR_INVALID_ARG),  # ... and a local layer
    (dict(lens=FAKE, flags=13, k=None, v=None, wsb=16), E.GEMMA_ERR_CAPACITY),  # int8 shared, source window
    (dict(W=0, cap=8), E.GEMMA_ERR_CAPACITY),          # global cache shorter than the chunk
    (dict(k=None), E.GEMMA_ERR_INVALID_ARG),           # unshared layer without new keys
    (dict(flags=1), E.GEMMA_ERR_INVALID_ARG),          # shared layer with new keys
    (dict(flags=16), E.GEMMA_ERR_INVALID_ARG),         # unknown flag
    (dict(flags=4, wsb=16), E.GEMMA_ERR_CAPACITY),     # int8 KV: accepted
    (dict(flags=4, W=0, cap=4095, wsb=16), E.GEMMA_ERR_INVALID_ARG),   # int8 KV: odd capacity
    (dict(flags=4, lens=FAKE, wsb=16), E.GEMMA_ERR_CAPACITY),          # int8 KV after cached tokens: accepted
    (dict(flags=4, W=0, cap=16384, lens=FAKE, wsb=PLAIN_WS_GLOBAL), E.GEMMA_ERR_CAPACITY),  # ... whose global
                                                                        # layers need the larger workspace
    (dict(flags=5, k=None, v=None, wsb=16), E.GEMMA_ERR_CAPACITY),     # int8 KV on a shared layer: accepted
    (dict(W=0, cap=4096, flags=6, v=None, wsb=16), E.GEMMA_ERR_CAPACITY),  # int8 K = V: accepted
    (dict(flags=2, v=None), E.GEMMA_ERR_UNSUPPORTED),  # K = V on a local layer
    (dict(W=0, cap=4096, flags=2), E.GEMMA_ERR_INVALID_ARG),             # K = V with v_new
    (dict(W=0, cap=4096, flags=2, v=None, vc=FAKE + 256), E.GEMMA_ERR_INVALID_ARG),  # v_cache != k_cache
    (dict(W=0, cap=4096, flags=3, k=None, v=None, vc=None, wsb=16), E.GEMMA_ERR_CAPACITY),  # shared K = V: flags pass
    (dict(q=None), E.GEMMA_ERR_INVALID_ARG),
    (dict(q=FAKE + 8), E.GEMMA_ERR_INVALID_ARG),       # misaligned
    (dict(wsb=16), E.GEMMA_ERR_CAPACITY),
    (dict(B=0), E.GEMMA_ERR_INVALID_ARG),
])
def test_prefill_validation(over, code):
    assert _prefill_raw(**over) == code
    assert native.gemma_last_error()


@pytest.mark.parametrize("over,code", [
    (dict(lens=None), E.GEMMA_ERR_INVALID_ARG),
    (dict(maxlen=0), E.GEMMA_ERR_INVALID_ARG),
    (dict(cap=1000), E.GEMMA_ERR_CAPACITY),            # global cache < max length
    (dict(W=1024, cap=4096), E.GEMMA_ERR_INVALID_ARG),
    (dict(D=384), E.GEMMA_ERR_UNSUPPORTED),
    (dict(k=None, v=None, flags=0), E.GEMMA_ERR_INVALID_ARG),
    (dict(wsb=1024), E.GEMMA_ERR_CAPACITY),
    (dict(out=None), E.GEMMA_ERR_INVALID_ARG),
    (dict(flags=2), E.GEMMA_ERR_INVALID_ARG),                          # K = V with v_new
    (dict(flags=2, v=None, vc=FAKE + 256), E.GEMMA_ERR_INVALID_ARG),   # v_cache != k_cache
    (dict(W=1024, cap=1024, flags=2, v=None), E.GEMMA_ERR_UNSUPPORTED),
    (dict(flags=2, v=None, vc=None, wsb=1024), E.GEMMA_ERR_CAPACITY),  # K = V accepted: v_cache optional
    (dict(flags=4, wsb=1024), E.GEMMA_ERR_CAPACITY),                   # int8 KV accepted
    (dict(flags=4, cap=4097, maxlen=4097, wsb=1024), E.GEMMA_ERR_INVALID_ARG),  # int8 KV: odd capacity
    (dict(flags=5, k=None, v=None, wsb=1024), E.GEMMA_ERR_CAPACITY),   # int8 KV on a shared layer: accepted
    (dict(flags=8), E.GEMMA_ERR_INVALID_ARG),                          # the source-window flag is not for decode
    (dict(flags=16), E.GEMMA_ERR_INVALID_ARG),                         # unknown flag
])
def test_decode_validation(over, code):
    assert _decode_raw(**over) == code


def _multi_raw(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, cap=4096, lens=FAKE, maxlen=4096, B=2, T=4, W=0,
             Hq=32, Hkv=4, D=512, frac=0.25, theta=1e6, scale=0.044, out=FAKE, ws=FAKE,
             wsb=16, flags=0)
    a.update(over)
    return native._multi(a["q"], a["k"], a["v"], a["kc"], a["vc"], a["cap"], a["lens"], a["maxlen"],
                         a["B"], a["T"], a["W"], a["Hq"], a["Hkv"], a["D"], a["frac"], a["theta"],
                         a["scale"], a["out"], a["ws"], a["wsb"], a["flags"], None)


@pytest.mark.parametrize("over,code", [
    (dict(), E.GEMMA_ERR_CAPACITY),                                   # the tensor-core path: accepted
    (dict(T=0), E.GEMMA_ERR_INVALID_ARG),
    (dict(T=5000, wsb=1 << 30), E.GEMMA_ERR_INVALID_ARG),             # more new tokens than any length allows
    (dict(lens=None), E.GEMMA_ERR_INVALID_ARG),
    (dict(maxlen=0), E.GEMMA_ERR_INVALID_ARG),
    (dict(cap=1000), E.GEMMA_ERR_CAPACITY),                           # global cache < max length
    (dict(D=384), E.GEMMA_ERR_UNSUPPORTED),
    (dict(k=None, v=None), E.GEMMA_ERR_INVALID_ARG),                  # unshared layer without new keys
    (dict(flags=1), E.GEMMA_ERR_INVALID_ARG),                         # shared layer with new keys
    (dict(flags=1, k=None, v=None), E.GEMMA_ERR_CAPACITY),            # shared global: accepted
    (dict(flags=2), E.GEMMA_ERR_INVALID_ARG),                         # K = V with v_new
    (dict(flags=2, v=None, vc=None), E.GEMMA_ERR_CAPACITY),           # K = V: accepted
    (dict(q=FAKE + 8, wsb=1 << 30), E.GEMMA_ERR_INVALID_ARG),         # misaligned
    (dict(out=None, wsb=1 << 30), E.GEMMA_ERR_INVALID_ARG),
    (dict(T=17), E.GEMMA_ERR_CAPACITY),                               # 8 x 17 rows: the prefill route
    (dict(T=17, out=None, wsb=1 << 30), E.GEMMA_ERR_INVALID_ARG),     # ... which validates as prefill
    (dict(W=1024, cap=1024, Hkv=16, D=256, frac=1.0, theta=1e4), E.GEMMA_ERR_CAPACITY),  # local: accepted
    (dict(W=1024, cap=4096, Hkv=16, D=256, frac=1.0, theta=1e4, wsb=1 << 30), E.GEMMA_ERR_INVALID_ARG),
    (dict(W=1024, cap=1024, Hkv=16, D=256, frac=1.0, theta=1e4, flags=1, k=None, v=None, wsb=1 << 30),
     E.GEMMA_ERR_UNSUPPORTED),                                        # shared local after cached tokens ...
    (dict(W=1024, cap=1024, Hkv=16, D=256, frac=1.0, theta=1e4, flags=9, k=None, v=None),
     E.GEMMA_ERR_CAPACITY),                                           # ... on its source's window: routed
    (dict(flags=8, wsb=1 << 30), E.GEMMA_ERR_INVALID_ARG),            # the source-window flag on a global layer
    (dict(flags=4), E.GEMMA_ERR_CAPACITY),                            # int8: route
])
def test_decode_multi_validation(over, code):
    assert _multi_raw(**over) == code
    assert native.gemma_last_error()


def test_decode_multi_workspace_sizes():
    """The tensor-core path holds the rotated queries and fp32 split
    partials (local layers also the new tokens' rotated keys); the routed
    layers a length buffer plus the chunked-prefill workspace."""
    n = native.gemma_attn_decode_multi_workspace_size(64, 4, 32, 4, 512, 0, 131072, 131072, 0)
    assert n >= 64 * 4 * 32 * 512 * (2 + 4)
    loc = native.gemma_attn_decode_multi_workspace_size(64, 4, 32, 16, 256, 1024, 131072, 1024, 0)
    assert loc >= 64 * 4 * 32 * 256 * (2 + 4) + 64 * 4 * 16 * 256 * 2
    routed = native.gemma_attn_decode_multi_workspace_size(1, 40, 32, 16, 256, 1024, 4096, 1024, 0)  # 80 rows
    assert routed >= 256 + native.gemma_attn_prefill_workspace_size_cached(1, 40, 32, 16, 256, 1024, 1024, 0)
    shared = native.gemma_attn_decode_multi_workspace_size(1, 4, 32, 16, 256, 1024, 4096, 1024, native.GEMMA_F_SHARED)
    assert shared >= 256 + native.gemma_attn_prefill_workspace_size_cached(1, 4, 32, 16, 256, 1024, 1024, 0)
    # int8 global layers decode the tokens one at a time: the decode workspace plus one token's rows,
    # whatever the cached length (a chunked prefill would need the whole prefix in bf16)
    q8 = native.gemma_attn_decode_multi_workspace_size(2, 4, 32, 4, 512, 0, 4096, 4096, native.GEMMA_F_KV_INT8)
    assert q8 >= native.gemma_attn_decode_workspace_size(2, 32, 4, 512, 0, 4096) + 2 * (32 + 4) * 512 * 2 * 2
    big = native.gemma_attn_decode_multi_workspace_size(64, 4, 32, 4, 512, 0, 131072, 131072, native.GEMMA_F_KV_INT8)
    assert big < 1 << 30 < native.gemma_attn_prefill_workspace_size_cached(64, 4, 32, 4, 512, 0, 131072,
                                                                             native.GEMMA_F_KV_INT8)
    assert native.gemma_attn_decode_multi_workspace_size(0, 4, 32, 4, 512, 0, 4096, 4096, 0) == 0
    assert native.gemma_attn_decode_multi_workspace_size(2, 0, 32, 4, 512, 0, 4096, 4096, 0) == 0


def test_cached_prefill_workspace_sizes():
    """Only an int8 global layer after cached tokens needs more: its keys and
    values up to the capacity in bf16."""
    for W in (512, 0):
        for D, Hkv in ((256, 4), (512, 1)):
            plain = native.gemma_attn_prefill_workspace_size(2, 1024, 8, Hkv, D, W)
            assert native.gemma_attn_prefill_workspace_size_cached(2, 1024, 8, Hkv, D, W, 16384, 0) == plain
            q8 = native.gemma_attn_prefill_workspace_size_cached(2, 1024, 8, Hkv, D, W, 16384,
                                                                 native.GEMMA_F_KV_INT8)
            if W:
                assert q8 == plain
            else:
                assert q8 >= 2 * 1024 * 8 * D * 2 + 2 * (2 * 16384 * Hkv * D * 2)
    assert native.gemma_attn_prefill_workspace_size_cached(2, 1024, 8, 4, 256, 0, 0, 0) == 0


def test_workspace_sizes_cover_the_configs():
    assert native.gemma_attn_prefill_workspace_size(1, 8192, 8, 4, 256, 512) >= 8192 * 8 * 256 * 2 + 8192 * 4 * 256 * 2
    assert native.gemma_attn_prefill_workspace_size(1, 8192, 8, 1, 512, 0) >= 8192 * 8 * 512 * 2
    n = native.gemma_attn_decode_workspace_size(64, 32, 4, 512, 0, 131072)
    assert n >= 64 * 32 * 512 * 2
    assert native.gemma_attn_decode_workspace_size(0, 32, 4, 512, 0, 131072) == 0


def test_kv_cache_bytes():
    """bf16: one element per (row, dim); int8: the codes padded to 256 bytes,
    then one (min, step) float pair per row."""
    assert native.gemma_kv_cache_bytes(2, 4, 4096, 512) == 2 * 4 * 4096 * 512 * 2
    codes = native.gemma_kv_codes_bytes(2, 4, 4096, 512)
    assert codes == 2 * 4 * 4096 * 512
    assert native.gemma_kv_cache_bytes(2, 4, 4096, 512, native.GEMMA_F_KV_INT8) == codes + 2 * 4 * 4096 * 8
    assert native.gemma_kv_codes_bytes(1, 1, 2, 256) == 512
    assert native.gemma_kv_codes_bytes(1, 3, 2, 16) == 256        # 96 bytes of codes, padded
    assert native.gemma_kv_cache_bytes(1, 3, 2, 16, native.GEMMA_F_KV_INT8) == 256 + 6 * 8
    assert native.gemma_kv_cache_bytes(0, 4, 4096, 512) == 0
    assert native.gemma_kv_codes_bytes(1, 1, 0, 256) == 0


# the plain workspace of the paged prefill harness's shapes
PAGED_PLAIN_WS = native.gemma_attn_prefill_workspace_size(2, 16, 8, 1, 512, 0)


def _prefill_paged_raw(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, table=FAKE, ps=128, pps=64, npages=256, lens=None, B=2,
             S=16, Hq=8, Hkv=1, D=512, frac=0.25, theta=1e6, scale=0.044, out=FAKE, lse=None, ws=FAKE,
             wsb=1 << 30, flags=0)
    a.update(over)
    return native._prefill_paged(a["q"], a["k"], a["v"], a["kc"], a["vc"], a["table"], a["ps"], a["pps"],
                                 a["npages"], a["lens"], a["B"], a["S"], a["Hq"], a["Hkv"], a["D"], a["frac"],
                                 a["theta"], a["scale"], a["out"], a["lse"], a["ws"], a["wsb"], a["flags"], None)


def _decode_paged_raw(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kc=FAKE, vc=FAKE, table=FAKE, ps=256, pps=32, npages=64, lens=FAKE,
             maxlen=4096, B=2, Hq=32, Hkv=4, D=512, frac=0.25, theta=1e6, scale=0.044, out=FAKE, ws=FAKE,
             wsb=1 << 30, flags=0)
    a.update(over)
    return native._decode_paged(a["q"], a["k"], a["v"], a["kc"], a["vc"], a["table"], a["ps"], a["pps"],
                                a["npages"], a["lens"], a["maxlen"], a["B"], a["Hq"], a["Hkv"], a["D"], a["frac"],
                                a["theta"], a["scale"], a["out"], a["ws"], a["wsb"], a["flags"], None)


@pytest.mark.parametrize("over,code", [
    (dict(wsb=16), E.GEMMA_ERR_CAPACITY),                  # accepted
    (dict(table=None), E.GEMMA_ERR_INVALID_ARG),
    (dict(ps=100), E.GEMMA_ERR_INVALID_ARG),               # not a multiple of 128
    (dict(ps=0), E.GEMMA_ERR_INVALID_ARG),
    (dict(pps=0), E.GEMMA_ERR_INVALID_ARG),
    (dict(npages=0), E.GEMMA_ERR_INVALID_ARG),
    (dict(flags=4, wsb=16), E.GEMMA_ERR_CAPACITY),         # int8 pools accepted
    (dict(flags=4, lens=FAKE, wsb=PAGED_PLAIN_WS), E.GEMMA_ERR_CAPACITY),  # ... after cached tokens they
                                                                          # need the larger workspace
    (dict(pps=1, S=200), E.GEMMA_ERR_CAPACITY),            # chunk beyond pages_per_seq * page_size
    (dict(flags=2, v=None, vc=None, wsb=16), E.GEMMA_ERR_CAPACITY),   # K = V accepted
])
def test_prefill_paged_validation(over, code):
    assert _prefill_paged_raw(**over) == code
    assert native.gemma_last_error()


@pytest.mark.parametrize("over,code", [
    (dict(wsb=1024), E.GEMMA_ERR_CAPACITY),                # accepted
    (dict(table=None), E.GEMMA_ERR_INVALID_ARG),
    (dict(ps=192), E.GEMMA_ERR_INVALID_ARG),
    (dict(flags=4, wsb=1024), E.GEMMA_ERR_CAPACITY),      # int8 pools accepted
    (dict(pps=8), E.GEMMA_ERR_CAPACITY),                   # 8 pages of 256 < max_seq_len 4096
    (dict(flags=1, k=None, v=None, wsb=1024), E.GEMMA_ERR_CAPACITY),  # shared layer accepted
])
def test_decode_paged_validation(over, code):
    assert _decode_paged_raw(**over) == code
    assert native.gemma_last_error()


def test_binding_rejects_mixed_cache_kinds():
    """An int8 key cache with a bf16 value cache (or the reverse) would be read
    with the wrong layout: the binding refuses it before any call."""
    import torch
    i8 = native.Int8KVCache(1, 1, 16, 256, "cpu")
    bf = torch.zeros((1, 1, 16, 256), dtype=torch.bfloat16)
    assert native._kv_kind(i8, i8) == native.GEMMA_F_KV_INT8
    assert native._kv_kind(i8, None) == native.GEMMA_F_KV_INT8   # K = V
    assert native._kv_kind(bf, bf) == 0
    for k, v in ((i8, bf), (bf, i8)):
        with pytest.raises(TypeError):
            native._kv_kind(k, v)


# --------------------------------------------------------------------------- binding vs header
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_prototypes():
    """{name: (return type, [parameter types])} of every function the C
    header declares, types with names and comments stripped."""
    import re
    text = open(os.path.join(ROOT, "include", "gemma_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"#[^\n]*", " ", text)
    protos = {}
    for m in re.finditer(r"([A-Za-z_][\w\s\*]*?)\b(gemma_\w+)\s*\(([^;{}]*?)\)\s*;", text):
        ret, name, params = m.group(1), m.group(2), m.group(3)
        ret = " ".join(ret.replace("*", " * ").split())
        types = []
        for p in params.split(","):
            p = " ".join(p.replace("*", " * ").split())
            if not p or p == "void":
                continue
            words = p.split(" ")
            if words[-1] != "*":
                words = words[:-1]  # drop the parameter name
            types.append(" ".join(w for w in words if w != "const"))
        protos[name] = (ret.replace("const ", ""), types)
    return protos


def _ctype_of(c):
    """ctypes class of a C type from the header; "pointer" for any data
    pointer (void*, int32_t*, float*, double*, a struct pointer)."""
    import ctypes
    table = {"int": ctypes.c_int, "unsigned": ctypes.c_uint, "float": ctypes.c_float,
             "size_t": ctypes.c_size_t, "long long": ctypes.c_longlong, "char *": ctypes.c_char_p,
             "gemma_status": ctypes.c_int}
    if c in table:
        return table[c]
    if c.endswith("*"):
        return "pointer"
    raise AssertionError("no ctypes mapping for %r" % c)


def test_binding_signatures_match_the_header():
    """Every function native.py binds has the header's arity and argument
    types (a pointer for every pointer: void*, int32_t*, float*, double*,
    a struct pointer), and its return type."""
    import ctypes
    protos = _header_prototypes()
    bound = {f.__name__: f for f in vars(native).values() if isinstance(f, ctypes._CFuncPtr)}
    assert len(bound) >= 20
    for name, f in sorted(bound.items()):
        assert name in protos, "%s is bound but not declared in the header" % name
        ret, params = protos[name]
        assert len(f.argtypes) == len(params), "%s: %d ctypes args, header has %d" % (
            name, len(f.argtypes), len(params))
        for i, (a, c) in enumerate(zip(f.argtypes, params)):
            want = _ctype_of(c)
            if want == "pointer":
                assert a is ctypes.c_void_p or issubclass(a, ctypes._Pointer), "%s arg %d (%s): %r" % (name, i, c, a)
            else:
                assert a is want, "%s arg %d (%s): %r" % (name, i, c, a)
        assert f.restype is _ctype_of(ret), "%s returns %r, header %r" % (name, f.restype, ret)


def test_every_declared_function_is_bound_and_exported():
    protos = _header_prototypes()
    import ctypes
    bound = {f.__name__ for f in vars(native).values() if isinstance(f, ctypes._CFuncPtr)}
    assert set(protos) == bound, (sorted(set(protos) - bound), sorted(bound - set(protos)))


def test_kv_desc_struct_matches_the_header():
    import ctypes
    import re
    text = open(os.path.join(ROOT, "include", "gemma_attn.h")).read()
    body = re.search(r"typedef struct gemma_kv_desc \{(.*?)\} gemma_kv_desc;", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", " ", body, flags=re.S)
    fields = []
    for decl in body.split(";"):
        words = decl.replace("*", " * ").split()
        if words:
            fields.append((words[-1], " ".join(words[:-1])))
    got = native.gemma_kv_desc._fields_
    assert [n for n, _ in fields] == [n for n, _ in got]
    for (n, c), (_, t) in zip(fields, got):
        want = _ctype_of(c)
        assert (t is ctypes.c_void_p) if want == "pointer" else (t is want), (n, c, t)
