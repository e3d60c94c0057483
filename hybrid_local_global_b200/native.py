"""ctypes binding of ``libgemma_attn.so`` -- argument marshalling only.

Every function carries the name of the C entry point it calls (declared in
``include/gemma_attn.h``). Tensors are torch CUDA tensors; their device
pointers, the shapes read off them and the current CUDA stream are passed
through unchanged. There is no fallback: if the shared library is missing
the import fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgemma_attn.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        "libgemma_attn.so is not built (run `python -m hybrid_local_global_b200.build`); "
        "there is no fallback implementation")
_lib = ctypes.CDLL(_LIB_PATH)
LIB_PATH = _LIB_PATH

GEMMA_OK = 0
GEMMA_ERR_INVALID_ARG = 1
GEMMA_ERR_UNSUPPORTED = 2
GEMMA_ERR_SHARE_MISMATCH = 3
GEMMA_ERR_CAPACITY = 4
GEMMA_ERR_CUDA = 5
GEMMA_ERR_DEVICE_TIMEOUT = 6
GEMMA_ERR_DEVICE_RANGE = 7
GEMMA_F_SHARED = 1
GEMMA_F_KEQV = 2  # K = V on a global layer: no v_new, values read from the key cache
GEMMA_F_KV_INT8 = 4  # int8 KV cache (Int8KVCache buffers); added automatically for those
GEMMA_F_SOURCE_WINDOW = 8  # shared local layer after cached tokens: attend to the source call's window

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t


class gemma_kv_desc(ctypes.Structure):
    _fields_ = [("k_cache", _P), ("v_cache", _P), ("layer", _I), ("cache_cap", _I),
                ("window", _I), ("n_kv_heads", _I), ("head_dim", _I), ("rope_frac", _F),
                ("rope_theta", _F), ("shared_from", _I), ("k_eq_v", _I), ("kv_int8", _I)]


def _sig(name, restype, argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = argtypes
    return f


_prefill_ws = _sig("gemma_attn_prefill_workspace_size", _SZ, [_I, _I, _I, _I, _I, _I])
_prefill_ws_cached = _sig("gemma_attn_prefill_workspace_size_cached", _SZ,
                          [_I, _I, _I, _I, _I, _I, _I, ctypes.c_uint])
_prefill = _sig("gemma_attn_prefill", _I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                           _F, _F, _F, _P, _P, _P, _SZ, ctypes.c_uint, _P])
_decode_ws = _sig("gemma_attn_decode_workspace_size", _SZ, [_I, _I, _I, _I, _I, _I])
_decode = _sig("gemma_attn_decode", _I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                         _F, _F, _F, _P, _P, _SZ, ctypes.c_uint, _P])
_bind = _sig("gemma_kv_share_bind", _I, [ctypes.POINTER(gemma_kv_desc), ctypes.POINTER(gemma_kv_desc)])
_sched = _sig("gemma_layer_schedule", _I, [_I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)])
_ranges = _sig("gemma_attn_visible_ranges", _I, [_P, _I, _I, _I, _P, _P])
_sync = _sig("gemma_attn_sync_status", _I, [_P])
_last = _sig("gemma_last_error", ctypes.c_char_p, [])
_wait = _sig("gemma_attn_set_wait_limit", _I, [ctypes.c_longlong])
_drop = _sig("gemma_attn_debug_drop_next_copy", _I, [_I])
_kv_bytes = _sig("gemma_kv_cache_bytes", _SZ, [_I, _I, _I, _I, ctypes.c_uint])
_prefill_paged = _sig("gemma_attn_prefill_paged", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _I, _I,
                                                       _I, _F, _F, _F, _P, _P, _P, _SZ, ctypes.c_uint, _P])
_decode_paged = _sig("gemma_attn_decode_paged", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _I, _I, _I,
                                                     _F, _F, _F, _P, _P, _SZ, ctypes.c_uint, _P])
_kv_codes = _sig("gemma_kv_codes_bytes", _SZ, [_I, _I, _I, _I])
_multi_ws = _sig("gemma_attn_decode_multi_workspace_size", _SZ, [_I, _I, _I, _I, _I, _I, _I, _I, ctypes.c_uint])
_multi = _sig("gemma_attn_decode_multi", _I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I,
                                              _F, _F, _F, _P, _P, _SZ, ctypes.c_uint, _P])
_multi_paged = _sig("gemma_attn_decode_multi_paged", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _I, _I,
                                                          _I, _I, _F, _F, _F, _P, _P, _SZ, ctypes.c_uint, _P])

EXPORTED = ["gemma_attn_prefill_workspace_size", "gemma_attn_prefill",
            "gemma_attn_decode_workspace_size", "gemma_attn_decode", "gemma_kv_share_bind",
            "gemma_layer_schedule", "gemma_attn_visible_ranges", "gemma_attn_sync_status",
            "gemma_last_error", "gemma_attn_set_wait_limit", "gemma_attn_debug_drop_next_copy",
            "gemma_kv_cache_bytes", "gemma_kv_codes_bytes", "gemma_attn_prefill_paged",
            "gemma_attn_decode_paged", "gemma_attn_prefill_workspace_size_cached"]


class GemmaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("gemma_attn error %d: %s" % (code, msg))
        self.code = code


def _check(rc: int) -> int:
    if rc != GEMMA_OK:
        raise GemmaError(rc, gemma_last_error())
    return rc


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def gemma_kv_cache_bytes(batch, n_kv_heads, cache_cap, head_dim, flags=0) -> int:
    return int(_kv_bytes(batch, n_kv_heads, cache_cap, head_dim, flags))


def gemma_kv_codes_bytes(batch, n_kv_heads, cache_cap, head_dim) -> int:
    return int(_kv_codes(batch, n_kv_heads, cache_cap, head_dim))


class Int8KVCache:
    """One layer's int8 K (or V) cache buffer (GEMMA_F_KV_INT8 layout):
    ``codes`` uint8 [B, Hkv, cap, D], then ``params`` float32 [B, Hkv, cap, 2]
    = (min, step) per row, a row's value being min + code * step."""

    def __init__(self, batch, n_kv_heads, cache_cap, head_dim, device, fill=0):
        n = gemma_kv_cache_bytes(batch, n_kv_heads, cache_cap, head_dim, GEMMA_F_KV_INT8)
        if n == 0:
            raise ValueError("bad int8 cache shape")
        self.shape = (batch, n_kv_heads, cache_cap, head_dim)
        self.buf = torch.full((n,), fill, dtype=torch.uint8, device=device)
        rows = batch * n_kv_heads * cache_cap
        off = gemma_kv_codes_bytes(batch, n_kv_heads, cache_cap, head_dim)
        self.codes = self.buf[:rows * head_dim].view(batch, n_kv_heads, cache_cap, head_dim)
        self.params = self.buf[off:off + rows * 8].view(torch.float32).view(batch, n_kv_heads, cache_cap, 2)
        self.device = self.buf.device

    def data_ptr(self):
        return self.buf.data_ptr()

    def numel(self):
        return self.buf.numel()


def _kv_kind(k_cache, v_cache) -> int:
    """GEMMA_F_KV_INT8 when the caches are Int8KVCache buffers, else 0; both
    caches (v_cache may be None under K = V) must be of one kind."""
    q8 = isinstance(k_cache, Int8KVCache)
    if v_cache is not None and isinstance(v_cache, Int8KVCache) != q8:
        raise TypeError("k_cache and v_cache must both be Int8KVCache buffers or both bf16 tensors")
    return GEMMA_F_KV_INT8 if q8 else 0


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bf16(t, name):
    if t is None or isinstance(t, Int8KVCache):
        return
    if t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda:
        raise TypeError("%s must be a contiguous bf16 CUDA tensor" % name)


def gemma_last_error() -> str:
    s = _last()
    return s.decode() if s else ""


def gemma_attn_prefill_workspace_size(batch, s_new, n_q_heads, n_kv_heads, head_dim, window) -> int:
    return int(_prefill_ws(batch, s_new, n_q_heads, n_kv_heads, head_dim, window))


def gemma_attn_prefill_workspace_size_cached(batch, s_new, n_q_heads, n_kv_heads, head_dim, window, cache_cap,
                                             flags=0) -> int:
    return int(_prefill_ws_cached(batch, s_new, n_q_heads, n_kv_heads, head_dim, window, cache_cap, flags))


def gemma_attn_prefill(q, k_new, v_new, k_cache, v_cache, *, window, rope_frac, rope_theta, scale,
                       out, seq_lens_before=None, lse=None, workspace=None, flags=0, stream=None):
    """q [B,S,Hq,D]; k_new/v_new [B,S,Hkv,D] (None if shared); caches [B,Hkv,cap,D]."""
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"),
                 (v_cache, "v_cache"), (out, "out")):
        _bf16(t, n)
    B, S, Hq, D = q.shape
    _, Hkv, cap, _ = k_cache.shape
    flags |= _kv_kind(k_cache, v_cache)
    if workspace is None:
        n = (gemma_attn_prefill_workspace_size_cached(B, S, Hq, Hkv, D, window, cap, flags)
             if seq_lens_before is not None or flags & GEMMA_F_SHARED
             else gemma_attn_prefill_workspace_size(B, S, Hq, Hkv, D, window))
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    return _check(_prefill(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), cap,
                           _ptr(seq_lens_before), B, S, window, Hq, Hkv, D, rope_frac, rope_theta,
                           scale, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), flags,
                           _stream(stream)))


def gemma_attn_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, window, max_seq_len) -> int:
    return int(_decode_ws(batch, n_q_heads, n_kv_heads, head_dim, window, max_seq_len))


def gemma_attn_decode(q, k_new, v_new, k_cache, v_cache, *, seq_lens, max_seq_len, window,
                      rope_frac, rope_theta, scale, out, workspace=None, flags=0, stream=None):
    """q [B,Hq,D]; k_new/v_new [B,Hkv,D] (None if shared); caches [B,Hkv,cap,D];
    seq_lens int32 [B] on the device (length including the new token)."""
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"),
                 (v_cache, "v_cache"), (out, "out")):
        _bf16(t, n)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    B, Hq, D = q.shape
    _, Hkv, cap, _ = k_cache.shape
    flags |= _kv_kind(k_cache, v_cache)
    if workspace is None:
        n = gemma_attn_decode_workspace_size(B, Hq, Hkv, D, window, max_seq_len)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    return _check(_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), cap,
                          _ptr(seq_lens), max_seq_len, B, window, Hq, Hkv, D, rope_frac,
                          rope_theta, scale, _ptr(out), _ptr(workspace), workspace.numel(), flags,
                          _stream(stream)))


def gemma_attn_decode_multi_workspace_size(batch, tokens, n_q_heads, n_kv_heads, head_dim, window, max_seq_len,
                                           cache_cap, flags=0) -> int:
    return int(_multi_ws(batch, tokens, n_q_heads, n_kv_heads, head_dim, window, max_seq_len, cache_cap, flags))


def gemma_attn_decode_multi(q, k_new, v_new, k_cache, v_cache, *, seq_lens, max_seq_len, window,
                            rope_frac, rope_theta, scale, out, workspace=None, flags=0, stream=None):
    """q [B,T,Hq,D]; k_new/v_new [B,T,Hkv,D] (None if shared); caches [B,Hkv,cap,D];
    seq_lens int32 [B] on the device (length including the T new tokens)."""
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"),
                 (v_cache, "v_cache"), (out, "out")):
        _bf16(t, n)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    B, T, Hq, D = q.shape
    _, Hkv, cap, _ = k_cache.shape
    flags |= _kv_kind(k_cache, v_cache)
    if workspace is None:
        n = gemma_attn_decode_multi_workspace_size(B, T, Hq, Hkv, D, window, max_seq_len, cap, flags)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    return _check(_multi(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), cap,
                         _ptr(seq_lens), max_seq_len, B, T, window, Hq, Hkv, D, rope_frac,
                         rope_theta, scale, _ptr(out), _ptr(workspace), workspace.numel(), flags,
                         _stream(stream)))


def _paged_args(k_pool, page_table):
    if page_table.dtype != torch.int32 or not page_table.is_cuda or page_table.dim() != 2:
        raise TypeError("page_table must be an int32 CUDA tensor [batch, pages_per_seq]")
    n_pages, Hkv, page_size, _ = k_pool.shape
    return n_pages, Hkv, page_size, page_table.shape[1]


def gemma_attn_prefill_paged(q, k_new, v_new, k_pool, v_pool, page_table, *, rope_frac, rope_theta, scale, out,
                             seq_lens_before=None, lse=None, workspace=None, flags=0, stream=None):
    """Global layer on a paged cache: pools [n_pages, Hkv, page_size, D]
    (bf16, or Int8KVCache(n_pages, Hkv, page_size, D) buffers), page_table
    int32 [B, pages_per_seq] on the device."""
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_pool, "k_pool"), (v_pool, "v_pool"),
                 (out, "out")):
        _bf16(t, n)
    B, S, Hq, D = q.shape
    n_pages, Hkv, ps, pps = _paged_args(k_pool, page_table)
    flags |= _kv_kind(k_pool, v_pool)
    if workspace is None:
        n = (gemma_attn_prefill_workspace_size_cached(B, S, Hq, Hkv, D, 0, ps * pps, flags)
             if seq_lens_before is not None or flags & GEMMA_F_SHARED
             else gemma_attn_prefill_workspace_size(B, S, Hq, Hkv, D, 0))
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    return _check(_prefill_paged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(page_table),
                                 ps, pps, n_pages, _ptr(seq_lens_before), B, S, Hq, Hkv, D, rope_frac, rope_theta,
                                 scale, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), flags,
                                 _stream(stream)))


def gemma_attn_decode_paged(q, k_new, v_new, k_pool, v_pool, page_table, *, seq_lens, max_seq_len, rope_frac,
                            rope_theta, scale, out, workspace=None, flags=0, stream=None):
    """Global-layer decode on a paged cache (see gemma_attn_prefill_paged)."""
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_pool, "k_pool"), (v_pool, "v_pool"),
                 (out, "out")):
        _bf16(t, n)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    B, Hq, D = q.shape
    n_pages, Hkv, ps, pps = _paged_args(k_pool, page_table)
    flags |= _kv_kind(k_pool, v_pool)
    if workspace is None:
        n = gemma_attn_decode_workspace_size(B, Hq, Hkv, D, 0, max_seq_len)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    return _check(_decode_paged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(page_table),
                                ps, pps, n_pages, _ptr(seq_lens), max_seq_len, B, Hq, Hkv, D, rope_frac,
                                rope_theta, scale, _ptr(out), _ptr(workspace), workspace.numel(), flags,
                                _stream(stream)))


def gemma_attn_decode_multi_paged(q, k_new, v_new, k_pool, v_pool, page_table, *, seq_lens, max_seq_len, rope_frac,
                                  rope_theta, scale, out, workspace=None, flags=0, stream=None):
    """Multi-token decode of a global layer on a paged cache: q [B,T,Hq,D],
    k_new/v_new [B,T,Hkv,D]; pools and page table as gemma_attn_prefill_paged."""
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_pool, "k_pool"), (v_pool, "v_pool"),
                 (out, "out")):
        _bf16(t, n)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    B, T, Hq, D = q.shape
    n_pages, Hkv, ps, pps = _paged_args(k_pool, page_table)
    flags |= _kv_kind(k_pool, v_pool)
    if workspace is None:
        n = gemma_attn_decode_multi_workspace_size(B, T, Hq, Hkv, D, 0, max_seq_len, ps * pps, flags)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    return _check(_multi_paged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(page_table),
                               ps, pps, n_pages, _ptr(seq_lens), max_seq_len, B, T, Hq, Hkv, D, rope_frac,
                               rope_theta, scale, _ptr(out), _ptr(workspace), workspace.numel(), flags,
                               _stream(stream)))


def gemma_kv_share_bind(dst: gemma_kv_desc, src: gemma_kv_desc) -> int:
    return _check(_bind(ctypes.byref(dst), ctypes.byref(src)))


def gemma_layer_schedule(n_layers: int, ratio: int, n_shared: int = 0):
    g = (_I * n_layers)()
    s = (_I * n_layers)()
    _check(_sched(n_layers, ratio, n_shared, g, s))
    return [bool(x) for x in g], [int(x) for x in s]


def gemma_attn_visible_ranges(batch, s_new, window, ranges, seq_lens_before=None, stream=None):
    if ranges.dtype != torch.int32 or not ranges.is_cuda or ranges.numel() < batch * s_new * 3:
        raise TypeError("ranges must be an int32 CUDA tensor of batch*s_new*3 elements")
    return _check(_ranges(_ptr(seq_lens_before), batch, s_new, window, _ptr(ranges), _stream(stream)))


def gemma_attn_sync_status(stream=None) -> int:
    """Returns the status code (does not raise)."""
    return int(_sync(_stream(stream)))


def gemma_attn_set_wait_limit(max_ns: int) -> int:
    return _check(_wait(max_ns))


def gemma_attn_debug_drop_next_copy(enable: bool) -> int:
    return _check(_drop(int(bool(enable))))


GEMMA_KERNEL_PREFILL_ROPE = 0
GEMMA_KERNEL_PREFILL_ATTN = 1
GEMMA_KERNEL_DECODE_APPEND = 2
GEMMA_KERNEL_DECODE_SPLIT = 3
GEMMA_KERNEL_DECODE_COMBINE = 4
KERNEL_NAMES = {0: "prefill_rope", 1: "prefill_attn", 2: "decode_append", 3: "decode_split",
                4: "decode_combine"}

_prof = _sig("gemma_attn_profile", _I, [_I])
_prof_read = _sig("gemma_attn_profile_read", _I, [_I, ctypes.POINTER(ctypes.c_double),
                                                  ctypes.POINTER(ctypes.c_longlong)])
_tinfo = _sig("gemma_attn_debug_timeout_info", _I, [ctypes.POINTER(ctypes.c_longlong)])
EXPORTED += ["gemma_attn_profile", "gemma_attn_profile_read", "gemma_attn_debug_timeout_info"]


def gemma_attn_debug_timeout_info():
    """-> list of 8 ints describing the first bounded wait that gave up (cleared on read)."""
    buf = (ctypes.c_longlong * 8)()
    _check(_tinfo(buf))
    return [int(x) for x in buf]


def gemma_attn_profile(enable: bool) -> int:
    return _check(_prof(int(bool(enable))))


def gemma_attn_profile_read(kernel: int):
    """-> (total device ms, launches) of one kernel kind since profiling began."""
    ms = ctypes.c_double()
    n = ctypes.c_longlong()
    _check(_prof_read(kernel, ctypes.byref(ms), ctypes.byref(n)))
    return float(ms.value), int(n.value)


_decode_noalloc = _sig("gemma_attn_decode_noalloc", _I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I,
                                                         _I, _F, _F, _F, _P, ctypes.c_uint, _P])
EXPORTED += ["gemma_attn_decode_noalloc", "gemma_attn_decode_multi_workspace_size", "gemma_attn_decode_multi",
             "gemma_attn_decode_multi_paged"]
NOALLOC_SCRATCH_BYTES = 32 << 20


def gemma_attn_decode_noalloc(q, k_new, v_new, k_cache, v_cache, *, seq_lens, max_seq_len, window,
                              rope_frac, rope_theta, scale, out, flags=0, stream=None):
    """gemma_attn_decode for callers that cannot allocate device memory: the
    split-K scratch is the library's fixed 32 MiB array (shared by all calls;
    overlapping calls race). Same arguments as gemma_attn_decode without the
    workspace."""
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"),
                 (v_cache, "v_cache"), (out, "out")):
        _bf16(t, n)
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda:
        raise TypeError("seq_lens must be an int32 CUDA tensor")
    B, Hq, D = q.shape
    _, Hkv, cap, _ = k_cache.shape
    flags |= _kv_kind(k_cache, v_cache)
    return _check(_decode_noalloc(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), cap,
                                  _ptr(seq_lens), max_seq_len, B, window, Hq, Hkv, D, rope_frac,
                                  rope_theta, scale, _ptr(out), flags, _stream(stream)))
