"""fp64 CPU oracle for interleaved local/global causal GQA attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The product (``hybrid_local_global_b200``) never imports it and
shares no code with it; the arithmetic lives in ``hlg_oracle.c`` (plain C,
fp64, no blocking or reordering beyond the definition).

Inputs are bf16 bit patterns (``numpy.uint16``); outputs are fp64. The
int8 KV pieces (``quantize_rows_u8``, ``dequantize_rows_u8``) take their
code decision in fp32, and ``attend_rows`` attends over given fp64 keys and
values (already rotated), e.g. dequantized cache rows.
Citations of the pages are in the C file next to each function.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hlg_oracle.c")
_LIB = os.path.join(_HERE, "libhlg_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp64: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        p = ctypes.c_void_p
        lib.hlg_layer_is_global.argtypes = [i32, i32, i32]
        lib.hlg_share_source.argtypes = [i32, i32, i32, i32]
        lib.hlg_cache_slot.argtypes = [i64, i32]
        lib.hlg_cache_slot.restype = i64
        lib.hlg_visible_range.argtypes = [i64, i32, i64, p, p]
        lib.hlg_visible_range.restype = i64
        lib.hlg_rope_n_rotated_pairs.argtypes = [i32, f64]
        lib.hlg_rope.argtypes = [p, p, i32, f64, f64, i64]
        lib.hlg_rope.restype = None
        lib.hlg_rope_bf16.argtypes = [p, p, i32, f64, f64, i64]
        lib.hlg_rope_bf16.restype = None
        lib.hlg_attention.argtypes = [p, p, p, p, p, p, i32, i32, i32, i32, i32, i32, i32,
                                      f64, f64, f64, i64, p, p, p, i32]
        lib.hlg_default_threads.argtypes = []
        lib.hlg_layer_cache_bytes.argtypes = [i64, i32, i64, i32, i32, i32]
        lib.hlg_layer_cache_bytes.restype = i64
        lib.hlg_stack_cache_bytes.argtypes = [i32, i32, i32, i64, i32, i32, i32, i64,
                                              i32, i32, i64, i32, i32]
        lib.hlg_stack_cache_bytes.restype = i64
        lib.hlg_quantize_rows_u8.argtypes = [p, i64, i32, p, p, p]
        lib.hlg_dequantize_rows_u8.argtypes = [p, p, p, i64, i32, p]
        lib.hlg_dequantize_rows_u8.restype = None
        lib.hlg_attend_rows.argtypes = [p, p, p, i64, p, p, i64, i32, f64, p, p]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return int(_load().hlg_default_threads())


def layer_is_global(n_layers: int, ratio: int, layer: int) -> int:
    return int(_load().hlg_layer_is_global(n_layers, ratio, layer))


def layer_schedule(n_layers: int, ratio: int) -> list[bool]:
    return [layer_is_global(n_layers, ratio, l) == 1 for l in range(n_layers)]


def share_source(n_layers: int, ratio: int, n_shared: int, layer: int) -> int:
    return int(_load().hlg_share_source(n_layers, ratio, n_shared, layer))


def cache_slot(pos: int, window: int) -> int:
    return int(_load().hlg_cache_slot(pos, window))


def visible_range(pos: int, window: int, n_keys: int) -> tuple[int, int, int]:
    lo = ctypes.c_int64()
    hi = ctypes.c_int64()
    cnt = _load().hlg_visible_range(pos, window, n_keys, ctypes.byref(lo), ctypes.byref(hi))
    return int(lo.value), int(hi.value), int(cnt)


def rope_n_rotated_pairs(head_dim: int, rope_frac: float) -> int:
    return int(_load().hlg_rope_n_rotated_pairs(head_dim, rope_frac))


def rope(x: np.ndarray, pos: int, rope_frac: float, theta: float) -> np.ndarray:
    """(p-)RoPE of one fp64 vector."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _load().hlg_rope(_ptr(x), _ptr(y), x.shape[0], rope_frac, theta, pos)
    return y


def rope_bf16(x_bits: np.ndarray, pos: int, rope_frac: float, theta: float) -> np.ndarray:
    """(p-)RoPE of one bf16 vector (given as uint16 bits), fp64 result."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    y = np.empty(x_bits.shape[0], dtype=np.float64)
    _load().hlg_rope_bf16(_ptr(x_bits), _ptr(y), x_bits.shape[0], rope_frac, theta, pos)
    return y


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray | None, *, q_pos0, n_keys, rot_from,
              window: int, rope_frac: float, theta: float, scale: float,
              rows: np.ndarray | None = None, n_threads: int = 0):
    """Exact attention rows.

    q: uint16 [B,S,Hq,D]; k, v: uint16 [B,T,Hkv,D] in position order.
    q_pos0[b]: absolute position of query row 0; n_keys[b]: keys 0..n_keys-1
    exist; keys at positions >= rot_from[b] are rotated here, earlier keys
    arrive rotated. v = None: K = V, the values are the keys as cached
    (rotated). rows: int32 [R,3] (b, h, i); None = every row.
    Returns (out fp64 [R,D], lse fp64 [R]).
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    if v is not None:
        v = np.ascontiguousarray(v, dtype=np.uint16)
    B, S, Hq, D = q.shape
    Bk, T, Hkv, Dk = k.shape
    if Bk != B or Dk != D or (v is not None and v.shape != k.shape):
        raise ValueError("shape mismatch")
    if rows is None:
        bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(S), indexing="ij")
        rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    rows = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    q_pos0 = np.ascontiguousarray(np.broadcast_to(np.asarray(q_pos0, np.int64), (B,)))
    n_keys = np.ascontiguousarray(np.broadcast_to(np.asarray(n_keys, np.int64), (B,)))
    rot_from = np.ascontiguousarray(np.broadcast_to(np.asarray(rot_from, np.int64), (B,)))
    out = np.zeros((rows.shape[0], D), dtype=np.float64)
    lse = np.zeros(rows.shape[0], dtype=np.float64)
    rc = _load().hlg_attention(_ptr(q), _ptr(k), _ptr(v) if v is not None else None, _ptr(q_pos0), _ptr(n_keys),
                               _ptr(rot_from), B, S, T, Hq, Hkv, D, window, rope_frac,
                               theta, scale, rows.shape[0], _ptr(rows), _ptr(out), _ptr(lse),
                               n_threads)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out, lse


def layer_cache_bytes(batch: int, n_kv_heads: int, capacity: int, head_dim: int,
                      elem_bytes: int = 2, k_equals_v: bool = False) -> int:
    return int(_load().hlg_layer_cache_bytes(batch, n_kv_heads, capacity, head_dim,
                                             elem_bytes, int(k_equals_v)))


def stack_cache_bytes(n_layers: int, ratio: int, n_shared: int, batch: int, *,
                      local_kv_heads: int, local_head_dim: int, local_capacity: int,
                      global_kv_heads: int, global_head_dim: int, global_capacity: int,
                      elem_bytes: int = 2, global_k_equals_v: bool = False,
                      which: str = "all") -> int:
    w = {"all": 0, "local": 1, "global": 2}[which]
    return int(_load().hlg_stack_cache_bytes(n_layers, ratio, n_shared, batch, elem_bytes,
                                             local_kv_heads, local_head_dim, local_capacity,
                                             global_kv_heads, global_head_dim, global_capacity,
                                             int(global_k_equals_v), w))


def quantize_rows_u8(x_bits: np.ndarray):
    """int8 KV rows (see hlg_quantize_rows_u8): x_bits uint16 bf16 [..., D] ->
    (codes uint8 [..., D], lo float32 [...], step float32 [...])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    D = x.shape[-1]
    n = x.size // D
    codes = np.zeros(x.shape, dtype=np.uint8)
    lo = np.zeros(x.shape[:-1], dtype=np.float32)
    step = np.zeros(x.shape[:-1], dtype=np.float32)
    if _load().hlg_quantize_rows_u8(_ptr(x), n, D, _ptr(codes), _ptr(lo), _ptr(step)) != 0:
        raise ValueError("oracle rejected the arguments")
    return codes, lo, step


def dequantize_rows_u8(codes: np.ndarray, lo: np.ndarray, step: np.ndarray) -> np.ndarray:
    """min + code * step, fp64, same shape as codes."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    lo = np.ascontiguousarray(lo, dtype=np.float32)
    step = np.ascontiguousarray(step, dtype=np.float32)
    D = c.shape[-1]
    out = np.zeros(c.shape, dtype=np.float64)
    _load().hlg_dequantize_rows_u8(_ptr(c), _ptr(lo), _ptr(step), c.size // D, D, _ptr(out))
    return out


def attend_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, key_begin, key_count, scale: float):
    """Attention of fp64 query rows q [R, D] over keys/values k, v [N, D]
    (fp64, already rotated): row r reads rows key_begin[r] .. +key_count[r].
    Returns (out fp64 [R, D], lse fp64 [R])."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    R, D = q.shape
    kb = np.ascontiguousarray(np.broadcast_to(np.asarray(key_begin, np.int64), (R,)))
    kc = np.ascontiguousarray(np.broadcast_to(np.asarray(key_count, np.int64), (R,)))
    out = np.zeros((R, D), dtype=np.float64)
    lse = np.zeros(R, dtype=np.float64)
    if _load().hlg_attend_rows(_ptr(q), _ptr(k), _ptr(v), k.shape[0], _ptr(kb), _ptr(kc), R, D, scale,
                               _ptr(out), _ptr(lse)) != 0:
        raise ValueError("oracle rejected the arguments")
    return out, lse
