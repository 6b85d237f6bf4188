"""Python wrapper of the fp64 CPU oracle (oracle.c) via ctypes.

TEST INFRASTRUCTURE: only tests/, the package's smoke() check and bench.py's
CPU-baseline / reference leg import this package.  The product library never
imports, links or calls it, and it imports nothing from the product library.

Functions take bf16 inputs as uint16 bit patterns (the exact values the CUDA
path consumes) and return float64 results.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, f64, i32 = ctypes.c_int64, ctypes.c_double, ctypes.c_int
        vp = ctypes.c_void_p
        L.oracle_softmax.argtypes = [vp, i64, vp]
        L.oracle_softmax.restype = None
        L.oracle_logsumexp.argtypes = [vp, i64]
        L.oracle_logsumexp.restype = f64
        L.oracle_rope.argtypes = [vp, vp, i64, i64, i64, i64, f64, i64, i32]
        L.oracle_rope.restype = None
        L.oracle_visible_prefix.argtypes = [i64, i64, i64, i32, i64]
        L.oracle_visible_prefix.restype = i64
        L.oracle_attn_rows.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, i32, i64, i32,
                                       f64, vp, i32, f64, i32, i32, i64, i64, vp, i64, vp, vp,
                                       i32]
        L.oracle_attn_rows.restype = i32
        L.oracle_attn_online_rows.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, i32,
                                              i64, i32, f64, vp, i64, vp, i64, vp, vp, i32]
        L.oracle_attn_online_rows.restype = i32
        L.oracle_kv_tiles.argtypes = [i64, i64, i32, i64, i64, i64, i64, vp, vp, vp]
        L.oracle_kv_tiles.restype = None
        L.oracle_kv_tiles_window.argtypes = [i64, i64, i32, i64, i64, i64, i64, i64, vp, vp, vp]
        L.oracle_kv_tiles_window.restype = None
        L.oracle_visible_range.argtypes = [i64, i64, i64, i32, i64, i64, vp, vp]
        L.oracle_visible_range.restype = None
        L.oracle_visible_range_ex.argtypes = [i64, i64, i64, i32, i64, i64, i32, vp, vp]
        L.oracle_visible_range_ex.restype = None
        L.oracle_query_position.argtypes = [i64, i64, i64, i64, i32]
        L.oracle_query_position.restype = i64
        L.oracle_kv_tiles_ex.argtypes = [i64, i64, i32, i64, i64, i32, i64, i64, i64, vp, vp,
                                         vp]
        L.oracle_kv_tiles_ex.restype = None
        L.oracle_gather_paged.argtypes = [vp, i64, i64, i64, i64, vp, i64, vp, i64, i64, vp]
        L.oracle_gather_paged.restype = i32
        _lib = L
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def softmax(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib().oracle_softmax(_ptr(x), x.size, _ptr(out))
    return out


def logsumexp(x) -> float:
    x = np.ascontiguousarray(x, dtype=np.float64)
    return float(lib().oracle_logsumexp(_ptr(x), x.size))


def rope(x_bits, base=10000.0, pos_offset=0, pairing=0) -> np.ndarray:
    """x_bits: uint16 [B,H,N,d] -> float64 rotated copy."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    B, H, N, d = x.shape
    out = np.empty(x.shape, np.float64)
    lib().oracle_rope(_ptr(x), _ptr(out), B, H, N, d, float(base), int(pos_offset), int(pairing))
    return out


def visible_prefix(i, Nq, Nk, causal, key_len) -> int:
    return int(lib().oracle_visible_prefix(i, Nq, Nk, int(bool(causal)), key_len))


def kv_tiles(Nq, Nk, causal, key_len, Br, Bc, qt, window=0, align=0):
    f, l, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    if align:
        lib().oracle_kv_tiles_ex(Nq, Nk, int(bool(causal)), key_len, window, int(align), Br, Bc,
                                 qt, ctypes.byref(f), ctypes.byref(l), ctypes.byref(c))
    else:
        lib().oracle_kv_tiles_window(Nq, Nk, int(bool(causal)), key_len, window, Br, Bc, qt,
                                     ctypes.byref(f), ctypes.byref(l), ctypes.byref(c))
    return f.value, l.value, c.value


def query_position(i, Nq, Nk, key_len, align=0) -> int:
    return int(lib().oracle_query_position(i, Nq, Nk, key_len, int(align)))


def visible_range(i, Nq, Nk, causal, key_len, window=0, align=0):
    lo, hi = ctypes.c_int64(), ctypes.c_int64()
    if align:
        lib().oracle_visible_range_ex(i, Nq, Nk, int(bool(causal)), key_len, window, int(align),
                                      ctypes.byref(lo), ctypes.byref(hi))
    else:
        lib().oracle_visible_range(i, Nq, Nk, int(bool(causal)), key_len, window,
                                   ctypes.byref(lo), ctypes.byref(hi))
    return lo.value, hi.value


def _prep(q, k, v, key_lens, rows):
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    kl = None if key_lens is None else np.ascontiguousarray(key_lens, dtype=np.int32)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = B * Hq * Nq if r is None else r.size
    return q, k, v, kl, r, (B, Hq, Hkv, Nq, Nk, d), nrows


def attn_rows(q, k, v, causal, scale, key_lens=None, rows=None, rope_cfg=None,
              nthreads=None, window=0, align=0):
    """Naive fp64 attention for the listed flat rows (all rows if None).

    q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] as bf16 bit patterns.  rope_cfg: None or
    dict(base=, pairing=, q_pos_offset=, k_pos_offset=, round_bf16=) -- round_bf16
    rounds the rotated rows to bf16 (a RoPE pass with bf16 output feeding the
    attention).  window: sliding window (0 = none).  align: 0 puts query row i
    at key position i + Nk - Nq, 1 at i + key_lens[b] - Nq.
    Returns (o [n,d], lse [n]).
    """
    q, k, v, kl, r, (B, Hq, Hkv, Nq, Nk, d), nrows = _prep(q, k, v, key_lens, rows)
    o = np.empty((nrows, d), np.float64)
    lse = np.empty(nrows, np.float64)
    rc = rope_cfg or {}
    st = lib().oracle_attn_rows(
        _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Nq, Nk, d, int(bool(causal)), int(window),
        int(align), float(scale), _ptr(kl), int(rope_cfg is not None),
        float(rc.get("base", 10000.0)),
        int(rc.get("pairing", 0)), int(bool(rc.get("round_bf16", False))),
        int(rc.get("q_pos_offset", 0)), int(rc.get("k_pos_offset", 0)),
        _ptr(r), nrows, _ptr(o), _ptr(lse), int(nthreads or default_threads()))
    if st != 0:
        raise ValueError("oracle_attn_rows rejected its arguments")
    return o, lse


def attn_online_rows(q, k, v, causal, scale, block, key_lens=None, rows=None, nthreads=None,
                     window=0, align=0):
    """Online-recurrence fp64 attention over key blocks of size `block`."""
    q, k, v, kl, r, (B, Hq, Hkv, Nq, Nk, d), nrows = _prep(q, k, v, key_lens, rows)
    o = np.empty((nrows, d), np.float64)
    lse = np.empty(nrows, np.float64)
    st = lib().oracle_attn_online_rows(
        _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Nq, Nk, d, int(bool(causal)), int(window),
        int(align), float(scale), _ptr(kl), int(block), _ptr(r), nrows, _ptr(o), _ptr(lse),
        int(nthreads or default_threads()))
    if st != 0:
        raise ValueError("oracle_attn_online_rows rejected its arguments")
    return o, lse


def gather_paged(cache, block_table, key_lens, Nk):
    """Paged cache bf16 bits [num_pages, Hkv, page_size, d] + block table
    int32 [B, max_pages] -> contiguous bf16 bits [B, Hkv, Nk, d] (keys beyond
    key_lens[b] zero)."""
    c = np.ascontiguousarray(cache, dtype=np.uint16)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    kl = np.ascontiguousarray(key_lens, dtype=np.int32)
    num_pages, Hkv, ps, d = c.shape
    B, max_pages = bt.shape
    out = np.empty((B, Hkv, Nk, d), np.uint16)
    st = lib().oracle_gather_paged(_ptr(c), num_pages, Hkv, ps, d, _ptr(bt), max_pages, _ptr(kl),
                                   B, Nk, _ptr(out))
    if st != 0:
        raise ValueError("oracle_gather_paged rejected its arguments")
    return out


def attn_paged_rows(q, k_cache, v_cache, block_table, key_lens, causal, scale, rows=None,
                    window=0, nthreads=None):
    """Attention of q [B, Hq, Nq, d] over a paged cache: the gathered logical
    cache with each sequence's query rows at its newest positions (align 1)."""
    B, _, Nq, _ = np.shape(q)
    max_pages = np.shape(block_table)[1]
    Nk = int(max(1, max_pages * np.shape(k_cache)[2]))
    k = gather_paged(k_cache, block_table, key_lens, Nk)
    v = gather_paged(v_cache, block_table, key_lens, Nk)
    return attn_rows(q, k, v, causal, scale, key_lens=key_lens, rows=rows, window=window,
                     align=1, nthreads=nthreads)
