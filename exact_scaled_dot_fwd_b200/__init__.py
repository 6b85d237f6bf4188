"""exact_scaled_dot_fwd_b200 -- exact scaled dot-product attention forward on
B200 (sm_100a).

Thin Python binding over the C ABI of libattn_b200.so (include/attn.h).  It
only marshals arguments: torch tensors supply device pointers and the current
CUDA stream; every step of the computation runs in the library's kernels.
There is no CPU or library fallback: if the shared library is missing or a
call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = ["attn_fwd", "attn_fwd_ws", "attn_workspace_size", "attn_set_workspace",
           "attn_fwd_paged", "attn_fwd_rope", "attn_fwd_decode_static", "rope_apply",
           "prefill_tile_shape", "tile_plan", "device_status", "attn_last_device_status",
           "AttnError", "lib", "STATUS_NAMES"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_b200.so")

STATUS_NAMES = {0: "ATTN_OK", 1: "ATTN_EINVAL", 2: "ATTN_EUNSUPPORTED", 3: "ATTN_EALIGN",
                4: "ATTN_EWORKSPACE", 5: "ATTN_ECUDA", 6: "ATTN_ETIMEOUT"}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


def lib():
    """Load libattn_b200.so (raises OSError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is missing: build it with "
                          "`python -m exact_scaled_dot_fwd_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, vp]
        L.attn_fwd.restype = i
        L.attn_fwd_ws.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, vp, sz, vp]
        L.attn_fwd_ws.restype = i
        L.attn_fwd_window.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp, vp, sz,
                                      vp]
        L.attn_fwd_window.restype = i
        L.attn_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, vp, vp, sz, vp]
        L.attn_fwd_ex.restype = i
        L.attn_fwd_paged.argtypes = [vp, vp, vp, vp, i, i, i, vp, vp, i, i, i, i, i, i, i, f, vp,
                                     vp, sz, vp]
        L.attn_fwd_paged.restype = i
        L.attn_fwd_rope.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, f, i, i, vp, sz,
                                    vp]
        L.attn_fwd_rope.restype = i
        L.attn_rope_workspace_size.argtypes = [i, i, i, i, i, i]
        L.attn_rope_workspace_size.restype = sz
        L.attn_workspace_size.argtypes = [i, i, i, i, i, i]
        L.attn_workspace_size.restype = sz
        L.attn_set_workspace.argtypes = [vp, sz]
        L.attn_set_workspace.restype = i
        L.rope_apply.argtypes = [vp, vp, i, i, i, i, f, i, i, vp]
        L.rope_apply.restype = i
        L.attn_prefill_tile_shape.argtypes = [i, ctypes.POINTER(i), ctypes.POINTER(i)]
        L.attn_prefill_tile_shape.restype = i
        L.attn_fwd_tile_plan.argtypes = [i, i, i, i, i, vp, vp, vp, vp]
        L.attn_fwd_tile_plan.restype = i
        L.attn_fwd_tile_plan_window.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp]
        L.attn_fwd_tile_plan_window.restype = i
        L.attn_fwd_tile_plan_ex.argtypes = [i, i, i, i, i, i, i, vp, vp, vp, vp]
        L.attn_fwd_tile_plan_ex.restype = i
        L.attn_device_status.argtypes = [vp, i]
        L.attn_device_status.restype = i
        L.attn_last_device_status.argtypes = [vp]
        L.attn_last_device_status.restype = i
        L.attn_strerror.argtypes = [i]
        L.attn_strerror.restype = ctypes.c_char_p
        L.attn_abi_version.argtypes = []
        L.attn_abi_version.restype = i
        L.attn_fwd_decode_static.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, vp]
        L.attn_fwd_decode_static.restype = i
        L.attn_decode_static_max_bytes.argtypes = []
        L.attn_decode_static_max_bytes.restype = sz
        L.attn_debug_timeout_probe.argtypes = [ctypes.c_ulonglong, vp]
        L.attn_debug_timeout_probe.restype = i
        _lib = L
    return _lib


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_tensor(t, name, dtype, ndim=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


def _raise(rc, what):
    if rc != 0:
        raise AttnError(rc, what)


def _shapes(q, k, v):
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    return B, Hq, Hkv, Nq, Nk, d


def attn_fwd(q, k, v, causal=False, scale=None, key_lens=None, out=None, lse=None,
             return_lse=True, stream=None, window=0, align=0):
    """O = softmax(Q K^T * scale + M) V on the GPU.

    q: bf16 [B, Hq, Nq, d]; k, v: bf16 [B, Hkv, Nk, d]; key_lens: int32 [B]
    (device) or None; window: sliding window in keys (0 = none); align: 0
    puts query row i at key position i + Nk - Nq, 1 at i + key_lens[b] - Nq
    (multi-token decode over ragged caches).  Returns (o, lse) (lse fp32
    [B, Hq, Nq], natural log) or o alone when return_lse is False.  Plain
    calls use the library's own workspace; with a window or align = 1 a
    workspace tensor is allocated here and passed to attn_fwd_ex.
    """
    if window or align:
        B, Hq, Hkv, Nq, Nk, d = _shapes(q, k, v)
        torch = _torch()
        ws = torch.empty(max(attn_workspace_size(B, Hq, Hkv, Nq, Nk, d), 256),
                         dtype=torch.uint8, device=q.device)
        return attn_fwd_ws(q, k, v, ws, causal=causal, scale=scale, key_lens=key_lens, out=out,
                           lse=lse, return_lse=return_lse, stream=stream, window=window,
                           align=align)
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_tensor(t, n, torch.bfloat16, 4)
    B, Hq, Hkv, Nq, Nk, d = _shapes(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if key_lens is not None:
        _check_tensor(key_lens, "key_lens", torch.int32, 1)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse if return_lse else None),
                        B, Hq, Hkv, Nq, Nk, d, int(bool(causal)), float(scale), _ptr(key_lens),
                        _stream(stream))
    _raise(rc, "attn_fwd")
    return (out, lse) if return_lse else out


_registered_ws = {}   # device index -> the tensor registered there (kept alive)


def attn_set_workspace(workspace=None, device=None):
    """Register a caller-owned uint8 CUDA tensor (256-byte aligned) as the
    workspace of attn_fwd on its device, or, with None, go back to the
    library's own workspace on `device` (default: the current device).  The
    tensor is kept referenced here while it is registered."""
    torch = _torch()
    if workspace is None:
        dev = torch.cuda.current_device() if device is None else torch.device(device).index
        with torch.cuda.device(dev):
            rc = lib().attn_set_workspace(None, 0)
        _raise(rc, "attn_set_workspace")
        _registered_ws.pop(dev, None)
        return
    _check_tensor(workspace, "workspace", torch.uint8, 1)
    dev = workspace.device.index
    with torch.cuda.device(dev):
        rc = lib().attn_set_workspace(_ptr(workspace), workspace.numel())
    _raise(rc, "attn_set_workspace")
    _registered_ws[dev] = workspace


def attn_workspace_size(B, Hq, Hkv, Nq, Nk, d) -> int:
    return int(lib().attn_workspace_size(B, Hq, Hkv, Nq, Nk, d))


def attn_fwd_ws(q, k, v, workspace, causal=False, scale=None, key_lens=None, out=None,
                lse=None, return_lse=True, stream=None, window=0, align=0):
    """attn_fwd with a caller-owned workspace (uint8 CUDA tensor); a window or
    align = 1 calls attn_fwd_ex."""
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_tensor(t, n, torch.bfloat16, 4)
    B, Hq, Hkv, Nq, Nk, d = _shapes(q, k, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if key_lens is not None:
        _check_tensor(key_lens, "key_lens", torch.int32, 1)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if window or align:
        rc = lib().attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                               _ptr(lse if return_lse else None), B, Hq, Hkv, Nq, Nk, d,
                               int(bool(causal)), int(window), int(align), float(scale),
                               _ptr(key_lens), _ptr(workspace), ws_bytes, _stream(stream))
        _raise(rc, "attn_fwd_ex")
    else:
        rc = lib().attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                               _ptr(lse if return_lse else None), B, Hq, Hkv, Nq, Nk, d,
                               int(bool(causal)), float(scale), _ptr(key_lens), _ptr(workspace),
                               ws_bytes, _stream(stream))
        _raise(rc, "attn_fwd_ws")
    return (out, lse) if return_lse else out


def attn_fwd_paged(q, k_cache, v_cache, block_table, key_lens, causal=True, scale=None,
                   window=0, workspace=None, out=None, lse=None, return_lse=True, stream=None):
    """Decode over a paged KV cache: q bf16 [B, Hq, Nq, d] (each sequence's
    newest Nq tokens), k_cache/v_cache bf16 [num_pages, Hkv, page_size, d],
    block_table int32 [B, max_pages], key_lens int32 [B] (sequence lengths)."""
    torch = _torch()
    _check_tensor(q, "q", torch.bfloat16, 4)
    _check_tensor(k_cache, "k_cache", torch.bfloat16, 4)
    _check_tensor(v_cache, "v_cache", torch.bfloat16, 4)
    _check_tensor(block_table, "block_table", torch.int32, 2)
    _check_tensor(key_lens, "key_lens", torch.int32, 1)
    B, Hq, Nq, d = q.shape
    num_pages, Hkv, page_size, dk = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or dk != d or block_table.shape[0] != B:
        raise ValueError("paged cache shapes do not match q / block_table")
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = attn_workspace_size(B, Hq, Hkv, Nq, max_pages * page_size, d)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().attn_fwd_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                              max_pages, page_size, num_pages, _ptr(out),
                              _ptr(lse if return_lse else None), B, Hq, Hkv, Nq, d,
                              int(bool(causal)), int(window), float(scale), _ptr(key_lens),
                              _ptr(workspace), ws_bytes, _stream(stream))
    _raise(rc, "attn_fwd_paged")
    return (out, lse) if return_lse else out


def attn_fwd_rope(q, k_rot, v, causal=False, scale=None, key_lens=None, rope_base=10000.0,
                  rope_pairing=0, q_pos_offset=0, workspace=None, out=None, lse=None,
                  return_lse=True, stream=None):
    """Attention with q's RoPE fused in: q un-rotated [B, Hq, Nq, d], k_rot
    keys already rotated (rope_apply), v [B, Hkv, Nk, d]."""
    torch = _torch()
    for t, n in ((q, "q"), (k_rot, "k_rot"), (v, "v")):
        _check_tensor(t, n, torch.bfloat16, 4)
    B, Hq, Hkv, Nq, Nk, d = _shapes(q, k_rot, v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if key_lens is not None:
        _check_tensor(key_lens, "key_lens", torch.int32, 1)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = int(lib().attn_rope_workspace_size(B, Hq, Hkv, Nq, Nk, d))
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().attn_fwd_rope(_ptr(q), _ptr(k_rot), _ptr(v), _ptr(out),
                             _ptr(lse if return_lse else None), B, Hq, Hkv, Nq, Nk, d,
                             int(bool(causal)), float(scale), _ptr(key_lens), float(rope_base),
                             int(rope_pairing), int(q_pos_offset), _ptr(workspace), ws_bytes,
                             _stream(stream))
    _raise(rc, "attn_fwd_rope")
    return (out, lse) if return_lse else out


def attn_fwd_decode_static(q, k, v, scale=None, key_lens=None, out=None, lse=None,
                           return_lse=True, stream=None):
    """Decode (Nq == 1) through the entry point that allocates nothing: its
    scratch is a fixed device array inside the library (see
    attn_fwd_decode_static in include/attn.h).  Same result as attn_fwd."""
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_tensor(t, n, torch.bfloat16, 4)
    B, Hq, Hkv, Nq, Nk, d = _shapes(q, k, v)
    if Nq != 1:
        raise ValueError("attn_fwd_decode_static takes one query row per sequence (Nq == 1)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if key_lens is not None:
        _check_tensor(key_lens, "key_lens", torch.int32, 1)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device=q.device)
    rc = lib().attn_fwd_decode_static(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                      _ptr(lse if return_lse else None), B, Hq, Hkv, Nk, d,
                                      float(scale), _ptr(key_lens), _stream(stream))
    _raise(rc, "attn_fwd_decode_static")
    return (out, lse) if return_lse else out


def rope_apply(x, base=10000.0, pos_offset=0, pairing=0, out=None, stream=None):
    """RoPE on bf16 [B, H, N, d]; out=x rotates in place."""
    torch = _torch()
    _check_tensor(x, "x", torch.bfloat16, 4)
    if out is None:
        out = torch.empty_like(x)
    B, H, N, d = x.shape
    rc = lib().rope_apply(_ptr(x), _ptr(out), B, H, N, d, float(base), int(pos_offset),
                          int(pairing), _stream(stream))
    _raise(rc, "rope_apply")
    return out


def prefill_tile_shape(d):
    br, bc = ctypes.c_int(), ctypes.c_int()
    _raise(lib().attn_prefill_tile_shape(d, ctypes.byref(br), ctypes.byref(bc)),
           "attn_prefill_tile_shape")
    return br.value, bc.value


def tile_plan(B, Nq, Nk, d, causal, key_lens=None, device="cuda", stream=None, window=0,
              align=0):
    """(first, count) int32 [B, nqt] tensors: the KV tiles the prefill kernel
    visits for each (b, query tile), optionally under a sliding window."""
    torch = _torch()
    br, _ = prefill_tile_shape(d)
    nqt = -(-Nq // br)
    first = torch.empty((B, nqt), dtype=torch.int32, device=device)
    count = torch.empty((B, nqt), dtype=torch.int32, device=device)
    rc = lib().attn_fwd_tile_plan_ex(B, Nq, Nk, d, int(bool(causal)), int(window), int(align),
                                     _ptr(key_lens), _ptr(first), _ptr(count), _stream(stream))
    _raise(rc, "attn_fwd_tile_plan_ex")
    return first, count


def device_status(reset=True, stream=None) -> int:
    """Synchronise and read the library's device status word (0 = OK)."""
    return int(lib().attn_device_status(_stream(stream), int(bool(reset))))


def attn_last_device_status(stream=None) -> int:
    """Synchronise, return the status since the last read and clear it."""
    return int(lib().attn_last_device_status(_stream(stream)))
