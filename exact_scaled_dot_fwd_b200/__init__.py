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
           "prefill_tile_shape", "tile_plan", "prefill_trace", "device_status", "attn_last_device_status",
           "AttnError", "lib", "STATUS_NAMES"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_b200.so")

STATUS_NAMES = {0: "ATTN_OK", 1: "ATTN_EINVAL", 2: "ATTN_EUNSUPPORTED", 3: "ATTN_EALIGN",
                4: "ATTN_EWORKSPACE", 5: "ATTN_ECUDA", 6: "ATTN_ETIMEOUT", 7: "ATTN_ERANGE"}

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
        L.attn_fwd_trace.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, vp, vp, sz,
                                     vp, vp]
        L.attn_fwd_trace.restype = i
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


def _torch_stream(stream):
    """The torch stream a call is enqueued on (default: the current one)."""
    return _torch().cuda.current_stream() if stream is None else stream


def _stream(stream):
    return ctypes.c_void_p(_torch_stream(stream).cuda_stream)


def _check_tensor(t, name, dtype, ndim=None):
    """Type, dtype, rank and contiguity of one argument (no device check:
    _check_devices does that once every argument is known)."""
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


def _check_devices(ref, named):
    """Every tensor in `named` ((tensor or None, name) pairs) on ref's CUDA
    device."""
    if not ref.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    for t, n in named:
        if t is not None and t.device != ref.device:
            raise ValueError(f"{n} is on {t.device}, expected {ref.device}")


def _check_io(q, key_lens, out, lse, B, Hq, Nq, extra=()):
    """The arguments every attention wrapper shares: key_lens int32 [B];
    out bf16 with q's shape; lse fp32 [B, Hq, Nq]; all on q's device.
    Shapes are checked before devices, so a mismatch is reported the same way
    on any machine.  A short key_lens or a small out / lse would make the
    kernels read or write past the buffers."""
    torch = _torch()
    if key_lens is not None:
        _check_tensor(key_lens, "key_lens", torch.int32, 1)
        if key_lens.numel() != B:
            raise ValueError(f"key_lens has {key_lens.numel()} entries, expected B = {B}")
    if out is not None:
        _check_tensor(out, "out", torch.bfloat16)
        if tuple(out.shape) != tuple(q.shape):
            raise ValueError(f"out has shape {tuple(out.shape)}, expected {tuple(q.shape)}")
    if lse is not None:
        _check_tensor(lse, "lse", torch.float32)
        if tuple(lse.shape) != (B, Hq, Nq):
            raise ValueError(f"lse has shape {tuple(lse.shape)}, expected {(B, Hq, Nq)}")
    _check_devices(q, [(key_lens, "key_lens"), (out, "out"), (lse, "lse"), *extra])


def _outputs(q, out, lse, return_lse, B, Hq, Nq):
    torch = _torch()
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    return out, lse


def _scratch(nbytes, device, stream):
    """A temporary uint8 workspace for one call on `stream`.  It is allocated
    on the current stream, so it is marked as used by `stream` too: the
    caching allocator then keeps it until `stream` has passed the call."""
    torch = _torch()
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    s = _torch_stream(stream)
    if s != torch.cuda.current_stream(device):
        ws.record_stream(s)
    return ws


def _raise(rc, what):
    if rc != 0:
        raise AttnError(rc, what)


def _shapes(q, k, v):
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    return B, Hq, Hkv, Nq, Nk, d


def _qkv(q, k, v, names=("q", "k", "v")):
    torch = _torch()
    for t, n in zip((q, k, v), names):
        _check_tensor(t, n, torch.bfloat16, 4)
    return _shapes(q, k, v)


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
        B, Hq, Hkv, Nq, Nk, d = _qkv(q, k, v)
        _check_devices(q, [(k, "k"), (v, "v")])
        ws = _scratch(attn_workspace_size(B, Hq, Hkv, Nq, Nk, d), q.device, stream)
        return attn_fwd_ws(q, k, v, ws, causal=causal, scale=scale, key_lens=key_lens, out=out,
                           lse=lse, return_lse=return_lse, stream=stream, window=window,
                           align=align)
    B, Hq, Hkv, Nq, Nk, d = _qkv(q, k, v)
    _check_io(q, key_lens, out, lse if return_lse else None, B, Hq, Nq,
              extra=[(k, "k"), (v, "v")])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse, return_lse, B, Hq, Nq)
    torch = _torch()
    with torch.cuda.device(q.device):
        rc = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                            _ptr(lse if return_lse else None), B, Hq, Hkv, Nq, Nk, d,
                            int(bool(causal)), float(scale), _ptr(key_lens), _stream(stream))
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
    _check_devices(workspace, [])
    dev = workspace.device.index
    with torch.cuda.device(dev):
        rc = lib().attn_set_workspace(_ptr(workspace), workspace.numel())
    _raise(rc, "attn_set_workspace")
    _registered_ws[dev] = workspace


def attn_workspace_size(B, Hq, Hkv, Nq, Nk, d) -> int:
    return int(lib().attn_workspace_size(B, Hq, Hkv, Nq, Nk, d))


def _check_workspace(workspace):
    if workspace is not None:
        _check_tensor(workspace, "workspace", _torch().uint8, 1)


def attn_fwd_ws(q, k, v, workspace, causal=False, scale=None, key_lens=None, out=None,
                lse=None, return_lse=True, stream=None, window=0, align=0):
    """attn_fwd with a caller-owned workspace (uint8 CUDA tensor); a window or
    align = 1 calls attn_fwd_ex."""
    B, Hq, Hkv, Nq, Nk, d = _qkv(q, k, v)
    _check_workspace(workspace)
    _check_io(q, key_lens, out, lse if return_lse else None, B, Hq, Nq,
              extra=[(k, "k"), (v, "v"), (workspace, "workspace")])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse, return_lse, B, Hq, Nq)
    ws_bytes = 0 if workspace is None else workspace.numel()
    torch = _torch()
    with torch.cuda.device(q.device):
        if window or align:
            rc = lib().attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                   _ptr(lse if return_lse else None), B, Hq, Hkv, Nq, Nk, d,
                                   int(bool(causal)), int(window), int(align), float(scale),
                                   _ptr(key_lens), _ptr(workspace), ws_bytes, _stream(stream))
            what = "attn_fwd_ex"
        else:
            rc = lib().attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                   _ptr(lse if return_lse else None), B, Hq, Hkv, Nq, Nk, d,
                                   int(bool(causal)), float(scale), _ptr(key_lens),
                                   _ptr(workspace), ws_bytes, _stream(stream))
            what = "attn_fwd_ws"
    _raise(rc, what)
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
    if key_lens is None:
        raise ValueError("attn_fwd_paged needs key_lens (the sequence lengths)")
    _check_workspace(workspace)
    B, Hq, Nq, d = q.shape
    num_pages, Hkv, page_size, dk = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or dk != d or block_table.shape[0] != B:
        raise ValueError("paged cache shapes do not match q / block_table")
    _check_io(q, key_lens, out, lse if return_lse else None, B, Hq, Nq,
              extra=[(k_cache, "k_cache"), (v_cache, "v_cache"), (block_table, "block_table"),
                     (workspace, "workspace")])
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse, return_lse, B, Hq, Nq)
    if workspace is None:
        workspace = _scratch(attn_workspace_size(B, Hq, Hkv, Nq, max_pages * page_size, d),
                             q.device, stream)
    ws_bytes = workspace.numel()
    with torch.cuda.device(q.device):
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
    keys already rotated (rope_apply), v [B, Hkv, Nk, d].  Row i of every
    sequence is rotated at position q_pos_offset + i."""
    B, Hq, Hkv, Nq, Nk, d = _qkv(q, k_rot, v, ("q", "k_rot", "v"))
    _check_workspace(workspace)
    _check_io(q, key_lens, out, lse if return_lse else None, B, Hq, Nq,
              extra=[(k_rot, "k_rot"), (v, "v"), (workspace, "workspace")])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse, return_lse, B, Hq, Nq)
    if workspace is None:
        workspace = _scratch(lib().attn_rope_workspace_size(B, Hq, Hkv, Nq, Nk, d), q.device,
                             stream)
    ws_bytes = workspace.numel()
    torch = _torch()
    with torch.cuda.device(q.device):
        rc = lib().attn_fwd_rope(_ptr(q), _ptr(k_rot), _ptr(v), _ptr(out),
                                 _ptr(lse if return_lse else None), B, Hq, Hkv, Nq, Nk, d,
                                 int(bool(causal)), float(scale), _ptr(key_lens),
                                 float(rope_base), int(rope_pairing), int(q_pos_offset),
                                 _ptr(workspace), ws_bytes, _stream(stream))
    _raise(rc, "attn_fwd_rope")
    return (out, lse) if return_lse else out


def attn_fwd_decode_static(q, k, v, scale=None, key_lens=None, out=None, lse=None,
                           return_lse=True, stream=None):
    """Decode (Nq == 1) through the entry point that allocates nothing: its
    scratch is a fixed device array inside the library (see
    attn_fwd_decode_static in include/attn.h).  Same result as attn_fwd."""
    B, Hq, Hkv, Nq, Nk, d = _qkv(q, k, v)
    if Nq != 1:
        raise ValueError("attn_fwd_decode_static takes one query row per sequence (Nq == 1)")
    _check_io(q, key_lens, out, lse if return_lse else None, B, Hq, Nq,
              extra=[(k, "k"), (v, "v")])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse, return_lse, B, Hq, Nq)
    torch = _torch()
    with torch.cuda.device(q.device):
        rc = lib().attn_fwd_decode_static(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                          _ptr(lse if return_lse else None), B, Hq, Hkv, Nk, d,
                                          float(scale), _ptr(key_lens), _stream(stream))
    _raise(rc, "attn_fwd_decode_static")
    return (out, lse) if return_lse else out


def rope_apply(x, base=10000.0, pos_offset=0, pairing=0, out=None, stream=None):
    """RoPE on bf16 [B, H, N, d]; out=x rotates in place."""
    torch = _torch()
    _check_tensor(x, "x", torch.bfloat16, 4)
    if out is not None:
        _check_tensor(out, "out", torch.bfloat16, 4)
        if tuple(out.shape) != tuple(x.shape):
            raise ValueError(f"out has shape {tuple(out.shape)}, expected {tuple(x.shape)}")
    _check_devices(x, [(out, "out")])
    if out is None:
        out = torch.empty_like(x)
    B, H, N, d = x.shape
    with torch.cuda.device(x.device):
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


def prefill_trace(q, k, v, causal=False, scale=None, key_lens=None, window=0, align=0,
                  stream=None):
    """Run the prefill kernel with its trace hook: returns (o, lse, trace),
    trace int32 [B, Hq, nqt, 3] = {first, last, count} of the KV tiles whose
    scores the kernel computed for each query tile ({-1, -1, 0} for none)."""
    B, Hq, Hkv, Nq, Nk, d = _qkv(q, k, v)
    _check_io(q, key_lens, None, None, B, Hq, Nq, extra=[(k, "k"), (v, "v")])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    torch = _torch()
    br, _ = prefill_tile_shape(d)
    nqt = -(-Nq // br)
    trace = torch.tensor([-1, -1, 0], dtype=torch.int32, device=q.device).repeat(B * Hq * nqt)
    out, lse = _outputs(q, None, None, True, B, Hq, Nq)
    ws = _scratch(attn_workspace_size(B, Hq, Hkv, Nq, Nk, d), q.device, stream)
    with torch.cuda.device(q.device):
        rc = lib().attn_fwd_trace(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv,
                                  Nq, Nk, d, int(bool(causal)), int(window), int(align),
                                  float(scale), _ptr(key_lens), _ptr(ws), ws.numel(),
                                  _ptr(trace), _stream(stream))
    _raise(rc, "attn_fwd_trace")
    return out, lse, trace.view(B, Hq, nqt, 3)


def device_status(reset=True, stream=None) -> int:
    """Synchronise and read the library's device status word (0 = OK)."""
    return int(lib().attn_device_status(_stream(stream), int(bool(reset))))


def attn_last_device_status(stream=None) -> int:
    """Synchronise, return the status since the last read and clear it."""
    return int(lib().attn_last_device_status(_stream(stream)))
