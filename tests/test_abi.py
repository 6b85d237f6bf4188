"""The C ABI without a GPU: the library loads, exports every function that
include/attn.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re

import pytest

import exact_scaled_dot_fwd_b200 as eb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"ATTN_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    return eb.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert L.attn_abi_version() == 1


def test_strerror(L):
    for code, name in eb.STATUS_NAMES.items():
        assert L.attn_strerror(code).decode().startswith(name)
    assert L.attn_strerror(99) == b"unknown attn status"


P = ctypes.c_void_p(0x1000)      # aligned, never dereferenced by these calls
U = ctypes.c_void_p(0x1001)      # misaligned


def fwd(L, q=P, k=P, v=P, o=P, lse=None, B=1, Hq=2, Hkv=2, Nq=8, Nk=8, d=64, causal=0,
        scale=0.125, key_lens=None):
    return L.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, key_lens, None)


def test_attn_fwd_rejects_bad_arguments_on_host(L):
    assert fwd(L, q=None) == 1
    assert fwd(L, o=None) == 1
    assert fwd(L, B=0) == 1
    assert fwd(L, Nk=-1) == 1
    assert fwd(L, Hq=3, Hkv=2) == 1
    assert fwd(L, causal=2) == 1
    assert fwd(L, scale=0.0) == 1
    assert fwd(L, scale=float("nan")) == 1
    assert fwd(L, scale=float("inf")) == 1
    assert fwd(L, d=96) == 2
    assert fwd(L, d=32) == 2
    assert fwd(L, q=U) == 3
    assert fwd(L, v=U) == 3


def test_attn_fwd_ws_rejects_missing_workspace(L):
    # decode needs a workspace (its size query needs a device, so on a
    # CPU-only host the call fails before any launch either way)
    rc = L.attn_fwd_ws(P, P, P, P, None, 2, 4, 1, 1, 64, 64, 0, 0.125, None, None, 0, None)
    assert rc in (4, 5)
    # prefill (more than 64 query rows per kv head) needs 256 bytes for its
    # scheduler counter
    assert L.attn_workspace_size(1, 2, 2, 128, 128, 64) == 256
    assert L.attn_workspace_size(1, 64, 1, 2, 128, 64) == 256
    rc = L.attn_fwd_ws(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 0, 0.125, None, None, 0, None)
    assert rc == 4
    rc = L.attn_fwd_ws(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 0, 0.125, None, P, 128, None)
    assert rc == 4
    rc = L.attn_fwd_ws(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 0, 0.125, None,
                       ctypes.c_void_p(0x1010), 256, None)
    assert rc == 3


def test_rope_rejects_bad_arguments_on_host(L):
    r = L.rope_apply
    assert r(None, P, 1, 1, 8, 64, 1e4, 0, 0, None) == 1
    assert r(P, P, 1, 1, 8, 63, 1e4, 0, 0, None) == 1       # odd d
    assert r(P, P, 1, 1, 8, 64, -1.0, 0, 0, None) == 1      # base
    assert r(P, P, 1, 1, 8, 64, 1e4, 0, 2, None) == 1       # pairing
    assert r(P, P, 1, 1, 8, 64, 1e4, -1, 0, None) == 1      # negative position
    assert r(P, P, 1, 1, 8, 512, 1e4, 0, 0, None) == 2
    assert r(U, U, 1, 1, 8, 64, 1e4, 0, 0, None) == 3
    # partial overlap of input and output
    assert r(ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1010), 1, 1, 8, 64, 1e4, 0, 0, None) == 1


def test_tile_shape_and_plan_args(L):
    br, bc = ctypes.c_int(), ctypes.c_int()
    assert L.attn_prefill_tile_shape(128, ctypes.byref(br), ctypes.byref(bc)) == 0
    assert br.value > 0 and bc.value > 0
    assert L.attn_prefill_tile_shape(96, ctypes.byref(br), ctypes.byref(bc)) == 2
    assert L.attn_fwd_tile_plan(1, 8, 8, 64, 0, None, None, P, None) == 1
    assert L.attn_fwd_tile_plan(1, 8, 8, 64, 3, None, P, P, None) == 1


def test_timeout_probe_rejects_bad_limits_on_host(L):
    assert L.attn_debug_timeout_probe(ctypes.c_ulonglong(0), None) == 1
    assert L.attn_debug_timeout_probe(ctypes.c_ulonglong(2_000_000_000), None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(eb, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(eb, "_lib", None)
    with pytest.raises(OSError):
        eb.lib()


def test_window_entry_points_reject_bad_arguments_on_host(L):
    w = L.attn_fwd_window
    # negative window
    assert w(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 1, -1, 0.125, None, P, 256, None) == 1
    # the checks shared with attn_fwd_ws come first
    assert w(None, P, P, P, None, 1, 2, 2, 128, 128, 64, 1, 16, 0.125, None, P, 256, None) == 1
    assert w(P, P, P, P, None, 1, 2, 2, 128, 128, 96, 1, 16, 0.125, None, P, 256, None) == 2
    assert w(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 1, 16, 0.125, None, None, 0, None) == 4
    assert w(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 1, 16, 0.125, None,
             ctypes.c_void_p(0x1010), 256, None) == 3
    t = L.attn_fwd_tile_plan_window
    assert t(1, 8, 8, 64, 1, -1, None, P, P, None) == 1
    assert t(1, 8, 8, 64, 1, 16, None, None, P, None) == 1
    assert t(1, 8, 8, 96, 1, 16, None, P, P, None) == 2


def test_ex_entry_points_reject_bad_arguments_on_host(L):
    x = L.attn_fwd_ex
    # align must be 0 or 1, window >= 0
    assert x(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 1, 0, 2, 0.125, None, P, 256, None) == 1
    assert x(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 1, -3, 1, 0.125, None, P, 256, None) == 1
    assert x(P, P, P, P, None, 1, 2, 2, 128, 128, 64, 1, 0, 1, 0.125, None, None, 0, None) == 4
    t = L.attn_fwd_tile_plan_ex
    assert t(1, 8, 8, 64, 1, 0, 2, None, P, P, None) == 1
    assert t(1, 8, 8, 64, 1, 0, 1, None, None, P, None) == 1


def test_paged_rejects_bad_arguments_on_host(L):
    f = L.attn_fwd_paged
    # q, k_cache, v_cache, table, max_pages, page_size, num_pages, o, lse, B, Hq, Hkv, Nq,
    # d, causal, window, scale, key_lens, workspace, bytes, stream
    assert f(P, P, P, None, 4, 16, 8, P, None, 1, 4, 1, 1, 128, 1, 0, 0.1, P, P, 1 << 20,
             None) == 1                                      # no block table
    assert f(P, P, P, P, 4, 16, 8, P, None, 1, 4, 1, 1, 128, 1, 0, 0.1, None, P, 1 << 20,
             None) == 1                                      # no key lengths
    assert f(P, P, P, P, 4, 12, 8, P, None, 1, 4, 1, 1, 128, 1, 0, 0.1, P, P, 1 << 20,
             None) == 2                                      # page size not a multiple of 8
    assert f(P, P, P, P, 2, 256, 8, P, None, 1, 4, 1, 1, 128, 1, 0, 0.1, P, P, 1 << 20,
             None) == 2                                      # page larger than a tile
    assert f(P, P, P, P, 4, 128, 8, P, None, 1, 4, 1, 1, 64, 1, 0, 0.1, P, P, 1 << 20,
             None) == 2                                      # d = 64 tiles hold 64 keys
    assert f(P, P, P, P, 4, 16, 8, P, None, 1, 64, 1, 2, 128, 1, 0, 0.1, P, P, 1 << 20,
             None) == 2                                      # 128 query rows per kv head
    assert f(P, P, P, P, 4, 16, 8, P, None, 1, 4, 1, 1, 128, 1, -1, 0.1, P, P, 1 << 20,
             None) == 1                                      # negative window


def test_fused_rope_rejects_bad_arguments_on_host(L):
    f = L.attn_fwd_rope
    # prefill shape: workspace = 256 (counter) + the (cos, sin) table of 128 rows
    need = L.attn_rope_workspace_size(1, 2, 2, 128, 128, 64)
    assert need == 256 + 128 * 32 * 8
    args = (P, P, P, P, None, 1, 2, 2, 128, 128, 64, 1, 0.125, None)
    assert f(*args, 0.0, 0, 0, P, need, None) == 1            # base
    assert f(*args, 1e4, 2, 0, P, need, None) == 1            # pairing
    assert f(*args, 1e4, 0, -1, P, need, None) == 1           # position offset
    assert f(*args, 1e4, 0, 0, P, need - 1, None) == 4        # workspace too small
    assert f(*args, 1e4, 0, 0, ctypes.c_void_p(0x1010), need, None) == 3


def test_set_workspace_rejects_bad_arguments_on_host(L):
    # only the checks made before any CUDA call: a pointer without a size, a
    # size without a pointer, a pointer off a 256-byte boundary
    assert L.attn_set_workspace(P, 0) == 1
    assert L.attn_set_workspace(None, 256) == 1
    assert L.attn_set_workspace(ctypes.c_void_p(0x1010), 256) == 3
    assert L.attn_set_workspace(ctypes.c_void_p(0x1080), 4096) == 3


def test_size_limits_rejected_on_host(L):
    # flat row counts must stay below 2^31 (int32 indexing inside the kernels)
    assert fwd(L, B=1 << 16, Hq=1 << 14, Hkv=1 << 14, Nq=2, Nk=2) == 2      # B*Hq*Nq = 2^31
    assert fwd(L, B=1, Hq=2, Hkv=2, Nq=8, Nk=1 << 30) == 2                # B*Hkv*Nk = 2^31
    # paged: logical capacity and physical cache rows
    pg = L.attn_fwd_paged
    assert pg(P, P, P, P, 1 << 20, 1 << 11, 4, P, None, 1, 2, 1, 1, 128, 0, 0, 0.1, P,
              None, 0, None) == 2                                           # max_pages*page = 2^31
    assert pg(P, P, P, P, 4, 16, 1 << 27, P, None, 1, 2, 1, 1, 128, 0, 0, 0.1, P,
              None, 0, None) == 2                                           # num_pages*Hkv*page = 2^31
