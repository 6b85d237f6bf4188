"""The prefill kernel's tile plan (csrc/tile_plan.cuh), compiled as host C++,
against brute force over the oracle's visible ranges (no GPU).

Checked on random shapes, with and without a sliding window ("Attention
mechanisms ...", section 11), key padding and both query alignments:
  - every row's visible range [lo, hi) equals the oracle's;
  - the KV-tile range of each query tile equals the oracle's
    (first, count), i.e. it covers every visible key and no tile without one;
  - every tile the plan marks as needing no element mask is fully visible
    to every row of the query tile (soundness), and every tile fully visible
    to all rows inside the range is marked (no masking work left on);
  - the decode key range [lo, L) covers every row's visible keys and starts
    at row 0's first visible key.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_scaled_dot_fwd_b200", "csrc")

WRAPPER = r"""
#define __host__
#define __device__
#define __forceinline__ inline
#include "tile_plan.cuh"
extern "C" {
void plan(int qt, int Br, int Bc, int Nq, int Nk, int causal, int L, int window, int align,
          int* out) {
  const int off = attn::query_offset(Nq, Nk, L, align);
  const attn::KvRange r = attn::kv_tile_range(qt, Br, Bc, Nq, off, causal, L, window);
  out[0] = r.begin; out[1] = r.count; out[2] = r.um_begin; out[3] = r.um_end;
}
void vrange(int i, int Nq, int Nk, int causal, int L, int window, int align, int* out) {
  attn::visible_range(i, attn::query_offset(Nq, Nk, L, align), causal, L, window, &out[0],
                      &out[1]);
}
int dkr(int Nq, int Nk, int L, int window, int align, int* lo) {
  return attn::decode_key_range(L, attn::query_offset(Nq, Nk, L, align), window, lo);
}
}
"""


@pytest.fixture(scope="module")
def P(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("tile_plan")
    src = d / "wrapper.cpp"
    src.write_text(WRAPPER)
    so = d / "libplan.so"
    subprocess.run([gxx, "-std=c++17", "-O1", "-fPIC", "-shared", "-I", CSRC, str(src), "-o",
                    str(so)], check=True, capture_output=True)
    L = ctypes.CDLL(str(so))
    L.plan.argtypes = [ctypes.c_int] * 9 + [ctypes.POINTER(ctypes.c_int)]
    L.vrange.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_int)]
    L.dkr.argtypes = [ctypes.c_int] * 5 + [ctypes.POINTER(ctypes.c_int)]
    L.dkr.restype = ctypes.c_int
    return L


def _plan(P, *args):
    out = (ctypes.c_int * 4)()
    P.plan(*args, out)
    return tuple(out)


def _vrange(P, *args):
    out = (ctypes.c_int * 2)()
    P.vrange(*args, out)
    return tuple(out)


def _cases(n, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    for _ in range(n):
        Nq = int(rng.integers(1, 700))
        Nk = int(rng.integers(1, 700))
        causal = int(rng.integers(0, 2))
        L = int(rng.integers(0, Nk + 1)) if rng.random() < 0.5 else Nk
        window = 0 if rng.random() < 0.25 else int(rng.integers(1, 400))
        Br, Bc = (128, 128) if rng.random() < 0.7 else (64, 32)
        align = int(rng.integers(0, 2))
        yield Nq, Nk, causal, L, window, Br, Bc, align


def test_visible_range_matches_oracle(P):
    for Nq, Nk, causal, L, window, _, _, align in _cases(80, 1):
        for i in range(Nq):
            lo, hi = _vrange(P, i, Nq, Nk, causal, L, window, align)
            rlo, rhi = oracle.visible_range(i, Nq, Nk, causal, L, window, align)
            what = (i, Nq, Nk, causal, L, window, align)
            if rhi > rlo:
                assert (lo, hi) == (rlo, rhi), what
            else:
                assert hi <= lo, what


def test_tile_ranges_and_unmasked_tiles(P):
    for Nq, Nk, causal, L, window, Br, Bc, align in _cases(200, 2):
        ranges = [oracle.visible_range(i, Nq, Nk, causal, L, window, align) for i in range(Nq)]
        for qt in range(-(-Nq // Br)):
            begin, count, umb, ume = _plan(P, qt, Br, Bc, Nq, Nk, causal, L, window, align)
            f, last, c = oracle.kv_tiles(Nq, Nk, causal, L, Br, Bc, qt, window=window,
                                         align=align)
            what = (qt, Nq, Nk, causal, L, window, Br, Bc, align)
            assert count == c, what
            if c:
                assert begin == f and begin + count - 1 == last, what
            rows = ranges[qt * Br: min(Nq, qt * Br + Br)]
            for t in range(begin, begin + count):
                full = all(lo <= t * Bc and (t + 1) * Bc <= hi for lo, hi in rows)
                marked = umb <= t < ume
                assert not marked or full, ("masked tile marked unmasked", t, what)
                assert marked or not full, ("fully visible tile left masked", t, what)


def test_decode_key_range_covers_every_row(P):
    rng = np.random.Generator(np.random.PCG64(3))
    for _ in range(3000):
        Nq = int(rng.integers(1, 17))
        Nk = int(rng.integers(1, 400))
        L = int(rng.integers(0, Nk + 1))
        window = 0 if rng.random() < 0.3 else int(rng.integers(1, 300))
        causal = int(rng.integers(0, 2))
        align = int(rng.integers(0, 2))
        lo = ctypes.c_int()
        n = P.dkr(Nq, Nk, L, window, align, ctypes.byref(lo))
        what = (Nq, Nk, L, window, causal, align)
        assert n == L - lo.value and 0 <= lo.value <= L, what
        for i in range(Nq):
            rlo, rhi = oracle.visible_range(i, Nq, Nk, causal, L, window, align)
            if rhi > rlo:
                assert lo.value <= rlo and rhi <= L, what
        r0 = oracle.visible_range(0, Nq, Nk, causal, L, window, align)
        if r0[1] > r0[0]:
            assert lo.value == r0[0], what
