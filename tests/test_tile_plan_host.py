"""The prefill kernel's tile plan (csrc/tile_plan.cuh), compiled as host C++,
against brute force over the oracle's visible ranges (no GPU).

Checked on random shapes, with and without a sliding window ("Attention
mechanisms ...", section 11) and key padding:
  - every row's visible range [lo, hi) equals the oracle's;
  - the KV-tile range of each query tile equals the oracle's
    (first, count), i.e. it covers every visible key and no tile without one;
  - every tile the plan marks as needing no element mask is fully visible
    to every row of the query tile (soundness), and every tile fully visible
    to all rows inside the range is marked (no masking work left on).
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

DRIVER = r"""
#define __host__
#define __device__
#define __forceinline__ inline
#include "tile_plan.cuh"
extern "C" {
void plan(int qt, int Br, int Bc, int Nq, int Nk, int causal, int L, int window, int* out) {
  const attn::KvRange r = attn::kv_tile_range(qt, Br, Bc, Nq, Nk, causal, L, window);
  out[0] = r.begin; out[1] = r.count; out[2] = r.um_begin; out[3] = r.um_end;
}
void vrange(int i, int Nq, int Nk, int causal, int L, int window, int* out) {
  attn::visible_range(i, Nq, Nk, causal, L, window, &out[0], &out[1]);
}
}
"""


@pytest.fixture(scope="module")
def P(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("tile_plan")
    src = d / "driver.cpp"
    src.write_text(DRIVER)
    so = d / "libplan.so"
    subprocess.run([gxx, "-std=c++17", "-O1", "-fPIC", "-shared", "-I", CSRC, str(src), "-o",
                    str(so)], check=True, capture_output=True)
    L = ctypes.CDLL(str(so))
    L.plan.argtypes = [ctypes.c_int] * 8 + [ctypes.POINTER(ctypes.c_int)]
    L.vrange.argtypes = [ctypes.c_int] * 6 + [ctypes.POINTER(ctypes.c_int)]
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
        yield Nq, Nk, causal, L, window, Br, Bc


def test_visible_range_matches_oracle(P):
    for Nq, Nk, causal, L, window, _, _ in _cases(60, 1):
        for i in range(Nq):
            lo, hi = _vrange(P, i, Nq, Nk, causal, L, window)
            rlo, rhi = oracle.visible_range(i, Nq, Nk, causal, L, window)
            if rhi > rlo:
                assert (lo, hi) == (rlo, rhi), (i, Nq, Nk, causal, L, window)
            else:
                assert hi <= lo, (i, Nq, Nk, causal, L, window)


def test_tile_ranges_and_unmasked_tiles(P):
    for Nq, Nk, causal, L, window, Br, Bc in _cases(150, 2):
        ranges = [oracle.visible_range(i, Nq, Nk, causal, L, window) for i in range(Nq)]
        for qt in range(-(-Nq // Br)):
            begin, count, umb, ume = _plan(P, qt, Br, Bc, Nq, Nk, causal, L, window)
            f, last, c = oracle.kv_tiles(Nq, Nk, causal, L, Br, Bc, qt, window=window)
            what = (qt, Nq, Nk, causal, L, window, Br, Bc)
            assert count == c, what
            if c:
                assert begin == f and begin + count - 1 == last, what
            rows = ranges[qt * Br: min(Nq, qt * Br + Br)]
            for t in range(begin, begin + count):
                full = all(lo <= t * Bc and (t + 1) * Bc <= hi for lo, hi in rows)
                marked = umb <= t < ume
                assert not marked or full, ("masked tile marked unmasked", t, what)
                assert marked or not full, ("fully visible tile left masked", t, what)
