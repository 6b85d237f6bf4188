"""The decode entry point that allocates nothing (attn_fwd_decode_static).

It exists for callers that cannot call cudaMalloc -- code running under a
fixed, preallocated memory budget, inside an allocator hook or another
runtime's callback, or on latency-critical paths where cudaMalloc's implicit
device synchronisation is not acceptable.  Its scratch is a device array
built into the library.  Here it is called through the C ABI and checked
against the regular entry point (attn_fwd) on two calls in a row (the array
keeps the first call's contents, which the second call must not depend on).
Both entry points run the same decode plan and kernels on the same inputs,
so the results must be equal bit for bit; the parity tolerances are
reported in the failure message.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest

from exact_scaled_dot_fwd_b200 import synth

pytestmark = pytest.mark.gpu

TOL_O_MAX, TOL_O_MEAN, TOL_LSE = 2e-2, 2e-3, 1e-3


def _dev(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _call_static(L, torch, q, k, v, o, lse, key_lens, scale):
    B, Hq, _, d = q.shape
    _, Hkv, Nk, _ = k.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.attn_fwd_decode_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, Nk, d, ctypes.c_float(scale),
        ctypes.c_void_p(key_lens.data_ptr()) if key_lens is not None else None, stream)


def test_decode_static_matches_regular_entry_twice():
    import torch
    import exact_scaled_dot_fwd_b200 as eb
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    L = eb.lib()
    assert L.attn_decode_static_max_bytes() == 8 << 20

    # two different decode problems, one after the other, sharing the array
    cases = [
        (64, 32, 1, 16384, 128, (1024, 16384), 4001),   # MQA over a ragged cache
        (8, 16, 4, 3000, 64, (1, 3000), 4002),          # GQA, d = 64
    ]
    for B, Hq, Hkv, Nk, d, (lo, hi), seed in cases:
        q = _dev(torch, synth.normal_bf16((B, Hq, 1, d), seed))
        k = _dev(torch, synth.normal_bf16((B, Hkv, Nk, d), seed + 1))
        v = _dev(torch, synth.normal_bf16((B, Hkv, Nk, d), seed + 2))
        kl = torch.from_numpy(synth.uniform_key_lens(B, lo, hi, seed + 3)).cuda()
        scale = 1.0 / math.sqrt(d)
        o_ref, lse_ref = eb.attn_fwd(q, k, v, scale=scale, key_lens=kl)
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
        rc = _call_static(L, torch, q, k, v, o, lse, kl, scale)
        assert rc == 0, eb.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        err = (o.float() - o_ref.float()).abs()
        lerr = (lse - lse_ref).abs().max().item()
        msg = (f"O max {err.max().item():.3g} (tol {TOL_O_MAX}), mean {err.mean().item():.3g} "
               f"(tol {TOL_O_MEAN}), lse {lerr:.3g} (tol {TOL_LSE})")
        assert torch.isfinite(o.float()).all()
        assert torch.equal(o, o_ref), msg
        assert torch.equal(lse, lse_ref), msg


def test_decode_static_rejects_sizes_beyond_its_array():
    import torch
    import exact_scaled_dot_fwd_b200 as eb
    L = eb.lib()
    B, Hq, Hkv, Nk, d = 2048, 64, 1, 16, 128   # partials far beyond 8 MiB
    q = torch.zeros((B, Hq, 1, d), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, Hkv, Nk, d), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
    rc = _call_static(L, torch, q, k, k, o, lse, None, 0.1)
    assert rc == 4   # ATTN_EWORKSPACE, before any launch
