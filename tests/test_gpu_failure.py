"""Failure detection without a GPU fault: a barrier wait whose limit runs out.

Every barrier wait in the attention kernels is bounded; when the limit runs
out the kernel records ATTN_ETIMEOUT in a device status word and winds down.
The hook attn_debug_timeout_probe runs that path on a barrier nothing ever
completes, with a 20 ms limit; the test reads the status back and checks the
context still computes correct attention afterwards."""
import ctypes
import math

import numpy as np
import pytest

import oracle
from exact_scaled_dot_fwd_b200 import synth

pytestmark = pytest.mark.gpu


def test_wait_limit_reports_timeout_and_context_survives():
    import torch
    import exact_scaled_dot_fwd_b200 as eb
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    L = eb.lib()
    assert eb.device_status(reset=True) == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.attn_debug_timeout_probe(ctypes.c_ulonglong(20_000_000), stream) == 0
    assert eb.device_status(reset=True) == 6          # ATTN_ETIMEOUT
    assert eb.device_status(reset=True) == 0          # cleared
    # the same through the read-and-clear entry point
    assert L.attn_debug_timeout_probe(ctypes.c_ulonglong(20_000_000), stream) == 0
    assert eb.attn_last_device_status() == 6
    assert eb.attn_last_device_status() == 0
    # the context is intact: a normal call still matches the oracle
    B, H, N, d = 1, 2, 200, 64
    q = synth.normal_bf16((B, H, N, d), 1)
    k = synth.normal_bf16((B, H, N, d), 2)
    v = synth.normal_bf16((B, H, N, d), 3)

    def dev(x):
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    o, lse = eb.attn_fwd(dev(q), dev(k), dev(v), causal=True)
    torch.cuda.synchronize()
    ref, _ = oracle.attn_rows(q, k, v, True, 1 / math.sqrt(d))
    got = synth.bf16_bits_to_f32(o.cpu().view(torch.int16).numpy().view(np.uint16))
    assert np.abs(got.reshape(-1, d) - ref).max() <= 2e-2
    assert eb.device_status(reset=True) == 0
