"""The KV tiles the prefill kernel actually scores, observed in the kernel.

attn_fwd_trace runs the prefill kernel with its trace hook: the thread that
issues the tensor-core MMAs records, for every query tile, the first and last
KV tile whose scores it computed and how many.  That set must equal, bit for
bit, the oracle's brute-force set of KV tiles holding a key visible to one of
the tile's rows (causal mask: "Attention mechanisms ...", section 5; sliding
window: section 11; key padding; query alignment of multi-token decode:
"Coding interview (14)", self-test 5) -- no tile with a visible key skipped,
no tile without one scored, including under a window, where the two query
tiles of a work item start at different KV tiles.  The outputs of the traced
launch are also checked against the oracle on every row."""
import math

import numpy as np
import pytest

import oracle

from parity import compare, from_dev, rand_inputs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    return t


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window, align, key_lens
    (2, 2, 2, 1000, 1000, 128, True, 0, 0, [1000, 300]),      # causal + padding, row-tile pairs
    (2, 8, 2, 300, 300, 128, True, 0, 0, None),               # GQA: head pairs
    (3, 2, 1, 333, 1500, 64, True, 0, 0, [1500, 1499, 1]),    # Nq < Nk (bottom-right), d = 64
    (2, 2, 2, 500, 200, 128, True, 0, 0, None),               # Nq > Nk: leading tiles score nothing
    (2, 4, 4, 500, 777, 128, False, 0, 0, [777, 129]),        # padded cross attention
    (1, 2, 2, 2000, 2000, 128, True, 300, 0, None),           # causal window, tiles start apart
    (2, 2, 2, 1000, 1000, 64, False, 200, 0, [1000, 650]),    # two-sided window + padding
    (2, 4, 4, 1200, 1200, 128, True, 128, 0, None),           # window of exactly one tile
    (3, 8, 1, 70, 900, 128, True, 0, 1, [900, 70, 300]),      # align 1: newest rows of each sequence
    (2, 4, 2, 150, 2000, 128, True, 256, 1, [2000, 700]),     # align 1 under a window
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:9])))
def test_scored_tiles_equal_the_visible_tile_set(torch, case):
    import exact_scaled_dot_fwd_b200 as eb
    B, Hq, Hkv, Nq, Nk, d, causal, window, align, kl = case
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=5100 + Nq + Nk + window, key_lens=kl)
    q, k, v = (to_dev(x[n], torch) for n in ("q", "k", "v"))
    kl_t = None if kl is None else torch.tensor(kl, dtype=torch.int32, device="cuda")
    scale = 1 / math.sqrt(d)
    o, lse, trace = eb.prefill_trace(q, k, v, causal=causal, scale=scale, key_lens=kl_t,
                                     window=window, align=align)
    torch.cuda.synchronize()
    assert eb.device_status() == 0
    trace = trace.cpu().numpy()
    br, bc = eb.prefill_tile_shape(d)
    nqt = trace.shape[2]
    assert nqt == -(-Nq // br)
    for b in range(B):
        L = Nk if kl is None else kl[b]
        for qt in range(nqt):
            want = oracle.kv_tiles(Nq, Nk, causal, L, br, bc, qt, window=window, align=align)
            for h in range(Hq):
                got = tuple(int(t) for t in trace[b, h, qt])
                assert got == want, (b, h, qt, got, want)
    o_ref, lse_ref = oracle.attn_rows(x["q"], x["k"], x["v"], causal, scale,
                                      key_lens=x["key_lens"], window=window, align=align)
    compare(from_dev(o).reshape(-1, d), lse.cpu().numpy().astype(np.float64).reshape(-1),
            o_ref, lse_ref, what=str(case))
    # the same bits as the untraced launch
    o2, l2 = eb.attn_fwd(q, k, v, causal=causal, scale=scale, key_lens=kl_t, window=window,
                         align=align)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)
