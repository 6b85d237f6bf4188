"""GPU parity of multi-token decode ("Coding interview (14)", self-test 5: t
new tokens after a cache of len keys see the cache and a lower triangle among
themselves) against the fp64 oracle on the same seeded inputs.

With align = 1 each sequence's Nq query rows are its newest Nq tokens: row i
sits at key position key_lens[b] - Nq + i.  Calls with at most 64 query rows
per kv head run the decode kernels (tcgen05 for d = 128, mma.sync for
d = 64); larger ones run the prefill kernel with the same alignment.

Values: O max-abs <= 2e-2, mean-abs <= 2e-3, lse <= 1e-3 against fp64.
Bit-exact: visible-key counts per row, the prefill tile plan under align = 1,
and both alignments agreeing when every cache is full."""
import math

import numpy as np
import pytest

import oracle
from exact_scaled_dot_fwd_b200 import synth

from parity import check_workload, compare, rand_inputs, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    return t


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window, align, key_lens
    (4, 32, 8, 4, 2000, 128, True, 0, 1, [2000, 1500, 37, 900]),     # GQA, 16 rows per kv head
    (3, 32, 1, 2, 3000, 128, True, 0, 1, [3000, 2047, 129]),        # MQA, 64 rows per kv head
    (2, 8, 8, 7, 500, 128, True, 0, 1, [500, 260]),                 # 7 tokens, MHA
    (3, 16, 4, 5, 1000, 64, True, 0, 1, [1000, 640, 77]),           # d = 64 (mma.sync)
    (2, 4, 1, 16, 900, 64, True, 0, 1, [900, 333]),                 # d = 64, 64 rows
    (2, 16, 1, 3, 1500, 128, True, 0, 1, [1500, 777]),              # 48 rows: S read in two parts, 32 % Nq != 0
    (3, 8, 1, 5, 1200, 128, True, 150, 1, [1200, 600, 40]),         # 40 rows, sliding window
    (2, 16, 2, 8, 1024, 128, True, 0, 0, None),                     # full caches, align 0
    (2, 8, 2, 3, 700, 128, False, 0, 1, [700, 300]),                # not causal
    (3, 16, 4, 4, 2000, 128, True, 300, 1, [2000, 1000, 200]),      # sliding window
    (3, 8, 2, 5, 600, 128, True, 0, 1, [3, 0, 600]),                # caches shorter than Nq
    (4, 32, 1, 1, 5000, 128, True, 1000, 1, [5000, 4000, 999, 1]),  # single token, window at L
    (2, 32, 1, 4, 3000, 128, True, 0, 1, [3000, 1234]),             # 128 rows: prefill kernel
    (2, 4, 4, 300, 900, 128, True, 200, 1, [900, 500]),             # prefill, window, align 1
    (2, 4, 2, 100, 700, 64, True, 0, 1, [700, 64]),                 # prefill d = 64, L < Nq
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:9])))
def test_multi_token_parity_all_rows(torch, case):
    B, Hq, Hkv, Nq, Nk, d, causal, w, align, kl = case
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=9500 + Nq * 7 + Nk, key_lens=kl)
    o, lse = run_gpu(x, causal, 1 / math.sqrt(d), window=w, align=align)
    o_ref, lse_ref = oracle.attn_rows(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d),
                                      key_lens=x["key_lens"], window=w, align=align)
    compare(o.reshape(-1, d), lse.reshape(-1), o_ref, lse_ref, what=str(case))


@pytest.mark.parametrize("Nq,Hq,Hkv,w,d", [(4, 8, 2, 0, 128), (6, 4, 4, 100, 128),
                                           (3, 8, 4, 0, 64), (2, 2, 1, 0, 128)])
def test_multi_token_visible_count_exact(torch, Nq, Hq, Hkv, w, d):
    """Q = 0: lse = log(count) for every row; the rounded count must equal
    the oracle's visible range length."""
    B, Nk = 4, 900
    kl = [900, 513, 2, 0]
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=51, key_lens=kl)
    x["q"][:] = 0
    _, lse = run_gpu(x, True, 0.125, window=w, align=1)
    for b in range(B):
        for i in range(Nq):
            lo, hi = oracle.visible_range(i, Nq, Nk, True, kl[b], w, 1)
            got = lse[b, :, i]
            if hi <= lo:
                assert np.all(np.isneginf(got)), (b, i)
            else:
                assert np.all(np.rint(np.exp(got)) == hi - lo), (b, i, lo, hi, got)


def test_alignments_agree_on_full_caches(torch):
    B, Hq, Hkv, Nq, Nk, d = 3, 16, 4, 4, 1500, 128
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=61, key_lens=[Nk] * B)
    o0, l0 = run_gpu(x, True, 1 / math.sqrt(d), align=0)
    o1, l1 = run_gpu(x, True, 1 / math.sqrt(d), align=1)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


@pytest.mark.parametrize("Nq,Nk,w,kl,d", [(300, 2000, 0, [2000, 700, 0, 150], 128),
                                          (200, 1500, 129, [1500, 300, 1, 1499], 64)])
def test_tile_plan_align_exact(torch, Nq, Nk, w, kl, d):
    import exact_scaled_dot_fwd_b200 as eb
    br, bc = eb.prefill_tile_shape(d)
    kl_t = torch.tensor(kl, dtype=torch.int32, device="cuda")
    first, count = eb.tile_plan(len(kl), Nq, Nk, d, True, key_lens=kl_t, window=w, align=1)
    first, count = first.cpu().numpy(), count.cpu().numpy()
    for b, L in enumerate(kl):
        for qt in range(first.shape[1]):
            f, last, c = oracle.kv_tiles(Nq, Nk, True, L, br, bc, qt, window=w, align=1)
            assert first[b, qt] == f and count[b, qt] == c, (b, qt, f, last, c)


def test_spec_decode_workload_all_rows(torch):
    w = synth.WORKLOADS["spec_decode"]
    x = synth.make_inputs(w)
    check_workload(x, (w.B, w.Hq, w.Nq, w.d), w.causal, w.scale, what=w.name, align=w.align)
