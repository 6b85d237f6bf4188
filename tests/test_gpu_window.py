"""GPU parity of the sliding-window path ("Attention mechanisms ...", section
11: key j is legal for query position p iff |p - j| < w, and j <= p when
causal; p = i + Nk - Nq) against the fp64 oracle on the same seeded inputs.

Values: O max-abs <= 2e-2, mean-abs <= 2e-3, lse <= 1e-3 against fp64.
Bit-exact: each row's visible-key count, its smallest and its largest
visible key index, the KV-tile range of every query tile, and equality with
the unwindowed result when the window covers every key."""
import math

import numpy as np
import pytest

import oracle
from exact_scaled_dot_fwd_b200 import synth

from parity import check_workload, rand_inputs, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    return t


WINDOW = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window, key_lens
    (1, 2, 2, 300, 300, 128, True, 1, None),           # each row sees itself only
    (1, 2, 2, 300, 300, 128, True, 128, None),         # window = one KV tile
    (2, 4, 4, 700, 700, 128, True, 200, None),         # MHA: row-tile pairs walk a union
    (2, 8, 2, 700, 700, 128, True, 200, None),         # GQA: head pairs share one range
    (1, 3, 3, 513, 513, 64, True, 129, None),          # d = 64, odd head count
    (2, 4, 2, 400, 400, 128, False, 100, None),        # two-sided window
    (2, 4, 4, 257, 900, 128, True, 300, None),         # Nq < Nk, bottom-right
    (2, 2, 2, 300, 100, 64, True, 50, None),           # Nq > Nk: leading rows see nothing
    (3, 4, 2, 600, 600, 128, True, 256, [600, 100, 0]),  # padding and an empty batch
    (2, 4, 4, 500, 800, 64, False, 333, [800, 450]),   # non-causal, padded
    (1, 2, 2, 1000, 1000, 128, True, 5000, None),      # window wider than the sequence
]


@pytest.mark.parametrize("case", WINDOW, ids=lambda c: "x".join(map(str, c[:8])))
def test_window_parity_all_rows(torch, case):
    B, Hq, Hkv, Nq, Nk, d, causal, w, kl = case
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=9100 + Nq + w, key_lens=kl)
    check_workload(x, (B, Hq, Nq, d), causal, 1 / math.sqrt(d), what=str(case), window=w)


DECODE_WINDOW = [
    # B, Hq, Hkv, Nk, d, window, key_lens
    (4, 32, 1, 5000, 128, 1000, None),                 # MQA, tcgen05 split kernel
    (3, 16, 4, 3000, 64, 700, [3000, 2500, 2000]),     # d = 64; one cache ends before Nk - w
    (2, 8, 8, 300, 128, 1, [300, 300]),                # only the newest key
    (2, 8, 2, 400, 128, 10000, [400, 17]),             # window beyond the cache
]


@pytest.mark.parametrize("case", DECODE_WINDOW, ids=lambda c: "x".join(map(str, c[:6])))
def test_window_decode(torch, case):
    B, Hq, Hkv, Nk, d, w, kl = case
    x = rand_inputs(B, Hq, Hkv, 1, Nk, d, seed=9300 + Nk + w, key_lens=kl)
    check_workload(x, (B, Hq, 1, d), False, 1 / math.sqrt(d), what=str(case), window=w)


@pytest.mark.parametrize("Nq,Nk,causal,w,kl", [(600, 600, True, 200, [600, 333]),
                                               (300, 700, False, 150, [700, 500]),
                                               (1, 900, True, 100, [900, 850])])
def test_window_visible_count_exact(torch, Nq, Nk, causal, w, kl):
    """Q = 0: every visible score is 0 and lse = log(count); the rounded
    count must equal the oracle's window range length for every row."""
    B, H, d = 2, 2, 128
    x = rand_inputs(B, H, H, Nq, Nk, d, seed=31, key_lens=kl)
    x["q"][:] = 0
    _, lse = run_gpu(x, causal, 0.125, window=w)
    for b in range(B):
        for i in range(Nq):
            lo, hi = oracle.visible_range(i, Nq, Nk, causal, kl[b], w)
            got = lse[b, :, i]
            if hi <= lo:
                assert np.all(np.isneginf(got)), (b, i)
            else:
                assert np.all(np.rint(np.exp(got)) == hi - lo), (b, i, lo, hi, got)


def _index_inputs(B, H, Nq, Nk, d, sign, kl):
    """K_j holds the hex digits of j; q_c = sign * 20 * 16^c with scale 1
    gives key j the score sign * 20 j, so O reads back the largest (sign +1)
    or the smallest (sign -1) visible key index."""
    kf = np.zeros((B, H, Nk, d), np.float32)
    j = np.arange(Nk)
    for c in range(4):
        kf[:, :, :, c] = (j >> (4 * c)) & 15
    qf = np.zeros((B, H, Nq, d), np.float32)
    for c in range(4):
        qf[:, :, :, c] = sign * 20.0 * 16.0 ** c
    return {"q": synth.bf16_bits_from_f32(qf), "k": synth.bf16_bits_from_f32(kf),
            "v": synth.bf16_bits_from_f32(kf), "key_lens": np.array(kl, np.int32)}


@pytest.mark.parametrize("Nq,Nk,causal,w,kl,d", [(700, 700, True, 300, [700, 450], 128),
                                                 (400, 1000, False, 129, [1000, 900], 64),
                                                 (1, 3000, False, 1000, [3000, 2500], 128)])
def test_window_extreme_visible_indices_exact(torch, Nq, Nk, causal, w, kl, d):
    B, H = 2, 2
    got = {}
    for sign in (+1, -1):
        o, _ = run_gpu(_index_inputs(B, H, Nq, Nk, d, sign, kl), causal, 1.0, window=w)
        dig = np.rint(o[..., :4]).astype(np.int64)
        got[sign] = dig[..., 0] + 16 * dig[..., 1] + 256 * dig[..., 2] + 4096 * dig[..., 3]
    for b in range(B):
        for i in range(Nq):
            lo, hi = oracle.visible_range(i, Nq, Nk, causal, kl[b], w)
            if hi > lo:
                assert np.all(got[+1][b, :, i] == hi - 1), (b, i, lo, hi, got[+1][b, :, i])
                assert np.all(got[-1][b, :, i] == lo), (b, i, lo, hi, got[-1][b, :, i])


@pytest.mark.parametrize("Nq,Nk,causal,w,kl,d", [(2000, 2000, True, 300, [2000, 700, 0], 128),
                                                 (1000, 3000, True, 129, [3000, 2999, 5], 64),
                                                 (900, 1300, False, 256, [1300, 128, 1], 128),
                                                 (640, 640, True, 1, [640, 640, 640], 64)])
def test_window_tile_plan_exact(torch, Nq, Nk, causal, w, kl, d):
    import exact_scaled_dot_fwd_b200 as eb
    br, bc = eb.prefill_tile_shape(d)
    kl_t = torch.tensor(kl, dtype=torch.int32, device="cuda")
    first, count = eb.tile_plan(len(kl), Nq, Nk, d, causal, key_lens=kl_t, window=w)
    first, count = first.cpu().numpy(), count.cpu().numpy()
    for b, L in enumerate(kl):
        for qt in range(first.shape[1]):
            f, last, c = oracle.kv_tiles(Nq, Nk, causal, L, br, bc, qt, window=w)
            assert first[b, qt] == f and count[b, qt] == c, (b, qt, f, last, c)
            if c:
                assert last == f + c - 1


def test_window_covering_everything_equals_no_window(torch):
    B, Hq, Hkv, N, d = 2, 4, 2, 777, 128
    x = rand_inputs(B, Hq, Hkv, N, N, d, seed=41, key_lens=[777, 500])
    for causal in (True, False):
        o0, l0 = run_gpu(x, causal, 1 / math.sqrt(d))
        o1, l1 = run_gpu(x, causal, 1 / math.sqrt(d), window=2 * N)
        assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_long_window_sampled_rows(torch):
    w = synth.WORKLOADS["long_window"]
    x = synth.make_inputs(w)
    rows = synth.sample_rows(w, per_head_random=5)
    check_workload(x, (w.B, w.Hq, w.Nq, w.d), w.causal, w.scale, rows=rows, what=w.name,
                   window=w.window)
