"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded bf16 inputs.  Tolerances: O max-abs <= 2e-2 and mean-abs
<= 2e-3 against fp64, lse <= 1e-3; masks, visible-key counts and the skipped
tile set are compared bit-exactly."""
import math

import numpy as np
import pytest

import oracle
from exact_scaled_dot_fwd_b200 import synth

from parity import check_workload, compare, from_dev, rand_inputs, run_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    return t


# ------------------------------------------------------ named workloads -----

@pytest.mark.parametrize("name", ["tiny", "tiny_causal"])
def test_tiny_all_rows(torch, name):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    check_workload(x, (w.B, w.Hq, w.Nq, w.d), w.causal, w.scale, what=name)


def test_mha_prefill_all_rows(torch):
    w = synth.WORKLOADS["mha_prefill"]
    x = synth.make_inputs(w)
    check_workload(x, (w.B, w.Hq, w.Nq, w.d), w.causal, w.scale, what=w.name)


def test_gqa_rope_prefill_sampled_rows(torch):
    w = synth.WORKLOADS["gqa_rope_prefill"]
    x = synth.make_inputs(w)
    # rope_apply stores bf16, so the composed pipeline attends over the
    # bf16-rounded rotated q/k; the oracle models that rounding
    rope = dict(base=synth.ROPE_BASE, pairing=synth.ROPE_PAIRING_HALF, q_pos_offset=0,
                k_pos_offset=0, round_bf16=True)
    rows = synth.sample_rows(w, per_head_random=23)
    check_workload(x, (w.B, w.Hq, w.Nq, w.d), w.causal, w.scale, rows=rows, rope=rope,
                   what=w.name)


def test_mqa_decode_all_rows(torch):
    w = synth.WORKLOADS["mqa_decode"]
    x = synth.make_inputs(w)
    check_workload(x, (w.B, w.Hq, w.Nq, w.d), w.causal, w.scale, what=w.name)


def test_long_causal_sampled_rows(torch):
    w = synth.WORKLOADS["long_causal"]
    x = synth.make_inputs(w)
    rows = synth.sample_rows(w, per_head_random=7)
    check_workload(x, (w.B, w.Hq, w.Nq, w.d), w.causal, w.scale, rows=rows, what=w.name)


def test_cross_padded_sampled_rows(torch):
    w = synth.WORKLOADS["cross_padded"]
    x = synth.make_inputs(w)
    rows = synth.sample_rows(w, per_head_random=40)
    check_workload(x, (w.B, w.Hq, w.Nq, w.d), w.causal, w.scale, rows=rows, what=w.name)


# ------------------------------------------------ ragged shapes, all rows ---

RAGGED = [
    # B, Hq, Hkv, Nq, Nk, d, causal, key_lens
    (1, 2, 2, 2, 2, 64, True, None),
    (1, 2, 1, 3, 5, 64, False, None),
    (2, 4, 2, 63, 63, 128, True, None),
    (2, 4, 2, 65, 65, 128, True, None),
    (1, 3, 3, 129, 129, 64, True, None),
    (2, 4, 4, 127, 300, 128, True, None),      # Nq < Nk, bottom-right causal
    (2, 2, 2, 200, 77, 64, True, None),        # Nq > Nk: leading rows see nothing
    (3, 8, 2, 100, 257, 128, False, [257, 1, 130]),
    (3, 8, 2, 257, 257, 64, True, [0, 256, 100]),
    (2, 2, 1, 512, 512, 128, False, [511, 64]),
]


@pytest.mark.parametrize("case", RAGGED, ids=lambda c: "x".join(map(str, c[:7])))
def test_ragged_prefill(torch, case):
    B, Hq, Hkv, Nq, Nk, d, causal, kl = case
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=7000 + Nq + Nk, key_lens=kl)
    check_workload(x, (B, Hq, Nq, d), causal, 1 / math.sqrt(d), what=str(case))


DECODE = [
    # B, Hq, Hkv, Nk, d, key_lens
    (1, 1, 1, 1, 64, None),
    (3, 8, 8, 100, 128, [100, 1, 37]),         # MHA decode
    (4, 16, 2, 1000, 64, [1000, 0, 999, 513]), # GQA, an empty cache
    (2, 64, 1, 3000, 128, [3000, 2048]),       # 64 query heads on one kv head
    (5, 12, 3, 700, 128, None),                # group of 4, not a multiple of 16
    (300, 32, 1, 50, 128, None),               # more units than CTAs
    (2, 4, 4, 300, 128, [2, 2]),               # fewer keys than CTAs: empty ranges
]


@pytest.mark.parametrize("case", DECODE, ids=lambda c: "x".join(map(str, c[:5])))
def test_ragged_decode(torch, case):
    B, Hq, Hkv, Nk, d, kl = case
    x = rand_inputs(B, Hq, Hkv, 1, Nk, d, seed=8000 + Nk + Hq, key_lens=kl)
    check_workload(x, (B, Hq, 1, d), False, 1 / math.sqrt(d), what=str(case))


# ------------------------------------------------------- bit-exact masks ----

@pytest.mark.parametrize("Nq,Nk,causal,kl", [(300, 300, True, [300, 77]),
                                             (64, 500, True, [500, 450]),
                                             (1, 700, False, [700, 3]),
                                             (130, 260, False, [260, 129])])
def test_visible_key_count_exact(torch, Nq, Nk, causal, kl):
    """Q = 0: every visible score is 0, lse = log(count) -> round(exp(lse))
    must equal the oracle's visible-key count for every row."""
    B, H, d = 2, 2, 64
    x = rand_inputs(B, H, H, Nq, Nk, d, seed=11, key_lens=kl)
    x["q"][:] = 0
    _, lse = run_gpu(x, causal, 0.125)
    for b in range(B):
        for i in range(Nq):
            n = oracle.visible_prefix(i, Nq, Nk, causal, kl[b])
            got = lse[b, :, i]
            if n == 0:
                assert np.all(np.isneginf(got))
            else:
                assert np.all(np.rint(np.exp(got)) == n), (b, i, n, got)


@pytest.mark.parametrize("Nq,Nk,causal,kl,d", [(300, 300, True, [300, 77], 128),
                                               (1, 4000, False, [4000, 1234], 128),
                                               (200, 700, True, [700, 690], 64)])
def test_max_visible_index_exact(torch, Nq, Nk, causal, kl, d):
    """K_j holds the hex digits of j and q_c = 20*16^c (scale 1): the score of
    key j is exactly 20 j, so O reads back the largest visible key index."""
    B, H = 2, 2
    kf = np.zeros((B, H, Nk, d), np.float32)
    j = np.arange(Nk)
    for c in range(4):
        kf[:, :, :, c] = (j >> (4 * c)) & 15
    qf = np.zeros((B, H, Nq, d), np.float32)
    for c in range(4):
        qf[:, :, :, c] = 20.0 * 16.0 ** c
    x = {"q": synth.bf16_bits_from_f32(qf), "k": synth.bf16_bits_from_f32(kf),
         "v": synth.bf16_bits_from_f32(kf), "key_lens": np.array(kl, np.int32)}
    o, _ = run_gpu(x, causal, 1.0)
    dig = np.rint(o[..., :4]).astype(np.int64)
    idx = dig[..., 0] + 16 * dig[..., 1] + 256 * dig[..., 2] + 4096 * dig[..., 3]
    for b in range(B):
        for i in range(Nq):
            n = oracle.visible_prefix(i, Nq, Nk, causal, kl[b])
            if n > 0:
                assert np.all(idx[b, :, i] == n - 1), (b, i, n, idx[b, :, i])


@pytest.mark.parametrize("Nq,Nk,causal,kl,d", [(1000, 1000, True, [1000, 300, 0], 128),
                                               (333, 1500, True, [1500, 1499, 1], 64),
                                               (500, 777, False, [777, 129, 0], 128)])
def test_skipped_tile_set_exact(torch, Nq, Nk, causal, kl, d):
    import exact_scaled_dot_fwd_b200 as eb
    br, bc = eb.prefill_tile_shape(d)
    kl_t = torch.tensor(kl, dtype=torch.int32, device="cuda")
    first, count = eb.tile_plan(len(kl), Nq, Nk, d, causal, key_lens=kl_t)
    first, count = first.cpu().numpy(), count.cpu().numpy()
    for b, L in enumerate(kl):
        for qt in range(first.shape[1]):
            f, last, c = oracle.kv_tiles(Nq, Nk, causal, L, br, bc, qt)
            assert first[b, qt] == f and count[b, qt] == c, (b, qt, f, last, c)
            if c:
                assert last == f + c - 1


# -------------------------------------------------- properties / pages ------

def test_gqa_equals_mha_with_repeated_kv(torch):
    B, Hq, Hkv, N, d = 2, 8, 2, 300, 128
    x = rand_inputs(B, Hq, Hkv, N, N, d, seed=21)
    o1, l1 = run_gpu(x, True, 1 / math.sqrt(d))
    xr = dict(x, k=np.repeat(x["k"], Hq // Hkv, axis=1), v=np.repeat(x["v"], Hq // Hkv, axis=1))
    o2, l2 = run_gpu(xr, True, 1 / math.sqrt(d))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_decode_equals_causal_prefill_row(torch):
    """Incremental decode over a cache of length i+1 equals row i of causal
    prefill ('Coding interview (14)', section 3.6)."""
    B, H, N, d = 2, 4, 300, 128
    x = rand_inputs(B, H, H, N, N, d, seed=31)
    o_full, l_full = run_gpu(x, True, 1 / math.sqrt(d))
    for i in (0, 1, 63, 64, 65, 128, 299):
        xi = dict(x, q=np.ascontiguousarray(x["q"][:, :, i:i + 1]),
                  key_lens=np.full(B, i + 1, np.int32))
        o, l = run_gpu(xi, False, 1 / math.sqrt(d))
        assert np.max(np.abs(o[:, :, 0] - o_full[:, :, i])) <= 2e-2
        assert np.max(np.abs(l[:, :, 0] - l_full[:, :, i])) <= 1e-3


def test_large_scores_stay_finite(torch):
    """Scores near 1000 (the pages' overflow example) must not produce NaN."""
    B, H, N, d = 1, 2, 200, 64
    x = rand_inputs(B, H, H, N, N, d, seed=41, std=12.0)
    check_workload(x, (B, H, N, d), True, 1.0, what="large scores")


@pytest.mark.parametrize("B,H,N,d,causal,window", [(2, 2, 1000, 128, True, 0),
                                                  (1, 2, 700, 64, False, 0),
                                                  (1, 2, 1200, 128, True, 300)])
def test_max_rises_inside_a_tile(torch, B, H, N, d, causal, window):
    """Scores 12 t (natural units, scale 1) on the second half of KV tile t's
    keys and about 0 on the first: in every unmasked tile after a row's first
    the max rises by ~17 log2 units within the tile's second half, the case in
    which the kernel rescales the first half's P in place.  Compared with the
    oracle (fp64, the definition without any running max) on every row."""
    rng = np.random.default_rng(77 + d)
    q = rng.normal(0.0, 0.25, (B, H, N, d))
    k = rng.normal(0.0, 0.25, (B, H, N, d))
    v = rng.normal(0.0, 1.0, (B, H, N, d))
    q[..., 0] = 1.0
    j = np.arange(N)
    k[..., 0] = np.where(j % 128 >= 64, 12.0 * (j // 128), 0.0)
    x = {"q": synth.bf16_bits_from_f32(q.astype(np.float32)),
         "k": synth.bf16_bits_from_f32(k.astype(np.float32)),
         "v": synth.bf16_bits_from_f32(v.astype(np.float32)), "key_lens": None}
    check_workload(x, (B, H, N, d), causal, 1.0, what="max rising in a tile", window=window)


@pytest.mark.parametrize("B,causal", [(64, True), (65, False)])
def test_ragged_batch_at_the_ordering_limit(torch, B, causal):
    """Batches of up to 64 sequences with key lengths run longest first (the
    kernel ranks them at launch), larger ones in index order: both sides of
    that limit, ragged lengths, every row against the oracle."""
    rng = np.random.default_rng(900 + B)
    kl = [int(x) for x in rng.integers(0, 301, size=B)]
    x = rand_inputs(B, 2, 2, 300, 300, 64, seed=61 + B, key_lens=kl)
    check_workload(x, (B, 2, 300, 64), causal, 0.125, what=f"B={B} ragged")


def test_deterministic(torch):
    w = synth.WORKLOADS["tiny_causal"]
    x = synth.make_inputs(w)
    o1, l1 = run_gpu(x, True, w.scale)
    o2, l2 = run_gpu(x, True, w.scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    xd = rand_inputs(4, 32, 1, 1, 5000, 128, seed=5, key_lens=[5000, 100, 4000, 2500])
    o1, l1 = run_gpu(xd, False, 0.088)
    o2, l2 = run_gpu(xd, False, 0.088)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ------------------------------------------------------------------ RoPE ----

@pytest.mark.parametrize("pairing,d,off", [(0, 128, 0), (1, 128, 5), (0, 64, 8000),
                                           (1, 40, 3), (0, 24, 0)])
def test_rope_matches_oracle(torch, pairing, d, off):
    import exact_scaled_dot_fwd_b200 as eb
    B, H, N = 2, 3, 300
    x = synth.normal_bf16((B, H, N, d), 91 + d)
    ref = oracle.rope(x, base=10000.0, pos_offset=off, pairing=pairing)
    y = from_dev(eb.rope_apply(to_dev(x, torch), base=10000.0, pos_offset=off, pairing=pairing))
    # bf16 output rounding (2^-9 relative) plus fp32 arithmetic
    tol = np.abs(ref) * 2.0 ** -8 + 1e-5
    assert np.all(np.abs(y - ref) <= tol)
    # in place gives the same bits
    t = to_dev(x, torch)
    eb.rope_apply(t, base=10000.0, pos_offset=off, pairing=pairing, out=t)
    assert np.array_equal(from_dev(t), y)


def test_rope_relative_position_on_gpu(torch):
    import exact_scaled_dot_fwd_b200 as eb
    d = 128
    q = synth.normal_bf16((1, 1, 1, d), 95)
    k = synth.normal_bf16((1, 1, 1, d), 96)
    dots = []
    for t in (0, 3, 6):
        rq = from_dev(eb.rope_apply(to_dev(q, torch), pos_offset=t))
        rk = from_dev(eb.rope_apply(to_dev(k, torch), pos_offset=t + 2))
        dots.append(float((rq * rk).sum()))
    # equal up to the bf16 rounding of the rotated vectors
    assert max(dots) - min(dots) < 0.05 * (1 + abs(dots[0]))


# Shapes the decode kernels do not take (more than 64 query rows per kv head,
# or more than 2048 sequences) run the prefill kernel, Nq = 1 included.
ROUTED_TO_PREFILL = [
    # B, Hq, Hkv, Nq, Nk, d, causal, key_lens
    (2, 128, 1, 1, 300, 128, False, [300, 17]),     # 128 query heads on one kv head
    (2, 64, 2, 3, 500, 64, True, [500, 250]),       # 96 rows per kv head, d = 64
    (2100, 2, 2, 1, 40, 128, False, None),          # more sequences than the decode scan holds
]


@pytest.mark.parametrize("case", ROUTED_TO_PREFILL, ids=lambda c: "x".join(map(str, c[:6])))
def test_decode_shapes_routed_to_prefill(torch, case):
    B, Hq, Hkv, Nq, Nk, d, causal, kl = case
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=8800 + B + Hq, key_lens=kl)
    rows = None
    if B * Hq * Nq > 20000:   # sample rows of the large batch
        rows = np.arange(0, B * Hq * Nq, 37, dtype=np.int64)
    check_workload(x, (B, Hq, Nq, d), causal, 1 / math.sqrt(d), rows=rows, what=str(case))
