"""Pins for the fp64 CPU oracle (no GPU).

Each test ties the oracle to something other than itself: values printed on
the pages (tests/golden/), closed forms, invariants, library routines that the
definition reduces to (torch's fp64 scaled_dot_product_attention on CPU,
scipy's softmax / logsumexp), and brute force on tiny inputs.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from exact_scaled_dot_fwd_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def f64(bits):
    return torch.from_numpy(synth.bf16_bits_to_f32(bits).astype(np.float64))


def page_mask(Nq, Nk, causal, key_len):
    """Visibility mask assembled the way the pages draw it: all-visible
    history columns beside a lower-triangular block over the last Nq keys
    (multi-token decode, 'Coding interview (14)' self-test 5; Nq == Nk gives
    np.tril), then key-padding columns cut off."""
    if causal:
        hist = max(Nk - Nq, 0)
        tri = np.tril(np.ones((Nq, Nq), dtype=bool))
        m = np.hstack([np.ones((Nq, hist), dtype=bool), tri])[:, -Nk:] if Nk >= Nq else \
            np.tril(np.ones((Nq, Nk), dtype=bool), k=Nk - Nq)
    else:
        m = np.ones((Nq, Nk), dtype=bool)
    m = m.copy()
    m[:, key_len:] = False
    return m


def torch_sdpa(q, k, v, scale, causal, key_lens=None):
    """fp64 library attention with an explicit boolean mask; returns O and
    lse (lse via scipy logsumexp of the library's scaled scores)."""
    Q, K, V = f64(q), f64(k), f64(v)
    B, Hq, Nq, d = Q.shape
    Hkv, Nk = K.shape[1], K.shape[2]
    rep = Hq // Hkv
    K = K.repeat_interleave(rep, dim=1)
    V = V.repeat_interleave(rep, dim=1)
    masks = torch.stack([torch.from_numpy(page_mask(Nq, Nk, causal,
                                                    Nk if key_lens is None else int(key_lens[b])))
                         for b in range(B)])[:, None]
    O = F.scaled_dot_product_attention(Q, K, V, attn_mask=masks, scale=scale)
    S = torch.matmul(Q, K.transpose(-1, -2)) * scale
    S = S.masked_fill(~masks, -math.inf)
    lse = scipy.special.logsumexp(S.numpy(), axis=-1)
    return O.numpy(), lse, masks.numpy()


# ---------------------------------------------------------------- softmax ---

def test_softmax_printed_values_and_no_nan():
    rows = _golden_rows("softmax_stability.txt")
    x = np.array([float(r[0]) for r in rows])
    want = np.array([float(r[1]) for r in rows])
    with np.errstate(over="ignore", invalid="ignore"):
        naive = np.exp(x) / np.exp(x).sum()
    assert np.all(np.isnan(naive))            # the page's failure case
    got = oracle.softmax(x)
    assert np.all(np.isfinite(got))
    assert np.array_equal(np.round(got, 3), want)
    e = math.e
    closed = np.array([1.0, e, e * e]) / (1 + e + e * e)
    assert np.max(np.abs(got - closed)) < 1e-15


def test_softmax_and_logsumexp_match_library():
    rng = np.random.default_rng(7)
    for n in (1, 2, 3, 17, 1000):
        x = rng.standard_normal(n) * 30
        assert np.max(np.abs(oracle.softmax(x) - scipy.special.softmax(x))) < 1e-15
        assert abs(oracle.logsumexp(x) - scipy.special.logsumexp(x)) < 1e-12
        assert abs(oracle.softmax(x).sum() - 1.0) < 1e-14
    assert oracle.logsumexp(np.array([1000.0, 1001.0, 1002.0])) == pytest.approx(
        1002 + math.log(1 + math.exp(-1) + math.exp(-2)), abs=1e-12)
    assert oracle.logsumexp(np.array([])) == -math.inf


def test_softmax_shift_invariance():
    rng = np.random.default_rng(8)
    x = rng.standard_normal(50)
    for c in (-700.0, -3.0, 5.0, 900.0):
        # x + c is itself rounded (ulp(900) ~ 1e-13), hence the tolerance
        assert np.max(np.abs(oracle.softmax(x + c) - oracle.softmax(x))) < 1e-12


# ------------------------------------------------------ whole attention -----

CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, key_lens
    (1, 2, 2, 33, 33, 16, False, None),
    (1, 2, 2, 33, 33, 16, True, None),
    (2, 4, 2, 19, 19, 32, True, None),          # GQA
    (2, 4, 1, 5, 40, 8, False, [40, 7]),         # MQA + padding
    (2, 2, 2, 6, 21, 16, True, None),            # Nq < Nk, bottom-right causal
    (3, 4, 2, 12, 12, 16, True, [12, 5, 9]),     # causal + padding
    (2, 2, 1, 1, 50, 64, False, [50, 13]),       # decode
]


@pytest.mark.parametrize("case", CASES)
def test_attention_matches_library_sdpa(case):
    B, Hq, Hkv, Nq, Nk, d, causal, kl = case
    seed = 100 + sum(case[:6])
    q = synth.normal_bf16((B, Hq, Nq, d), seed)
    k = synth.normal_bf16((B, Hkv, Nk, d), seed + 1)
    v = synth.normal_bf16((B, Hkv, Nk, d), seed + 2)
    key_lens = None if kl is None else np.array(kl, np.int32)
    scale = 1 / math.sqrt(d)
    o, lse = oracle.attn_rows(q, k, v, causal, scale, key_lens=key_lens)
    O, LSE, masks = torch_sdpa(q, k, v, scale, causal, key_lens)
    O = O.reshape(-1, d)
    LSE = LSE.reshape(-1)
    rows_ok = np.broadcast_to(masks.any(-1), (B, Hq, Nq)).reshape(-1)
    assert np.max(np.abs(o[rows_ok] - O[rows_ok])) < 1e-13
    assert np.max(np.abs(lse[rows_ok] - LSE[rows_ok])) < 1e-12
    # no visible key: the pages' NaN case, resolved as O = 0, lse = -inf
    assert np.all(o[~rows_ok] == 0.0)
    assert np.all(np.isneginf(lse[~rows_ok]))


def test_fully_masked_rows_and_zero_length():
    q = synth.normal_bf16((2, 2, 4, 8), 1)
    k = synth.normal_bf16((2, 1, 9, 8), 2)
    v = synth.normal_bf16((2, 1, 9, 8), 3)
    o, lse = oracle.attn_rows(q, k, v, False, 0.3, key_lens=np.array([0, 9], np.int32))
    o = o.reshape(2, 2, 4, 8)
    lse = lse.reshape(2, 2, 4)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(o[1])) and np.all(np.isfinite(lse[1]))
    # causal with Nq > Nk: the first Nq - Nk rows see nothing
    q = synth.normal_bf16((1, 1, 6, 8), 4)
    k = synth.normal_bf16((1, 1, 3, 8), 5)
    o, lse = oracle.attn_rows(q, k, k, True, 0.3)
    assert np.all(o[:3] == 0) and np.all(np.isneginf(lse[:3]))
    assert np.all(np.isfinite(lse[3:]))


def test_weights_form_a_convex_combination():
    """Rows of P sum to one: V = 1 gives O = 1; any O lies inside the
    per-dimension range of the visible V rows."""
    B, H, N, d = 1, 2, 40, 16
    q = synth.normal_bf16((B, H, N, d), 11, std=3.0)
    k = synth.normal_bf16((B, H, N, d), 12, std=3.0)
    ones = synth.bf16_bits_from_f32(np.ones((B, H, N, d), np.float32))
    o, _ = oracle.attn_rows(q, k, ones, True, 0.5)
    assert np.max(np.abs(o - 1.0)) < 1e-14
    v = synth.normal_bf16((B, H, N, d), 13)
    o, _ = oracle.attn_rows(q, k, v, True, 0.5)
    V = synth.bf16_bits_to_f32(v).astype(np.float64)
    o = o.reshape(B, H, N, d)
    for h in range(H):
        for i in range(N):
            lo = V[0, h, :i + 1].min(0) - 1e-12
            hi = V[0, h, :i + 1].max(0) + 1e-12
            assert np.all(o[0, h, i] >= lo) and np.all(o[0, h, i] <= hi)


def test_uniform_weights_count_visible_keys_exactly():
    """Q = 0 makes every visible score 0: O is the mean of the visible V rows
    and lse = log(count), so round(exp(lse)) recovers the visible-set size."""
    B, Hq, Hkv, Nq, Nk, d = 3, 4, 2, 17, 23, 8
    zero = np.zeros((B, Hq, Nq, d), np.uint16)
    k = synth.normal_bf16((B, Hkv, Nk, d), 21)
    v = synth.normal_bf16((B, Hkv, Nk, d), 22)
    kl = np.array([23, 0, 11], np.int32)
    V = synth.bf16_bits_to_f32(v).astype(np.float64)
    for causal in (False, True):
        o, lse = oracle.attn_rows(zero, k, v, causal, 0.7, key_lens=kl)
        o = o.reshape(B, Hq, Nq, d)
        lse = lse.reshape(B, Hq, Nq)
        for b in range(B):
            for h in range(Hq):
                g = h // (Hq // Hkv)
                for i in range(Nq):
                    n = int(kl[b])
                    if causal:
                        n = min(n, i + (Nk - Nq) + 1)
                    n = max(n, 0)
                    if n == 0:
                        assert np.isneginf(lse[b, h, i]) and np.all(o[b, h, i] == 0)
                        continue
                    assert round(math.exp(lse[b, h, i])) == n
                    assert abs(lse[b, h, i] - math.log(n)) < 1e-15
                    assert np.max(np.abs(o[b, h, i] - V[b, g, :n].mean(0))) < 1e-14


def hex_digit_inputs(B, H, Nq, Nk, d):
    """K_j carries the four hex digits of j, q_c = 20 * 16^c: with scale 1 the
    score of key j is exactly 20*j, so the largest visible key takes all but
    ~e^-20 of the weight and V_j (the same digits) reads back its index."""
    kf = np.zeros((B, H, Nk, d), np.float32)
    j = np.arange(Nk)
    for c in range(4):
        kf[:, :, :, c] = (j >> (4 * c)) & 15
    qf = np.zeros((B, H, Nq, d), np.float32)
    for c in range(4):
        qf[:, :, :, c] = 20.0 * 16.0 ** c
    q = synth.bf16_bits_from_f32(qf)
    k = synth.bf16_bits_from_f32(kf)
    assert np.array_equal(synth.bf16_bits_to_f32(k), kf)   # exact in bf16
    return q, k, k.copy()


def decode_index(o_rows):
    dig = np.rint(o_rows[:, :4]).astype(np.int64)
    return dig[:, 0] + 16 * dig[:, 1] + 256 * dig[:, 2] + 4096 * dig[:, 3]


def test_max_visible_index_readback():
    B, H, Nq, Nk, d = 2, 2, 37, 300, 8
    q, k, v = hex_digit_inputs(B, H, Nq, Nk, d)
    kl = np.array([300, 123], np.int32)
    for causal in (False, True):
        o, _ = oracle.attn_rows(q, k, v, causal, 1.0, key_lens=kl)
        idx = decode_index(o).reshape(B, H, Nq)
        for b in range(B):
            for i in range(Nq):
                n = int(kl[b])
                if causal:
                    n = min(n, i + (Nk - Nq) + 1)
                assert np.all(idx[b, :, i] == n - 1)


def test_masked_keys_get_exactly_zero_weight():
    """Changing K/V beyond the key length (or above the diagonal) to huge
    finite values leaves the output bit-identical."""
    B, H, N, d = 2, 2, 30, 16
    q = synth.normal_bf16((B, H, N, d), 31)
    k = synth.normal_bf16((B, H, N, d), 32)
    v = synth.normal_bf16((B, H, N, d), 33)
    kl = np.array([30, 12], np.int32)
    o1, l1 = oracle.attn_rows(q, k, v, False, 0.25, key_lens=kl)
    k2, v2 = k.copy(), v.copy()
    sent = synth.bf16_bits_from_f32(np.array([3.0e4], np.float32))[0]
    k2[1, :, 12:] = sent
    v2[1, :, 12:] = sent
    o2, l2 = oracle.attn_rows(q, k2, v2, False, 0.25, key_lens=kl)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # causal: the future of row i does not matter
    o3, _ = oracle.attn_rows(q, k, v, True, 0.25)
    k3, v3 = k.copy(), v.copy()
    k3[:, :, 20:] = sent
    v3[:, :, 20:] = sent
    o4, _ = oracle.attn_rows(q, k3, v3, True, 0.25)
    o3 = o3.reshape(B, H, N, d)
    o4 = o4.reshape(B, H, N, d)
    assert np.array_equal(o3[:, :, :20], o4[:, :, :20])


def test_gqa_equals_mha_with_repeated_kv():
    B, Hq, Hkv, N, d = 2, 8, 2, 24, 16
    q = synth.normal_bf16((B, Hq, N, d), 41)
    k = synth.normal_bf16((B, Hkv, N, d), 42)
    v = synth.normal_bf16((B, Hkv, N, d), 43)
    o1, l1 = oracle.attn_rows(q, k, v, True, 0.25)
    kr = np.repeat(k, Hq // Hkv, axis=1)     # np.repeat along heads
    vr = np.repeat(v, Hq // Hkv, axis=1)
    o2, l2 = oracle.attn_rows(q, kr, vr, True, 0.25)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # a wrong grouping (h % Hkv) would differ
    kw = np.tile(k, (1, Hq // Hkv, 1, 1))
    vw = np.tile(v, (1, Hq // Hkv, 1, 1))
    o3, _ = oracle.attn_rows(q, kw, vw, True, 0.25)
    assert np.max(np.abs(o1 - o3)) > 1e-3


def test_online_block2_seven_keys():
    n_keys, block, tol = _golden_rows("online_block2_seven_keys.txt")[0]
    n_keys, block = int(n_keys), int(block)
    q = synth.normal_bf16((1, 1, 1, 16), 51)
    k = synth.normal_bf16((1, 1, n_keys, 16), 52)
    v = synth.normal_bf16((1, 1, n_keys, 16), 53)
    o1, l1 = oracle.attn_rows(q, k, v, False, 0.25)
    o2, l2 = oracle.attn_online_rows(q, k, v, False, 0.25, block)
    assert np.max(np.abs(o1 - o2)) < 10 * float(tol)
    assert np.max(np.abs(l1 - l2)) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_online_equals_naive_every_block(causal):
    w = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(w)
    rows = np.arange(0, w.B * w.Hq * w.Nq, 5)
    o1, l1 = oracle.attn_rows(x["q"], x["k"], x["v"], causal, w.scale, rows=rows)
    for block in (1, 2, 3, 7, 64, 128, 255, 256, 1000):
        o2, l2 = oracle.attn_online_rows(x["q"], x["k"], x["v"], causal, w.scale, block,
                                         rows=rows)
        assert np.max(np.abs(o1 - o2)) < 1e-13
        assert np.max(np.abs(l1 - l2)) < 1e-13


def test_incremental_decode_equals_causal_row():
    (tol,) = _golden_rows("decode_vs_causal.txt")[0]
    B, H, N, d = 2, 4, 48, 32
    q = synth.normal_bf16((B, H, N, d), 61)
    k = synth.normal_bf16((B, H, N, d), 62)
    v = synth.normal_bf16((B, H, N, d), 63)
    o_full, l_full = oracle.attn_rows(q, k, v, True, 1 / math.sqrt(d))
    o_full = o_full.reshape(B, H, N, d)
    for i in range(N):
        qi = np.ascontiguousarray(q[:, :, i:i + 1])
        o, l = oracle.attn_rows(qi, k, v, False, 1 / math.sqrt(d),
                                key_lens=np.full(B, i + 1, np.int32))
        assert np.max(np.abs(o.reshape(B, H, d) - o_full[:, :, i])) < 100 * float(tol)


def test_scaled_score_variance_is_about_one():
    """With N(0,1) inputs, scores scaled by 1/sqrt(d) have variance ~1 and the
    unscaled ones ~d ('Transformer Architecture Breakdown', section 1.2)."""
    w = synth.WORKLOADS["mha_prefill"]
    q = synth.bf16_bits_to_f32(synth.normal_bf16((4096, 128), w.seed + 1)).astype(np.float64)
    k = synth.bf16_bits_to_f32(synth.normal_bf16((4096, 128), w.seed + 2)).astype(np.float64)
    s = (q * k).sum(1)
    assert abs(s.var() / 128 - 1) < 0.1
    assert abs((s / math.sqrt(128)).var() - 1) < 0.1


# -------------------------------------------------------------------- RoPE --

def _unit_bits(shape, idx, value=1.0):
    x = np.zeros(shape, np.float32)
    x[idx] = value
    return synth.bf16_bits_from_f32(x)


@pytest.mark.parametrize("pairing", [0, 1])
def test_rope_relative_position(pairing):
    shift, *positions = (int(t) for t in _golden_rows("rope_relative_shift.txt")[0])
    d = 64
    q = synth.normal_bf16((1, 1, 1, d), 71)
    k = synth.normal_bf16((1, 1, 1, d), 72)
    dots = []
    for t in positions:
        rq = oracle.rope(q, pos_offset=t, pairing=pairing)
        rk = oracle.rope(k, pos_offset=t + shift, pairing=pairing)
        dots.append(float((rq * rk).sum()))
    assert max(dots) - min(dots) < 1e-12
    # and it is not the unrotated product
    plain = float((synth.bf16_bits_to_f32(q).astype(np.float64) *
                   synth.bf16_bits_to_f32(k).astype(np.float64)).sum())
    assert abs(dots[0] - plain) > 1e-6


def test_rope_closed_forms():
    # position 0 is the identity
    x = synth.normal_bf16((1, 2, 3, 16), 73)
    xr = oracle.rope(x, pos_offset=0)[:, :, :1]
    assert np.array_equal(xr, synth.bf16_bits_to_f32(x[:, :, :1]).astype(np.float64))
    # d = 2: theta_0 = 1, (1, 0) at position t -> (cos t, sin t) (counter-clockwise)
    e = _unit_bits((1, 1, 1, 2), (0, 0, 0, 0))
    for t in (1, 2, 5, 1000):
        r = oracle.rope(e, pos_offset=t)[0, 0, 0]
        assert abs(r[0] - math.cos(t)) < 1e-15 and abs(r[1] - math.sin(t)) < 1e-15
    # d = 4, half pairing: pair 1 is (x1, x3) with theta_1 = base^(-2/4) = 0.01
    e = _unit_bits((1, 1, 1, 4), (0, 0, 0, 1))
    r = oracle.rope(e, pos_offset=7, base=10000.0, pairing=0)[0, 0, 0]
    assert abs(r[1] - math.cos(0.07)) < 1e-15 and abs(r[3] - math.sin(0.07)) < 1e-15
    assert r[0] == 0 and r[2] == 0
    # adjacent pairing: pair 1 is (x2, x3)
    e = _unit_bits((1, 1, 1, 4), (0, 0, 0, 2))
    r = oracle.rope(e, pos_offset=7, base=10000.0, pairing=1)[0, 0, 0]
    assert abs(r[2] - math.cos(0.07)) < 1e-15 and abs(r[3] - math.sin(0.07)) < 1e-15
    # rotations keep each pair's norm
    x = synth.normal_bf16((1, 1, 5, 32), 74)
    xr = oracle.rope(x, pos_offset=123)
    x0 = synth.bf16_bits_to_f32(x).astype(np.float64)
    n0 = x0[..., :16] ** 2 + x0[..., 16:] ** 2
    n1 = xr[..., :16] ** 2 + xr[..., 16:] ** 2
    assert np.max(np.abs(n0 - n1)) < 1e-12


def test_rope_pairings_are_a_permutation_of_each_other():
    d = 32
    x = synth.normal_bf16((1, 2, 6, d), 75)
    perm = np.empty(d, np.int64)          # half-split slot -> adjacent slot
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    half = oracle.rope(x, pos_offset=3, pairing=0)
    adj = oracle.rope(np.ascontiguousarray(x[..., perm]), pos_offset=3, pairing=1)
    assert np.max(np.abs(half[..., perm] - adj)) < 1e-15


def test_attention_with_rope_matches_library_on_rotated_inputs():
    B, Hq, Hkv, N, d = 1, 4, 2, 40, 32
    q = synth.normal_bf16((B, Hq, N, d), 81)
    k = synth.normal_bf16((B, Hkv, N, d), 82)
    v = synth.normal_bf16((B, Hkv, N, d), 83)
    for pairing in (0, 1):
        cfg = dict(base=10000.0, pairing=pairing, q_pos_offset=5, k_pos_offset=5)
        o, lse = oracle.attn_rows(q, k, v, True, 1 / math.sqrt(d), rope_cfg=cfg)
        Q = torch.from_numpy(oracle.rope(q, pos_offset=5, pairing=pairing))
        K = torch.from_numpy(oracle.rope(k, pos_offset=5, pairing=pairing)).repeat_interleave(2, 1)
        V = f64(v).repeat_interleave(2, 1)
        O = F.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=1 / math.sqrt(d))
        assert np.max(np.abs(o - O.numpy().reshape(-1, d))) < 1e-13
        # round_bf16: the rotated rows pass through a bf16 store first
        cfg["round_bf16"] = True
        o_r, _ = oracle.attn_rows(q, k, v, True, 1 / math.sqrt(d), rope_cfg=cfg)

        def rnd(a):
            return torch.from_numpy(synth.bf16_bits_to_f32(
                synth.bf16_bits_from_f32(a.astype(np.float32))).astype(np.float64))
        Qr = rnd(oracle.rope(q, pos_offset=5, pairing=pairing))
        Kr = rnd(oracle.rope(k, pos_offset=5, pairing=pairing)).repeat_interleave(2, 1)
        Or = F.scaled_dot_product_attention(Qr, Kr, V, is_causal=True, scale=1 / math.sqrt(d))
        assert np.max(np.abs(o_r - Or.numpy().reshape(-1, d))) < 1e-13
        assert np.max(np.abs(o_r - o)) > 1e-6


# ------------------------------------------------------------- tile plan ----

def test_kv_tile_sets_closed_forms():
    Br = Bc = 128
    for qt in range(8):
        assert oracle.kv_tiles(1024, 1024, False, 1024, Br, Bc, qt) == (0, 7, 8)
        assert oracle.kv_tiles(1024, 1024, True, 1024, Br, Bc, qt) == (0, qt, qt + 1)
    for L in (1, 127, 128, 129, 1000):
        n = -(-L // Bc)
        assert oracle.kv_tiles(1024, 1024, False, L, Br, Bc, 3) == (0, n - 1, n)
    assert oracle.kv_tiles(1024, 1024, False, 0, Br, Bc, 0) == (-1, -1, 0)
    # Br = 2 * Bc, causal: q tile qt covers rows up to 256*qt + 255
    assert oracle.kv_tiles(1024, 1024, True, 1024, 256, 128, 1) == (0, 3, 4)
    # bottom-right alignment with Nq < Nk shifts the diagonal right by Nk - Nq
    assert oracle.kv_tiles(128, 1024, True, 1024, 128, 128, 0) == (0, 7, 8)
    assert oracle.visible_prefix(0, 128, 1024, True, 1024) == 897


# -------------------------------------------------------- sliding window ----

def window_mask(Nq, Nk, w, causal):
    """The pages' sliding-window legality ('Attention mechanisms ...', section
    11: abs(i - j) < w, plus j <= i when causal), written with np.ogrid as on
    the page, with query positions bottom-right aligned when Nq < Nk."""
    i, j = np.ogrid[:Nq, :Nk]
    p = i + (Nk - Nq)
    allowed = np.abs(p - j) < w
    if causal:
        allowed &= (j <= p)
    return allowed


@pytest.mark.parametrize("Nq,Nk,w,causal", [(40, 40, 5, True), (40, 40, 5, False),
                                            (16, 50, 7, True), (33, 33, 1, True),
                                            (33, 33, 100, False)])
def test_window_matches_library_sdpa(Nq, Nk, w, causal):
    B, H, d = 2, 2, 16
    q = synth.normal_bf16((B, H, Nq, d), 201)
    k = synth.normal_bf16((B, H, Nk, d), 202)
    v = synth.normal_bf16((B, H, Nk, d), 203)
    o, lse = oracle.attn_rows(q, k, v, causal, 0.25, window=w)
    m = torch.from_numpy(window_mask(Nq, Nk, w, causal))
    O = F.scaled_dot_product_attention(f64(q), f64(k), f64(v), attn_mask=m, scale=0.25)
    S = (torch.matmul(f64(q), f64(k).transpose(-1, -2)) * 0.25).masked_fill(~m, -math.inf)
    L = scipy.special.logsumexp(S.numpy(), axis=-1).reshape(-1)
    ok = np.broadcast_to(m.numpy().any(-1), (B, H, Nq)).reshape(-1)
    assert np.max(np.abs(o[ok] - O.numpy().reshape(-1, d)[ok])) < 1e-13
    assert np.max(np.abs(lse[ok] - L[ok])) < 1e-12


def test_window_counts_closed_form():
    N, d, w = 60, 8, 9
    zero = np.zeros((1, 1, N, d), np.uint16)
    k = synth.normal_bf16((1, 1, N, d), 211)
    _, lse = oracle.attn_rows(zero, k, k, True, 1.0, window=w)
    for i in range(N):
        assert round(math.exp(lse[i])) == min(i + 1, w)
    _, lse = oracle.attn_rows(zero, k, k, False, 1.0, window=w)
    for i in range(N):
        assert round(math.exp(lse[i])) == min(i + w, N) - max(0, i - w + 1)


def test_window_online_equals_naive():
    B, H, N, d = 1, 2, 70, 16
    q = synth.normal_bf16((B, H, N, d), 221)
    k = synth.normal_bf16((B, H, N, d), 222)
    v = synth.normal_bf16((B, H, N, d), 223)
    for w in (1, 3, 17, 70):
        o1, l1 = oracle.attn_rows(q, k, v, True, 0.25, window=w)
        for block in (1, 4, 16):
            o2, l2 = oracle.attn_online_rows(q, k, v, True, 0.25, block, window=w)
            assert np.max(np.abs(o1 - o2)) < 1e-13 and np.max(np.abs(l1 - l2)) < 1e-13


def test_window_tile_sets_closed_forms():
    Br = Bc = 128
    for kk in (1, 2, 3):
        w = 128 * kk
        for qt in range(8):
            first = max(0, qt - kk)
            assert oracle.kv_tiles(1024, 1024, True, 1024, Br, Bc, qt, window=w) == \
                (first, qt, qt - first + 1)
    # a window of one key: each row sees only itself
    for i in (0, 5, 127, 128):
        assert oracle.visible_range(i, 256, 256, True, 256, 1) == (i, i + 1)


# ------------------------------------------- multi-token decode alignment ----

def multi_token_mask(lens, t, Nk):
    """The pages' speculative-decode mask ('Coding interview (14)', self-test
    5), per sequence: t new tokens after a cache of len keys see the whole
    cache and a lower triangle among themselves, [ones(t, len) | tril(t, t)];
    the row is padded with invisible columns up to Nk."""
    rows = []
    for n in lens:
        m = np.concatenate([np.ones((t, n), bool), np.tril(np.ones((t, t), bool))], axis=1)
        rows.append(np.concatenate([m, np.zeros((t, Nk - n - t), bool)], axis=1))
    return np.stack(rows)[:, None]          # [B, 1, t, Nk]


@pytest.mark.parametrize("t", [1, 2, 4, 7])
def test_multi_token_decode_matches_page_mask(t):
    """align = 1 places each sequence's t query rows at the end of its own
    key_lens[b] keys (cache + new tokens)."""
    B, Hq, Hkv, d, Nk = 4, 4, 2, 16, 40
    lens = [0, 5, 20, Nk - t]               # cache lengths before the new tokens
    key_lens = np.array([n + t for n in lens], np.int32)
    q = synth.normal_bf16((B, Hq, t, d), 301)
    k = synth.normal_bf16((B, Hkv, Nk, d), 302)
    v = synth.normal_bf16((B, Hkv, Nk, d), 303)
    o, lse = oracle.attn_rows(q, k, v, True, 0.25, key_lens=key_lens, align=1)
    m = torch.from_numpy(multi_token_mask(lens, t, Nk))
    kr = f64(k).repeat_interleave(Hq // Hkv, dim=1)
    vr = f64(v).repeat_interleave(Hq // Hkv, dim=1)
    O = F.scaled_dot_product_attention(f64(q), kr, vr, attn_mask=m, scale=0.25)
    S = (torch.matmul(f64(q), kr.transpose(-1, -2)) * 0.25).masked_fill(~m, -math.inf)
    L = scipy.special.logsumexp(S.numpy(), axis=-1).reshape(-1)
    assert np.max(np.abs(o - O.numpy().reshape(-1, d))) < 1e-13
    assert np.max(np.abs(lse - L)) < 1e-12
    # the online recurrence agrees under the same alignment
    o2, l2 = oracle.attn_online_rows(q, k, v, True, 0.25, 3, key_lens=key_lens, align=1)
    assert np.max(np.abs(o - o2)) < 1e-13 and np.max(np.abs(lse - l2)) < 1e-13


def test_alignment_special_cases():
    B, H, Nq, Nk, d = 2, 2, 6, 30, 8
    q = synth.normal_bf16((B, H, Nq, d), 311)
    k = synth.normal_bf16((B, H, Nk, d), 312)
    v = synth.normal_bf16((B, H, Nk, d), 313)
    # full-length sequences: both alignments put the rows at the end of Nk
    full = np.array([Nk, Nk], np.int32)
    a0 = oracle.attn_rows(q, k, v, True, 0.3, key_lens=full)
    a1 = oracle.attn_rows(q, k, v, True, 0.3, key_lens=full, align=1)
    assert np.array_equal(a0[0], a1[0]) and np.array_equal(a0[1], a1[1])
    # one new token: causal changes nothing, it sees its whole sequence
    q1 = q[:, :, :1]
    kl = np.array([17, 30], np.int32)
    c1 = oracle.attn_rows(q1, k, v, True, 0.3, key_lens=kl, align=1)
    c0 = oracle.attn_rows(q1, k, v, False, 0.3, key_lens=kl, align=1)
    assert np.array_equal(c1[0], c0[0]) and np.array_equal(c1[1], c0[1])
    # closed forms: row i of a sequence of L keys sees L - Nq + i + 1 keys
    # (causal), and its window ends at its own position
    for L in (6, 9, 30):
        for i in range(Nq):
            assert oracle.query_position(i, Nq, Nk, L, 1) == L - Nq + i
            assert oracle.visible_range(i, Nq, Nk, True, L, 0, 1) == (0, L - Nq + i + 1)
            p = L - Nq + i
            assert oracle.visible_range(i, Nq, Nk, True, L, 4, 1) == (max(0, p - 3), p + 1)
    # fewer keys than query rows: the leading rows see nothing when causal
    assert oracle.visible_range(0, Nq, Nk, True, 3, 0, 1) == (0, 0)
    assert oracle.visible_range(Nq - 1, Nq, Nk, True, 3, 0, 1) == (0, 3)
    # decode under a window over a ragged cache reads its last w keys
    assert oracle.visible_range(0, 1, 1000, False, 700, 64, 1) == (636, 700)
    # tile sets follow each sequence's own length
    assert oracle.kv_tiles(8, 4096, True, 1000, 128, 128, 0, align=1) == (0, 7, 8)
    assert oracle.kv_tiles(8, 4096, True, 1000, 128, 128, 0, window=300, align=1) == (5, 7, 3)


# ------------------------------------------------------- paged KV cache ----

def _interleaved_page_claims(lens, page_size, pool):
    """Physical pages of sequences that grow one token at a time, in turn:
    a sequence claims the next page of `pool` exactly when its next token
    opens a new block of page_size positions ('Attention mechanisms ...',
    section 20; 'Transformer internals', PagedAttention).  Returns one page
    list per sequence; logical block n of sequence b is pages[b][n]."""
    claims = iter(pool)
    pages = [[] for _ in lens]
    for pos in range(max(lens)):
        for b, n in enumerate(lens):
            if pos < n and pos % page_size == 0:
                pages[b].append(int(next(claims)))
    return pages


@pytest.mark.parametrize("page_size", [8, 16, 32])
def test_paged_cache_built_token_by_token(page_size):
    """Append every sequence's tokens one at a time in an interleaved order,
    writing K/V into kv_cache[phys, :, offset, :] as the pages do; the
    oracle's gather and paged attention must reproduce the contiguous cache
    and its attention exactly."""
    B, Hq, Hkv, Nq, d = 3, 4, 2, 3, 16
    lens = [37, 5, 64]
    Nk = max(lens)
    max_pages = -(-Nk // page_size)
    k = synth.normal_bf16((B, Hkv, Nk, d), 401)
    v = synth.normal_bf16((B, Hkv, Nk, d), 402)
    q = synth.normal_bf16((B, Hq, Nq, d), 403)
    num_blocks = sum(-(-n // page_size) for n in lens) + 4
    k_cache = np.full((num_blocks, Hkv, page_size, d), 0x7fc0, np.uint16)   # NaN filler
    v_cache = k_cache.copy()
    pool = np.random.Generator(np.random.PCG64(404)).permutation(num_blocks)
    pages = _interleaved_page_claims(lens, page_size, pool)
    for pos in range(Nk):                      # interleave the sequences
        for b in range(B):
            if pos < lens[b]:
                # the token's block and its row inside the block
                phys, off = pages[b][pos // page_size], pos % page_size
                k_cache[phys, :, off, :] = k[b, :, pos, :]
                v_cache[phys, :, off, :] = v[b, :, pos, :]
    table = np.zeros((B, max_pages), np.int32)
    for b in range(B):
        table[b, :len(pages[b])] = pages[b]
    kl = np.array(lens, np.int32)
    kg = oracle.gather_paged(k_cache, table, kl, Nk)
    for b in range(B):
        assert np.array_equal(kg[b, :, :lens[b]], k[b, :, :lens[b]])
        assert not kg[b, :, lens[b]:].any()
    o1, l1 = oracle.attn_paged_rows(q, k_cache, v_cache, table, kl, True, 0.3)
    o2, l2 = oracle.attn_rows(q, k, v, True, 0.3, key_lens=kl, align=1)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_paged_gather_rejects_bad_table_entries():
    cache = np.zeros((2, 1, 16, 8), np.uint16)
    table = np.array([[0, 5]], np.int32)       # block 5 does not exist
    with pytest.raises(ValueError):
        oracle.gather_paged(cache, table, np.array([20], np.int32), 32)
    # entries past the sequence's length are never read
    assert oracle.gather_paged(cache, table, np.array([16], np.int32), 32).shape == (1, 1, 32, 8)
