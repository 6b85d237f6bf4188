"""Seeded synthetic inputs shared by the tests, smoke() and bench.py.

This module holds no attention arithmetic: it draws i.i.d. N(0, 1) samples,
rounds them to bf16 (round-to-nearest-even on the fp32 bit pattern), draws
uniform integer key lengths and picks sample rows.  Both the CUDA path and the
fp64 oracle consume exactly the bf16 bit patterns produced here.

Workload table: the shapes of the configurations the pages' method is measured
on (tiny MHA, MHA prefill, GQA prefill with RoPE, MQA decode over a padded KV
cache, long-context causal, padded cross attention).  Seeds follow one rule:
S = 1000 * config number; Q uses S+1, K S+2, V S+3, key lengths S+4 and the
sampled rows S+5.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    """i.i.d. N(0, std^2) samples rounded to bf16, as uint16 bit patterns."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return bf16_bits_from_f32(x)


def uniform_key_lens(B: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """B integer lengths drawn uniformly from [lo, hi] inclusive (int32)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(lo, hi + 1, size=B, dtype=np.int64).astype(np.int32)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    number: int          # configuration number (seed base = 1000 * number)
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    rope: bool = False
    key_lens: tuple | None = None   # (lo, hi) inclusive uniform range
    note: str = ""
    window: int = 0                 # sliding window in keys (0 = none)
    align: int = 0                  # 1: query rows are each sequence's newest Nq tokens

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def seed(self) -> int:
        return 1000 * self.number

    def flops(self) -> float:
        """Formula FLOPs: 4*B*Hq*Nq*Nk*d, halved for causal.  With a causal
        sliding window over Nq == Nk keys (no padding): 4*B*Hq*d times the
        number of (row, key) pairs inside the window, sum_i min(i + 1, w)."""
        if self.window:
            if not (self.causal and self.Nq == self.Nk and self.key_lens is None):
                raise NotImplementedError("window FLOPs: causal, Nq == Nk, no padding")
            n, w = self.Nq, min(self.window, self.Nq)
            pairs = w * (w + 1) // 2 + (n - w) * w
            return 4.0 * self.B * self.Hq * self.d * pairs
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d
        return f / 2 if self.causal else f


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 2, 2, 256, 256, 64, False,
                     note="tiny MHA, run non-causal and causal"),
    "tiny_causal": Workload("tiny_causal", 1, 1, 2, 2, 256, 256, 64, True),
    "mha_prefill": Workload("mha_prefill", 2, 4, 16, 16, 2048, 2048, 128, True),
    "gqa_rope_prefill": Workload("gqa_rope_prefill", 3, 2, 32, 8, 8192, 8192, 128, True,
                                 rope=True),
    "mqa_decode": Workload("mqa_decode", 4, 64, 32, 1, 1, 16384, 128, False,
                           key_lens=(1024, 16384)),
    "long_causal": Workload("long_causal", 5, 1, 32, 32, 32768, 32768, 128, True),
    "cross_padded": Workload("cross_padded", 6, 8, 16, 16, 1024, 4096, 64, False,
                             key_lens=(2048, 4096)),
    # long causal context under a sliding window of 4096 keys (the pages give
    # the rule but no size; 4096 is a common choice)
    "long_window": Workload("long_window", 7, 1, 32, 32, 32768, 32768, 128, True,
                            window=4096),
    # multi-token decode (draft verification): 4 new tokens per sequence after
    # a ragged cache, GQA 32/8; key_lens count cache + new tokens
    "spec_decode": Workload("spec_decode", 8, 16, 32, 8, 4, 16384, 128, True,
                            key_lens=(1028, 16384), align=1),
}

ROPE_BASE = 10000.0
ROPE_PAIRING_HALF = 0       # (i, i + d/2)
ROPE_PAIRING_ADJACENT = 1   # (2i, 2i + 1)

# Fill value for K/V rows beyond a sequence's key length: large and finite, so
# any weight leaking onto a masked key shows up in the output.
PAD_SENTINEL = 30000.0


def make_inputs(w: Workload, pad_sentinel: bool = True):
    """Host inputs of a workload: dict of q, k, v (bf16 bits) and key_lens."""
    s = w.seed
    q = normal_bf16((w.B, w.Hq, w.Nq, w.d), s + 1)
    k = normal_bf16((w.B, w.Hkv, w.Nk, w.d), s + 2)
    v = normal_bf16((w.B, w.Hkv, w.Nk, w.d), s + 3)
    key_lens = None
    if w.key_lens is not None:
        key_lens = uniform_key_lens(w.B, w.key_lens[0], w.key_lens[1], s + 4)
        if pad_sentinel:
            sent = bf16_bits_from_f32(np.array([PAD_SENTINEL], np.float32))[0]
            for b in range(w.B):
                k[b, :, key_lens[b]:, :] = sent
                v[b, :, key_lens[b]:, :] = sent
    return {"q": q, "k": k, "v": v, "key_lens": key_lens}


def sample_rows(w: Workload, per_head_random: int = 55, seed_offset: int = 5) -> np.ndarray:
    """Flat row ids (b*Hq + h)*Nq + i: every (b, h) x the edge rows
    {0, 1, 127, 128, 129, 255, 256, N-129, N-1} plus `per_head_random`
    uniformly drawn rows, sorted and unique."""
    rng = np.random.Generator(np.random.PCG64(w.seed + seed_offset))
    N = w.Nq
    edge = [r for r in (0, 1, 127, 128, 129, 255, 256, N - 129, N - 1) if 0 <= r < N]
    out = []
    for bh in range(w.B * w.Hq):
        rows = set(edge)
        rows.update(int(x) for x in rng.integers(0, N, size=per_head_random))
        out.extend(bh * N + r for r in sorted(rows))
    return np.array(out, dtype=np.int64)


def paged_layout(key_lens, page_size: int, seed: int, spare_pages: int = 3,
                 shuffle: bool = True):
    """A seeded paged-cache layout for sequences of the given lengths: each
    sequence gets ceil(L / page_size) physical pages drawn in random order
    (or in order, shuffle=False) from a pool with `spare_pages` unused ones.
    Returns (block_table int32 [B, max_pages] with -1 in unused entries,
    num_pages)."""
    kl = np.asarray(key_lens, np.int64)
    need = [int(-(-int(n) // page_size)) for n in kl]
    max_pages = max(1, max(need))
    num_pages = sum(need) + spare_pages
    rng = np.random.Generator(np.random.PCG64(seed))
    perm = rng.permutation(num_pages) if shuffle else np.arange(num_pages)
    table = np.full((len(kl), max_pages), -1, np.int32)
    at = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[at:at + n]
        at += n
    return table, num_pages


def to_paged(x, block_table, key_lens, num_pages: int, page_size: int, fill_bits: int):
    """Copy a contiguous cache [B, Hkv, Nk, d] (bf16 bits) into a paged one
    [num_pages, Hkv, page_size, d]: key j of sequence b goes to block
    block_table[b, j // page_size], row j % page_size.  Rows of a sequence's
    last page past its length keep x's values there (x's padding) or, past
    Nk, the finite PAD_SENTINEL; pages no sequence owns hold `fill_bits`."""
    B, Hkv, Nk, d = x.shape
    out = np.full((num_pages, Hkv, page_size, d), fill_bits, np.uint16)
    pad = bf16_bits_from_f32(np.array([PAD_SENTINEL], np.float32))[0]
    for b in range(B):
        n = int(-(-int(key_lens[b]) // page_size))
        for p in range(n):
            j0, j1 = p * page_size, min((p + 1) * page_size, Nk)
            out[block_table[b, p]] = pad
            out[block_table[b, p], :, :j1 - j0, :] = x[b, :, j0:j1, :]
    return out
