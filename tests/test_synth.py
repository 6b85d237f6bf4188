"""The seeded input generators (exact_scaled_dot_fwd_b200/synth.py) on the
CPU: bf16 rounding against torch's own conversion, determinism per seed,
key-length ranges, and the paged-cache layout used by the paged tests and
bench (every owned page distinct, spare pages unowned, the contiguous cache
recoverable page by page)."""
import numpy as np
import pytest
import torch

from exact_scaled_dot_fwd_b200 import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.Generator(np.random.PCG64(11))
    x = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32) * np.float32(3.0),
        # halfway cases: the low 16 bits exactly 0x8000, both parities of bit 16
        (np.arange(1000, dtype=np.uint32) << 17 | np.uint32(0x3F808000)).view(np.float32),
        (np.arange(1000, dtype=np.uint32) << 17 | np.uint32(0x3F818000)).view(np.float32),
        np.array([0.0, -0.0, 1e-40, -1e-40, 3.0e38, 65504.0], np.float32),
    ])
    ours = synth.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # bits -> fp32 -> bits is the identity on finite patterns
    assert np.array_equal(synth.bf16_bits_from_f32(synth.bf16_bits_to_f32(ours)), ours)


def test_generators_are_deterministic_per_seed():
    a = synth.normal_bf16((3, 5, 7), 42)
    assert np.array_equal(a, synth.normal_bf16((3, 5, 7), 42))
    assert not np.array_equal(a, synth.normal_bf16((3, 5, 7), 43))
    s = synth.bf16_bits_to_f32(synth.normal_bf16((200_000,), 7, std=2.0)).astype(np.float64)
    assert abs(s.mean()) < 0.03 and abs(s.std() - 2.0) < 0.03
    kl = synth.uniform_key_lens(5000, 10, 20, 3)
    assert kl.dtype == np.int32 and kl.min() == 10 and kl.max() == 20
    assert np.array_equal(kl, synth.uniform_key_lens(5000, 10, 20, 3))


@pytest.mark.parametrize("page_size,shuffle", [(8, True), (16, True), (16, False), (128, True)])
def test_paged_layout_owns_distinct_pages(page_size, shuffle):
    lens = [0, 1, 15, 16, 17, 300, 1024]
    table, num_pages = synth.paged_layout(lens, page_size, seed=5, spare_pages=3,
                                          shuffle=shuffle)
    need = [-(-n // page_size) for n in lens]
    assert table.dtype == np.int32 and table.shape == (len(lens), max(need))
    assert num_pages == sum(need) + 3
    owned = []
    for b, n in enumerate(need):
        assert np.all(table[b, n:] == -1)
        owned += list(table[b, :n])
    assert len(owned) == len(set(owned)) == sum(need)
    assert all(0 <= p < num_pages for p in owned)
    if not shuffle:
        assert owned == list(range(sum(need)))


def test_to_paged_round_trip():
    page_size, fill = 16, 0x7FC0                       # unowned pages: NaN
    B, Hkv, Nk, d = 3, 2, 70, 8
    lens = np.array([70, 5, 33], np.int32)
    x = synth.normal_bf16((B, Hkv, Nk, d), 9)
    table, num_pages = synth.paged_layout(lens, page_size, seed=2)
    cache = synth.to_paged(x, table, lens, num_pages, page_size, fill)
    assert cache.shape == (num_pages, Hkv, page_size, d)
    owned = set()
    for b in range(B):
        for j in range(int(lens[b])):
            page, row = table[b, j // page_size], j % page_size
            owned.add(int(page))
            assert np.array_equal(cache[page, :, row, :], x[b, :, j, :])
    for p in range(num_pages):
        if p not in owned:
            assert np.all(cache[p] == fill)
    # rows of sequence 0's last page past Nk hold the finite pad sentinel
    last = table[0, (Nk - 1) // page_size]
    pad = synth.bf16_bits_from_f32(np.array([synth.PAD_SENTINEL], np.float32))[0]
    assert np.all(cache[last, :, Nk % page_size:, :] == pad)


def test_sample_rows_cover_edges_of_every_head():
    w = synth.WORKLOADS["gqa_rope_prefill"]
    rows = synth.sample_rows(w, per_head_random=23)
    N = w.Nq
    assert np.all(np.diff(rows) > 0)                     # sorted, unique
    assert rows.min() >= 0 and rows.max() < w.B * w.Hq * N
    by_head = {}
    for r in rows:
        by_head.setdefault(int(r) // N, set()).add(int(r) % N)
    assert sorted(by_head) == list(range(w.B * w.Hq))
    edges = {0, 1, 127, 128, 129, 255, 256, N - 129, N - 1}
    for bh, got in by_head.items():
        assert edges <= got, bh
        assert len(got) <= len(edges) + 23
    assert np.array_equal(rows, synth.sample_rows(w, per_head_random=23))
    # short sequences keep only the edge rows that exist
    tiny = synth.WORKLOADS["tiny"]
    t = synth.sample_rows(tiny, per_head_random=0)
    assert set(int(r) % tiny.Nq for r in t) == {0, 1, 127, 128, 129, 255, tiny.Nq - 129}
