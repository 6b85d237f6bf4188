"""GPU parity of decode over a paged KV cache ("Attention mechanisms ...",
section 20; "Transformer internals", PagedAttention: key j of a sequence in
block block_table[b][j / page_size] at offset j % page_size) against the fp64
oracle, which gathers the paged cache into a contiguous one.

The physical pages are shuffled; pages no sequence owns hold NaN and unused
table entries are -1, so a read of a wrong page shows up as NaN; rows of a
sequence's last page past its length hold a large finite sentinel, which
must get zero weight.  Tolerances: O max-abs <= 2e-2, mean-abs <= 2e-3,
lse <= 1e-3 against fp64."""
import math

import numpy as np
import pytest

import oracle
from exact_scaled_dot_fwd_b200 import synth

from parity import compare, from_dev, rand_inputs, to_dev

pytestmark = pytest.mark.gpu

NAN_BITS = 0x7FC0


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    return t


def run_paged(torch, x, page_size, causal, window, seed):
    import exact_scaled_dot_fwd_b200 as eb
    kl = x["key_lens"]
    table, num_pages = synth.paged_layout(kl, page_size, seed)
    kc = synth.to_paged(x["k"], table, kl, num_pages, page_size, NAN_BITS)
    vc = synth.to_paged(x["v"], table, kl, num_pages, page_size, NAN_BITS)
    q = to_dev(x["q"], torch)
    o, lse = eb.attn_fwd_paged(q, to_dev(kc, torch), to_dev(vc, torch),
                               torch.from_numpy(table).cuda(), torch.from_numpy(kl).cuda(),
                               causal=causal, window=window, scale=1 / math.sqrt(x["q"].shape[-1]))
    torch.cuda.synchronize()
    assert eb.device_status() == 0
    return from_dev(o), lse.cpu().numpy().astype(np.float64), (kc, vc, table)


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, page_size, causal, window, key_lens
    (4, 32, 1, 1, 3000, 128, 16, True, 0, [3000, 1, 16, 1234]),      # MQA, page-multiple and 1
    (3, 16, 4, 1, 2000, 128, 8, True, 0, [2000, 0, 777]),            # smallest pages, an empty cache
    (3, 16, 4, 1, 2000, 128, 32, True, 0, [129, 2000, 640]),
    (2, 8, 8, 1, 1500, 128, 64, True, 0, [1500, 65]),
    (2, 32, 8, 1, 1000, 128, 128, True, 0, [1000, 127]),             # one page per tile
    (3, 32, 8, 4, 2500, 128, 16, True, 0, [2500, 5, 1024]),          # multi-token, GQA
    (2, 16, 4, 2, 3000, 128, 16, True, 500, [3000, 700]),            # window
    (2, 16, 1, 3, 1800, 128, 32, True, 0, [1800, 900]),              # 48 rows per kv head
    (3, 16, 4, 1, 1200, 64, 16, True, 0, [1200, 33, 64]),            # d = 64 (mma.sync)
    (2, 8, 2, 3, 900, 64, 64, True, 0, [900, 100]),                  # d = 64, multi-token
    (2, 8, 2, 1, 900, 64, 8, False, 200, [900, 500]),                # d = 64, window
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:9])))
def test_paged_decode_parity(torch, case):
    B, Hq, Hkv, Nq, Nk, d, ps, causal, w, kl = case
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=9700 + Nk + ps, key_lens=kl)
    o, lse, (kc, vc, table) = run_paged(torch, x, ps, causal, w, seed=11 + ps)
    o_ref, lse_ref = oracle.attn_paged_rows(x["q"], kc, vc, table, x["key_lens"], causal,
                                            1 / math.sqrt(d), window=w)
    compare(o.reshape(-1, d), lse.reshape(-1), o_ref, lse_ref, what=str(case))
    # the same attention as the contiguous cache
    o_c, lse_c = oracle.attn_rows(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d),
                                  key_lens=x["key_lens"], window=w, align=1)
    assert np.array_equal(o_c, o_ref) and np.array_equal(lse_c, lse_ref)


def test_paged_rejects_bad_arguments(torch):
    import exact_scaled_dot_fwd_b200 as eb
    q = torch.zeros((1, 4, 1, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((4, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    table = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    kl = torch.tensor([20], dtype=torch.int32, device="cuda")
    with pytest.raises(eb.AttnError) as e:     # page size not a multiple of 8
        k12 = kc[:, :, :12].contiguous()
        eb.attn_fwd_paged(q, k12, k12, table, kl)
    assert e.value.status == 2
    q2 = torch.zeros((1, 64, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eb.AttnError) as e:     # 128 query rows per kv head
        eb.attn_fwd_paged(q2, kc, kc, table, kl)
    assert e.value.status == 2


@pytest.mark.parametrize("d,bad", [(128, 10 ** 6), (128, -3), (64, 1 << 30)])
def test_out_of_range_table_entry_is_reported_not_used(torch, d, bad):
    """A block-table entry outside [0, num_pages) inside a sequence's range:
    the kernels check it before using it as an address, read that page's
    keys and values as zeros, and record ATTN_ERANGE in the device status
    word.  (The check runs on the entry the kernel reads; no load leaves the
    cache.)  The output equals attention over the cache with those keys and
    values set to zero."""
    import exact_scaled_dot_fwd_b200 as eb
    B, Hq, Hkv, Nq, Nk, ps = 2, 16, 2, 1, 700, 16
    kl = [700, 300]
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=9900 + d, key_lens=kl)
    table, num_pages = synth.paged_layout(np.array(kl, np.int32), ps, 77)
    kc = synth.to_paged(x["k"], table, x["key_lens"], num_pages, ps, NAN_BITS)
    vc = synth.to_paged(x["v"], table, x["key_lens"], num_pages, ps, NAN_BITS)
    b_bad, p_bad = 1, 5                       # keys 80..95 of sequence 1
    table[b_bad, p_bad] = bad
    assert eb.device_status() == 0
    o, lse = eb.attn_fwd_paged(to_dev(x["q"], torch), to_dev(kc, torch), to_dev(vc, torch),
                               torch.from_numpy(table).cuda(), torch.from_numpy(x["key_lens"]).cuda(),
                               causal=True, scale=1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert eb.device_status() == 7            # ATTN_ERANGE, read and cleared
    assert eb.device_status() == 0
    k0, v0 = x["k"].copy(), x["v"].copy()
    k0[b_bad, :, p_bad * ps:(p_bad + 1) * ps] = 0
    v0[b_bad, :, p_bad * ps:(p_bad + 1) * ps] = 0
    o_ref, lse_ref = oracle.attn_rows(x["q"], k0, v0, True, 1 / math.sqrt(d),
                                      key_lens=x["key_lens"], align=1)
    compare(from_dev(o).reshape(-1, d), lse.cpu().numpy().astype(np.float64).reshape(-1),
            o_ref, lse_ref, what=f"bad entry {bad}")
