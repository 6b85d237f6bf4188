"""attn_fwd with a caller-registered workspace (attn_set_workspace): the
same results as with the library's own, ATTN_EWORKSPACE when the registered
buffer is too small (the library does not allocate in its place), and the
library's own workspace again after unregistering."""
import numpy as np
import pytest

from parity import rand_inputs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    from exact_scaled_dot_fwd_b200 import build
    build.build()
    return t


@pytest.mark.parametrize("shape", [(2, 4, 1, 1, 700, 128),      # decode: split partials
                                   (1, 2, 2, 200, 200, 64)])    # prefill: scheduler counter
def test_registered_workspace(torch, shape):
    import exact_scaled_dot_fwd_b200 as eb
    B, Hq, Hkv, Nq, Nk, d = shape
    lens = [Nk, Nk // 2 + 1][:B]
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=61, key_lens=lens)
    q, k, v = (to_dev(x[n], torch) for n in ("q", "k", "v"))
    kl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    causal = Nq > 1
    o_own, l_own = eb.attn_fwd(q, k, v, causal=causal, key_lens=kl)
    need = eb.attn_workspace_size(B, Hq, Hkv, Nq, Nk, d)
    assert need >= 256
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    eb.attn_set_workspace(ws)
    try:
        o_reg, l_reg = eb.attn_fwd(q, k, v, causal=causal, key_lens=kl)
        torch.cuda.synchronize()
        if need > 256:
            eb.attn_set_workspace(ws[:256])
            with pytest.raises(eb.AttnError) as e:
                eb.attn_fwd(q, k, v, causal=causal, key_lens=kl)
            assert e.value.status == 4
    finally:
        eb.attn_set_workspace(None)
    o_back, l_back = eb.attn_fwd(q, k, v, causal=causal, key_lens=kl)
    torch.cuda.synchronize()
    assert eb.device_status() == 0
    for o, l in ((o_reg, l_reg), (o_back, l_back)):
        assert torch.equal(o, o_own) and torch.equal(l, l_own)
    assert np.all(np.isfinite(o_own.float().cpu().numpy()))


@pytest.mark.parametrize("shape", [(2, 4, 1, 1, 700, 128),      # decode: temporary partials
                                   (1, 2, 2, 200, 200, 64)])    # prefill
def test_side_stream_matches_default_stream(torch, shape):
    """A call enqueued on a side stream with a workspace the binding allocates
    for it (window / align calls and paged decode do) gives the same bits as
    on the default stream: the temporary stays reserved for the side stream
    until the stream has passed the call, even after other work on the
    current stream reuses freed memory."""
    import exact_scaled_dot_fwd_b200 as eb
    B, Hq, Hkv, Nq, Nk, d = shape
    lens = [Nk, Nk // 3 + 1][:B]
    x = rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed=71, key_lens=lens)
    q, k, v = (to_dev(x[n], torch) for n in ("q", "k", "v"))
    kl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    causal = Nq > 1
    o_ref, l_ref = eb.attn_fwd(q, k, v, causal=causal, key_lens=kl, align=1)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    outs = []
    for _ in range(4):
        o, l = eb.attn_fwd(q, k, v, causal=causal, key_lens=kl, align=1, stream=side)
        outs.append((o, l))
        # current-stream work that would grab a freed temporary
        junk = torch.full((1 << 20,), 7, dtype=torch.uint8, device="cuda")
        del junk
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert eb.device_status() == 0
    for o, l in outs:
        assert torch.equal(o, o_ref) and torch.equal(l, l_ref)
