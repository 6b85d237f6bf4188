"""The Python binding's argument checks, on the CPU.

Shapes, dtypes and lengths are checked before devices and before the library
is called, so these run without a GPU: a key_lens shorter than B or an out /
lse buffer of the wrong shape would otherwise let a kernel read or write past
the end of a buffer."""
import pytest
import torch

import exact_scaled_dot_fwd_b200 as eb


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


B, H, N, D = 2, 4, 8, 64


@pytest.fixture
def qkv():
    return bf16(B, H, N, D), bf16(B, H, N, D), bf16(B, H, N, D)


@pytest.mark.parametrize("fn", ["attn_fwd", "attn_fwd_decode_static", "attn_fwd_rope"])
def test_key_lens_must_have_B_entries(qkv, fn):
    q, k, v = qkv
    kl = torch.zeros(B + 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="key_lens has 3 entries"):
        if fn == "attn_fwd":
            eb.attn_fwd(q, k, v, key_lens=kl)
        elif fn == "attn_fwd_rope":
            eb.attn_fwd_rope(q, k, v, key_lens=kl)
        else:
            eb.attn_fwd_decode_static(bf16(B, H, 1, D), k, v, key_lens=kl)


def test_key_lens_dtype(qkv):
    q, k, v = qkv
    with pytest.raises(TypeError):
        eb.attn_fwd(q, k, v, key_lens=torch.zeros(B, dtype=torch.int64))


def test_out_shape_and_dtype(qkv):
    q, k, v = qkv
    with pytest.raises(ValueError, match="out has shape"):
        eb.attn_fwd(q, k, v, out=bf16(B, H, N - 1, D))
    with pytest.raises(TypeError):
        eb.attn_fwd(q, k, v, out=torch.zeros(q.shape, dtype=torch.float16))
    ws = torch.zeros(256, dtype=torch.uint8)
    with pytest.raises(ValueError, match="out has shape"):
        eb.attn_fwd_ws(q, k, v, ws, out=bf16(B, H, N, D // 2))


def test_lse_shape_and_dtype(qkv):
    q, k, v = qkv
    with pytest.raises(ValueError, match="lse has shape"):
        eb.attn_fwd(q, k, v, lse=torch.zeros((B, H, N - 1), dtype=torch.float32))
    with pytest.raises(TypeError):
        eb.attn_fwd(q, k, v, lse=torch.zeros((B, H, N), dtype=torch.float64))
    # a lse that is not returned is not checked (nor written)
    with pytest.raises(ValueError, match="CUDA device"):
        eb.attn_fwd(q, k, v, lse=torch.zeros(1), return_lse=False)


def test_paged_checks(qkv):
    q = bf16(B, H, 1, D)
    kc = bf16(10, H, 16, D)
    table = torch.zeros((B, 4), dtype=torch.int32)
    with pytest.raises(ValueError, match="needs key_lens"):
        eb.attn_fwd_paged(q, kc, kc, table, None)
    with pytest.raises(ValueError, match="key_lens has 1 entries"):
        eb.attn_fwd_paged(q, kc, kc, table, torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="lse has shape"):
        eb.attn_fwd_paged(q, kc, kc, table, torch.zeros(B, dtype=torch.int32),
                          lse=torch.zeros((B, H, 2), dtype=torch.float32))


def test_rope_apply_out_shape():
    x = bf16(1, 2, 4, 8)
    with pytest.raises(ValueError, match="out has shape"):
        eb.rope_apply(x, out=bf16(1, 2, 4, 4))


def test_well_formed_host_tensors_are_rejected_for_their_device(qkv):
    q, k, v = qkv
    with pytest.raises(ValueError, match="CUDA device"):
        eb.attn_fwd(q, k, v, key_lens=torch.zeros(B, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA device"):
        eb.rope_apply(q)
