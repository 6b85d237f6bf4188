"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare against the fp64 oracle on the same seeded bf16 inputs."""
import numpy as np

import oracle
from exact_scaled_dot_fwd_b200 import synth

# Tolerances of the method's result against fp64 (bf16 inputs, fp32
# accumulation, bf16 output): O max-abs / mean-abs, lse abs.
TOL_O_MAX = 2e-2
TOL_O_MEAN = 2e-3
TOL_LSE = 1e-3


def rand_inputs(B, Hq, Hkv, Nq, Nk, d, seed, key_lens=None, std=1.0):
    """Seeded bf16 q/k/v; keys at or beyond key_lens[b] hold a large finite
    sentinel (they must get zero weight)."""
    x = {"q": synth.normal_bf16((B, Hq, Nq, d), seed, std),
         "k": synth.normal_bf16((B, Hkv, Nk, d), seed + 1, std),
         "v": synth.normal_bf16((B, Hkv, Nk, d), seed + 2),
         "key_lens": None if key_lens is None else np.asarray(key_lens, np.int32)}
    if key_lens is not None:
        sent = synth.bf16_bits_from_f32(np.array([synth.PAD_SENTINEL], np.float32))[0]
        for b, L in enumerate(key_lens):
            x["k"][b, :, L:] = sent
            x["v"][b, :, L:] = sent
    return x


def to_dev(x, torch):
    """uint16 bf16 bits (numpy) -> CUDA bf16 tensor, bit-exact."""
    t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def from_dev(t):
    """CUDA bf16 tensor -> float64 numpy (exact)."""
    import torch
    bits = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def run_gpu(inputs, causal, scale, rope=None, window=0, align=0):
    """Attention through the C ABI; returns (o float64 [B,Hq,Nq,d], lse float64)."""
    import torch
    import exact_scaled_dot_fwd_b200 as eb
    q, k, v = (to_dev(inputs[n], torch) for n in ("q", "k", "v"))
    kl = inputs.get("key_lens")
    kl_t = None if kl is None else torch.from_numpy(np.asarray(kl, np.int32)).cuda()
    if rope is not None:
        q = eb.rope_apply(q, base=rope["base"], pos_offset=rope.get("q_pos_offset", 0),
                          pairing=rope["pairing"])
        k = eb.rope_apply(k, base=rope["base"], pos_offset=rope.get("k_pos_offset", 0),
                          pairing=rope["pairing"])
    o, lse = eb.attn_fwd(q, k, v, causal=causal, scale=scale, key_lens=kl_t, window=window,
                         align=align)
    torch.cuda.synchronize()
    assert eb.device_status() == 0
    return from_dev(o), lse.cpu().numpy().astype(np.float64)


def compare(o_gpu_rows, lse_gpu_rows, o_ref, lse_ref, what=""):
    """Element-wise check of selected rows.  Returns the error summary."""
    assert np.all(np.isfinite(o_gpu_rows)), f"{what}: NaN/Inf in O"
    err = np.abs(o_gpu_rows - o_ref)
    empty = np.isneginf(lse_ref)
    full = ~empty
    res = {"o_max": float(err.max()) if err.size else 0.0,
           "o_mean": float(err.mean()) if err.size else 0.0}
    if full.any():
        res["lse_max"] = float(np.abs(lse_gpu_rows[full] - lse_ref[full]).max())
    else:
        res["lse_max"] = 0.0
    assert res["o_max"] <= TOL_O_MAX, f"{what}: O max-abs {res['o_max']}"
    assert res["o_mean"] <= TOL_O_MEAN, f"{what}: O mean-abs {res['o_mean']}"
    assert res["lse_max"] <= TOL_LSE, f"{what}: lse abs {res['lse_max']}"
    # rows without a visible key: O = 0 exactly and lse = -inf
    if empty.any():
        assert np.all(o_gpu_rows[empty] == 0.0), f"{what}: empty rows not zero"
        assert np.all(np.isneginf(lse_gpu_rows[empty])), f"{what}: empty rows lse"
    return res


def check_workload(inputs, shape, causal, scale, rows=None, rope=None, what="", window=0,
                   align=0):
    """Run GPU + oracle on the same inputs; rows = flat row ids or None (all)."""
    B, Hq, Nq, d = shape
    o, lse = run_gpu(inputs, causal, scale, rope=rope, window=window, align=align)
    o = o.reshape(-1, d)
    lse = lse.reshape(-1)
    o_ref, lse_ref = oracle.attn_rows(inputs["q"], inputs["k"], inputs["v"], causal, scale,
                                      key_lens=inputs.get("key_lens"), rows=rows,
                                      rope_cfg=rope, window=window, align=align)
    sel = slice(None) if rows is None else rows
    return compare(o[sel], lse[sel], o_ref, lse_ref, what)
