"""bench.py's work accounting on the CPU: which workloads are measured in HBM
bytes, the algorithmic bytes of a decode step, and the FLOPs of a windowed
workload, each against a count made independently here."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from exact_scaled_dot_fwd_b200 import synth  # noqa: E402


def test_memory_bound_workloads():
    W = synth.WORKLOADS
    assert bench.memory_bound(W["mqa_decode"])        # 32 rows per kv head
    assert bench.memory_bound(W["spec_decode"])       # 4 heads x 4 tokens
    for name in ("mha_prefill", "gqa_rope_prefill", "long_causal", "cross_padded", "long_window"):
        assert not bench.memory_bound(W[name]), name


def test_decode_bytes_count_each_valid_key_once():
    w = synth.WORKLOADS["mqa_decode"]
    kl = synth.uniform_key_lens(w.B, w.key_lens[0], w.key_lens[1], w.seed + 4)
    kv = sum(int(L) * w.Hkv * w.d * 2 * 2 for L in kl)          # K and V, bf16
    qo = w.B * w.Hq * w.Nq * w.d * 2 * 2                           # Q and O, bf16
    lse = w.B * w.Hq * w.Nq * 4
    assert bench.decode_bytes(w, kl) == kv + qo + lse
    # the same formula at several rows per kv head (multi-token decode)
    s = synth.WORKLOADS["spec_decode"]
    kl2 = synth.uniform_key_lens(s.B, s.key_lens[0], s.key_lens[1], s.seed + 4)
    assert bench.decode_bytes(s, kl2) == (float(kl2.sum()) * s.Hkv * s.d * 4
                                           + s.B * s.Hq * s.Nq * (s.d * 4 + 4))


def test_window_flops_count_visible_pairs():
    """4 d FLOPs per (row, key) pair inside a causal window, counted by brute
    force on a small shape and by the closed form on the bench workload."""
    n, w, d, B, H = 300, 37, 8, 2, 3
    small = synth.Workload("t", 99, B, H, H, n, n, d, True, window=w)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    pairs = int(((j <= i) & (i - j < w)).sum())
    assert small.flops() == 4.0 * B * H * d * pairs
    lw = synth.WORKLOADS["long_window"]
    N, W = lw.Nq, lw.window
    assert lw.flops() == 4.0 * lw.B * lw.Hq * lw.d * (W * (W + 1) // 2 + (N - W) * W)


def test_cpu_baseline_entry_reports_rate_and_extrapolation():
    w = synth.WORKLOADS["tiny_causal"]
    e = bench.cpu_baseline_entry(w, "TFLOP/s", seconds=0.05)
    assert e["kind"] == "oracle" and e["cores"] >= 1 and e["value"] > 0
    assert e["unit"].startswith("TFLOP/s")
    # rows/s times the extrapolated time is the workload's row count
    total_rows = w.B * w.Hq * w.Nq
    assert abs(e["rows_per_s"] * e["full_workload_s_extrapolated"] - total_rows) < 1e-6 * total_rows
    g = bench.cpu_baseline_entry(w, "GB/s", seconds=0.05)
    assert g["unit"].startswith("GB/s") and g["value"] > 0


def test_traffic_hash_follows_code_not_comments():
    src = ('int f(int x) {  // doubles x\n'
           '  /* block\n     comment */ return 2 * x;\n}\n'
           'const char* s = "// kept: inside a string";\n')
    base = bench.code_tokens(src)
    assert "doubles" not in base and "block" not in base
    assert "// kept: inside a string" in base
    # comment text, comment layout and blank lines do not matter ...
    assert bench.code_tokens(src.replace("doubles x", "returns twice x\n\n// more")) == base
    assert bench.code_tokens(src.replace("  return", "\n\n  return")) == base
    # ... the code does
    assert bench.code_tokens(src.replace("2 * x", "3 * x")) != base
    assert bench.code_tokens(src.replace("inside a string", "inside a strinG")) != base


def test_stored_captures_are_reported_only_for_the_captured_code(monkeypatch):
    # A stored ncu capture belongs to the kernel code it was taken on: the
    # bench line reports it while the code hashes the same and null after
    # any change to the code, until the kernel is captured again.
    cur = bench.source_hash("prefill")
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"a": ("prefill", cur, 123),
                                               "b": ("prefill", "0" * 16, 456)})
    monkeypatch.setattr(bench, "NCU_COUNTERS", {"a": ("prefill", cur, {"tensor_pipe_pct": 50.0}),
                                                "b": ("prefill", "0" * 16, {"x": 1})})
    assert bench.ncu_traffic("a") == 123 and bench.ncu_traffic("b") is None
    assert bench.ncu_counters("a") == {"tensor_pipe_pct": 50.0} and bench.ncu_counters("b") == {}
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0}
    r = bench.roofline("tensor", 700.0, peaks, "measured", "a")
    assert r["traffic"] == 123 and r["ncu_tensor_pipe_pct"] == 50.0
    assert bench.roofline("tensor", 700.0, peaks, "measured", "b")["traffic"] is None
    # every stored entry names a kernel whose sources exist
    for table in (bench.NCU_TRAFFIC, bench.NCU_COUNTERS):
        for kernel, digest, _ in table.values():
            assert len(bench.source_hash(kernel)) == len(digest) == 16


def test_roofline_object_reports_measured_and_nominal_fractions():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0}
    t = bench.roofline("tensor", 750.0, peaks, "measured", "no_such_workload")
    assert t["unit"] == "TFLOP/s" and t["peak"] == 1500.0 and abs(t["frac"] - 0.5) < 1e-12
    assert t["nominal_peak"] == 2250.0 and abs(t["frac_of_nominal"] - 750.0 / 2250.0) < 1e-12
    assert t["traffic"] is None                     # no capture stored for this workload
    h = bench.roofline("hbm", 4800.0, peaks, "fallback", "mqa_decode")
    assert h["unit"] == "GB/s" and abs(h["frac"] - 0.8) < 1e-12 and h["peak_source"] == "fallback"
    assert abs(h["frac_of_nominal"] - 0.6) < 1e-12
    assert h["traffic"] == bench.ncu_traffic("mqa_decode")


def test_reference_arm_reports_the_same_config(capsys):
    """Both arms print the config object of config_of, so the driver can
    match the lines; input_copies sizes the rotation above twice the L2."""
    import argparse
    import json
    w = synth.WORKLOADS["tiny"]
    bench.run_reference(argparse.Namespace(config="tiny", steps=1, warmup=0))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.config_of(w, *bench.input_copies(w), 1)
    for name in ("mha_prefill", "long_causal", "tiny"):
        x = synth.WORKLOADS[name]
        copies, per_copy = bench.input_copies(x)
        nbytes = 2 * (x.B * x.Hq * x.Nq * x.d + 2 * x.B * x.Hkv * x.Nk * x.d)
        assert per_copy == nbytes
        assert copies * per_copy >= min(2 * bench.L2_BYTES, 8 * per_copy)
        assert copies == 1 or (copies - 1) * per_copy < 2 * bench.L2_BYTES


def test_profile_case_keeps_the_group_size():
    import pytest
    w = synth.WORKLOADS["long_causal"]
    c = bench.profile_case(w, 8)
    assert (c.Hq, c.Hkv, c.Nq, c.Nk, c.d, c.causal) == (8, 8, w.Nq, w.Nk, w.d, w.causal)
    g = bench.profile_case(synth.WORKLOADS["gqa_rope_prefill"], 8)
    assert (g.Hq, g.Hkv) == (8, 2)
    assert bench.profile_case(w, 0) is w
    # FLOPs scale with the heads (the capture's traffic is scaled the same way)
    assert c.flops() * 4 == w.flops()
    with pytest.raises(SystemExit):
        bench.profile_case(synth.WORKLOADS["gqa_rope_prefill"], 6)
