#!/usr/bin/env python
"""Benchmark of the exact attention forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one pass of the hot path over one batch of the workload (default:
the long-context causal prefill, B=1, H=32, N=32768, d=128, the largest
single-GPU configuration).  Inputs are resident in HBM; each step reads one
of several input copies whose total exceeds the 126 MB L2 (one copy when a
single one already does), so no step finds its inputs in cache.  W untimed
warm-up steps precede K timed steps bracketed by a barrier and a device
synchronisation; the time is the maximum over ranks of CUDA-event time on
the launching stream.  For N > 1 (torchrun) every rank runs an independent
batch (weak scaling, no collective on the data path).

The JSON line also carries: the roofline of the dominant kernel (with the
stored ncu counters of its capture while the kernel code is unchanged), the
end-to-end figure through the public API with host buffers, the oracle timed
on host cores (rank 0, N=1, bounded sample), SM clocks sampled during the
timed region, the decode workload (MQA over a ragged KV cache) in GB/s, the
sliding-window prefill workload in useful TFLOP/s, the multi-token and paged
decode workloads, the GQA RoPE prefill step with separate RoPE passes and
with q's RoPE fused into the attention kernel, and the attention kernel alone
on the other prefill workloads (MHA prefill, padded cross attention, GQA).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_scaled_dot_fwd_b200 import synth  # noqa: E402

METRIC = "attention fwd TFLOPS (bf16, causal) and decode GB/s; % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024

# DRAM traffic per launch of the dominant kernel, from one ncu capture each
# (dram__bytes_read.sum + dram__bytes_write.sum; summaries in profiles/),
# with a hash of the kernel's source files at capture time.  The figure is
# reported only while the sources still hash the same.  The hash covers the
# code only: comments are dropped and whitespace runs collapse to one space,
# so a comment edit keeps the capture while any change to the code voids it.
KERNEL_SOURCES = {
    "prefill": ["prefill.cu", "tcgen05.cuh", "common.cuh", "tile_plan.cuh", "rope_math.cuh"],
    "decode": ["decode_tc.cu", "tcgen05.cuh", "common.cuh", "tile_plan.cuh"],
}
# workload: (kernel, source hash, DRAM bytes read + written per launch).
# long_causal and long_window were captured on their 8-head cuts (bench.py
# --profile-heads 8; a full launch holds 805 MB of inputs) and are scaled by
# 32 / 8: every head is an independent set of items over its own K/V.
# paged_decode is mqa_decode over a cache of 16-token pages (the bench's
# paged_decode object); gqa_rope_prefill is its attention kernel on rotated
# inputs (the rotation passes are separate kernels).
NCU_TRAFFIC = {
    "long_causal": ("prefill", "cf9fb7b089ed0128", (362489088 + 53635072) * 4),
    "mha_prefill": ("prefill", "cf9fb7b089ed0128", 132578304 + 13372928),
    "long_window": ("prefill", "cf9fb7b089ed0128", (241136128 + 48871424) * 4),
    "cross_padded": ("prefill", "cf9fb7b089ed0128", 122257152 + 8826624),
    "gqa_rope_prefill": ("prefill", "cf9fb7b089ed0128", 406414848 + 104055808),
    "mqa_decode": ("decode", "5707f1bdfff62684", 322999296 + 4343040),
    "spec_decode": ("decode", "5707f1bdfff62684", 508918784 + 4852480),
    "paged_decode": ("decode", "5707f1bdfff62684", 319074560 + 4551936),
}
# Further counters of the same captures (same keys and hash rule): the
# tensor-pipe utilisation of a prefill launch (sm__pipe_tensor_cycles_active,
# % of peak over the launch) and the DRAM throughput of a decode launch
# (dram__bytes.sum.per_second, GB/s).
NCU_COUNTERS = {
    "long_causal": ("prefill", "cf9fb7b089ed0128", {"tensor_pipe_pct": 58.9}),
    "mha_prefill": ("prefill", "cf9fb7b089ed0128", {"tensor_pipe_pct": 35.5}),
    "long_window": ("prefill", "cf9fb7b089ed0128", {"tensor_pipe_pct": 46.5}),
    "cross_padded": ("prefill", "cf9fb7b089ed0128", {"tensor_pipe_pct": 27.2}),
    "gqa_rope_prefill": ("prefill", "cf9fb7b089ed0128", {"tensor_pipe_pct": 57.0}),
    "mqa_decode": ("decode", "5707f1bdfff62684", {"dram_gbs": 5470.3}),
    "spec_decode": ("decode", "5707f1bdfff62684", {"dram_gbs": 6081.6}),
    "paged_decode": ("decode", "5707f1bdfff62684", {"dram_gbs": 4926.1}),
}


_COMMENT_OR_LITERAL = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^\\"\n])*"|\'(?:\\.|[^\\\'\n])*\'',
                                 re.S)


def code_tokens(src):
    """C/C++/CUDA source without comments (string and character literals
    kept as written), whitespace runs collapsed to one space."""
    kept = _COMMENT_OR_LITERAL.sub(lambda m: m.group(0) if m.group(0)[0] in "\"'" else " ", src)
    return " ".join(kept.split())


def source_hash(kernel):
    import hashlib
    m = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "exact_scaled_dot_fwd_b200", "csrc", f)) as fh:
            m.update(code_tokens(fh.read()).encode())
    return m.hexdigest()[:16]


def _stored(table, workload):
    entry = table.get(workload)
    if entry is None:
        return None
    kernel, digest, value = entry
    try:
        return value if source_hash(kernel) == digest else None
    except OSError:
        return None


def ncu_traffic(workload):
    """Measured DRAM bytes per launch, or None when not captured for this
    workload or when the kernel changed since the capture."""
    return _stored(NCU_TRAFFIC, workload)


def ncu_counters(workload):
    """The other stored counters of the workload's capture ({} when none
    match the current code)."""
    return dict(_stored(NCU_COUNTERS, workload) or {})


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--config", default="long_causal", choices=sorted(synth.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-window", action="store_true")
    p.add_argument("--no-rope", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the other prefill workloads (MHA prefill, padded cross attention, "
                        "the GQA attention kernel alone)")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--profile-heads", type=int, default=0,
                   help="cut the workload down to this many query heads (kv heads in "
                        "proportion): the smaller case an ncu capture of a large workload "
                        "runs on; its DRAM traffic scales with the heads")
    return p.parse_args()


# B200 datasheet figures (dense bf16 tensor, HBM3e): context beside the
# measured peaks, which are the roofline denominators.
NOMINAL_PEAKS = {"tensor": 2250.0, "hbm": 8000.0}


def roofline(bound, achieved, peaks, peak_src, workload):
    """The roofline object of a bench line: `achieved` against the measured
    peak (frac) and, labelled separately, against the nominal one; with the
    stored ncu counters of the workload's dominant kernel when they match
    the current code."""
    peak = peaks["bf16_tflops"] if bound == "tensor" else peaks["hbm_gbs"]
    nominal = NOMINAL_PEAKS[bound]
    r = {"bound": bound, "achieved": achieved, "peak": peak,
         "unit": "TFLOP/s" if bound == "tensor" else "GB/s", "frac": achieved / peak,
         "traffic": ncu_traffic(workload), "peak_source": peak_src,
         "nominal_peak": nominal, "frac_of_nominal": achieved / nominal}
    c = ncu_counters(workload)
    if bound == "tensor":
        r["ncu_tensor_pipe_pct"] = c.get("tensor_pipe_pct")
    else:
        r["ncu_dram_gbs"] = c.get("dram_gbs")
    return r


def profile_case(w, heads):
    """The workload with `heads` query heads and the kv heads in proportion
    (heads = 0: unchanged)."""
    if not heads:
        return w
    g = w.Hq // w.Hkv
    if heads % g or heads > w.Hq:
        raise SystemExit(f"--profile-heads {heads}: must be a multiple of {g} and <= {w.Hq}")
    import dataclasses
    return dataclasses.replace(w, Hq=heads, Hkv=heads // g)


def config_of(w, copies, per_copy, world):
    """The line's config object; both arms report the same one."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq,
            "Nk": w.Nk, "d": w.d, "causal": w.causal, "rope": w.rope,
            "key_lens": list(w.key_lens) if w.key_lens else None,
            "window": w.window, "align": w.align,
            "l2": f"{copies} rotating input copies ({copies * per_copy / 1e6:.0f} MB > "
                  f"126 MB L2)",
            "parallelism": f"replicas x{world} (independent batch per GPU)"}


def input_copies(w):
    """Copies of the inputs a step rotates over so that their total exceeds
    twice the L2 (1 when one copy already does), and the bytes of one copy."""
    per_copy = 2 * (w.B * w.Hq * w.Nq * w.d + 2 * w.B * w.Hkv * w.Nk * w.d)
    return max(1, min(8, math.ceil(2 * L2_BYTES / per_copy))), per_copy


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return {k: float(j[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks --

def gpu_selector(torch, device):
    """nvidia-smi -i argument for the torch device: its PCI bus id."""
    try:
        p = torch.cuda.get_device_properties(device)
        return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id=None):
        self.bus_id = bus_id
        self.proc = None
        self.out = None

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.bus_id:
            cmd[1:1] = ["-i", self.bus_id]
        try:
            self.out = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception as e:  # noqa: BLE001
            self.proc = None
            self.err = repr(e)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": ["nvidia-smi unavailable: " + getattr(self, "err", "")]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.seek(0)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ oracle --

def oracle_sample(w, seconds, seed=12345, rows_per_batch=None):
    """Time the fp64 oracle on uniformly sampled rows of workload w.
    Returns (useful_flops, elapsed_s, rows, threads)."""
    import oracle
    x = synth.make_inputs(w)
    total_rows = w.B * w.Hq * w.Nq
    rng = np.random.Generator(np.random.PCG64(seed))
    threads = oracle.default_threads()
    kl = x["key_lens"]

    def flops(rows):
        f = 0.0
        for r in rows:
            i = int(r % w.Nq)
            b = int(r // (w.Nq * w.Hq))
            L = w.Nk if kl is None else int(kl[b])
            lo, hi = oracle.visible_range(i, w.Nq, w.Nk, w.causal, L, w.window, w.align)
            f += 4.0 * w.d * (hi - lo)
        return f

    rope = (dict(base=synth.ROPE_BASE, pairing=0, q_pos_offset=0, k_pos_offset=0)
            if w.rope else None)
    n = rows_per_batch or 8 * threads
    used_f, used_t, used_rows = 0.0, 0.0, 0
    while used_t < seconds:
        rows = np.sort(rng.integers(0, total_rows, size=n)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attn_rows(x["q"], x["k"], x["v"], w.causal, w.scale, key_lens=kl, rows=rows,
                         rope_cfg=rope, nthreads=threads, window=w.window, align=w.align)
        dt = time.perf_counter() - t0
        used_f += flops(rows)
        used_t += dt
        used_rows += n
        if dt < 0.5 * seconds:
            n = min(n * 2, 1 << 16)
    return used_f, used_t, used_rows, threads


def cpu_baseline_entry(w, unit, seconds):
    """The bench line's cpu_baseline object: the oracle on a uniform row
    sample of workload w, in the line's unit, with rows/s and the whole
    workload's time extrapolated from the sample."""
    f, t, rows, thr = oracle_sample(w, seconds)
    e = {"value": f / t / 1e12, "unit": "TFLOP/s (useful, sampled rows)",
         "cores": thr, "kind": "oracle",
         "sample": f"{rows} uniformly drawn query rows of {w.name}, fp64, {t:.1f} s",
         "rows_per_s": rows / t,
         # uniform row sample: the whole workload costs total_rows / rows times as much
         "full_workload_s_extrapolated": t * (w.B * w.Hq * w.Nq) / rows}
    if unit == "GB/s":
        # bytes the sampled rows read (K and V of the visible keys: 4 d bytes per key)
        e["value"] = (f / (4.0 * w.d)) * w.d * 4 / t / 1e9
        e["unit"] = "GB/s (K/V bytes of sampled rows)"
    return e


# ------------------------------------------------------------------- ours ---

def to_dev(bits, torch, device):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def memory_bound(w):
    """Decode-shaped workloads (at most 64 query rows per kv head) are measured
    in HBM bytes; the rest in tensor FLOPs."""
    return w.Nq * (w.Hq // w.Hkv) <= 64


def decode_bytes(w, key_lens):
    """Algorithmic bytes of a decode step: K and V of every valid key once
    per kv head, plus Q, O (bf16) and lse (fp32).  No window here."""
    assert w.window == 0
    kl = np.full(w.B, w.Nk) if key_lens is None else np.clip(key_lens, 0, w.Nk)
    kv = float(kl.sum()) * w.Hkv * w.d * 2 * 2
    return kv + w.B * w.Hq * w.Nq * (w.d * 2 * 2 + 4)


def time_steps(fn, steps, torch, dist, stream):
    """Barrier + sync, events around `steps` calls of fn(i), sync + barrier;
    returns the max over ranks of the elapsed ms."""
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return reduce_max(e0.elapsed_time(e1), dist)


def reduce_max(value, dist):
    """Maximum of `value` over all ranks (identity without a process group).
    The tensor lives where the backend wants it: CUDA for NCCL, CPU for gloo."""
    if dist is None:
        return value
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_ours(args):
    import torch
    import exact_scaled_dot_fwd_b200 as eb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    eb.lib()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()

    w = profile_case(synth.WORKLOADS[args.config], args.profile_heads)
    # every rank processes its own batch: shift the seed by the rank
    wr = synth.Workload(**{**w.__dict__, "number": w.number + 100 * rank}) if rank else w
    x = synth.make_inputs(wr)
    copies, per_copy = input_copies(w)
    Q = [to_dev(x["q"], torch, device) for _ in range(copies)]
    K = [to_dev(x["k"], torch, device) for _ in range(copies)]
    V = [to_dev(x["v"], torch, device) for _ in range(copies)]
    kl = None if x["key_lens"] is None else torch.from_numpy(x["key_lens"]).to(device)
    O = torch.empty_like(Q[0])
    LSE = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=device)
    ws = torch.empty(eb.attn_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d),
                     dtype=torch.uint8, device=device)

    if w.rope:
        QR = torch.empty_like(Q[0])
        KR = torch.empty_like(K[0])

    def attn_only(i):
        c = i % copies
        q, k = (QR, KR) if w.rope else (Q[c], K[c])
        eb.attn_fwd_ws(q, k, V[c], ws, causal=w.causal, scale=w.scale, key_lens=kl,
                       out=O, lse=LSE, window=w.window, align=w.align)

    def step(i):
        # one pass of the whole path: the RoPE prologue (when the workload has
        # one) rotates Q and K in two rope_apply passes -- measured faster than
        # the fused rotation of Q (the bench's rope_prefill object has both) --
        # then the attention forward
        if w.rope:
            c = i % copies
            eb.rope_apply(Q[c], base=synth.ROPE_BASE, pairing=synth.ROPE_PAIRING_HALF, out=QR)
            eb.rope_apply(K[c], base=synth.ROPE_BASE, pairing=synth.ROPE_PAIRING_HALF, out=KR)
        attn_only(i)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    # size K so that the timed region lasts about two seconds by default
    probe = time_steps(step, 3, torch, dist, stream) / 3
    steps = args.steps or max(10, int(2000.0 / max(probe, 1e-3)))
    sampler = ClockSampler(gpu_selector(torch, device))
    sampler.start()
    time.sleep(0.3)
    ms = time_steps(step, steps, torch, dist, stream)
    clocks = sampler.stop()
    ms_step = ms / steps
    # this library's kernels per step: decode = split + combine; prefill = the
    # attention kernel (its counter reset is a runtime memset, not a kernel
    # of ours); plus the two RoPE launches when the workload has RoPE
    launches_per_step = (2 if memory_bound(w) else 1) + (2 if w.rope else 0)
    # the dominant kernel alone (differs from the step only when RoPE runs)
    ms_kernel = ms if not w.rope else time_steps(attn_only, steps, torch, dist, stream)
    if memory_bound(w):
        unit, work = "GB/s", decode_bytes(w, x["key_lens"])
        value = world * work * steps / (ms / 1e3) / 1e9
        kval = work * steps / (ms_kernel / 1e3) / 1e9
        roof = roofline("hbm", kval, peaks, peak_src, w.name)
    else:
        unit, work = "TFLOP/s", w.flops()
        value = world * work * steps / (ms / 1e3) / 1e12
        kval = work * steps / (ms_kernel / 1e3) / 1e12
        roof = roofline("tensor", kval, peaks, peak_src, w.name)
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, copies, per_copy, world),
        "roofline": roof,
        "gpu_launches": steps * launches_per_step,
        "clocks": clocks,
    }
    if clocks.get("sm_mhz"):
        # step time x median SM clock: comparable across runs at different clocks
        clocks["ms_x_mhz"] = ms_step * clocks["sm_mhz"]

    # ---- end to end through the public API with pinned host buffers
    if not args.no_e2e:
        hq = torch.from_numpy(x["q"].view(np.int16)).view(torch.bfloat16).pin_memory()
        hk = torch.from_numpy(x["k"].view(np.int16)).view(torch.bfloat16).pin_memory()
        hv = torch.from_numpy(x["v"].view(np.int16)).view(torch.bfloat16).pin_memory()
        ho = [torch.empty(O.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        hl = [torch.empty(LSE.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2
        d2h = ho[0].numel() * 2 + hl[0].numel() * 4
        e_steps = max(3, min(steps, 20))

        def path(q, k, v, o, lse):
            # the step's operations on one set of device buffers
            if w.rope:
                eb.rope_apply(q, base=synth.ROPE_BASE, pairing=synth.ROPE_PAIRING_HALF, out=QR)
                eb.rope_apply(k, base=synth.ROPE_BASE, pairing=synth.ROPE_PAIRING_HALF, out=KR)
                q, k = QR, KR
            eb.attn_fwd_ws(q, k, v, ws, causal=w.causal, scale=w.scale, key_lens=kl,
                           out=o, lse=lse, window=w.window, align=w.align)

        # serial: each step copies its inputs in, computes, copies O and lse
        # back, one after the other on the compute stream
        def e2e_serial(i):
            Q[0].copy_(hq, non_blocking=True)
            K[0].copy_(hk, non_blocking=True)
            V[0].copy_(hv, non_blocking=True)
            path(Q[0], K[0], V[0], O, LSE)
            ho[0].copy_(O, non_blocking=True)
            hl[0].copy_(LSE, non_blocking=True)

        for i in range(2):
            e2e_serial(i)
        ems_serial = time_steps(e2e_serial, e_steps, torch, dist, stream)

        # pipelined, as a server streams batches: step i's host-to-device copy
        # (copy stream) overlaps step i-1's compute (compute stream) and step
        # i-2's device-to-host copy (a third stream); device inputs and outputs
        # are double-buffered, and events keep each buffer's reuse in order.
        # Every step's copies and compute lie inside the timed region.
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        dq = [Q[0], torch.empty_like(Q[0])]
        dk = [K[0], torch.empty_like(K[0])]
        dv = [V[0], torch.empty_like(V[0])]
        do = [O, torch.empty_like(O)]
        dl = [LSE, torch.empty_like(LSE)]

        def e2e_pipelined(n):
            loaded, computed, stored = [None] * n, [None] * n, [None] * n
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(computed[i - 2])   # buffer b's inputs read
                    dq[b].copy_(hq, non_blocking=True)
                    dk[b].copy_(hk, non_blocking=True)
                    dv[b].copy_(hv, non_blocking=True)
                    loaded[i] = torch.cuda.Event()
                    loaded[i].record(s_in)
                stream.wait_event(loaded[i])
                if i >= 2:
                    stream.wait_event(stored[i - 2])       # buffer b's outputs copied out
                path(dq[b], dk[b], dv[b], do[b], dl[b])
                computed[i] = torch.cuda.Event()
                computed[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(computed[i])
                    ho[b].copy_(do[b], non_blocking=True)
                    hl[b].copy_(dl[b], non_blocking=True)
                    stored[i] = torch.cuda.Event()
                    stored[i].record(s_out)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)                      # the last copies end the region

        e2e_pipelined(3)
        torch.cuda.synchronize()
        ems = time_steps(lambda i: e2e_pipelined(e_steps), 1, torch, dist, stream)
        ev = world * work * e_steps / (ems / 1e3) / (1e9 if unit == "GB/s" else 1e12)
        ev_serial = world * work * e_steps / (ems_serial / 1e3) / (1e9 if unit == "GB/s" else 1e12)
        line["e2e"] = {"value": ev, "unit": unit, "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "steps": e_steps,
                       "ms_per_step": ems / e_steps,
                       "overlap": "pipelined: host-to-device copy, compute and device-to-host "
                                  "copy of consecutive steps on three streams",
                       "serial": {"value": ev_serial, "ms_per_step": ems_serial / e_steps}}
        del dq[1], dk[1], dv[1], do[1], dl[1]

    # ---- decode workload (HBM-bound half of the metric), same run
    if not args.no_decode and not memory_bound(w) and rank == 0 and world == 1:
        line["decode"] = run_decode(torch, eb, device, stream, peaks, peak_src)
        line["multi_token_decode"] = run_decode(torch, eb, device, stream, peaks, peak_src,
                                                name="spec_decode")
        line["paged_decode"] = run_decode(torch, eb, device, stream, peaks, peak_src,
                                          page_size=16)
    # ---- sliding-window prefill, same run
    if not args.no_window and w.name != "long_window" and rank == 0 and world == 1:
        line["window"] = run_window(torch, eb, device, stream, peaks, peak_src)
    # ---- GQA prefill with RoPE: separate RoPE passes vs q's RoPE fused
    if not args.no_rope and not w.rope and rank == 0 and world == 1:
        line["rope_prefill"] = run_rope(torch, eb, device, stream, peaks, peak_src)
    # ---- the other prefill workloads, each its attention kernel alone
    if not args.no_extra and rank == 0 and world == 1:
        for name in ("mha_prefill", "cross_padded", "gqa_rope_prefill", "long_causal"):
            if name != w.name:
                line[name] = run_prefill(torch, eb, device, stream, peaks, peak_src, name)

    # ---- oracle on host cores (rank 0, N=1 only)
    if not args.no_cpu and rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline_entry(w, unit, args.cpu_seconds)

    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_decode(torch, eb, device, stream, peaks, peak_src, steps=None, name="mqa_decode",
               page_size=0):
    """A decode workload in GB/s; page_size > 0 stores its KV cache in pages
    of that many tokens, shuffled, and runs the paged entry point."""
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    if page_size:
        table, num_pages = synth.paged_layout(x["key_lens"], page_size, w.seed + 6)
        x["k"] = synth.to_paged(x["k"], table, x["key_lens"], num_pages, page_size, 0)
        x["v"] = synth.to_paged(x["v"], table, x["key_lens"], num_pages, page_size, 0)
        table_d = torch.from_numpy(table).to(device)
    per_copy = x["k"].nbytes + x["v"].nbytes
    copies = 2
    Q = to_dev(x["q"], torch, device)
    K = [to_dev(x["k"], torch, device) for _ in range(copies)]
    V = [to_dev(x["v"], torch, device) for _ in range(copies)]
    kl = torch.from_numpy(x["key_lens"]).to(device)
    O = torch.empty_like(Q)
    LSE = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=device)
    ws = torch.empty(eb.attn_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d),
                     dtype=torch.uint8, device=device)

    def step(i):
        if page_size:
            eb.attn_fwd_paged(Q, K[i % copies], V[i % copies], table_d, kl, causal=w.causal,
                              scale=w.scale, window=w.window, workspace=ws, out=O, lse=LSE)
        else:
            eb.attn_fwd_ws(Q, K[i % copies], V[i % copies], ws, causal=w.causal, scale=w.scale,
                           key_lens=kl, out=O, lse=LSE, window=w.window, align=w.align)

    for i in range(5):
        step(i)
    probe = time_steps(step, 5, torch, None, stream) / 5
    n = steps or max(20, int(1000.0 / max(probe, 1e-3)))
    ms = time_steps(step, n, torch, None, stream)
    gbs = decode_bytes(w, x["key_lens"]) * n / (ms / 1e3) / 1e9
    return {"metric": "decode GB/s (algorithmic bytes: K/V of valid keys + Q + O + lse)",
            "value": gbs, "unit": "GB/s", "workload": w.name, "steps": n, "ms_per_step": ms / n,
            "page_size": page_size or None,
            "algorithmic_bytes": decode_bytes(w, x["key_lens"]),
            "l2": f"{copies} rotating KV caches ({copies * per_copy / 1e6:.0f} MB allocated)",
            "roofline": roofline("hbm", gbs, peaks, peak_src,
                                 "paged_decode" if page_size else w.name),
            "gpu_launches": 2 * n}


def run_rope(torch, eb, device, stream, peaks, peak_src, steps=None):
    """The GQA RoPE prefill step two ways (inputs larger than L2, one copy):
    rope_apply on Q and K then attention, and rope_apply on K then attention
    with q's RoPE fused in.  Useful FLOPs of the attention (4*B*Hq*N*N*d / 2)
    over the whole step."""
    w = synth.WORKLOADS["gqa_rope_prefill"]
    x = synth.make_inputs(w)
    q, k, v = (to_dev(x[n], torch, device) for n in ("q", "k", "v"))
    qr, kr = torch.empty_like(q), torch.empty_like(k)
    O = torch.empty_like(q)
    LSE = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=device)
    ws = torch.empty(eb.attn_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d),
                     dtype=torch.uint8, device=device)
    wsr = torch.empty(eb.lib().attn_rope_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d),
                      dtype=torch.uint8, device=device)
    rb, rp = synth.ROPE_BASE, synth.ROPE_PAIRING_HALF

    def separate(i):
        eb.rope_apply(q, base=rb, pairing=rp, out=qr)
        eb.rope_apply(k, base=rb, pairing=rp, out=kr)
        eb.attn_fwd_ws(qr, kr, v, ws, causal=True, scale=w.scale, out=O, lse=LSE)

    def fused(i):
        eb.rope_apply(k, base=rb, pairing=rp, out=kr)
        eb.attn_fwd_rope(q, kr, v, causal=True, scale=w.scale, rope_base=rb, rope_pairing=rp,
                         workspace=wsr, out=O, lse=LSE)

    out = {"metric": "useful TFLOP/s of the whole step (RoPE + attention)", "unit": "TFLOP/s",
           "workload": w.name}
    for name, fn in (("separate", separate), ("fused_q", fused)):
        for i in range(3):
            fn(i)
        probe = time_steps(fn, 2, torch, None, stream) / 2
        n = steps or max(5, int(1000.0 / max(probe, 1e-3)))
        ms = time_steps(fn, n, torch, None, stream)
        out[name] = {"value": w.flops() * n / (ms / 1e3) / 1e12, "ms_per_step": ms / n,
                     # separate: 2 rope_apply + attention; fused: rope_apply on K,
                     # the cos/sin table, attention
                     "steps": n, "gpu_launches": 3 * n}
    out["value"] = out["fused_q"]["value"]
    return out


def run_prefill(torch, eb, device, stream, peaks, peak_src, name, steps=None):
    """The attention kernel alone on a prefill workload (inputs rotating over
    copies larger than L2; a RoPE workload's q and k are rotated once,
    outside the timed region)."""
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    copies, per_copy = input_copies(w)
    Q = [to_dev(x["q"], torch, device) for _ in range(copies)]
    K = [to_dev(x["k"], torch, device) for _ in range(copies)]
    V = [to_dev(x["v"], torch, device) for _ in range(copies)]
    if w.rope:
        for c in range(copies):
            eb.rope_apply(Q[c], base=synth.ROPE_BASE, pairing=synth.ROPE_PAIRING_HALF, out=Q[c])
            eb.rope_apply(K[c], base=synth.ROPE_BASE, pairing=synth.ROPE_PAIRING_HALF, out=K[c])
    kl = None if x["key_lens"] is None else torch.from_numpy(x["key_lens"]).to(device)
    O = torch.empty_like(Q[0])
    LSE = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=device)
    ws = torch.empty(eb.attn_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d),
                     dtype=torch.uint8, device=device)

    def step(i):
        c = i % copies
        eb.attn_fwd_ws(Q[c], K[c], V[c], ws, causal=w.causal, scale=w.scale, key_lens=kl,
                       out=O, lse=LSE, window=w.window, align=w.align)

    for i in range(3):
        step(i)
    probe = time_steps(step, 3, torch, None, stream) / 3
    n = steps or max(10, int(1000.0 / max(probe, 1e-3)))
    ms = time_steps(step, n, torch, None, stream)
    tf = w.flops() * n / (ms / 1e3) / 1e12
    return {"metric": "attention fwd TFLOPS (formula FLOPs 4*B*Hq*Nq*Nk*d, halved for causal)",
            "value": tf, "unit": "TFLOP/s", "workload": w.name, "steps": n,
            "ms_per_step": ms / n, "flops_per_step": w.flops(),
            "config": config_of(w, copies, per_copy, 1),
            "roofline": roofline("tensor", tf, peaks, peak_src, w.name),
            "gpu_launches": n}


def run_window(torch, eb, device, stream, peaks, peak_src, steps=None):
    """The sliding-window prefill workload (inputs larger than L2, one copy)."""
    w = synth.WORKLOADS["long_window"]
    x = synth.make_inputs(w)
    q, k, v = (to_dev(x[n], torch, device) for n in ("q", "k", "v"))
    O = torch.empty_like(q)
    LSE = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=device)
    ws = torch.empty(eb.attn_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d),
                     dtype=torch.uint8, device=device)

    def step(i):
        eb.attn_fwd_ws(q, k, v, ws, causal=w.causal, scale=w.scale, out=O, lse=LSE,
                       window=w.window)

    for i in range(3):
        step(i)
    probe = time_steps(step, 3, torch, None, stream) / 3
    n = steps or max(10, int(1000.0 / max(probe, 1e-3)))
    ms = time_steps(step, n, torch, None, stream)
    tf = w.flops() * n / (ms / 1e3) / 1e12
    mb = (x["q"].nbytes + x["k"].nbytes + x["v"].nbytes) / 1e6
    return {"metric": "useful TFLOP/s (4 d per visible (row, key) pair)", "value": tf,
            "unit": "TFLOP/s", "workload": w.name, "window": w.window, "steps": n,
            "ms_per_step": ms / n, "flops_per_step": w.flops(),
            "l2": f"inputs {mb:.0f} MB > 126 MB L2",
            "roofline": roofline("tensor", tf, peaks, peak_src, w.name),
            "gpu_launches": n}


# -------------------------------------------------------------- reference ---

def run_reference(args):
    """The oracle as the reference arm: each step is a bounded sample of rows
    of the same workload, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    w = synth.WORKLOADS[args.config]
    threads = oracle.default_threads()
    x = synth.make_inputs(w)
    kl = x["key_lens"]
    rng = np.random.Generator(np.random.PCG64(777))
    rope = (dict(base=synth.ROPE_BASE, pairing=0, q_pos_offset=0, k_pos_offset=0)
            if w.rope else None)
    rows_per_step = 4 * threads
    total_rows = w.B * w.Hq * w.Nq

    def one(rows):
        oracle.attn_rows(x["q"], x["k"], x["v"], w.causal, w.scale, key_lens=kl, rows=rows,
                         rope_cfg=rope, nthreads=threads, window=w.window, align=w.align)

    def flops(rows):
        f = 0.0
        for r in rows:
            i = int(r % w.Nq)
            b = int(r // (w.Nq * w.Hq))
            L = w.Nk if kl is None else int(kl[b])
            lo, hi = oracle.visible_range(i, w.Nq, w.Nk, w.causal, L, w.window, w.align)
            f += 4.0 * w.d * (hi - lo)
        return f

    steps = args.steps or 5
    for _ in range(args.warmup):
        one(np.sort(rng.integers(0, total_rows, size=rows_per_step)))
    t_total, f_total = 0.0, 0.0
    for _ in range(steps):
        rows = np.sort(rng.integers(0, total_rows, size=rows_per_step)).astype(np.int64)
        t0 = time.perf_counter()
        one(rows)
        t_total += time.perf_counter() - t0
        f_total += flops(rows)
    if memory_bound(w):
        unit = "GB/s"
        value = (f_total / (4.0 * w.d)) * w.d * 4 / t_total / 1e9
    else:
        unit = "TFLOP/s"
        value = f_total / t_total / 1e12
    sample = f"{rows_per_step} uniformly drawn query rows of {w.name} per step, fp64 oracle"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit,
            "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t_total / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, *input_copies(w), world),
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                             "sample": sample,
                             "rows_per_s": steps * rows_per_step / t_total,
                             "full_workload_s_extrapolated":
                                 t_total * total_rows / (steps * rows_per_step)},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
