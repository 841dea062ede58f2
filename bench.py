"""Benchmark of the joint (prefix-LM) attention on B200: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one joint-prefill call (pi_attn_prefill) over one batch of the pi0
workload: B=8, Hq=8, Hkv=1, d=256, S=611 (2 x 256 image patches + 48 text
tokens, ar_mask False; 1 state token True; 50 action tokens, the first True).
`value` is unmasked attention pairs per second, counted per (batch, query
head, query token, visible key), for the whole job; FLOPs are 4 * d per pair.
Inputs rotate over enough distinct sets that each step reads HBM-cold inputs
(more than twice the 126 MB L2); the timed loop replays CUDA graphs of the
ABI calls, timed with CUDA events on the launching stream.

The same line also carries the suffix-pass figure of the pi0 Euler loop
(B=32, 816-token prefix cache, 10 steps x 51 suffix tokens): microseconds per
10-step control, and the roofline, e2e (host buffers through the C ABI),
clocks and CPU-oracle baseline objects.

N > 1 (torchrun, one process per GPU): every rank runs its own batch shard of
the same per-rank size (weak scaling, no data-path collective); the timed
region is bracketed by barriers and the max over ranks is reported.

--impl reference times the CPU oracle (numpy float64) on a bounded sample of
the same workload; under torchrun only rank 0 runs it.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "unmasked attn pairs/s + TFLOP/s vs bf16 TC peak; suffix-pass µs per 10-step ctrl"
L2_BYTES = 126 * 2**20

# DRAM traffic of the prefill kernel per launch on the pi0 workload, from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum); valid only for the
# kernel sources whose digest is recorded beside it.
TRAFFIC = {"bytes": 25184896, "src_sha": "f6025ed41baa6bac"}
KERNEL_SOURCES = ("vla_prefix_lm_b200/csrc/tc_pair.cu", "vla_prefix_lm_b200/csrc/common.cuh",
                  "vla_prefix_lm_b200/csrc/mask.cuh")


def kernel_digest() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------------ counts


def visible_pairs_per_bh(ar, seg=None, P=0):
    """Unmasked (query, key) pairs of one (batch, head), by the prefix-LM rule.

    Counted from the per-token block index: with cs non-decreasing, query i
    sees every key j with cs[j] <= cs[i], minus FAST keys for expert queries;
    suffix queries also see all P cached keys.
    """
    ar = np.asarray(ar) != 0
    cs = np.cumsum(ar)
    n_le = np.searchsorted(cs, cs, side="right")          # keys with cs <= cs[i]
    total = int(n_le.sum()) + P * len(cs)
    if seg is not None:
        seg = np.asarray(seg)
        fast_cs = np.sort(cs[seg == 1])
        total -= int(np.searchsorted(fast_cs, cs[seg == 2], side="right").sum())
    return total


# ------------------------------------------------------------------ clocks


class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        use = inside if inside else rows
        reasons = sorted({n for r in use for n, v in zip(self.NAMES, r[3]) if v == "Active"})
        return {"sm_mhz": float(np.median([r[1] for r in use])) if use else None,
                "sm_max_mhz": max((r[2] for r in use), default=None),
                "reasons": reasons, "samples": len(inside),
                "window": "timed region" if inside else "whole run (region shorter than a sample)"}


def gpu_id(dev) -> str:
    """An nvidia-smi -i selector for this device (UUID, else PCI id, else index)."""
    import torch
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    if uuid is not None:
        u = str(uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    try:
        return "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    except AttributeError:
        return str(dev.index or 0)


# ------------------------------------------------------------------ our arm


def run_ours(args, rank, ws, local):
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    binding.lib()  # fails loudly without the CUDA library
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    P = peaks()

    w = W.workload(2)
    B = w.B                                   # per-rank batch (weak scaling)
    pairs_bh = visible_pairs_per_bh(w.ar)
    pairs_step = pairs_bh * B * w.Hq
    flops_step = 4.0 * w.d * pairs_step
    bytes_step = (B * w.Sq * w.Hq * w.d * 2) * 2 + (B * w.Sq * w.d * 2) * 2 + w.Sq

    # rotating device-resident input sets: > 2 x L2 in total
    set_bytes = B * w.Sq * (w.Hq + 2) * w.d * 2
    n_sets = max(3, int(np.ceil(2 * L2_BYTES / set_bytes)))
    sets = []
    for i in range(n_sets):
        x = W.prefill_inputs(w, W.seed_for(2, 100 + rank * 1000 + i), B=B)
        sets.append((x.q.to(dev), x.k.to(dev), x.v.to(dev), x.ar.to(dev)))
    outs = [torch.empty_like(s[0]) for s in sets]

    def step(i):
        q, k, v, ar = sets[i % n_sets]
        binding.pi_attn_prefill(q, k, v, ar, out=outs[i % n_sets], stream=stream)

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 1)):
            step(i)
    torch.cuda.synchronize()
    assert binding.pi_attn_read_status(stream) == binding.PI_OK

    # one graph per chunk of steps (a whole number of input rotations)
    chunk = n_sets * max(1, min(64 // n_sets, args.steps // n_sets or 1))
    graphs = {}

    def graph_for(n):
        if n not in graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    step(i)
            graphs[n] = g
        return graphs[n]

    plan = [chunk] * (args.steps // chunk) + ([args.steps % chunk] if args.steps % chunk else [])
    # CUDAGraph.replay() launches on torch's current stream: make it `stream`,
    # the stream the timing events are recorded on.
    with torch.cuda.stream(stream):
        for n in set(plan):
            graph_for(n).replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(gpu_id(dev)) if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for n in plan:
            graph_for(n).replay()
        e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    dist.barrier()
    ms = e0.elapsed_time(e1)
    clocks = sampler.stop(t_wall0, t_wall1) if sampler else None
    ms_max = dist.max_over_ranks(ms)
    status = binding.pi_attn_read_status(stream)
    if status != binding.PI_OK:
        raise RuntimeError(f"device status after timing: {binding.status_string(status)}")

    value = ws * pairs_step * args.steps / (ms_max / 1e3)
    ms_step = ms_max / args.steps
    achieved_tflops = flops_step / (ms / args.steps / 1e3) / 1e12

    # e2e: host (pinned) buffers through the public API, copies inside the region
    n_e2e = max(3, min(args.steps, 200))
    hq = [s[0].cpu().pin_memory() for s in sets[:2]]
    hk = [s[1].cpu().pin_memory() for s in sets[:2]]
    hv = [s[2].cpu().pin_memory() for s in sets[:2]]
    har = [s[3].cpu().pin_memory() for s in sets[:2]]
    dq, dk, dv, dar = (torch.empty_like(sets[0][j]) for j in range(4))
    hout = torch.empty(outs[0].shape, dtype=outs[0].dtype, pin_memory=True)
    h2d = hq[0].nbytes + hk[0].nbytes + hv[0].nbytes + har[0].nbytes
    d2h = hout.nbytes

    def e2e_step(i):
        j = i % 2
        with torch.cuda.stream(stream):
            dq.copy_(hq[j], non_blocking=True)
            dk.copy_(hk[j], non_blocking=True)
            dv.copy_(hv[j], non_blocking=True)
            dar.copy_(har[j], non_blocking=True)
            o = binding.pi_attn_prefill(dq, dk, dv, dar, out=outs[0], stream=stream)
            hout.copy_(o, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    dist.barrier()
    e0.record(stream)
    for i in range(n_e2e):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    e2e_ms = dist.max_over_ranks(e0.elapsed_time(e1))
    e2e_value = ws * pairs_step * n_e2e / (e2e_ms / 1e3)

    # suffix pass: 10 Euler steps against the prefix cache (warm L2, back to back)
    suffix = suffix_control(args, dev, stream, rank)
    decode = decode_steps(args, dev, stream, rank)
    prepost = prepost_steps(args, dev, stream, rank)
    bwd = backward_steps(args, dev, stream, rank)

    traffic = TRAFFIC["bytes"] if TRAFFIC["src_sha"] == kernel_digest() else None
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "pairs/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)*d^-0.25 q/k/v rounded to bf16)",
        "config": {
            "workload": "pi0_joint_prefill: B=8 per rank, Hq=8, Hkv=1, d=256, S=611 "
                        "(560 prefix False | state True | 50 actions True,False*49)",
            "per_rank_batch": B,
            "global_batch": B * ws,
            "seq_len": w.Sq,
            "parallelism": f"batch replicas x{ws} (no data-path collective)",
            "l2": f"inputs rotate over {n_sets} device-resident sets "
                  f"({n_sets * set_bytes / 2**20:.0f} MiB > 2 x L2)",
            "timing": "CUDA events on the launching stream around CUDA-graph replays "
                      f"of {chunk} calls; max over ranks",
        },
        "tflops": ws * flops_step * args.steps / (ms_max / 1e3) / 1e12,
        "gb_per_s_algorithmic": bytes_step / (ms_step / 1e3) / 1e9,
        "roofline": {
            "bound": "tensor",
            "kernel": "tc_pair_kernel<prefill>",
            "achieved": achieved_tflops,
            "peak": P["bf16_tflops"],
            "unit": "TFLOP/s",
            "frac": achieved_tflops / P["bf16_tflops"],
            "peak_source": f"{P['source']} bf16 dense (burst)",
            "frac_of_sustained": (achieved_tflops / P["bf16_tflops_sustained"]
                                  if P["bf16_tflops_sustained"] else None),
            "traffic": traffic,
            "algorithmic_flop_per_launch": flops_step,
        },
        "e2e": {"value": e2e_value, "unit": "pairs/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n_e2e,
                "what": "pinned host q/k/v/ar -> device, pi_attn_prefill, out -> pinned host"},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "suffix_ctrl": suffix,
        "decode": decode,
        "prepost": prepost,
        "backward": bwd,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, seconds=args.cpu_seconds)
    return line


def _cold_graph_us(fn, stream, reps=20):
    """Median device time of one graph replay of ``fn`` with L2 flushed before each."""
    import torch

    with torch.cuda.stream(stream):
        for _ in range(3):
            fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=stream.device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t = []
    for _ in range(reps):
        with torch.cuda.stream(stream):
            flush.fill_(1.0)
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        t.append(e0.elapsed_time(e1) * 1e3)
    del g, flush
    return float(np.median(t))


def prepost_steps(args, dev, stream, rank):
    """RoPE and the Euler update around the attention, each timed alone (cold
    L2), and the whole pi0 sampling loop -- per step RoPE of the suffix q/k at
    the continued positions, the suffix pass, the Euler update -- as one graph."""
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    P_ = peaks()
    hbm = P_["hbm_gbs"]
    res = {}
    # prefill: q [8, 611, 8, 256], k [8, 611, 1, 256] bf16, all tokens valid
    B, S, Hq, d = 8, 611, 8, 256
    q, _ = W.draw((B, S, Hq, d), 9101 + rank, d, "bf16")
    k, _ = W.draw((B, S, 1, d), 9102 + rank, d, "bf16")
    q, k = q.to(dev), k.to(dev)
    tm = torch.ones((B, S), dtype=torch.uint8, device=dev)
    us = dist.max_over_ranks(_cold_graph_us(
        lambda: binding.pi_rope_inplace(q, k, tm, stream=stream), stream))
    nb = 2 * (q.numel() + k.numel()) * 2 + tm.numel()
    res["rope_prefill"] = {"shape": "q [8,611,8,256], k [8,611,1,256] bf16", "us_cold_l2": us,
                           "algorithmic_bytes": nb, "gb_per_s": nb / us / 1e3,
                           "hbm_frac": nb / us / 1e3 / hbm}
    del q, k, tm

    # suffix loop of the pi0 workload: B=32, 51 suffix tokens, cache 816, 10 steps
    w = W.workload(3)
    c = W.cache_inputs(w, W.seed_for(3, 999) + rank * 7, B=w.B)
    kc, vc = c.k.to(dev), c.v.to(dev)
    steps = [W.suffix_inputs(w, W.seed_for(3, s) + rank * 7, B=w.B) for s in range(w.calls)]
    ins = [(x.q.to(dev), x.k.to(dev), x.v.to(dev), x.ar.to(dev)) for x in steps]
    outs = [torch.empty_like(x[0]) for x in ins]
    pm = torch.ones((w.B, w.P), dtype=torch.uint8, device=dev)
    sm_ = torch.ones((w.B, w.Sq), dtype=torch.uint8, device=dev)
    A, D = w.Sq - 1, 32
    x = torch.zeros((w.B, A, D), dtype=torch.float32, device=dev)
    vel = [torch.randn((w.B, A, D), dtype=torch.float32, device=dev) for _ in range(w.calls)]
    need = binding.pi_attn_suffix_workspace_bytes(ins[0][0], ins[0][1], kc, ins[0][3])
    wsb = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    q0, k0 = ins[0][0], ins[0][1]
    us = dist.max_over_ranks(_cold_graph_us(
        lambda: binding.pi_rope_inplace(q0, k0, sm_, prefix_mask=pm, stream=stream), stream))
    nb = 2 * (q0.numel() + k0.numel()) * 2 + sm_.numel() + pm.numel()
    res["rope_suffix"] = {"shape": "q [32,51,8,256], k [32,51,1,256] bf16, prefix mask [32,816]",
                          "us_cold_l2": us, "algorithmic_bytes": nb, "gb_per_s": nb / us / 1e3,
                          "hbm_frac": nb / us / 1e3 / hbm}
    us = dist.max_over_ranks(_cold_graph_us(
        lambda: binding.pi_euler_update(x, vel[0], -0.1, stream=stream), stream))
    nb = 3 * x.numel() * 4
    res["euler"] = {"shape": "x, v [32,50,32] fp32", "us_cold_l2": us, "algorithmic_bytes": nb,
                    "gb_per_s": nb / us / 1e3}

    def ctrl():
        for s, (q, k, v, ar) in enumerate(ins):
            binding.pi_rope_inplace(q, k, sm_, prefix_mask=pm, stream=stream)
            binding.pi_attn_suffix(q, k, v, kc, vc, ar, out=outs[s], workspace=wsb, stream=stream)
            binding.pi_euler_update(x, vel[s], -1.0 / w.calls, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            ctrl()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        ctrl()
    reps = max(5, min(200, args.steps // 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us_ctrl = dist.max_over_ranks(e0.elapsed_time(e1) * 1e3 / reps)
    del g
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    res["sampling_loop"] = {
        "workload": "pi0 10-step loop: RoPE(suffix q/k) + suffix pass + Euler per step, B=32",
        "us_per_ctrl": us_ctrl, "gpu_launches_per_ctrl": 3 * w.calls,
        "timing": f"one graph of 30 launches replayed {reps}x (warm L2)"}
    return res


def backward_steps(args, dev, stream, rank):
    """Gradient of the pi0 joint prefill (B=8, S=611): dq, dk, dv from the
    forward's out and lse, fp32 SIMT.  Visible-pair work: five dot products or
    updates of length d per (query head, visible key) -- the scores, dP, dV,
    dQ and dK -- 10 * d FLOP per pair."""
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    w = W.workload(2)
    x = W.prefill_inputs(w, W.seed_for(2, 555) + rank * 7, B=w.B)
    q, k, v, ar = x.q.to(dev), x.k.to(dev), x.v.to(dev), x.ar.to(dev)
    dout, _ = W.draw(tuple(x.q.shape), 9201 + rank, w.d, w.dtype, 0.5)
    dout = dout.to(dev)
    lse = torch.empty((w.B, w.Sq, w.Hq), dtype=torch.float32, device=dev)
    out = binding.pi_attn_prefill(q, k, v, ar, lse=lse, stream=stream)
    wsb = torch.empty(binding.pi_attn_prefill_backward_workspace_bytes(q, k, ar),
                      dtype=torch.uint8, device=dev)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(v.shape, dtype=torch.float32, device=dev)

    def step():
        binding.pi_attn_prefill_backward(q, k, v, ar, out, lse, dout, dq=dq, dk=dk, dv=dv,
                                         workspace=wsb, stream=stream)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    reps = 3
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            step()
        e1.record(stream)
    torch.cuda.synchronize()
    us = dist.max_over_ranks(e0.elapsed_time(e1) * 1e3 / reps)
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    pairs = visible_pairs_per_bh(w.ar) * w.B * w.Hq
    flops = 10 * w.d * pairs
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            sm_mhz = float(json.load(f).get("sm_max_mhz", 1965.0))
    except (OSError, ValueError):
        sm_mhz = 1965.0
    fp32_peak = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12       # FFMA lanes x 2 FLOP x clock
    return {
        "workload": "pi0 joint prefill backward: B=8, S=611, Hq=8, d=256, bf16 in, fp32 grads",
        "us_per_call": us,
        "tflops": flops / (us / 1e6) / 1e12,
        "bound": "alu",
        "fp32_fma_peak_tflops": fp32_peak,
        "frac_of_fp32_peak": flops / (us / 1e6) / 1e12 / fp32_peak,
        "algorithmic_flop_per_call": flops,
        "gpu_launches_per_call": 3,
        "timing": f"{reps} calls back to back after one warm-up (warm L2)",
    }


def decode_steps(args, dev, stream, rank):
    """FAST-style single-token decode: B=32 queries of one token (8 heads)
    against a cache of 880 tokens (816 prefix + 64 generated), cold L2.  Each
    step reads the whole cache once: HBM-bound."""
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    B, P, Hq, d = 32, 880, 8, 256
    P_ = peaks()
    kc, _ = W.draw((B, P, 1, d), 9001 + rank, d, "bf16")
    vc, _ = W.draw((B, P, 1, d), 9002 + rank, d, "bf16")
    q, _ = W.draw((B, 1, Hq, d), 9003 + rank, d, "bf16")
    k, _ = W.draw((B, 1, 1, d), 9004 + rank, d, "bf16")
    v, _ = W.draw((B, 1, 1, d), 9005 + rank, d, "bf16")
    kc, vc, q, k, v = (t.to(dev) for t in (kc, vc, q, k, v))
    ar = torch.ones(1, dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    need = binding.pi_attn_suffix_workspace_bytes(q, k, kc, ar)
    wsb = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            binding.pi_attn_suffix(q, k, v, kc, vc, ar, out=out, workspace=wsb, stream=stream)
    torch.cuda.synchronize()
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        binding.pi_attn_suffix(q, k, v, kc, vc, ar, out=out, workspace=wsb, stream=stream)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cold = []
    dist.barrier()
    for _ in range(20):
        with torch.cuda.stream(stream):
            flush.fill_(1.0)
            e0.record(stream)
            g1.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        cold.append(e0.elapsed_time(e1) * 1e3)
    us = dist.max_over_ranks(float(np.median(cold)))
    del flush
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    bytes_step = 2 * B * P * d * 2 + 2 * B * Hq * d * 2 + 2 * B * d * 2
    return {
        "workload": "single-token decode: B=32, Hq=8, d=256, cache 880 (pi_attn_suffix, Sq=1)",
        "us_per_step_cold_l2": us,
        "gb_per_s_algorithmic": bytes_step / (us / 1e6) / 1e9,
        "hbm_frac": bytes_step / (us / 1e6) / 1e9 / P_["hbm_gbs"],
        "algorithmic_bytes_per_step": bytes_step,
        "splits": binding.pi_attn_suffix_workspace_bytes(q, k, kc, ar) > 0,
    }


def suffix_control(args, dev, stream, rank):
    """pi0 Euler loop: 10 suffix passes (fresh suffix q/k/v each) against one cache."""
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    w = W.workload(3)
    P = peaks()
    c = W.cache_inputs(w, W.seed_for(3, 999) + rank * 7, B=w.B)
    kc, vc = c.k.to(dev), c.v.to(dev)
    steps = [W.suffix_inputs(w, W.seed_for(3, s) + rank * 7, B=w.B) for s in range(w.calls)]
    ins = [(x.q.to(dev), x.k.to(dev), x.v.to(dev), x.ar.to(dev)) for x in steps]
    outs = [torch.empty_like(x[0]) for x in ins]
    need = binding.pi_attn_suffix_workspace_bytes(ins[0][0], ins[0][1], kc, ins[0][3])
    wsb = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    def ctrl():
        for s, (q, k, v, ar) in enumerate(ins):
            binding.pi_attn_suffix(q, k, v, kc, vc, ar, out=outs[s], workspace=wsb, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            ctrl()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        ctrl()
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    reps = max(5, min(200, args.steps // 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us_ctrl = dist.max_over_ranks(e0.elapsed_time(e1) * 1e3 / reps)

    # cold-L2 per step: flush (write > L2) before each single-step graph, outside the events
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        q, k, v, ar = ins[0]
        binding.pi_attn_suffix(q, k, v, kc, vc, ar, out=outs[0], workspace=wsb, stream=stream)
    cold = []
    for _ in range(20):
        with torch.cuda.stream(stream):
            flush.fill_(1.0)
            e0.record(stream)
            g1.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        cold.append(e0.elapsed_time(e1) * 1e3)
    us_cold = dist.max_over_ranks(float(np.median(cold)))
    del flush
    assert binding.pi_attn_read_status(stream) == binding.PI_OK

    pairs = visible_pairs_per_bh(w.ar, P=w.P) * w.B * w.Hq
    rows = w.B * w.Sq * w.Hq
    bytes_step = (2 * w.B * w.P * w.d * 2) + (2 * rows * w.d * 2) + (2 * w.B * w.Sq * w.d * 2)
    us_step = us_ctrl / w.calls
    return {
        "workload": "pi0_euler_suffix: B=32, Hq=8, d=256, prefix cache 816, 10 steps x 51 tokens",
        "us_per_ctrl": us_ctrl,
        "us_per_step_warm": us_step,
        "us_per_step_cold_l2": us_cold,
        "pairs_per_s": pairs / (us_step / 1e6),
        "tflops": 4 * w.d * pairs / (us_step / 1e6) / 1e12,
        "gb_per_s_algorithmic_cold": bytes_step / (us_cold / 1e6) / 1e9,
        "hbm_frac_cold": bytes_step / (us_cold / 1e6) / 1e9 / P["hbm_gbs"],
        "algorithmic_bytes_per_step": bytes_step,
        "gpu_launches_per_ctrl": w.calls,
        "timing": f"graph of 10 steps replayed {reps}x (warm); cold: L2 flushed before each step",
    }


# ------------------------------------------------------- per-config table


def oracle_seconds_per_call(w, x, max_rows, seconds=5.0):
    """The oracle's wall time for one whole call of workload ``w``, estimated
    from a bounded sample: ``max_rows`` query rows of batch element 0 (all
    heads), timed for about ``seconds``, scaled by B * S / rows."""
    import oracle

    ar = np.array(w.ar)
    seg = None if w.seg is None else np.array(w.seg)
    S = w.Sq
    n_rows = min(S, max_rows)
    rows = [(0, int(i)) for i in np.linspace(0, S - 1, n_rows).round().astype(int)]
    t0 = time.perf_counter()
    n = 0
    while n < 1 or time.perf_counter() - t0 < seconds:
        oracle.prefill(x.q64[:1], x.k64[:1], x.v64[:1], ar, seg, scale=w.scale, rows=rows)
        n += 1
    dt = (time.perf_counter() - t0) / n
    return dt * w.B * S / n_rows, (f"{n_rows} of {S} query rows (all heads) of 1 of {w.B} "
                                   f"batch elements, {n} repeats, scaled to the whole call")


def prefill_config_line(cfg, dev, stream, sets, reps, oracle_rows):
    """Device time per call of one prefill workload, rotating over ``sets``
    device-resident input sets, plus the oracle's estimated time per call."""
    import torch

    from vla_prefix_lm_b200 import binding
    from vla_prefix_lm_b200 import workloads as W

    w = W.workload(cfg)
    P_ = peaks()
    host = [W.prefill_inputs(w, W.seed_for(cfg, c), B=w.B) for c in range(sets)]
    ins = []
    for x in host:
        seg = None if x.seg is None else x.seg.to(dev)
        ins.append((x.q.to(dev), x.k.to(dev), x.v.to(dev), x.ar.to(dev), seg))
    outs = [torch.empty_like(t[0]) for t in ins]

    def call(i):
        q, k, v, ar, seg = ins[i % sets]
        binding.pi_attn_prefill(q, k, v, ar, segment_ids=seg, out=outs[i % sets],
                                softmax_scale=w.scale, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(max(3, sets)):
            call(i)
    torch.cuda.synchronize()
    n = sets * max(1, 8 // sets)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            call(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * n)
    del g
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    elt = 2 if w.dtype == "bf16" else 4
    pairs = visible_pairs_per_bh(w.ar, w.seg) * w.B * w.Hq
    flops = 4 * w.d * pairs
    nbytes = (2 * w.B * w.Sq * w.Hq * w.d + 2 * w.B * w.Sq * w.Hkv * w.d) * elt
    o_s, sample = oracle_seconds_per_call(w, host[0], oracle_rows)
    line = {
        "config": cfg, "workload": f"{w.name}: {w.note}",
        "shape": {"B": w.B, "S": w.Sq, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "dtype": w.dtype},
        "us_per_call": us, "pairs_per_call": pairs, "pairs_per_s": pairs / (us / 1e6),
        "tflops": flops / (us / 1e6) / 1e12, "gb_per_s_algorithmic": nbytes / (us / 1e6) / 1e9,
        "timing": f"CUDA graph of {n} calls over {sets} input sets, replayed {reps}x",
        "oracle_s_per_call": o_s, "oracle_sample": sample,
        "oracle_cores": len(os.sched_getaffinity(0)),
    }
    if w.dtype == "bf16":
        line["frac_of_bf16_peak"] = line["tflops"] / P_["bf16_tflops"]
        line["frac_of_bf16_sustained"] = line["tflops"] / P_["bf16_tflops_sustained"]
    if w.calls > 1:
        line["us_per_workload"] = us * w.calls
        line["calls"] = w.calls
    return line


def run_configs(args):
    """One JSON line per workload config: device time, rates, roofline
    fractions and the oracle's estimated time per call (one GPU, no ranks)."""
    import torch

    from vla_prefix_lm_b200 import binding

    binding.lib()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream()
    plan = {1: (1, 200, 49), 2: (6, 50, 611), 4: (2, 20, 256), 5: (2, 5, 64)}
    for cfg in (1, 2, 4, 5):
        sets, reps, rows = plan[cfg]
        print(json.dumps({"impl": "ours", "mode": "configs",
                          **prefill_config_line(cfg, dev, stream, sets, reps, rows)}),
              flush=True)
    suffix = suffix_control(args, dev, stream, 0)
    print(json.dumps({"impl": "ours", "mode": "configs", "config": 3, **suffix}), flush=True)


# ------------------------------------------------------------ CPU baselines


def cpu_baseline(w, seconds=10.0):
    """The oracle (numpy float64, as it stands) on a bounded sample of the workload."""
    import oracle
    from vla_prefix_lm_b200 import workloads as W

    x = W.prefill_inputs(w, W.seed_for(2), B=1)
    ar = np.array(w.ar)
    pairs = visible_pairs_per_bh(w.ar) * w.Hq
    t0 = time.perf_counter()
    n = 0
    while n < 3 or time.perf_counter() - t0 < seconds:
        oracle.prefill(x.q64, x.k64, x.v64, ar)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": pairs * n / dt, "unit": "pairs/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{n} oracle.prefill calls on 1 of the 8 batch elements (all 8 heads, "
                      f"S=611), {dt:.1f} s wall; numpy/BLAS threads = cores"}


def run_reference(args, rank, ws):
    import oracle
    from vla_prefix_lm_b200 import workloads as W

    if rank != 0:
        return None
    w = W.workload(2)
    x = W.prefill_inputs(w, W.seed_for(2), B=1)
    ar = np.array(w.ar)
    pairs = visible_pairs_per_bh(w.ar) * w.Hq
    for _ in range(args.warmup):
        oracle.prefill(x.q64, x.k64, x.v64, ar)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.prefill(x.q64, x.k64, x.v64, ar)
    dt = time.perf_counter() - t0
    value = pairs * args.steps / dt
    cores = len(os.sched_getaffinity(0))
    sample = "each step: oracle.prefill on 1 of the 8 batch elements of pi0_joint_prefill"
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "pairs/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1)*d^-0.25 q/k/v rounded to bf16, upcast)",
        "config": {"workload": "pi0_joint_prefill: Hq=8, Hkv=1, d=256, S=611; "
                               "sample of 1 batch element per step",
                   "seq_len": w.Sq, "parallelism": "rank 0 only (CPU)"},
        "cpu_baseline": {"value": value, "unit": "pairs/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "pairs/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--configs", action="store_true",
                    help="instead of the bench line: one line per workload config (1 GPU)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")

    from vla_prefix_lm_b200 import dist
    rank, ws, local = dist.world()
    if args.configs:
        dist.init()
        try:
            run_configs(args)
        finally:
            dist.shutdown()
        return
    if args.impl == "reference":
        line = run_reference(args, rank, ws)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    dist.init()
    try:
        line = run_ours(args, rank, ws, local)
    finally:
        dist.shutdown()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
