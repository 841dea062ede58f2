"""Benchmark of the joint (prefix-LM) attention on B200: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --case NAME [--launches N]     (a few launches, for ncu)

The headline workload is the largest configuration: MM-DiT-shaped full
bidirectional attention, B=4 per rank, Hq=8, Hkv=1, d=256, S=4096 patches +
154 text tokens (ar_mask all False), 28 calls with fresh inputs.  One step is
those 28 calls (pi_attn_prefill), each on its own device-resident input set,
so every call reads its inputs from HBM.  `value` is unmasked attention pairs
per second, counted per (batch, query head, query token, visible key), for the
whole job; FLOPs are 4 * d per pair.  The timed loop replays one CUDA graph of
the 28 ABI calls per step, timed with CUDA events on the launching stream.

The same line carries, as sub-objects, the other configurations (the tiny fp32
prefill, the pi0 prefill B=8 S=611, the pi0.5 three-segment prefill B=16
S=938, and the pi0 Euler suffix control B=32 with an 816-token cache), the
single-token decode, RoPE / Euler, the backward, and the roofline, e2e (host
buffers through the C ABI), clocks and CPU-oracle baseline objects.

N > 1 (one process per GPU): every rank runs its own batch of the same
per-rank size (weak scaling, no data-path collective); the timed region is
bracketed by barriers and the max over ranks is reported.  `--gpus N` started
without a launcher re-runs this script under torch.distributed.run.

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

# DRAM traffic of the prefill kernel per launch on the headline workload, from
# one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum); valid only for
# the kernel sources whose digest is recorded beside it.
TRAFFIC = {"bytes": 125614848, "src_sha": "d4a1a6103d0956fc", "workload": "mmdit"}
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


def _prefill_ws(q, k, ar):
    """Scratch that lets the prefill split its last round of query tiles over
    idle SM pairs (None if this geometry takes none)."""
    import torch

    from vla_prefix_lm_b200 import binding

    n = binding.pi_attn_prefill_workspace_bytes(q, k, ar)
    return torch.empty(n, dtype=torch.uint8, device=q.device) if n else None


def _mmdit_sets(w, dev, n, seed0):
    """``n`` fresh MM-DiT input sets (q, k, v, ar) drawn on the device."""
    import torch

    from vla_prefix_lm_b200 import workloads as W

    ar = torch.tensor(w.ar, dtype=torch.uint8, device=dev)
    sets = []
    for i in range(n):
        s = seed0 + 4 * i
        q = W.device_draw((w.B, w.Sq, w.Hq, w.d), s, w.d, w.dtype, dev)
        k = W.device_draw((w.B, w.Sq, w.Hkv, w.d), s + 1, w.d, w.dtype, dev)
        v = W.device_draw((w.B, w.Sq, w.Hkv, w.d), s + 2, w.d, w.dtype, dev)
        sets.append((q, k, v, ar))
    return sets


def timed_steps(step, steps, stream, rank):
    """Runs ``steps`` calls of ``step()`` between a barrier and a synchronize
    on both sides; returns (device ms on this rank from CUDA events on
    ``stream``, max over ranks, wall-clock bounds, clock record)."""
    import torch

    from vla_prefix_lm_b200 import dist

    sampler = ClockSampler(gpu_id(stream.device)) if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    dist.barrier()
    ms = e0.elapsed_time(e1)
    clocks = sampler.stop(t0, t1) if sampler else None
    return ms, dist.max_over_ranks(ms), clocks


def run_ours(args, rank, ws, local):
    """The bench line: the MM-DiT workload (the largest config) as the headline,
    the other configs, the suffix control, decode, RoPE/Euler and backward as
    sub-objects."""
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    binding.lib()  # fails loudly without the CUDA library
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    P = peaks()

    # --- headline: MM-DiT, B=4 per rank, S=4250, all False; one step = the
    # workload's 28 calls, each on its own fresh input set
    w = W.workload(5)
    calls = w.calls
    pairs_call = visible_pairs_per_bh(w.ar) * w.B * w.Hq
    flops_call = 4.0 * w.d * pairs_call
    bytes_call = 2 * (2 * w.B * w.Sq * w.Hq * w.d + 2 * w.B * w.Sq * w.Hkv * w.d) + w.Sq
    sets = _mmdit_sets(w, dev, calls, 5_000_000 + 1000 * rank)
    outs = [torch.empty_like(s_[0]) for s_ in sets]
    set_bytes = sum(t.nbytes for t in sets[0][:3]) + outs[0].nbytes

    pws = _prefill_ws(sets[0][0], sets[0][1], sets[0][3])
    # kernels per call: the attention kernel, plus the tail merge when the last
    # round of query tiles is split
    kernels_per_call = 1 if pws is None or binding.pi_attn_prefill_tail_splits(
        sets[0][0], sets[0][1], sets[0][3]) == 1 else 2

    def workload_calls():
        for i, (q, k, v, ar) in enumerate(sets):
            binding.pi_attn_prefill(q, k, v, ar, out=outs[i], stream=stream, workspace=pws)

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 1)):
            workload_calls()
    torch.cuda.synchronize()
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        workload_calls()
    # CUDAGraph.replay() launches on torch's current stream: timed_steps makes
    # it `stream`, the stream the events are recorded on.
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    ms, ms_max, clocks = timed_steps(g.replay, args.steps, stream, rank)
    status = binding.pi_attn_read_status(stream)
    if status != binding.PI_OK:
        raise RuntimeError(f"device status after timing: {binding.status_string(status)}")
    del g
    ms_step = ms_max / args.steps
    value = ws * pairs_call * calls * args.steps / (ms_max / 1e3)
    us_launch = ms / (args.steps * calls) * 1e3
    achieved_tflops = flops_call / (us_launch / 1e6) / 1e12

    e2e = e2e_mmdit(args, w, dev, stream, rank, ws, sets[:2])
    del sets, outs
    torch.cuda.empty_cache()

    configs = {
        "tiny_f32": prefill_config(1, dev, stream, rank, n_sets=1, reps=200),
        "pi0_prefill": prefill_config(2, dev, stream, rank, n_sets=6, reps=50),
        "pi05_prefill": prefill_config(4, dev, stream, rank, n_sets=3, reps=20),
        "pi0_euler_suffix": suffix_control(args, dev, stream, rank),
    }
    decode = decode_steps(args, dev, stream, rank)
    prepost = prepost_steps(args, dev, stream, rank)
    bwd = backward_steps(args, dev, stream, rank)

    traffic = None
    if TRAFFIC.get("src_sha") == kernel_digest() and TRAFFIC.get("workload") == "mmdit":
        traffic = TRAFFIC["bytes"]
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
        "data": "synthetic (seeded N(0,1)*d^-0.25 q/k/v, bf16)",
        "config": {
            "workload": "mmdit_full_bidirectional: B=4 per rank, Hq=8, Hkv=1, d=256, "
                        "S=4250 (4096 patches + 154 text, ar_mask all False); one step = "
                        "the workload's 28 calls, each on a fresh input set",
            "per_rank_batch": w.B,
            "global_batch": w.B * ws,
            "seq_len": w.Sq,
            "calls_per_step": calls,
            "parallelism": f"batch replicas x{ws} (no data-path collective)",
            "l2": f"inputs larger than L2: each step reads {calls} distinct input sets "
                  f"({calls * set_bytes / 2**30:.1f} GiB with outputs), so every call's "
                  "inputs come from HBM",
            "timing": "CUDA events on the launching stream around one CUDA-graph replay "
                      f"(the {calls} calls) per step; barrier + synchronize on both sides; "
                      "max over ranks",
        },
        "us_per_call": ms_step / calls * 1e3,
        "tflops": ws * flops_call * calls * args.steps / (ms_max / 1e3) / 1e12,
        "gb_per_s_algorithmic": bytes_call / (us_launch / 1e6) / 1e9,
        "roofline": {
            "bound": "tensor",
            "kernel": "tc_pair_kernel<prefill> (+ tail_combine_kernel: each call's time, "
                      "both kernels, is charged to it)",
            "achieved": achieved_tflops,
            "peak": P["bf16_tflops"],
            "unit": "TFLOP/s",
            "frac": achieved_tflops / P["bf16_tflops"],
            "peak_source": f"{P['source']} bf16 dense (burst)",
            "frac_of_sustained": (achieved_tflops / P["bf16_tflops_sustained"]
                                  if P["bf16_tflops_sustained"] else None),
            "traffic": traffic,
            "algorithmic_flop_per_launch": flops_call,
            "launch_us": us_launch,
        },
        "e2e": e2e,
        "gpu_launches": calls * args.steps * kernels_per_call,
        "clocks": clocks,
        "configs": configs,
        "decode": decode,
        "prepost": prepost,
        "backward": bwd,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, seconds=args.cpu_seconds)
    return line


def e2e_mmdit(args, w, dev, stream, rank, ws, dev_sets):
    """The headline metric end to end through the public API: every call's
    q/k/v/ar go from pinned host memory to the device, pi_attn_prefill runs,
    and out comes back to pinned host memory, all inside the timed region.
    Three streams (host-to-device, compute, device-to-host) and two buffer
    slots let the copies of neighbouring calls overlap with each other and
    with the kernel.  Also reports the copy-only floor: the same transfers with
    no kernel, both directions overlapped."""
    import torch

    from vla_prefix_lm_b200 import binding, dist

    calls = w.calls
    n_steps = max(1, min(args.steps, 2))
    host = []
    for q, k, v, ar in dev_sets:
        host.append(tuple(t.cpu().pin_memory() for t in (q, k, v, ar)))
    hout = [torch.empty(dev_sets[0][0].shape, dtype=torch.bfloat16, pin_memory=True)
            for _ in range(2)]
    din = [tuple(torch.empty_like(t) for t in dev_sets[0]) for _ in range(2)]
    pws = _prefill_ws(dev_sets[0][0], dev_sets[0][1], dev_sets[0][3])
    dout = [torch.empty_like(dev_sets[0][0]) for _ in range(2)]
    h2d_bytes = sum(t.nbytes for t in host[0])
    d2h_bytes = hout[0].nbytes
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n_calls, compute=True):
        for i in range(n_calls):
            j = i % 2
            if i >= 2:
                s_in.wait_event(ev_done[j])            # input slot j free again
            with torch.cuda.stream(s_in):
                for dst, src in zip(din[j], host[i % len(host)]):
                    dst.copy_(src, non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])           # output slot j copied out
            if compute:
                q, k, v, ar = din[j]
                binding.pi_attn_prefill(q, k, v, ar, out=dout[j], stream=stream, workspace=pws)
            ev_done[j].record(stream)
            s_out.wait_event(ev_done[j])
            with torch.cuda.stream(s_out):
                hout[j].copy_(dout[j], non_blocking=True)
                ev_out[j].record(s_out)
        stream.wait_stream(s_out)
        stream.wait_stream(s_in)

    run(4)
    torch.cuda.synchronize()
    res = {}
    for key, compute in (("value", True), ("copy_only", False)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        s_in.wait_stream(stream)
        run(n_steps * calls, compute)
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        res[key] = dist.max_over_ranks(e0.elapsed_time(e1))
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    pairs = ws * visible_pairs_per_bh(w.ar) * w.B * w.Hq * calls * n_steps
    return {
        "value": pairs / (res["value"] / 1e3),
        "unit": "pairs/s",
        "h2d_bytes_per_step": h2d_bytes * calls,
        "d2h_bytes_per_step": d2h_bytes * calls,
        "steps": n_steps,
        "ms_per_step": res["value"] / n_steps,
        "copy_floor_ms_per_step": res["copy_only"] / n_steps,
        "copy_floor_pairs_per_s": pairs / (res["copy_only"] / 1e3),
        "what": "per call: pinned host q/k/v/ar -> device, pi_attn_prefill, out -> pinned "
                "host; copies and kernel overlapped over three streams and two buffer "
                "slots; copy_floor = the same copies with no kernel",
    }


def prefill_config(cfg, dev, stream, rank, n_sets, reps):
    """Device time per call of one prefill workload: a CUDA graph of calls over
    ``n_sets`` device-resident input sets (together larger than L2 where the
    workload is large enough), replayed ``reps`` times."""
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    w = W.workload(cfg)
    P_ = peaks()
    ar = torch.tensor(w.ar, dtype=torch.uint8, device=dev)
    seg = None if w.seg is None else torch.tensor(w.seg, dtype=torch.int32, device=dev)
    ins = []
    for i in range(n_sets):
        s = 6_000_000 + 10_000 * cfg + 1000 * rank + 4 * i
        ins.append(tuple(W.device_draw((w.B, w.Sq, h, w.d), s + j, w.d, w.dtype, dev)
                         for j, h in enumerate((w.Hq, w.Hkv, w.Hkv))))
    outs = [torch.empty_like(t[0]) for t in ins]
    pws = _prefill_ws(ins[0][0], ins[0][1], ar)

    def call(i):
        q, k, v = ins[i % n_sets]
        binding.pi_attn_prefill(q, k, v, ar, segment_ids=seg, out=outs[i % n_sets],
                                softmax_scale=w.scale, stream=stream, workspace=pws)

    with torch.cuda.stream(stream):
        for i in range(max(3, n_sets)):
            call(i)
    torch.cuda.synchronize()
    n = n_sets * max(1, 8 // n_sets)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            call(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    with torch.cuda.stream(stream):
        g.replay()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = dist.max_over_ranks(e0.elapsed_time(e1) * 1e3 / (reps * n))
    del g
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    elt = 2 if w.dtype == "bf16" else 4
    pairs = visible_pairs_per_bh(w.ar, w.seg) * w.B * w.Hq
    flops = 4 * w.d * pairs
    nbytes = (2 * w.B * w.Sq * w.Hq * w.d + 2 * w.B * w.Sq * w.Hkv * w.d) * elt
    set_bytes = (2 * w.B * w.Sq * w.Hq * w.d + 2 * w.B * w.Sq * w.Hkv * w.d) * elt
    line = {
        "workload": f"{w.name}: B={w.B}, Hq={w.Hq}, Hkv={w.Hkv}, d={w.d}, {w.dtype}; {w.note}",
        "us_per_call": us, "pairs_per_call": pairs, "pairs_per_s": pairs / (us / 1e6),
        "tflops": flops / (us / 1e6) / 1e12, "gb_per_s_algorithmic": nbytes / (us / 1e6) / 1e9,
        "timing": f"CUDA graph of {n} calls over {n_sets} input sets "
                  f"({n_sets * set_bytes / 2**20:.0f} MiB with outputs), replayed {reps}x",
    }
    if w.dtype == "bf16":
        line["bound"] = "tensor"
        line["frac_of_bf16_peak"] = line["tflops"] / P_["bf16_tflops"]
        line["frac_of_bf16_sustained"] = line["tflops"] / P_["bf16_tflops_sustained"]
    else:
        line["bound"] = "launch latency (fp32 SIMT path; parity case, throughput not a target)"
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


def _rotating_us(calls, stream, reps=10):
    """Device time per call of ``calls`` (one per input set, the sets together
    larger than twice the L2), captured as one CUDA graph and replayed ``reps``
    times after one untimed replay: every call reads its inputs from HBM, and
    the L2 holds only the earlier calls' own data."""
    import torch

    with torch.cuda.stream(stream):
        for c in calls:
            c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / (reps * len(calls))


def _n_sets(set_bytes):
    return max(3, int(np.ceil(2 * L2_BYTES / set_bytes)) + 1)


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
    set_bytes = B * S * (Hq + 1) * d * 2
    n = _n_sets(set_bytes)
    qk = [(W.device_draw((B, S, Hq, d), 9100 + 10 * i + rank, d, "bf16", dev),
           W.device_draw((B, S, 1, d), 9101 + 10 * i + rank, d, "bf16", dev)) for i in range(n)]
    tm = torch.ones((B, S), dtype=torch.uint8, device=dev)
    us = dist.max_over_ranks(_rotating_us(
        [lambda q=q, k=k: binding.pi_rope_inplace(q, k, tm, stream=stream) for q, k in qk],
        stream))
    nb = 2 * set_bytes + tm.numel()
    res["rope_prefill"] = {"shape": "q [8,611,8,256], k [8,611,1,256] bf16", "us_cold": us,
                           "algorithmic_bytes": nb, "gb_per_s": nb / us / 1e3,
                           "hbm_frac": nb / us / 1e3 / hbm,
                           "timing": f"graph over {n} input sets ({n * set_bytes / 2**20:.0f} "
                                     "MiB > 2 x L2): every call reads HBM"}
    del qk, tm

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

    set_bytes = w.B * w.Sq * (w.Hq + 1) * w.d * 2
    n = _n_sets(set_bytes)
    qk = [(W.device_draw((w.B, w.Sq, w.Hq, w.d), 9200 + 10 * i + rank, w.d, "bf16", dev),
           W.device_draw((w.B, w.Sq, 1, w.d), 9201 + 10 * i + rank, w.d, "bf16", dev))
          for i in range(n)]
    us = dist.max_over_ranks(_rotating_us(
        [lambda q=q, k=k: binding.pi_rope_inplace(q, k, sm_, prefix_mask=pm, stream=stream)
         for q, k in qk], stream))
    nb = 2 * set_bytes + sm_.numel() + pm.numel()
    res["rope_suffix"] = {"shape": "q [32,51,8,256], k [32,51,1,256] bf16, prefix mask [32,816]",
                          "us_cold": us, "algorithmic_bytes": nb, "gb_per_s": nb / us / 1e3,
                          "hbm_frac": nb / us / 1e3 / hbm,
                          "timing": f"graph over {n} input sets ({n * set_bytes / 2**20:.0f} "
                                    "MiB > 2 x L2): every call reads HBM"}
    del qk
    us = dist.max_over_ranks(_cold_graph_us(
        lambda: binding.pi_euler_update(x, vel[0], -0.1, stream=stream), stream))
    nb = 3 * x.numel() * 4
    res["euler"] = {"shape": "x, v [32,50,32] fp32", "us_cold_l2": us, "algorithmic_bytes": nb,
                    "gb_per_s": nb / us / 1e3,
                    "timing": "median of 20 single-call graph replays, L2 flushed before each "
                              "(launch-bound: 0.6 MB)"}

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
    forward's out and lse, on tensor cores (a row-dot pass, the score pass,
    the dK/dV pass and its chunk sum, the dQ pass).  Algorithmic work: the
    five contractions of length d per (query head, visible key) -- the
    scores, dP, dV, dK and dQ -- 10 * d FLOP per pair."""
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    w = W.workload(2)
    P_ = peaks()
    q, k, v = (W.device_draw((w.B, w.Sq, h, w.d), 8_000_000 + 10 * rank + j, w.d, w.dtype, dev)
               for j, h in enumerate((w.Hq, w.Hkv, w.Hkv)))
    dout = W.device_draw(tuple(q.shape), 8_000_003 + 10 * rank, w.d, w.dtype, dev, 0.5)
    ar = torch.tensor(w.ar, dtype=torch.uint8, device=dev)
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
        for _ in range(3):
            step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    reps = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    with torch.cuda.stream(stream):
        g.replay()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = dist.max_over_ranks(e0.elapsed_time(e1) * 1e3 / reps)
    del g
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    pairs = visible_pairs_per_bh(w.ar) * w.B * w.Hq
    flops = 10 * w.d * pairs
    tf = flops / (us / 1e6) / 1e12
    return {
        "workload": "pi0 joint prefill backward: B=8, S=611, Hq=8, d=256, bf16 in, fp32 grads",
        "us_per_call": us,
        "tflops": tf,
        "bound": "tensor",
        "frac_of_bf16_peak": tf / P_["bf16_tflops"],
        "peak_source": f"{P_['source']} bf16 dense (burst)",
        "algorithmic_flop_per_call": flops,
        "workspace_bytes": int(wsb.numel()),
        "timing": f"CUDA graph of one call replayed {reps}x (warm L2)",
    }


def decode_steps(args, dev, stream, rank):
    """FAST-style single-token decode: B=32 queries of one token (8 heads)
    against a cache of 880 tokens (816 prefix + 64 generated).  Each step reads
    the whole cache once: HBM-bound.  Timed over rotating caches larger than
    twice the L2, so every step reads HBM."""
    import torch

    from vla_prefix_lm_b200 import binding, dist
    from vla_prefix_lm_b200 import workloads as W

    B, P, Hq, d = 32, 880, 8, 256
    P_ = peaks()
    set_bytes = 2 * B * P * d * 2
    n = _n_sets(set_bytes)
    sets = []
    for i in range(n):
        s0 = 9000 + 10 * i + 1000 * rank
        sets.append((W.device_draw((B, 1, Hq, d), s0, d, "bf16", dev),
                     W.device_draw((B, 1, 1, d), s0 + 1, d, "bf16", dev),
                     W.device_draw((B, 1, 1, d), s0 + 2, d, "bf16", dev),
                     W.device_draw((B, P, 1, d), s0 + 3, d, "bf16", dev),
                     W.device_draw((B, P, 1, d), s0 + 4, d, "bf16", dev)))
    ar = torch.ones(1, dtype=torch.uint8, device=dev)
    outs = [torch.empty_like(x[0]) for x in sets]
    need = binding.pi_attn_suffix_workspace_bytes(sets[0][0], sets[0][1], sets[0][3], ar)
    wsb = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    dist.barrier()
    us = dist.max_over_ranks(_rotating_us(
        [lambda x=x, o=o: binding.pi_attn_suffix(x[0], x[1], x[2], x[3], x[4], ar, out=o,
                                                 workspace=wsb, stream=stream)
         for x, o in zip(sets, outs)], stream, reps=20))
    assert binding.pi_attn_read_status(stream) == binding.PI_OK
    bytes_step = 2 * B * P * d * 2 + 2 * B * Hq * d * 2 + 2 * B * d * 2
    return {
        "workload": "single-token decode: B=32, Hq=8, d=256, cache 880 (pi_attn_suffix, Sq=1)",
        "us_per_step_cold": us,
        "gb_per_s_algorithmic": bytes_step / (us / 1e6) / 1e9,
        "hbm_frac": bytes_step / (us / 1e6) / 1e9 / P_["hbm_gbs"],
        "algorithmic_bytes_per_step": bytes_step,
        "kernel": "decode_kernel: a cluster of 8 CTAs per batch element, mma.sync, on-chip merge",
        "timing": f"graph over {n} caches ({n * set_bytes / 2**20:.0f} MiB > 2 x L2), "
                  "replayed 20x: every step reads HBM",
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

    # cold: one step per input set (its own cache, suffix q/k/v and output), the
    # sets together larger than twice the L2, so every step reads HBM
    set_bytes = 2 * w.B * w.P * w.d * 2 + 2 * w.B * w.Sq * w.Hq * w.d * 2 + 2 * w.B * w.Sq * w.d * 2
    n = _n_sets(set_bytes)
    cold_sets = []
    for i in range(n):
        s0 = 9500 + 10 * i + 1000 * rank
        cold_sets.append((W.device_draw((w.B, w.Sq, w.Hq, w.d), s0, w.d, "bf16", dev),
                          W.device_draw((w.B, w.Sq, 1, w.d), s0 + 1, w.d, "bf16", dev),
                          W.device_draw((w.B, w.Sq, 1, w.d), s0 + 2, w.d, "bf16", dev),
                          W.device_draw((w.B, w.P, 1, w.d), s0 + 3, w.d, "bf16", dev),
                          W.device_draw((w.B, w.P, 1, w.d), s0 + 4, w.d, "bf16", dev)))
    cold_outs = [torch.empty_like(x[0]) for x in cold_sets]
    ar0 = ins[0][3]
    us_cold = dist.max_over_ranks(_rotating_us(
        [lambda x=x, o=o: binding.pi_attn_suffix(x[0], x[1], x[2], x[3], x[4], ar0, out=o,
                                                 workspace=wsb, stream=stream)
         for x, o in zip(cold_sets, cold_outs)], stream, reps=20))
    del cold_sets, cold_outs
    assert binding.pi_attn_read_status(stream) == binding.PI_OK

    pairs = visible_pairs_per_bh(w.ar, P=w.P) * w.B * w.Hq
    rows = w.B * w.Sq * w.Hq
    bytes_step = (2 * w.B * w.P * w.d * 2) + (2 * rows * w.d * 2) + (2 * w.B * w.Sq * w.d * 2)
    us_step = us_ctrl / w.calls
    return {
        "workload": "pi0_euler_suffix: B=32, Hq=8, d=256, prefix cache 816, 10 steps x 51 tokens",
        "us_per_ctrl": us_ctrl,
        "us_per_step_warm": us_step,
        "us_per_step_cold": us_cold,
        "pairs_per_s": pairs / (us_step / 1e6),
        "tflops": 4 * w.d * pairs / (us_step / 1e6) / 1e12,
        "gb_per_s_algorithmic_cold": bytes_step / (us_cold / 1e6) / 1e9,
        "hbm_frac_cold": bytes_step / (us_cold / 1e6) / 1e9 / P["hbm_gbs"],
        "algorithmic_bytes_per_step": bytes_step,
        "gpu_launches_per_ctrl": w.calls,
        "timing": f"warm: graph of 10 steps against one cache replayed {reps}x; cold: graph "
                  f"over {n} input sets ({n * set_bytes / 2**20:.0f} MiB > 2 x L2, each with "
                  "its own cache) replayed 20x, every step reading HBM",
    }


# ------------------------------------------------------------ CPU baselines


def _oracle_rows_sample(w, n_tok, i0):
    """The oracle on ``n_tok`` query tokens (all heads) of batch element 0 of
    the MM-DiT workload, starting at token ``i0``: its own mask builder and
    attention, as they stand.  Returns the visible pairs it computed."""
    import oracle
    from vla_prefix_lm_b200 import workloads as W

    x = _ORACLE_INPUTS.get(w.name)
    if x is None:
        x = _ORACLE_INPUTS[w.name] = W.prefill_inputs(w, W.seed_for(5, 0), B=1)
    ar = np.array(w.ar)
    rows = np.arange(i0, min(i0 + n_tok, w.Sq))
    M = oracle.prefill_mask(ar, rows=rows)
    oracle.attention(x.q64[:, rows], x.k64, x.v64, M, scale=w.scale)
    return int(M.sum()) * w.Hq


_ORACLE_INPUTS = {}


def cpu_baseline(w, seconds=10.0, n_tok=512):
    """The oracle (numpy float64, as it stands) on a bounded sample of the
    headline workload: blocks of ``n_tok`` query tokens of one batch element."""
    _oracle_rows_sample(w, 8, 0)                       # inputs drawn outside the clock
    t0 = time.perf_counter()
    n, pairs = 0, 0
    while n < 2 or time.perf_counter() - t0 < seconds:
        pairs += _oracle_rows_sample(w, n_tok, (n * n_tok) % w.Sq)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": pairs / dt, "unit": "pairs/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{n} blocks of {n_tok} query tokens x 8 heads x 4250 keys of batch "
                      f"element 0 of the MM-DiT workload (oracle.prefill_mask + "
                      f"oracle.attention), {dt:.1f} s wall; numpy/BLAS threads = cores"}


def run_reference(args, rank, ws):
    """The oracle arm: each step is a bounded sample of the headline workload
    (512 query tokens x 8 heads of one batch element against all 4250 keys)."""
    from vla_prefix_lm_b200 import workloads as W

    if rank != 0:
        return None
    w = W.workload(5)
    n_tok = 512
    _oracle_rows_sample(w, 8, 0)
    for i in range(args.warmup):
        _oracle_rows_sample(w, n_tok, (i * n_tok) % w.Sq)
    t0 = time.perf_counter()
    pairs = 0
    for i in range(args.steps):
        pairs += _oracle_rows_sample(w, n_tok, (i * n_tok) % w.Sq)
    dt = time.perf_counter() - t0
    value = pairs / dt
    cores = len(os.sched_getaffinity(0))
    sample = (f"each step: oracle.prefill_mask + oracle.attention on {n_tok} query tokens "
              "(all 8 heads, all 4250 keys) of batch element 0 of the MM-DiT workload")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "pairs/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / max(args.steps, 1) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1)*d^-0.25 q/k/v rounded to bf16, upcast)",
        "config": {"workload": "mmdit_full_bidirectional: Hq=8, Hkv=1, d=256, S=4250, "
                               f"ar_mask all False; sample of {n_tok} query tokens per step",
                   "seq_len": w.Sq, "parallelism": "rank 0 only (CPU)"},
        "cpu_baseline": {"value": value, "unit": "pairs/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "pairs/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------- profiling


CASES = ("mmdit_prefill", "pi0_prefill", "pi05_prefill", "pi0_suffix_step", "decode_step",
         "pi0_backward", "rope_prefill")


def run_case(args):
    """A few launches of one workload on one input set, for ncu captures:
    little device memory (one set, no rotation) and no timing."""
    import torch

    from vla_prefix_lm_b200 import binding
    from vla_prefix_lm_b200 import workloads as W

    binding.lib()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    name = args.case
    if name == "rope_prefill":
        q = W.device_draw((8, 611, 8, 256), 7_300_000, 256, "bf16", dev)
        k = W.device_draw((8, 611, 1, 256), 7_300_001, 256, "bf16", dev)
        tm = torch.ones((8, 611), dtype=torch.uint8, device=dev)

        def call():
            binding.pi_rope_inplace(q, k, tm, stream=stream)
    elif name == "pi0_backward":
        w = W.workload(2)
        q, k, v = (W.device_draw((w.B, w.Sq, h, w.d), 7_200_000 + j, w.d, w.dtype, dev)
                   for j, h in enumerate((w.Hq, w.Hkv, w.Hkv)))
        dout = W.device_draw(tuple(q.shape), 7_200_003, w.d, w.dtype, dev, 0.5)
        ar = torch.tensor(w.ar, dtype=torch.uint8, device=dev)
        lse = torch.empty((w.B, w.Sq, w.Hq), dtype=torch.float32, device=dev)
        out = binding.pi_attn_prefill(q, k, v, ar, lse=lse, stream=stream)
        wsb = torch.empty(binding.pi_attn_prefill_backward_workspace_bytes(q, k, ar),
                          dtype=torch.uint8, device=dev)
        grads = [torch.empty(t.shape, dtype=torch.float32, device=dev) for t in (q, k, v)]

        def call():
            binding.pi_attn_prefill_backward(q, k, v, ar, out, lse, dout, dq=grads[0],
                                             dk=grads[1], dv=grads[2], workspace=wsb,
                                             stream=stream)
    elif name.endswith("_prefill"):
        w = W.workload({"mmdit_prefill": 5, "pi0_prefill": 2, "pi05_prefill": 4}[name])
        B = args.case_batch or w.B
        q, k, v = (W.device_draw((B, w.Sq, h, w.d), 7_000_000 + j, w.d, w.dtype, dev)
                   for j, h in enumerate((w.Hq, w.Hkv, w.Hkv)))
        ar = torch.tensor(w.ar, dtype=torch.uint8, device=dev)
        seg = None if w.seg is None else torch.tensor(w.seg, dtype=torch.int32, device=dev)
        out = torch.empty_like(q)
        pws = _prefill_ws(q, k, ar)

        def call():
            binding.pi_attn_prefill(q, k, v, ar, segment_ids=seg, out=out, stream=stream,
                                    workspace=pws)
    else:
        if name == "pi0_suffix_step":
            w = W.workload(3)
            B, P, Sq, ar_np = w.B, w.P, w.Sq, np.array(w.ar, np.uint8)
        else:
            B, P, Sq, ar_np = 32, 880, 1, np.ones(1, np.uint8)
        d = 256
        kc, vc = (W.device_draw((B, P, 1, d), 7_100_000 + j, d, "bf16", dev) for j in (0, 1))
        q = W.device_draw((B, Sq, 8, d), 7_100_002, d, "bf16", dev)
        k, v = (W.device_draw((B, Sq, 1, d), 7_100_003 + j, d, "bf16", dev) for j in (0, 1))
        ar = torch.from_numpy(ar_np).to(dev)
        out = torch.empty_like(q)
        need = binding.pi_attn_suffix_workspace_bytes(q, k, kc, ar)
        wsb = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

        def call():
            binding.pi_attn_suffix(q, k, v, kc, vc, ar, out=out, workspace=wsb, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(args.launches):
            call()
    torch.cuda.synchronize()
    st = binding.pi_attn_read_status(stream)
    print(json.dumps({"case": name, "launches": args.launches,
                      "status": binding.status_string(st)}), flush=True)
    if st != binding.PI_OK:
        raise SystemExit(1)


# ------------------------------------------------------------ rank plumbing


def run_plumbing_check(args, rank, ws):
    """The bench's multi-rank plumbing on CPU (gloo): the same barrier / max
    over ranks / whole-job value arithmetic as the GPU arm, around a fixed
    host workload; rank 0 prints the line.  Used by the host tests."""
    from vla_prefix_lm_b200 import dist

    units_per_step = 1000
    a = np.random.default_rng(rank).standard_normal((256, 256))
    for _ in range(args.warmup):
        a = np.tanh(a @ a.T / 256)
    dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        a = np.tanh(a @ a.T / 256)
    ms = (time.perf_counter() - t0) * 1e3 + 5.0 * rank   # ranks differ: the max must win
    dist.barrier()
    ms_max = dist.max_over_ranks(ms)
    return {"metric": "plumbing check", "value": ws * units_per_step * args.steps / (ms_max / 1e3),
            "unit": "units/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "rank_ms": ms, "max_rank_ms": ms_max}


def relaunch_under_torchrun(n):
    """``--gpus N`` without a launcher: start N ranks of this script with
    torch.distributed.run (one process per GPU, rendezvous on 127.0.0.1)."""
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--case", choices=CASES,
                    help="run --launches calls of one workload on one input set (for ncu)")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--case-batch", type=int, default=0,
                    help="with a prefill --case: this batch size instead of the workload's "
                         "(a smaller case of the same kernel for multi-pass captures)")
    ap.add_argument("--plumbing-check", action="store_true",
                    help="CPU-only multi-rank check of the timing plumbing (gloo)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours" and not args.case:
        ap.error("--warmup must be >= 3")

    from vla_prefix_lm_b200 import dist
    rank, ws, local = dist.world()
    if args.case:
        run_case(args)
        return
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if ws == 1 and args.gpus > 1 and "LOCAL_RANK" not in os.environ:
        raise SystemExit(relaunch_under_torchrun(args.gpus))
    if ws != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started WORLD_SIZE={ws} ranks")
    if args.impl == "reference":
        line = run_reference(args, rank, ws)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    dist.init(backend="gloo" if args.plumbing_check else None)
    try:
        line = (run_plumbing_check(args, rank, ws) if args.plumbing_check
                else run_ours(args, rank, ws, local))
    finally:
        dist.shutdown()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
