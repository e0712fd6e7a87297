#!/usr/bin/env python
"""Benchmark: KDA prefill tokens/s and decode tokens/s on one B200 (replicas for N > 1).

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill leg: kda_chunk_fwd over B=2 sequences x T=2048 tokens, H=32 heads,
    dk = dv = 128, chunk 64, bf16 q/k/v/o, fp32 g/beta/state (steps a1-a4);
  * decode leg: kda_decode_step for N=256 sequences x H=32 heads, 128 x 128 fp32
    state updated in place (step a5); the 8 pre-drawn input sets are cycled.
Each leg is timed with CUDA events on the stream it is launched on.  `value` is
the prefill leg's tokens/s (sum of sequence lengths, not x heads); the decode
leg's tokens/s (sequences x steps) is reported in `decode`.  L2 is flushed
(a 256 MiB write) before each leg of each step, outside the leg's events.

Multi-GPU: every rank runs an independent replica (no data-path collective;
the path shards by sequence and head).  value = sum over ranks of the tokens
divided by the max over ranks of the time.

`--impl reference` times the fp64 CPU oracle (the correctness reference; there
is no other implementation of this method to run) on the host cores, on a
bounded sample of the same prefill workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s and decode tokens/s; % of tensor / HBM roofline (1 B200)"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch from one
# ncu capture of each kernel on a workload (summaries in profiles/), keyed by
# (kernel, workload).  Reported only while the kernel's source still matches the
# capture; null once it has changed, or for a workload never captured.
_SPLIT = "gated_delta_rule_124_b200/csrc/kda_chunk_split.cu"
_CFG1 = "prefill: B=2 H=32 T=2048 d=128 C=64 bf16"
_CFG2 = "long prefill: B=1 H=32 T=65536 d=128 C=64 bf16 slow decay"
_DECODE = "gated_delta_rule_124_b200/csrc/kda_decode.cu"
_DEC = "decode: N=256 H=32 d=128 bf16, fp32 state, 8 input sets cycled"
MEASURED_TRAFFIC = {
    ("split_intra", _CFG1): (_SPLIT, "0b693b66fe9f5011f077ea95ae6503d88abc4208", 222362880),
    ("split_chain", _CFG1): (_SPLIT, "0b693b66fe9f5011f077ea95ae6503d88abc4208", 195830272),
    # captured on B=1 x T=16384 (a quarter of the tokens) and scaled by 4
    ("chunk_fwd_overlap", _CFG2): (_SPLIT, "0b693b66fe9f5011f077ea95ae6503d88abc4208", 5597298688),
    ("decode", _DEC): (_DECODE, "e97a0fa46338f7541982499a4e97d31ac9101889", 1027143936),
}


def measured_traffic(name, workload):
    import hashlib
    entry = MEASURED_TRAFFIC.get((name, workload))
    if entry is None:
        return None
    path, sha, nbytes = entry
    try:
        with open(os.path.join(ROOT, path), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != sha:
                return None
    except OSError:
        return None
    return nbytes


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return d, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


# ----------------------------------------------------------- algorithmic cost

def prefill_bytes(tokens_x_heads: int, n_seq_heads: int, dk=128, dv=128, in_bytes=2) -> int:
    """q, k (dk) and v (dv) in the input dtype, g fp32 (dk), beta fp32, o (dv);
    plus the initial and final state (fp32) once per (sequence, head)."""
    per = in_bytes * (2 * dk + dv) + 4 * dk + 4 + in_bytes * dv
    return tokens_x_heads * per + n_seq_heads * 2 * 4 * dk * dv


def prefill_flops(tokens_x_heads: int, d=128, C=64) -> int:
    """Per head and token: 6 d^2 + 3 C d + C^2 (Kimi Linear, aiwiki.ai, 'The
    constrained DPLR form and the chunkwise algorithm', training cost)."""
    return tokens_x_heads * (6 * d * d + 3 * C * d + C * C)


def decode_bytes(units: int, dk=128, dv=128, in_bytes=2) -> int:
    """State read + write (fp32) + q, k, v, o (input dtype) + g fp32 + beta."""
    return units * (2 * 4 * dk * dv + in_bytes * (2 * dk + 2 * dv) + 4 * dk + 4)


# ------------------------------------------------------------- multi-rank

def max_over_ranks(vals, world, device="cpu"):
    """Element-wise max of per-rank device times over all ranks (replicas)."""
    if world <= 1:
        return [float(v) for v in vals]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(units_per_rank_step, world, steps, time_ms):
    """Whole-job units/s: every rank's units over the slowest rank's time."""
    return units_per_rank_step * world * steps / (time_ms / 1e3)


# ------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


# ------------------------------------------------------------------ ours

def prefill_case(wl, args):
    """The prefill workload of this run (a named configuration, or --prefill-shape)."""
    if args.prefill_shape:
        B, T, H = (int(x) for x in args.prefill_shape.split(","))
        return wl.make_prefill(1100, [T] * B, H=H, dk=128, dv=128, chunk=64, dtype="bf16",
                               name=f"prefill: B={B} H={H} T={T} d=128 C=64 bf16")
    return wl.prefill_config(args.prefill_config)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import gated_delta_rule_124_b200 as kda
    from gated_delta_rule_124_b200 import workloads as wl

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    kda.load()

    # ---- inputs (resident in HBM before timing)
    pc = prefill_case(wl, args)
    P = pc.to(dev)
    dcase = wl.decode_config()
    D = [{k: v.to(dev) for k, v in s.items()} for s in dcase.steps]
    state = dcase.state0.to(dev)
    Np, H, dk, dv, C = P.N, P.H, P.dk, P.dv, P.chunk
    total = P.total
    ws = kda.alloc_workspace(total, Np, H, dk, dv, C, "bf16", dev)
    o = torch.empty_like(P.v)
    hN = torch.empty(Np, H, dk, dv, dtype=torch.float32, device=dev)
    Nd = dcase.N
    od = torch.empty(Nd, H, dv, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    Bc, Tc = (1, total) if P.cu_seqlens is not None else (P.B, P.T)

    def prefill():
        kda.kda_chunk_fwd(P.q, P.k, P.v, P.g, P.beta, P.initial_state, P.cu_seqlens, Bc, Tc, Np,
                          H, dk, dv, C, "bf16", o, hN, ws)

    def decode(i):
        s = D[i % len(D)]
        kda.kda_decode_step(s["q"], s["k"], s["v"], s["g"], s["beta"], state, od, Nd, H, dk,
                            dv, "bf16")

    def step(i, ev=None):
        flush.zero_()
        if ev: ev[0].record(stream)
        prefill()
        if ev: ev[1].record(stream)
        flush.zero_()
        if ev: ev[2].record(stream)
        decode(i)
        if ev: ev[3].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status(ws) == kda.KDA_OK

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t0.elapsed_time(t1)
    pre_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[2].elapsed_time(e[3]) for e in evs]
    pre_sum, dec_sum = sum(pre_ms), sum(dec_ms)

    # ---- max over ranks (device time), whole-job throughput
    total_ms, pre_sum, dec_sum = max_over_ranks([total_ms, pre_sum, dec_sum], world, dev)
    value = job_throughput(total, world, args.steps, pre_sum)
    dec_value = job_throughput(Nd, world, args.steps, dec_sum)

    # ---- per-kernel times of the prefill (dominant kernel) with the step calls
    kern = prefill_kernel_times(kda, P, ws, dev, stream, reps=max(5, min(50, args.steps)))

    # ---- the steps around the operator (conv/Swish/L2-norm before, RMSNorm and
    # output gate after), on this workload's tensors, each timed alone
    layer = layer_times(kda, torch, P, dev, stream, reps=max(5, min(50, args.steps)))

    # ---- end to end through host buffers (pinned), copies inside the region
    e2e = run_e2e(kda, torch, pc, dcase, dev, stream, steps=max(3, min(args.steps, 50)))

    # ---- the backward (gradients of o and the final state) on the same workload,
    # last: a failure there is reported in its entry and leaves the line intact
    bwd = None
    if not args.no_backward:
        try:
            bwd = backward_times(
                kda, torch, P, pc, dev, stream, reps=max(3, min(20, args.steps)),
                sm_max_mhz=clk.get("sm_max_mhz") if isinstance(clk, dict) else None)
        except (kda.KdaError, RuntimeError, AssertionError) as e:
            bwd = {"error": f"{type(e).__name__}: {e}"}

    peaks, peak_kind = load_peaks()
    hbm = peaks["hbm_gbs"]
    tx = total * H
    pb = prefill_bytes(tx, Np * H)
    pf = prefill_flops(tx)
    pre_avg = pre_sum / args.steps / 1e3  # s
    dom_name, dom_s = kern["dominant"]
    # roofline of the dominant prefill kernel: its share of the algorithmic bytes
    dom_bytes = kern["bytes"][dom_name]
    roof = {"kernel": dom_name, "bound": "hbm", "achieved": dom_bytes / dom_s / 1e9,
            "peak": hbm, "unit": "GB/s", "frac": dom_bytes / dom_s / 1e9 / hbm,
            "traffic": measured_traffic(dom_name, pc.name),
            "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)",
            "per_launch_us": dom_s * 1e6, "algorithmic_bytes_per_launch": dom_bytes}
    dec_avg = dec_sum / args.steps / 1e3
    db = decode_bytes(Nd * H)
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; distributions of the pages' configurations)",
        "config": {"workload": pc.name, "B": pc.B, "T": pc.T, "H": H, "dk": dk, "dv": dv,
                   "chunk": C, "prefill_path": kern["path"], "decode_workload": dcase.name,
                   "l2": "flushed (256 MiB write) before each leg",
                   "parallelism": f"replicas x{world}"},
        "prefill": {"value": value, "unit": "tokens/s", "ms_per_call": pre_avg * 1e3,
                    "hbm_frac": pb / pre_avg / 1e9 / hbm,
                    "tensor_frac": pf / pre_avg / 1e12 / peaks["bf16_tflops"],
                    "algorithmic_bytes": pb, "paper_flops": pf,
                    "kernels_us": {k: v * 1e6 for k, v in kern["times"].items()}},
        "decode": {"value": dec_value, "unit": "tokens/s", "ms_per_step": dec_avg * 1e3,
                   "roofline": {"bound": "hbm", "achieved": db / dec_avg / 1e9, "peak": hbm,
                                "unit": "GB/s", "frac": db / dec_avg / 1e9 / hbm,
                                "traffic": measured_traffic("decode", dcase.name),
                                "algorithmic_bytes_per_launch": db}},
        "roofline": roof,
        "layer_steps": layer,
        "backward": bwd,
        "e2e": e2e,
        "gpu_launches": args.steps * (kern["launches_per_call"] + 1),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(pc, seconds=args.cpu_seconds)
        if isinstance(bwd, dict) and "error" not in bwd:
            bwd["cpu_oracle"] = cpu_baseline_backward(pc)
    return res


def prefill_path(kda, total, Np, H, dk, dv, C, packed, dtype="bf16"):
    """The plan kda_chunk_fwd runs for this problem (the library's own answer):
    'simt', 'fused', 'split' or 'overlap' (see include/kda.h)."""
    return kda.PLAN_NAMES[kda.kda_chunk_fwd_plan(total, Np, H, dk, dv, C, dtype, packed)]


def prefill_kernel_times(kda, P, ws, dev, stream, reps=20):
    """Device times of the prefill kernels, each from CUDA events around its own
    call on the launching stream, L2 flushed before each.  CUDA-core path: the
    four step calls (a1..a4); split plan: kda_chunk_split_intra and
    kda_chunk_split_chain; fused plan: the one kernel (the whole call).  Each
    call's time includes the chunk-table kernel that starts it, where it has
    one.  Algorithmic bytes are the pages' inputs and outputs that each kernel
    must move; the split plan's hand-over through the workspace is overhead."""
    import torch
    Np, H, dk, dv, C, total = P.N, P.H, P.dk, P.dv, P.chunk, P.total
    path = prefill_path(kda, total, Np, H, dk, dv, C, P.cu_seqlens is not None)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    in_b = 2
    tx = total * H
    Bc, Tc = (1, total) if P.cu_seqlens is not None else (P.B, P.T)

    def timed(calls):
        times = {}
        for name in calls:
            ts = []
            for _ in range(reps):
                for n2, f in calls.items():  # the whole sequence, so inputs are valid
                    if n2 == name:
                        flush.zero_()
                        e0 = torch.cuda.Event(enable_timing=True)
                        e1 = torch.cuda.Event(enable_timing=True)
                        e0.record(stream)
                        f()
                        e1.record(stream)
                        ts.append((e0, e1))
                    else:
                        f()
            torch.cuda.synchronize()
            times[name] = statistics.median(x.elapsed_time(y) for x, y in ts) / 1e3
        return times

    if path != "simt":
        o = torch.empty_like(P.v)
        hN = torch.empty(Np, H, dk, dv, device=dev)
        if path in ("fused", "overlap"):
            name = "chunk_fwd_tc" if path == "fused" else "chunk_fwd_overlap"
            calls = {name: lambda: kda.kda_chunk_fwd(
                P.q, P.k, P.v, P.g, P.beta, P.initial_state, P.cu_seqlens, Bc, Tc, Np, H, dk,
                dv, C, "bf16", o, hN, ws)}
            nbytes = {name: prefill_bytes(tx, Np * H)}
            launches = 2
        else:
            a = (P.cu_seqlens, Bc, Tc, Np, H)
            calls = {
                "split_intra": lambda: kda.kda_chunk_split_intra(P.q, P.k, P.g, P.beta, *a, ws),
                "split_chain": lambda: kda.kda_chunk_split_chain(P.v, P.initial_state, *a, o,
                                                                 hN, ws),
            }
            nbytes = {"split_intra": tx * (in_b * 2 * dk + 4 * dk + 4),
                      "split_chain": tx * in_b * 2 * dv + Np * H * 2 * 4 * dk * dv}
            launches = 3
        times = timed(calls)
        dom = max(times, key=times.get)
        return {"times": times, "bytes": nbytes, "dominant": (dom, times[dom]),
                "launches_per_call": launches, "path": path}
    G = torch.empty(total, H, dk, device=dev)
    W = torch.empty(total, H, dk, device=dev)
    U = torch.empty(total, H, dv, device=dev)
    maxc = kda.kda_num_chunks_upper_bound(total, Np, C)
    S = torch.empty(maxc, H, dk, dv, device=dev)
    hN = torch.empty(Np, H, dk, dv, device=dev)
    o = torch.empty_like(P.v)
    a = (P.cu_seqlens, Bc, Tc, Np, H)
    calls = {
        "a1_gate_cumsum": lambda: kda.kda_chunk_gate_cumsum(P.g, *a, dk, C, G, ws),
        "a2_intra": lambda: kda.kda_chunk_intra(P.k, P.v, G, P.beta, *a, dk, dv, C, "bf16", W,
                                                U, ws),
        "a3_inter": lambda: kda.kda_chunk_inter(P.k, G, W, U, P.initial_state, *a, dk, dv, C,
                                                "bf16", S, hN, ws),
        "a4_output": lambda: kda.kda_chunk_output(P.q, P.k, G, U, S, *a, dk, dv, C, "bf16", o,
                                                  ws),
    }
    tx = total * H
    nbytes = {
        "a1_gate_cumsum": tx * dk * 8,
        "a2_intra": tx * (in_b * (dk + dv) + 4 * dk + 4 + 4 * (dk + dv)),
        "a3_inter": tx * (in_b * dk + 4 * dk + 4 * dk + 8 * dv) + maxc * H * dk * dv * 4,
        "a4_output": tx * (in_b * 2 * dk + 4 * dk + 4 * dv + in_b * dv) + maxc * H * dk * dv * 4,
    }
    times = timed(calls)
    dom = max(times, key=times.get)
    return {"times": times, "bytes": nbytes, "dominant": (dom, times[dom]),
            "launches_per_call": 5, "path": path}


def layer_times(kda, torch, P, dev, stream, reps=20):
    """CUDA-event times of kda_qkv_conv_norm and kda_output_norm_gate on the
    prefill workload's shapes (bf16), L2 flushed before each, with their HBM
    fraction (bytes: every tensor read or written once; conv weights excluded)."""
    total, H, dk, dv = P.total, P.H, P.dk, P.dv
    Bc, Tc = (1, total) if P.cu_seqlens is not None else (P.B, P.T)
    g = torch.Generator(device=dev).manual_seed(7)
    xs = [torch.randn(total, H, d, device=dev, generator=g).to(torch.bfloat16)
          for d in (dk, dk, dv)]
    ws = [torch.randn(H * d, 4, device=dev, generator=g) for d in (dk, dk, dv)]
    outs = [torch.empty_like(x) for x in xs]
    gate = torch.randn(total, H, dv, device=dev, generator=g).to(torch.bfloat16)
    wn = torch.ones(dv, device=dev)
    y = torch.empty_like(gate)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    calls = {
        "qkv_conv_norm": (lambda: kda.kda_qkv_conv_norm(*xs, *ws, P.cu_seqlens, Bc, Tc, P.N, H,
                                                        dk, dv, "bf16", 1e-6, *outs),
                          2 * 2 * total * H * (2 * dk + dv)),
        "output_norm_gate": (lambda: kda.kda_output_norm_gate(outs[2], gate, wn, total, H, dv,
                                                              "bf16", 1e-6, y),
                             2 * 3 * total * H * dv),
    }
    peaks, _ = load_peaks()
    res = {}
    for name, (f, nbytes) in calls.items():
        f()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            f()
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        t = statistics.median(x.elapsed_time(z) for x, z in ts) / 1e3
        res[name] = {"us": t * 1e6, "bytes": nbytes, "gbs": nbytes / t / 1e9,
                     "hbm_frac": nbytes / t / 1e9 / peaks["hbm_gbs"]}
    return res


def backward_flops(head_tokens, dk, dv, C=64):
    """Floating-point operations of the chunked backward per call: per chunk
    of C tokens and one head, the multiply-adds of each step (the forward's
    A, P, W, Ut and chain recomputed, then E, F, the reverse chain, the back
    substitution, the products with U, S and dS', and the pair sums), two
    flops each."""
    tri, stri = C * (C + 1) // 2, C * (C - 1) // 2
    fma = (2 * tri * dk + stri * (dk + dv) + 2 * C * dk * dv      # A, P; [W | Ut]; chain
           + tri * dv + 2 * C * dk * dv + 2 * C * dk * dv        # E; F; reverse chain
           + stri * dv + 2 * C * C * dv + 3 * C * dk * dv        # Y; Y U^T, dO U^T; dense
           + 4 * tri * dk)                                        # pair sums
    return 2 * fma * head_tokens / C


def backward_times(kda, torch, P, pc, dev, stream, reps=10, sm_max_mhz=None):
    """kda_chunk_bwd on the prefill workload (fp32 gradients of o and the final
    state), timed with CUDA events on the launching stream, L2 flushed before
    each call.  Bound by fp32 arithmetic on the CUDA cores: the roofline peak
    is 148 SMs x 128 fp32 lanes x 2 flops x the SM clock."""
    total, H, dk, dv = P.total, P.H, P.dk, P.dv
    Bc, Tc = (1, total) if P.cu_seqlens is not None else (P.B, P.T)
    g = torch.Generator(device=dev).manual_seed(9)
    do = torch.randn(total, H, dv, device=dev, generator=g).to(torch.bfloat16)
    dhT = torch.randn(P.N, H, dk, dv, device=dev, generator=g)
    f32 = dict(dtype=torch.float32, device=dev)
    outs = [torch.empty(total, H, dk, **f32), torch.empty(total, H, dk, **f32),
            torch.empty(total, H, dv, **f32), torch.empty(total, H, dk, **f32),
            torch.empty(total, H, **f32), torch.empty(P.N, H, dk, dv, **f32)]
    ws = torch.empty(kda.kda_chunk_bwd_workspace_size(total, P.N, H, dk, dv), dtype=torch.uint8,
                     device=dev)
    call = lambda: kda.kda_chunk_bwd(P.q, P.k, P.v, P.g, P.beta, P.initial_state, do, dhT,
                                     P.cu_seqlens, Bc, Tc, P.N, H, dk, dv, "bf16", *outs, ws)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    call()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    t = statistics.median(x.elapsed_time(z) for x, z in ts) / 1e3
    fl = backward_flops(total * H, dk, dv)
    mhz = sm_max_mhz or 1965.0
    peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
    res = {"ms_per_call": t * 1e3, "tokens_per_s": total / t, "kernels_per_call": 9,
           "roofline": {"bound": "alu", "achieved": fl / t / 1e12, "peak": peak,
                        "unit": "TFLOP/s", "frac": fl / t / 1e12 / peak,
                        "peak_kind": f"fp32 CUDA cores, 148 SMs x 128 lanes x 2 x {mhz:.0f} MHz",
                        "algorithmic_flops_per_call": fl},
           "workspace_bytes": int(ws.numel())}
    return res


def run_e2e(kda, torch, pc, dcase, dev, stream, steps=10):
    """Prefill through the public call with pinned host buffers: H2D of the
    inputs, kda_chunk_fwd, D2H of o and the final state -- all inside the
    events; the same for one decode step (state resident on the device)."""
    pin = lambda t: None if t is None else t.pin_memory()
    hq, hk, hv, hg, hb, h0 = map(pin, (pc.q, pc.k, pc.v, pc.g, pc.beta, pc.initial_state))
    dq, dk_, dv_, dg, db, d0 = (torch.empty_like(x, device=dev) for x in (hq, hk, hv, hg, hb, h0))
    H, dk, dv, C, N, total = pc.H, pc.dk, pc.dv, pc.chunk, pc.N, pc.total
    o = torch.empty_like(dv_)
    hN = torch.empty(N, H, dk, dv, device=dev)
    ho = torch.empty_like(hv).pin_memory()
    hhN = torch.empty(N, H, dk, dv).pin_memory()
    ws = kda.alloc_workspace(total, N, H, dk, dv, C, "bf16", dev)

    hcu = None if pc.cu_seqlens is None else pc.cu_seqlens.pin_memory()
    dcu = None if hcu is None else torch.empty_like(hcu, device=dev)
    Bc, Tc = (1, total) if hcu is not None else (pc.B, pc.T)

    def one():
        for d, h in ((dq, hq), (dk_, hk), (dv_, hv), (dg, hg), (db, hb), (d0, h0), (dcu, hcu)):
            if d is not None:
                d.copy_(h, non_blocking=True)
        kda.kda_chunk_fwd(dq, dk_, dv_, dg, db, d0, dcu, Bc, Tc, N, H, dk, dv, C, "bf16",
                          o, hN, ws)
        ho.copy_(o, non_blocking=True)
        hhN.copy_(hN, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    t = a.elapsed_time(b) / 1e3 / steps
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hg, hb, h0, hcu)
              if x is not None)
    d2h = ho.numel() * ho.element_size() + hhN.numel() * hhN.element_size()

    # decode: per step the token's inputs go up and o comes back
    s0 = dcase.steps[0]
    hs = {k: v.pin_memory() for k, v in s0.items()}
    ds = {k: torch.empty_like(v, device=dev) for k, v in hs.items()}
    state = dcase.state0.to(dev)
    od = torch.empty(dcase.N, H, dv, dtype=torch.bfloat16, device=dev)
    hod = torch.empty_like(od, device="cpu").pin_memory()

    def dec():
        for kname in ds:
            ds[kname].copy_(hs[kname], non_blocking=True)
        kda.kda_decode_step(ds["q"], ds["k"], ds["v"], ds["g"], ds["beta"], state, od, dcase.N,
                            H, dk, dv, "bf16")
        hod.copy_(od, non_blocking=True)

    for _ in range(2):
        dec()
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(steps):
        dec()
    b.record(stream)
    torch.cuda.synchronize()
    td = a.elapsed_time(b) / 1e3 / steps
    dh2d = sum(x.numel() * x.element_size() for x in hs.values())
    return {"value": total / t, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "decode": {"value": dcase.N / td, "unit": "tokens/s", "h2d_bytes_per_step": dh2d,
                       "d2h_bytes_per_step": hod.numel() * hod.element_size()}}


# ------------------------------------------------------------- cpu baseline

def cpu_baseline(pc, seconds=15.0, heads=None):
    """The fp64 oracle (as it stands) on the host cores, on a bounded sample of
    the prefill workload.  With `heads` given: the first sequence, first
    `heads` heads, once.  Otherwise the whole workload (all sequences and
    heads), repeated until about `seconds` of CPU time have run.  Reported as
    tokens/s of the full workload (head-tokens/s / H)."""
    import oracle
    cores = oracle.max_threads()
    H = pc.H
    if heads is not None:
        T = pc.T
        t = time.perf_counter()
        oracle.forward(pc.q[:T, :heads], pc.k[:T, :heads], pc.v[:T, :heads], pc.g[:T, :heads],
                       pc.beta[:T, :heads], pc.initial_state[:1, :heads], num_threads=cores)
        el = time.perf_counter() - t
        return {"value": T * heads / el / H, "unit": "tokens/s", "cores": cores,
                "kind": "oracle", "sample": f"1 sequence x {T} tokens x {heads} of {H} heads, "
                                            f"fp64 token recurrence, {el:.1f} s"}
    cu = pc.cu_host()
    reps, el = 0, 0.0
    while el < seconds:
        t = time.perf_counter()
        oracle.forward(pc.q, pc.k, pc.v, pc.g, pc.beta, pc.initial_state, cu_seqlens=cu,
                       num_threads=cores)
        el += time.perf_counter() - t
        reps += 1
    # one thread, on the first sequence's first two heads
    T1, h1 = int(cu[1]) - int(cu[0]), min(2, H)
    t = time.perf_counter()
    oracle.forward(pc.q[:T1, :h1], pc.k[:T1, :h1], pc.v[:T1, :h1], pc.g[:T1, :h1],
                   pc.beta[:T1, :h1], pc.initial_state[:1, :h1], num_threads=1)
    el1 = time.perf_counter() - t
    return {"value": pc.total * reps / el, "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"whole prefill workload ({pc.N} x {pc.T} tokens x {H} heads) x {reps} "
                      f"repetitions, fp64 token recurrence, {el:.1f} s",
            "single_thread": {"value": T1 * h1 / el1 / H, "unit": "tokens/s",
                              "sample": f"1 sequence x {T1} tokens x {h1} of {H} heads, "
                                        f"1 thread, {el1:.2f} s"}}


def cpu_baseline_backward(pc, tokens=256):
    """The gradient oracle (fp64 token recurrence differentiated by autograd, as
    it stands) on a bounded sample of the prefill workload: the first `tokens`
    tokens of the first sequence, one head, one thread.  Reported as tokens/s of
    the full workload (head-tokens/s / H), beside the backward's GPU time."""
    import torch

    from oracle import backward as obwd
    H, dk, dv = pc.H, pc.dk, pc.dv
    Ts = min(tokens, int(pc.cu_host()[1]))
    hd = lambda x: x[:Ts, :1]  # noqa: E731
    g0 = torch.Generator().manual_seed(9)
    do0 = torch.randn(Ts, 1, dv, generator=g0).to(torch.bfloat16)
    h0 = pc.initial_state[:1, :1] if pc.initial_state is not None else torch.zeros(1, 1, dk, dv)
    t0 = time.perf_counter()
    obwd.backward(hd(pc.q), hd(pc.k), hd(pc.v), hd(pc.g), pc.beta[:Ts, :1], h0, do0, None,
                  [0, Ts])
    el = time.perf_counter() - t0
    return {"value": Ts / el / H, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"1 sequence x {Ts} tokens x 1 of {H} heads, fp64 token recurrence "
                      f"differentiated by autograd, {el:.2f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from gated_delta_rule_124_b200 import workloads as wl
    pc = wl.prefill_config(1)
    for _ in range(args.warmup):
        cpu_baseline(pc, heads=1)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = cpu_baseline(pc, heads=max(1, min(pc.H, args.ref_heads)))
        vals.append(r["value"])
    el = time.perf_counter() - t0
    v = statistics.median(vals)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": pc.name, "B": pc.B, "T": pc.T, "H": pc.H, "dk": pc.dk,
                       "dv": pc.dv, "chunk": pc.chunk},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": r["cores"],
                             "kind": "oracle", "sample": r["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_backward_only(args):
    """kda_chunk_bwd alone on the prefill workload (one GPU)."""
    import torch

    import gated_delta_rule_124_b200 as kda
    from gated_delta_rule_124_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    kda.load()
    pc = prefill_case(wl, args)
    P = pc.to(dev)
    bwd = backward_times(kda, torch, P, pc, dev, torch.cuda.current_stream(),
                         reps=max(3, min(20, args.steps)))
    if not args.no_cpu_baseline:
        bwd["cpu_oracle"] = cpu_baseline_backward(pc)
    return {"backward": bwd, "config": {"workload": pc.name, "B": pc.B, "T": pc.T, "H": pc.H,
                                        "dk": pc.dk, "dv": pc.dv}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-heads", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward timing beside the step")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only kda_chunk_bwd on the prefill workload and print its "
                         "entry (for profiling the backward kernels alone)")
    ap.add_argument("--prefill-config", type=int, default=1, choices=[1, 2, 3],
                    help="prefill workload: 1 = B=2 x T=2048 (default), 2 = B=1 x T=65536, "
                         "3 = 16 packed sequences of U[1024,16384] tokens")
    ap.add_argument("--prefill-shape", default=None, metavar="B,T,H",
                    help="instead of --prefill-config: B sequences of T tokens, H heads "
                         "(d = 128, chunk 64, bf16, the default configuration's distributions)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if args.backward_only:
        if rank == 0:
            print(json.dumps(run_backward_only(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_ours(args, rank, world, local)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
