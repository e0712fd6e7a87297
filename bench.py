#!/usr/bin/env python
"""Benchmark: KDA prefill tokens/s and decode tokens/s on one B200 (replicas for N > 1).

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill leg: kda_chunk_fwd over the varlen workload -- 16 packed sequences
    of U[1024, 16384] tokens (seeded), H=32 heads, dk = dv = 128, chunk 64,
    bf16 q/k/v/o, fp32 g/beta/state (steps a1-a4), the largest configuration;
  * decode leg: the decode workload, N=256 sequences x H=32 heads, 128 x 128
    fp32 states updated in place, all 1000 steps of its schedule (8 pre-drawn
    input sets cycled), one kda_decode_step launch per step (step a5).
Each leg is timed with CUDA events on the stream it is launched on.  `value` is
the prefill leg's tokens/s (sum of sequence lengths, not x heads); the decode
leg's tokens/s (sequences x steps) is reported in `decode`.  Both workloads are
larger than L2 (≈6 GB of prefill inputs, a 512 MiB state); L2 is also flushed
(a 256 MiB write) before each prefill leg.  The other prefill configurations
(B=2 x T=2048 and B=1 x T=65536) are timed outside the step and reported under
`configs`; `parity` holds the errors of the timed configurations against the
fp64 oracle.

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
_CFG3 = "varlen prefill: 16 seqs U[1024,16384] H=32 d=128 C=64 bf16"
_CFG2 = "long prefill: B=1 H=32 T=65536 d=128 C=64 bf16 slow decay"
_DECODE = "gated_delta_rule_124_b200/csrc/kda_decode.cu"
_DEC = "decode: N=256 H=32 d=128 bf16, fp32 state, 8 input sets cycled"
MEASURED_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch, captured on
    # B=8 x T=2048, H=32 (8192 (chunk, head) items, inputs larger than L2)
    # and scaled by the items of the varlen workload (62560): per item
    # 127.7 KB (intra) and 100.9 KB (chain)
    ("split_intra", _CFG3): (_SPLIT, "1dd5be2a9803eb0eceec8f921e9102c6fdb8dedc", 7986931585),
    ("split_chain", _CFG3): (_SPLIT, "1dd5be2a9803eb0eceec8f921e9102c6fdb8dedc", 6309916945),
    ("decode", _DEC): (_DECODE, "e97a0fa46338f7541982499a4e97d31ac9101889", 1027143936),
}


TRAFFIC_NOTE = {
    ("split_intra", _CFG3): "ncu DRAM bytes of B=8 x T=2048, H=32 scaled by (chunk, head) items",
    ("split_chain", _CFG3): "ncu DRAM bytes of B=8 x T=2048, H=32 scaled by (chunk, head) items",
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


def _events(torch, n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def time_calls(torch, stream, flush, f, reps):
    """Median device time (s) of f() over `reps` calls, CUDA events on the
    launching stream, L2 flushed before each call outside its events."""
    f()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = _events(torch, 2)
        a.record(stream)
        f()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(x.elapsed_time(y) for x, y in ts) / 1e3


def prefill_roofline(kern, pc, peaks, peak_kind):
    """Roofline of the dominant kernel of one prefill call: its algorithmic
    bytes per launch over its CUDA-event time, against the measured HBM copy
    bandwidth; `traffic` is its ncu DRAM bytes while the source matches."""
    hbm = peaks["hbm_gbs"]
    dom_name, dom_s = kern["dominant"]
    dom_bytes = kern["bytes"][dom_name]
    return {"kernel": dom_name, "bound": "hbm", "achieved": dom_bytes / dom_s / 1e9,
            "peak": hbm, "unit": "GB/s", "frac": dom_bytes / dom_s / 1e9 / hbm,
            "traffic": measured_traffic(dom_name, pc.name),
            "traffic_note": (TRAFFIC_NOTE.get((dom_name, pc.name))
                             if measured_traffic(dom_name, pc.name) else None),
            "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)",
            "per_launch_us": dom_s * 1e6, "algorithmic_bytes_per_launch": dom_bytes}


def prefill_summary(P, t, peaks):
    """tokens/s, HBM and tensor fractions of one prefill call of t seconds."""
    tx = P.total * P.H
    pb = prefill_bytes(tx, P.N * P.H)
    pf = prefill_flops(tx)
    return {"value": P.total / t, "unit": "tokens/s", "ms_per_call": t * 1e3,
            "hbm_frac": pb / t / 1e9 / peaks["hbm_gbs"],
            "tensor_frac": pf / t / 1e12 / peaks["bf16_tflops"],
            "algorithmic_bytes": pb, "paper_flops": pf}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import gated_delta_rule_124_b200 as kda
    from gated_delta_rule_124_b200 import workloads as wl

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    kda.load()
    peaks, peak_kind = load_peaks()
    hbm = peaks["hbm_gbs"]

    # ---- inputs (resident in HBM before timing)
    pc = prefill_case(wl, args)
    P = pc.to(dev)
    dcase = wl.decode_config()
    D = [{k: v.to(dev) for k, v in s.items()} for s in dcase.steps]
    state0 = dcase.state0.to(dev)
    state = state0.clone()
    Np, H, dk, dv, C = P.N, P.H, P.dk, P.dv, P.chunk
    total = P.total
    ws = kda.alloc_workspace(total, Np, H, dk, dv, C, "bf16", dev)
    o = torch.empty_like(P.v)
    hN = torch.empty(Np, H, dk, dv, dtype=torch.float32, device=dev)
    Nd = dcase.N
    dsteps = args.decode_steps
    od = torch.empty(Nd, H, dv, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    Bc, Tc = (1, total) if P.cu_seqlens is not None else (P.B, P.T)

    def prefill(out=o):
        kda.kda_chunk_fwd(P.q, P.k, P.v, P.g, P.beta, P.initial_state, P.cu_seqlens, Bc, Tc, Np,
                          H, dk, dv, C, "bf16", out, hN, ws)

    def decode_pass(st, outs=None):
        for i in range(dsteps):
            s = D[i % len(D)]
            kda.kda_decode_step(s["q"], s["k"], s["v"], s["g"], s["beta"], st,
                                od if outs is None else outs[i], Nd, H, dk, dv, "bf16")

    def step(ev=None):
        flush.zero_()
        if ev: ev[0].record(stream)
        prefill()
        if ev: ev[1].record(stream)
        if ev: ev[2].record(stream)
        decode_pass(state)
        if ev: ev[3].record(stream)

    for i in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert kda.kda_get_device_status(ws) == kda.KDA_OK

    evs = [_events(torch, 4) for _ in range(args.steps)]
    t0, t1 = _events(torch, 2)
    clocks = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
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
    dec_value = job_throughput(Nd * dsteps, world, args.steps, dec_sum)

    # ---- per-kernel times of the prefill (dominant kernel) with the step calls
    reps = max(5, min(20, args.steps))
    kern = prefill_kernel_times(kda, P, ws, dev, stream, reps=reps)
    pre_avg = pre_sum / args.steps / 1e3  # s
    prefill_entry = prefill_summary(P, pre_avg, peaks)
    prefill_entry["kernels_us"] = {k: v * 1e6 for k, v in kern["times"].items()}
    roof = prefill_roofline(kern, pc, peaks, peak_kind)

    # ---- parity of the timed configurations against the fp64 oracle (one
    # untimed call each), the oracle's time doubling as the CPU baseline
    do_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    parity, cpu = {}, None
    if do_cpu:
        o_chk = torch.full_like(P.v, float("nan"))
        prefill(o_chk)
        torch.cuda.synchronize()
        cpu, parity[pc.name] = oracle_prefill_parity(pc, o_chk, hN)
        del o_chk

    # ---- the other prefill configurations, each timed outside the step
    configs = {}
    if not args.only_headline:
        for idx in (1, 2):
            pcx = wl.prefill_config(idx)
            if pcx.name == pc.name:
                continue
            configs[str(idx)] = prefill_config_entry(kda, torch, pcx, dev, stream, flush, peaks,
                                                     peak_kind, reps, do_cpu, parity)

    # ---- decode: roofline and a parity pass from the initial state
    dec_avg = dec_sum / args.steps / dsteps / 1e3  # s per decode step
    db = decode_bytes(Nd * H)
    decode_entry = {"value": dec_value, "unit": "tokens/s", "ms_per_step": dec_avg * 1e3,
                    "steps_per_pass": dsteps,
                    "roofline": {"bound": "hbm", "achieved": db / dec_avg / 1e9, "peak": hbm,
                                 "unit": "GB/s", "frac": db / dec_avg / 1e9 / hbm,
                                 "traffic": measured_traffic("decode", dcase.name),
                                 "algorithmic_bytes_per_launch": db}}
    if do_cpu:
        outs = torch.empty(dsteps, Nd, H, dv, dtype=torch.bfloat16, device=dev)
        st = state0.clone()
        decode_pass(st, outs)
        torch.cuda.synchronize()
        decode_entry["cpu_baseline"], parity[dcase.name] = oracle_decode_parity(
            dcase, dsteps, outs, st, seqs=args.decode_parity_seqs)
        del outs, st

    # ---- the steps around the operator (conv/Swish/L2-norm before, RMSNorm and
    # output gate after), on this workload's tensors, each timed alone
    layer = layer_times(kda, torch, P, dcase, dev, stream, reps=reps)

    # ---- end to end through host buffers (pinned), copies inside the region
    e2e = run_e2e(kda, torch, pc, dcase, dev, stream, steps=6)

    # ---- the backward (gradients of o and the final state) on the B=2 x
    # T=2048 workload, last: a failure there is reported in its entry and
    # leaves the line intact
    bwd = None
    if not args.no_backward:
        try:
            pcb = wl.prefill_config(1)
            bwd = backward_times(
                kda, torch, pcb.to(dev), pcb, dev, stream, reps=max(3, min(20, args.steps)),
                sm_max_mhz=clk.get("sm_max_mhz") if isinstance(clk, dict) else None)
            bwd["workload"] = pcb.name
            if do_cpu:
                bwd["cpu_oracle"] = cpu_baseline_backward(pcb)
        except (kda.KdaError, RuntimeError, AssertionError) as e:
            bwd = {"error": f"{type(e).__name__}: {e}"}

    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; distributions of the pages' configurations)",
        "config": {"workload": pc.name, "B": pc.B, "T": pc.T, "N": Np, "tokens": total,
                   "H": H, "dk": dk, "dv": dv, "chunk": C, "prefill_path": kern["path"],
                   "decode_workload": dcase.name, "decode_steps_per_step": dsteps,
                   "l2": "inputs larger than L2; L2 also flushed (256 MiB write) before each "
                         "prefill leg",
                   "parallelism": f"replicas x{world}"},
        "prefill": prefill_entry,
        "decode": decode_entry,
        "roofline": roof,
        "configs": configs,
        "parity": parity,
        "layer_steps": layer,
        "backward": bwd,
        "e2e": e2e,
        "gpu_launches": args.steps * (kern["launches_per_call"] + dsteps),
        "clocks": clk,
    }
    if cpu is not None:
        res["cpu_baseline"] = cpu
    return res


def prefill_config_entry(kda, torch, pc, dev, stream, flush, peaks, peak_kind, reps, do_cpu,
                         parity):
    """One other prefill configuration: the default call timed alone (median of
    `reps`, L2 flushed before each), its plan, kernel times and dominant-kernel
    roofline, and (rank 0, one GPU) its parity and CPU-oracle baseline."""
    P = pc.to(dev)
    Bc, Tc = (1, P.total) if P.cu_seqlens is not None else (P.B, P.T)
    ws = kda.alloc_workspace(P.total, P.N, P.H, P.dk, P.dv, P.chunk, "bf16", dev)
    o = torch.empty_like(P.v)
    hN = torch.empty(P.N, P.H, P.dk, P.dv, device=dev)
    call = lambda: kda.kda_chunk_fwd(P.q, P.k, P.v, P.g, P.beta, P.initial_state,  # noqa: E731
                                     P.cu_seqlens, Bc, Tc, P.N, P.H, P.dk, P.dv, P.chunk, "bf16",
                                     o, hN, ws)
    t = time_calls(torch, stream, flush, call, reps)
    assert kda.kda_get_device_status(ws) == kda.KDA_OK
    kern = prefill_kernel_times(kda, P, ws, dev, stream, reps=reps)
    e = prefill_summary(P, t, peaks)
    e.update({"workload": pc.name, "prefill_path": kern["path"],
              "kernels_us": {k: v * 1e6 for k, v in kern["times"].items()},
              "roofline": prefill_roofline(kern, pc, peaks, peak_kind)})
    if do_cpu:
        o.fill_(float("nan"))
        call()
        torch.cuda.synchronize()
        e["cpu_baseline"], parity[pc.name] = oracle_prefill_parity(pc, o, hN)
    del P, ws, o, hN
    torch.cuda.empty_cache()
    return e


def _parity_entry(x, ref):
    """max |x - ref| / max |ref| and max |x - ref| / (|ref| + 1e-3 max |ref|)."""
    import numpy as np
    x = x.detach().to("cpu", dtype=__import__("torch").float64).numpy() \
        if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.abs(x - ref)
    m = float(np.abs(ref).max(initial=0.0))
    return {"max_abs_over_max_ref": float(d.max(initial=0.0)) / max(m, 1e-30),
            "elementwise": float((d / (np.abs(ref) + 1e-3 * m)).max(initial=0.0)),
            "finite": bool(np.isfinite(x).all())}


def oracle_prefill_parity(pc, o, hN):
    """The fp64 oracle (as it stands) on the whole prefill workload, on all host
    cores, once: its time is the CPU baseline and its result the parity
    reference of the GPU call's o and final state."""
    import oracle
    cores = oracle.max_threads()
    t = time.perf_counter()
    ro, rh = oracle.forward(pc.q, pc.k, pc.v, pc.g, pc.beta, pc.initial_state,
                            cu_seqlens=pc.cu_host(), num_threads=cores)
    el = time.perf_counter() - t
    tol = 2e-2 if pc.dtype == "bf16" else 1e-4
    par = {"o": _parity_entry(o, ro), "final_state": _parity_entry(hN, rh), "tolerance": tol,
           "sample": "every sequence, head and token"}
    par["pass"] = all(par[k]["max_abs_over_max_ref"] <= tol and par[k]["finite"]
                      for k in ("o", "final_state"))
    cpu = {"value": pc.total / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": f"whole workload ({pc.N} sequences, {pc.total} tokens x {pc.H} heads) "
                     f"once, fp64 token recurrence, {el:.1f} s"}
    return cpu, par


def oracle_decode_parity(dcase, steps, outs, state, seqs=32):
    """The fp64 oracle replays the first `seqs` sequences' `steps` decode steps
    (all heads) as one recurrence per sequence; its time is the decode CPU
    baseline, its outputs (every step) and final states the parity reference."""
    import numpy as np
    import torch

    import oracle
    cores = oracle.max_threads()
    sched = [t % len(dcase.steps) for t in range(steps)]
    H, dv = dcase.H, dcase.dv
    seqs = min(seqs, dcase.N)
    seq = {k: torch.stack([dcase.steps[i][k][:seqs] for i in sched], 1)
           for k in ("q", "k", "v", "g", "beta")}
    flat = {k: v.reshape(-1, *v.shape[2:]) for k, v in seq.items()}
    cu = np.arange(0, (seqs + 1) * steps, steps, dtype=np.int32)
    t = time.perf_counter()
    ro, rs = oracle.forward(flat["q"], flat["k"], flat["v"], flat["g"], flat["beta"],
                            dcase.state0[:seqs], cu_seqlens=cu, num_threads=cores)
    el = time.perf_counter() - t
    ro = ro.reshape(seqs, steps, H, dv).transpose(1, 0, 2, 3)
    par = {"o": _parity_entry(outs[:, :seqs], ro), "state": _parity_entry(state[:seqs], rs),
           "tolerance": 2e-2,
           "sample": f"{seqs} of {dcase.N} sequences x {H} heads, all {steps} steps"}
    par["pass"] = all(par[k]["max_abs_over_max_ref"] <= 2e-2 and par[k]["finite"]
                      for k in ("o", "state"))
    cpu = {"value": seqs * steps / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": f"{seqs} sequences x {H} heads x {steps} steps, fp64 recurrence, "
                     f"{el:.1f} s"}
    return cpu, par


def prefill_path(kda, total, Np, H, dk, dv, C, packed, dtype="bf16"):
    """The plan kda_chunk_fwd runs for this problem (the library's own answer):
    'simt', 'split' or 'overlap' (see include/kda.h)."""
    return kda.PLAN_NAMES[kda.kda_chunk_fwd_plan(total, Np, H, dk, dv, C, dtype, packed)]


def prefill_kernel_times(kda, P, ws, dev, stream, reps=20):
    """Device times of the prefill kernels, each from CUDA events around its own
    call on the launching stream, L2 flushed before each.  CUDA-core path: the
    four step calls (a1..a4); split plan: kda_chunk_split_intra and
    kda_chunk_split_chain; overlap plan: the one co-scheduled launch.  Each
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
        if path == "overlap":
            name = "chunk_fwd_overlap"
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


def layer_times(kda, torch, P, dcase, dev, stream, reps=20):
    """The steps around the operator on this workload's shapes (bf16), each
    timed with CUDA events, L2 flushed before each call: the three separate
    calls (kda_qkv_conv_norm, kda_output_norm_gate, with their HBM fraction --
    every tensor read or written once, filters excluded) and, for the whole
    layer core, the fused call (kda_layer_chunk_fwd) against the three
    separate launches around kda_chunk_fwd; the same for one decode step
    (kda_layer_decode_step against kda_qkv_conv_norm_step + kda_decode_step +
    kda_output_norm_gate) on the decode workload."""
    total, H, dk, dv = P.total, P.H, P.dk, P.dv
    N = P.N
    Bc, Tc = (1, total) if P.cu_seqlens is not None else (P.B, P.T)
    g = torch.Generator(device=dev).manual_seed(7)
    xs = [torch.randn(total, H, d, device=dev, generator=g).to(torch.bfloat16)
          for d in (dk, dk, dv)]
    ws = [torch.randn(H * d, 4, device=dev, generator=g) * 0.5 for d in (dk, dk, dv)]
    outs = [torch.empty_like(x) for x in xs]
    gate = torch.randn(total, H, dv, device=dev, generator=g).to(torch.bfloat16)
    wn = torch.ones(dv, device=dev)
    y = torch.empty_like(gate)
    o = torch.empty_like(gate)
    hN = torch.empty(N, H, dk, dv, device=dev)
    wsp = kda.alloc_workspace(total, N, H, dk, dv, P.chunk, "bf16", dev)
    wsl = torch.empty(kda.kda_layer_chunk_fwd_workspace_size(total, N, H, dk, dv, P.chunk, "bf16"),
                      dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    conv = lambda: kda.kda_qkv_conv_norm(*xs, *ws, P.cu_seqlens, Bc, Tc, N, H, dk, dv,  # noqa
                                         "bf16", 1e-6, *outs)
    norm = lambda: kda.kda_output_norm_gate(outs[2], gate, wn, total, H, dv, "bf16", 1e-6, y)  # noqa

    def separate():
        conv()
        kda.kda_chunk_fwd(*outs, P.g, P.beta, P.initial_state, P.cu_seqlens, Bc, Tc, N, H, dk,
                          dv, P.chunk, "bf16", o, hN, wsp)
        kda.kda_output_norm_gate(o, gate, wn, total, H, dv, "bf16", 1e-6, y)

    fused = lambda: kda.kda_layer_chunk_fwd(*xs, *ws, P.g, P.beta, P.initial_state,  # noqa
                                            P.cu_seqlens, Bc, Tc, N, H, dk, dv, P.chunk, "bf16",
                                            gate, wn, 1e-6, 1e-6, y, hN, wsl)
    peaks, _ = load_peaks()
    res = {}
    for name, f, nbytes in (("qkv_conv_norm", conv, 2 * 2 * total * H * (2 * dk + dv)),
                            ("output_norm_gate", norm, 2 * 3 * total * H * dv)):
        t = time_calls(torch, stream, flush, f, reps)
        res[name] = {"us": t * 1e6, "bytes": nbytes, "gbs": nbytes / t / 1e9,
                     "hbm_frac": nbytes / t / 1e9 / peaks["hbm_gbs"]}
    res["layer_prefill"] = {"workload": P.name if hasattr(P, "name") else None,
                            "fused_us": time_calls(torch, stream, flush, fused, reps) * 1e6,
                            "separate_launches_us": time_calls(torch, stream, flush, separate,
                                                               reps) * 1e6}
    assert kda.kda_get_device_status(wsl) == kda.KDA_OK
    # one decode step of the layer core
    Nd = dcase.N
    s0 = {k: v.to(dev) for k, v in dcase.steps[0].items()}
    st = dcase.state0.to(dev)
    dxs = [torch.randn(Nd, H, d, device=dev, generator=g).to(torch.bfloat16)
           for d in (dk, dk, dv)]
    cst = [torch.zeros(Nd, 3, H, d, device=dev, dtype=torch.bfloat16) for d in (dk, dk, dv)]
    dgate = torch.randn(Nd, H, dv, device=dev, generator=g).to(torch.bfloat16)
    dy = torch.empty_like(dgate)
    qkv = [torch.empty_like(x) for x in dxs]
    od = torch.empty_like(dgate)
    dfused = lambda: kda.kda_layer_decode_step(*dxs, *ws, *cst, s0["g"], s0["beta"], st,  # noqa
                                               dgate, wn, Nd, H, dk, dv, "bf16", 1e-6, 1e-6, dy)

    def dseparate():
        kda.kda_qkv_conv_norm_step(*dxs, *ws, *cst, Nd, H, dk, dv, "bf16", 1e-6, *qkv)
        kda.kda_decode_step(*qkv, s0["g"], s0["beta"], st, od, Nd, H, dk, dv, "bf16")
        kda.kda_output_norm_gate(od, dgate, wn, Nd, H, dv, "bf16", 1e-6, dy)

    res["layer_decode_step"] = {"workload": dcase.name,
                                "fused_us": time_calls(torch, stream, flush, dfused, reps) * 1e6,
                                "separate_launches_us": time_calls(torch, stream, flush,
                                                                   dseparate, reps) * 1e6}
    return res


def backward_flops(head_tokens, dk, dv, C=64):
    """Floating-point operations of the chunked backward per call: per chunk
    of C tokens and one head, the multiply-adds of each step (the forward's
    A, P, W, Ut and chain recomputed, then E, F, the reverse chain, the back
    substitution, the products with U, S and dS', and the pair sums), two
    flops each.  Returns (on the tensor cores, on the CUDA cores): for dk = dv
    = 128 every contraction runs as a tcgen05 product (the substitutions as
    products with T = (I + A)^-1); other shapes run everything on the CUDA
    cores."""
    tri, stri = C * (C + 1) // 2, C * (C - 1) // 2
    tensor = (2 * tri * dk                                         # A, P
              + stri * (dk + dv)                                   # [W | Ut]
              + 2 * C * dk * dv + 2 * C * dk * dv                  # the two chains
              + tri * dv + 2 * C * dk * dv                         # E; F
              + stri * dv + 2 * C * C * dv                         # Y; Y U^T, dO U^T
              + 3 * C * dk * dv                                    # dense
              + 4 * tri * dk)                                      # pair sums
    alu = 0
    if not (dk == 128 and dv == 128):
        tensor, alu = 0, tensor + alu
    return 2 * tensor * head_tokens / C, 2 * alu * head_tokens / C


def backward_times(kda, torch, P, pc, dev, stream, reps=10, sm_max_mhz=None):
    """kda_chunk_bwd on the prefill workload (fp32 gradients of o and the final
    state), timed with CUDA events on the launching stream, L2 flushed before
    each call.  Roofline: the kernels run one after another, so the bound is
    the tensor-core flops at the tf32 peak (the measured bf16 peak x the
    nominal tf32 / bf16 ratio 1.1 / 2.25) plus any CUDA-core flops at 148
    SMs x 128 fp32 lanes x 2 flops x the SM clock; `peak` is the total flops
    over that time."""
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
    fl_tc, fl_alu = backward_flops(total * H, dk, dv)
    fl = fl_tc + fl_alu
    mhz = sm_max_mhz or 1965.0
    alu_peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
    peaks, kind = load_peaks()
    tf32_peak = peaks["bf16_tflops"] * 1.1 / 2.25
    t_bound = fl_tc / tf32_peak / 1e12 + fl_alu / alu_peak / 1e12
    peak = fl / t_bound / 1e12
    res = {"ms_per_call": t * 1e3, "tokens_per_s": total / t, "kernels_per_call": 11,
           "roofline": {"bound": "tensor" if fl_alu == 0 else "alu",
                        "achieved": fl / t / 1e12, "peak": peak,
                        "unit": "TFLOP/s", "frac": fl / t / 1e12 / peak,
                        "peak_kind": (f"{fl_tc / 1e9:.1f} GFLOP at the tf32 tensor peak "
                                      f"{tf32_peak:.0f} TFLOP/s ({kind} bf16 x 1.1/2.25) + "
                                      f"{fl_alu / 1e9:.1f} GFLOP at the fp32 CUDA-core peak "
                                      f"{alu_peak:.1f} TFLOP/s (148 SMs x 128 lanes x 2 x "
                                      f"{mhz:.0f} MHz); the algorithm's count, not the three "
                                      f"tf32 passes of the products that use them"),
                        "bound_ms": t_bound * 1e3,
                        "algorithmic_flops_per_call": fl},
           "workspace_bytes": int(ws.numel())}
    return res


def run_e2e(kda, torch, pc, dcase, dev, stream, steps=10):
    """Prefill through the public call with pinned host buffers: every step
    copies its inputs host -> device, runs kda_chunk_fwd and copies o and the
    final state back, all inside the events.  Consecutive prefill batches are
    independent, so the steps are pipelined as a server would run them: two
    device buffer sets, the uploads on one stream, the calls on the launching
    stream, the downloads on a third, so that one step's download and call
    overlap the next step's upload (separate copy engines).  One decode step
    (state resident on the device) the same way but serially, since a decode
    step's inputs follow from the previous step's output."""
    pin = lambda t: None if t is None else t.pin_memory()
    hq, hk, hv, hg, hb, h0 = map(pin, (pc.q, pc.k, pc.v, pc.g, pc.beta, pc.initial_state))
    hcu = None if pc.cu_seqlens is None else pc.cu_seqlens.pin_memory()
    host_in = (hq, hk, hv, hg, hb, h0, hcu)
    H, dk, dv, C, N, total = pc.H, pc.dk, pc.dv, pc.chunk, pc.N, pc.total
    Bc, Tc = (1, total) if hcu is not None else (pc.B, pc.T)

    def buffers():
        d_in = tuple(None if h is None else torch.empty_like(h, device=dev) for h in host_in)
        return {"in": d_in, "o": torch.empty_like(d_in[2]),
                "hN": torch.empty(N, H, dk, dv, device=dev),
                "ho": torch.empty_like(hv).pin_memory(),
                "hhN": torch.empty(N, H, dk, dv).pin_memory()}

    sets = [buffers(), buffers()]
    ws = kda.alloc_workspace(total, N, H, dk, dv, C, "bf16", dev)
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    free_in = [ev(), ev()]    # the call that read set b has run
    up_done = [ev(), ev()]    # set b's inputs are on the device
    called = [ev(), ev()]     # set b's outputs are written
    down_done = [ev(), ev()]  # set b's outputs are on the host
    for b in range(2):  # nothing pending on either set at the start
        free_in[b].record(stream)
        down_done[b].record(stream)

    def one(i):
        bset = sets[i % 2]
        b = i % 2
        s_up.wait_event(free_in[b])
        with torch.cuda.stream(s_up):
            for d, h in zip(bset["in"], host_in):
                if d is not None:
                    d.copy_(h, non_blocking=True)
        up_done[b].record(s_up)
        stream.wait_event(up_done[b])
        stream.wait_event(down_done[b])  # o, hN of set b have been read back
        dq, dk_, dv_, dg, db, d0, dcu = bset["in"]
        kda.kda_chunk_fwd(dq, dk_, dv_, dg, db, d0, dcu, Bc, Tc, N, H, dk, dv, C, "bf16",
                          bset["o"], bset["hN"], ws)
        free_in[b].record(stream)
        called[b].record(stream)
        s_down.wait_event(called[b])
        with torch.cuda.stream(s_down):
            bset["ho"].copy_(bset["o"], non_blocking=True)
            bset["hhN"].copy_(bset["hN"], non_blocking=True)
        down_done[b].record(s_down)

    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_up.wait_event(a)
    for i in range(steps):
        one(i)
    stream.wait_event(down_done[(steps - 1) % 2])
    stream.wait_event(down_done[steps % 2])
    b_.record(stream)
    torch.cuda.synchronize()
    t = a.elapsed_time(b_) / 1e3 / steps
    h2d = sum(x.numel() * x.element_size() for x in host_in if x is not None)
    d2h = sets[0]["ho"].numel() * sets[0]["ho"].element_size() + \
        sets[0]["hhN"].numel() * sets[0]["hhN"].element_size()
    del sets

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
    b_.record(stream)
    torch.cuda.synchronize()
    td = a.elapsed_time(b_) / 1e3 / steps
    dh2d = sum(x.numel() * x.element_size() for x in hs.values())
    return {"value": total / t, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "decode": {"value": dcase.N / td, "unit": "tokens/s", "h2d_bytes_per_step": dh2d,
                       "d2h_bytes_per_step": hod.numel() * hod.element_size()}}


# ------------------------------------------------------------- cpu baseline

def cpu_baseline(pc, heads=1, tokens=None):
    """The fp64 oracle (as it stands) on the host cores, on a bounded sample of
    the prefill workload: the first sequence's first `tokens` tokens (all of
    them when None) on its first `heads` heads, once.  Reported as tokens/s of
    the full workload (head-tokens/s / H)."""
    import oracle
    cores = oracle.max_threads()
    H = pc.H
    T = int(pc.cu_host()[1])
    if tokens is not None:
        T = min(T, tokens)
    h0 = None if pc.initial_state is None else pc.initial_state[:1, :heads]
    t = time.perf_counter()
    oracle.forward(pc.q[:T, :heads], pc.k[:T, :heads], pc.v[:T, :heads], pc.g[:T, :heads],
                   pc.beta[:T, :heads], h0, num_threads=cores)
    el = time.perf_counter() - t
    return {"value": T * heads / el / H, "unit": "tokens/s", "cores": min(cores, heads),
            "kind": "oracle", "sample": f"1 sequence x {T} tokens x {heads} of {H} heads, "
                                        f"fp64 token recurrence, {el:.2f} s"}


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
    """The oracle as it stands on the host cores, on the headline prefill
    workload's configuration: each step one bounded sample (the first
    sequence's tokens on `--ref-heads` heads, one thread per head)."""
    if rank != 0:
        return None
    from gated_delta_rule_124_b200 import workloads as wl
    pc = prefill_case(wl, args)
    heads = max(1, min(pc.H, args.ref_heads))
    for _ in range(args.warmup):
        cpu_baseline(pc, heads=1, tokens=256)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = cpu_baseline(pc, heads=heads)
        vals.append(r["value"])
    el = time.perf_counter() - t0
    v = statistics.median(vals)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": pc.name, "B": pc.B, "T": pc.T, "N": pc.N,
                       "tokens": pc.total, "H": pc.H, "dk": pc.dk, "dv": pc.dv,
                       "chunk": pc.chunk},
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
    pc = wl.prefill_config(args.backward_config)
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-heads", type=int, default=4)
    ap.add_argument("--decode-steps", type=int, default=1000,
                    help="decode steps per bench step (the decode workload's schedule)")
    ap.add_argument("--decode-parity-seqs", type=int, default=32,
                    help="decode sequences the oracle replays for the parity entry")
    ap.add_argument("--only-headline", action="store_true",
                    help="skip the other prefill configurations (for profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward timing beside the step")
    ap.add_argument("--backward-config", type=int, default=1, choices=[1, 2, 3],
                    help="workload of --backward-only (default: B=2 x T=2048)")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only kda_chunk_bwd on the prefill workload and print its "
                         "entry (for profiling the backward kernels alone)")
    ap.add_argument("--prefill-config", type=int, default=3, choices=[1, 2, 3],
                    help="prefill workload: 3 = 16 packed sequences of U[1024,16384] tokens "
                         "(default, the largest), 1 = B=2 x T=2048, 2 = B=1 x T=65536")
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
