#!/usr/bin/env python
"""Benchmark of the q4f16 dequantizing GEMV hot path on B200.

One step = one Phi-3-mini-shaped decode weight pass at M = 1: 32 layers of
{qkv 3072->9216, o 3072->3072, gate_up 3072->2x8192 with SiLU(gate)*up,
down 8192->3072} plus the LM head 3072->32064 (f32 logits + argmax), on
seeded synthetic q4 weights (2.1 GB, larger than L2, so no flush is needed
between steps).  The step is one call of the library's pass entry point
(zt_q4_pass: one persistent kernel over all 129 projections plus the argmax
reduction), each bracketed by CUDA events.  The workload's activations are
independent inputs (x ~ N(0,1) per projection), so no projection waits on
another.  Reported beside it: the chained form (each projection reads its x
only after every earlier projection finished, as if each x were an earlier
output) and the pass issued as 130 separate calls (CUDA graph + programmatic
dependent launch).

Prints one JSON line (rank 0).  Metric: effective HBM GB/s of the pass
(algorithmic bytes / time); the line also carries us per pass, the roofline
of the dominant kernel, the CPU oracle baseline, an end-to-end figure with
host<->device copies, the SM clocks seen, and the launch count.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
  python bench.py --sweep-m        # gate_up single calls at M = 1, 2, 4, 8, 16
  python bench.py --prefill        # batched prefill: dequant + tensor-core GEMM

--impl reference times the float64 CPU oracle on the same workload (a bounded
sample per step) on the host cores.  With N > 1 (torchrun) every rank runs
its own replica (the path does not shard; weak scaling).  --prefill prints one
line per token count with the GEMM against the measured tensor peak, the
dequant against HBM, and the fused gate_up + SiLU on the same tokens.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from int4_group_quantized_q4f16_b200 import synth  # noqa: E402

METRIC = "q4 dequant-GEMV effective HBM GB/s & % of B200 peak; us per decode weight pass"
NOMINAL_HBM_GBS = 8000.0
def workload(layers: int, seed: int) -> str:
    return (f"Phi-3-mini decode weight pass, M=1: {layers} x (qkv 3072->9216, o 3072->3072, "
            "gate_up 3072->2x8192 +SiLU*up, down 8192->3072) + LM head 3072->32064 f32+argmax; "
            f"q4 group-32 weights, seed {seed}")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--layers", type=int, default=32)
    p.add_argument("--prefill", action="store_true",
                   help="instead of the pass: the batched prefill GEMM (binary16 dequant + tensor-core GEMM) on the "
                        "Phi-3-mini qkv projection (K 3072, N 9216) at M = 128, 512, 2048 tokens, one JSON line per M")
    p.add_argument("--prefill-m", type=str, default="128,512,2048")
    p.add_argument("--only-pass", action="store_true",
                   help="time the pass alone and print its line without the comparisons, the CPU baseline and the "
                        "other configurations (for profiling the pass kernel)")
    p.add_argument("--sweep-m", action="store_true",
                   help="instead of the pass: the fused gate_up projection (K 3072, 2 x 8192 rows) at M = 1, 2, 4, "
                        "8, 16, one JSON line per M")
    return p.parse_args()


MODELS = {
    "phi3": (synth.phi3_mini_layer, synth.phi3_mini_lm_head),
    "llama7b": (synth.llama7b_layer, synth.llama7b_lm_head),
}


def projections(layers: int, model: str = "phi3"):
    """(layer, Proj) for every launch of the pass, LM head last."""
    layer, head = MODELS[model]
    out = [(l, p) for l in range(layers) for p in layer()]
    out.append((0, head()))
    return out


def llama_workload(seed: int) -> str:
    return ("Llama-7B decode weight pass, M=1: 32 x (qkv 4096->12288, o 4096->4096, gate_up 4096->2x11008 +SiLU*up, "
            f"down 11008->4096) + LM head 4096->32000 f32+argmax; q4 group-32 weights, seed {seed}")


def alg_bytes(p: synth.Proj, M: int = 1) -> int:
    """Algorithmic bytes of one call: codes + scales + x + outputs."""
    out_bytes = 4 if p.kind == "lm_head" else 2
    return p.weight_bytes() + M * p.K * 2 + M * p.n_out * out_bytes + (4 * M if p.kind == "lm_head" else 0)


PASS_KERNEL_SOURCES = ("q4_common.cuh", "q4_mma.cuh", "q4_pass.cuh")


def kernel_sources_sha() -> str:
    """Hash of the device sources the pass kernel and the argmax reduction are
    compiled from; a recorded DRAM traffic figure is used only while it matches."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int4_group_quantized_q4f16_b200", "csrc")
    for f in PASS_KERNEL_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------- clocks ----
class ClockSampler:
    """nvidia-smi samples (200 ms) during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        mhz, max_mhz, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                max_mhz = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max_mhz, "reasons": sorted(reasons),
                "samples": len(mhz)}


# ---------------------------------------------------------- distributed ----
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def dist_max(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------- CPU side ----
def cpu_oracle_sample(seed: int, layers: int, threads: int):
    """Time the float64 oracle on `layers` full layers of the pass (all four
    projections each).  Returns (algorithmic bytes, seconds)."""
    import oracle
    o = oracle.get()
    nbytes, secs = 0, 0.0
    for l in range(layers):
        for p in synth.phi3_mini_layer():
            qw, s, x = synth.proj_inputs(seed, l, p)
            t0 = time.perf_counter()
            if p.kind == "gemv":
                o.gemv(qw, s, x, threads=threads)
            else:
                o.gate_up_silu(qw, s, x, threads=threads)
            secs += time.perf_counter() - t0
            nbytes += alg_bytes(p)
    return nbytes, secs


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, world, rank):
    """The oracle as the reference arm: each step = one layer of the pass on
    the host cores (a bounded sample of the same workload)."""
    if rank != 0:
        return
    cores = host_cores()
    for _ in range(args.warmup):
        cpu_oracle_sample(args.seed, 1, cores)
    nbytes, secs = 0, 0.0
    for _ in range(args.steps):
        b, s = cpu_oracle_sample(args.seed, 1, cores)
        nbytes += b
        secs += s
    gbs = nbytes / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload(32, args.seed), "sample_per_step": "layer 0: qkv, o, gate_up+SiLU, down (63.8 MB)"},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": "one Phi-3-mini layer (4 projections, 63.8 MB of q4 weights) per step"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- GPU side ----
def build_pass(args, device, model: str = "phi3"):
    """Allocate the pass on the device: weights, activations, outputs.  All
    activations live in one contiguous buffer and all outputs in another, so
    an end-to-end step moves them with one copy each way."""
    import torch
    from int4_group_quantized_q4f16_b200 import zt_q4
    projs = projections(args.layers, model)
    x_bytes = sum(p.K * 2 for _, p in projs)
    y_bytes = sum(p.n_out * (4 if p.kind == "lm_head" else 2) for _, p in projs) + 16
    xbuf = torch.empty((x_bytes,), dtype=torch.uint8, device=device)
    ybuf = torch.empty((y_bytes,), dtype=torch.uint8, device=device)
    calls, xo, yo = [], 0, 0
    for l, p in projs:
        qw, s, x = synth.proj_inputs(args.seed, l, p)
        xd = xbuf[xo:xo + p.K * 2].view(torch.float16).view(1, p.K)
        xd.copy_(torch.from_numpy(x))
        xo += p.K * 2
        d = {
            "p": p, "layer": l,
            "qw": torch.from_numpy(qw.view(np.int32)).to(device),
            "s": torch.from_numpy(s).to(device),
            "x": xd,
        }
        if p.kind == "lm_head":
            d["y"] = ybuf[yo:yo + p.n_out * 4].view(torch.float32).view(1, p.n_out)
            yo += p.n_out * 4
            d["am"] = ybuf[yo:yo + 4].view(torch.int32)
            yo += 16
            d["ws"] = torch.empty((zt_q4.lmhead_workspace_bytes(1, p.n_out, p.K),), dtype=torch.uint8,
                                  device=device)
        else:
            d["y"] = ybuf[yo:yo + p.n_out * 2].view(torch.float16).view(1, p.n_out)
            yo += p.n_out * 2
        calls.append(d)
    return calls, xbuf, ybuf


def batched_pass_results(seed: int, device, calls, stream, Ms, steps: int, hbm_peak: float):
    """Batched decode: the same pass (the weights of `calls`) with M tokens per projection -- x [M][K]
    ~ N(0,1) fp16, outputs [M][N] -- one zt_q4_pass call, each between its own events.  Returns per M
    (us per pass, GB/s of algorithmic bytes, fraction of the measured copy)."""
    import torch
    from int4_group_quantized_q4f16_b200 import zt_q4
    gen = torch.Generator(device=device).manual_seed(seed)
    out = []
    for M in Ms:
        projs, nbytes = [], 0
        for d in calls:
            p = d["p"]
            e = {"kind": p.kind, "qw": d["qw"], "scales": d["s"],
                 "x": torch.randn((M, p.K), generator=gen, device=device).half(),
                 "out": torch.empty((M, p.n_out), dtype=torch.float32 if p.kind == "lm_head" else torch.float16,
                                    device=device)}
            if p.kind == "lm_head":
                e["argmax"] = torch.empty((M,), dtype=torch.int32, device=device)
            projs.append(e)
            nbytes += alg_bytes(p, M)
        zp = zt_q4.Pass(projs)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with torch.cuda.stream(stream):
            for _ in range(3):
                zp.run(stream)
            for a_, b_ in ev:
                a_.record(stream)
                zp.run(stream)
                b_.record(stream)
            stream.synchronize()
        assert zp.errors() == 0, "a bounded wait of the pass kernel expired"
        us = statistics.mean(a_.elapsed_time(b_) for a_, b_ in ev) * 1e3
        out.append({"M": M, "us": round(us, 2), "GBps": round(nbytes / us / 1e3, 1),
                    "frac": round(nbytes / us / 1e3 / hbm_peak, 4), "bytes": nbytes})
        del zp, projs
    return out


def launch(zt_q4, d, stream):
    p = d["p"]
    if p.kind == "gemv":
        zt_q4.gemv(d["qw"], d["s"], d["x"], d["y"], stream=stream)
    elif p.kind == "gate_up":
        zt_q4.gate_up_silu(d["qw"], d["s"], d["x"], d["y"], stream=stream)
    else:
        zt_q4.lmhead_argmax(d["qw"], d["s"], d["x"], d["y"], d["am"], d["ws"], stream=stream)


def launches_per_step(calls) -> int:
    return sum(2 if d["p"].kind == "lm_head" else 1 for d in calls)


def run_ours(args, world, rank, local):
    import torch
    from int4_group_quantized_q4f16_b200 import zt_q4

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    calls, xbuf, ybuf = build_pass(args, device)
    total_bytes = sum(alg_bytes(d["p"]) for d in calls)
    stream = torch.cuda.Stream(device=device)

    # the pass: one persistent launch over all projections.  The workload's
    # activations are independent inputs, so no projection waits on another;
    # the chained form (each projection waits for all earlier ones, as when
    # every x were an earlier output) is timed below for comparison.
    def make_pass(chained, calls=calls):
        projs = []
        for i, d in enumerate(calls):
            e = {"kind": d["p"].kind, "qw": d["qw"], "scales": d["s"], "x": d["x"], "out": d["y"],
                 "wait": 1 if (chained and i) else 0}
            if d["p"].kind == "lm_head":
                e["argmax"] = d["am"]
            projs.append(e)
        return zt_q4.Pass(projs)

    zpass = make_pass(False)
    zchain = make_pass(True)

    def step():
        zpass.run(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert zpass.errors() == 0, "a bounded wait of the pass kernel expired"

    # ---- timed region: K steps, barrier + sync on both sides.  Each step is
    # one zt_q4_pass call (the pass kernel + the argmax reduction), bracketed
    # by its own event pair on the launching stream; the host enqueues far
    # ahead of the GPU (a step is ~0.5 ms), so the events add no gaps. ----
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.4)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    dist_barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for a0, a1 in evs:
            a0.record(stream)
            step()
            a1.record(stream)
    torch.cuda.synchronize()
    dist_barrier(world)
    ms = evs[0][0].elapsed_time(evs[-1][1])
    launch_ms = [a0.elapsed_time(a1) for a0, a1 in evs]
    clock_info = clocks.stop() if clocks else None
    ms_max = dist_max(ms, world, device)
    ms_per_step = ms_max / args.steps
    value = total_bytes * world * args.steps / (ms_max / 1e3) / 1e9
    assert zpass.errors() == 0, "a bounded wait of the pass kernel expired"
    if args.only_pass:
        if rank == 0:
            kms = statistics.mean(launch_ms)
            print(json.dumps({"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
                              "us_per_launch": round(kms * 1e3, 3), "bytes_per_step": total_bytes,
                              "config": {"workload": workload(args.layers, args.seed), "only_pass": True},
                              "clocks": clock_info}), flush=True)
        return

    # ---- the chained form of the pass, for comparison ----
    with torch.cuda.stream(stream):
        for _ in range(3):
            zchain.run(stream)
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        ch_steps = max(1, min(args.steps, 200))
        for _ in range(ch_steps):
            zchain.run(stream)
        c1.record(stream)
        stream.synchronize()
    chained_us = c0.elapsed_time(c1) / ch_steps * 1e3
    assert zchain.errors() == 0, "a bounded wait of the chained pass expired"

    # ---- the pass with the decoder layer's fusions, for comparison: every
    # qkv split into Q/K rows with a RoPE epilogue and V rows (one [1][9216]
    # output through ld_out), residual add + RMSNorm prologues on Q/K, V and
    # gate_up (x computed while staging; the V projection normalises the same
    # residual again) -- 161 projections, one launch ----
    def make_fused_pass():
        projs, gen = [], torch.Generator(device=device).manual_seed(args.seed)
        pos = torch.full((1,), 1234, dtype=torch.int32, device=device)

        def norm(K):
            return {"residual": torch.randn((1, K), generator=gen, device=device).half(),
                    "delta": torch.randn((1, K), generator=gen, device=device).half(),
                    "gamma": torch.rand((K,), generator=gen, device=device).half() + 0.5, "eps": 1e-5}

        for d in calls:
            name, K = d["p"].name, d["p"].K
            if name == "qkv":
                nm = norm(K)
                D = d["p"].n_out // 3
                projs.append({"kind": "gemv", "qw": d["qw"][:2 * D], "scales": d["s"][:2 * D], "out": d["y"],
                              "ld_out": 3 * D, "norm": nm, "rope": {"pos": pos, "head_dim": 96, "theta": 10000.0}})
                projs.append({"kind": "gemv", "qw": d["qw"][2 * D:], "scales": d["s"][2 * D:],
                              "out": d["y"][:, 2 * D:], "ld_out": 3 * D, "norm": nm})
                continue
            e = {"kind": d["p"].kind, "qw": d["qw"], "scales": d["s"], "x": d["x"], "out": d["y"]}
            if d["p"].kind == "lm_head":
                e["argmax"] = d["am"]
            if name == "gate_up":
                e["norm"] = norm(K)
            projs.append(e)
        return zt_q4.Pass(projs), len(projs)

    def time_alternating(pa, pb, steps):
        """Mean us per call of two passes run alternately, each call between
        its own events, so clock and power drift weigh on both alike."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        with torch.cuda.stream(stream):
            for _ in range(3):
                pa.run(stream)
                pb.run(stream)
            for e in ev:
                e[0].record(stream)
                pa.run(stream)
                e[1].record(stream)
                e[2].record(stream)
                pb.run(stream)
                e[3].record(stream)
            stream.synchronize()
        ta = statistics.mean(e[0].elapsed_time(e[1]) for e in ev) * 1e3
        tb = statistics.mean(e[2].elapsed_time(e[3]) for e in ev) * 1e3
        return ta, tb

    zfused, n_fused = make_fused_pass()
    fz_steps = max(1, min(args.steps, 200))
    plain_us_short, fused_us = time_alternating(zpass, zfused, fz_steps)
    assert zfused.errors() == 0

    # ---- the same pass with groups of 128 k per scale (the GPTQ / AWQ
    # grouping: 1/4 of the scale bytes), alternating with the group-32 pass ----
    g128 = []
    g128_bytes = 0
    for d in calls:
        sc = d["s"][:, ::4].contiguous()
        e = {"kind": d["p"].kind, "qw": d["qw"], "scales": sc, "x": d["x"], "out": d["y"], "group": 128}
        if d["p"].kind == "lm_head":
            e["argmax"] = d["am"]
        g128.append(e)
        g128_bytes += alg_bytes(d["p"]) - d["p"].n_rows * (d["p"].K // 32) * 2 + sc.numel() * 2
    zg128 = zt_q4.Pass(g128)
    plain_us_g, g128_us = time_alternating(zpass, zg128, fz_steps)
    assert zg128.errors() == 0

    # ---- the same pass as 130 separate calls (graph + PDL), for comparison ----
    def capture(fn):
        with torch.cuda.stream(stream):
            fn()
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
        torch.cuda.synchronize()
        return g

    def per_call_step():
        for d in calls:
            launch(zt_q4, d, stream)

    pc_graph = capture(per_call_step)
    with torch.cuda.stream(stream):
        for _ in range(5):
            pc_graph.replay()
        p0 = torch.cuda.Event(enable_timing=True)
        p1 = torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        pc_steps = max(1, min(args.steps, 200))
        for _ in range(pc_steps):
            pc_graph.replay()
        p1.record(stream)
        stream.synchronize()
    per_call_us = p0.elapsed_time(p1) / pc_steps * 1e3
    pc_graph.reset()

    # ---- the pass launch alone, after an idle GPU (queued behind a GPU delay),
    # for comparison with its duration inside the sustained timed region ----
    pass_ms = []
    with torch.cuda.stream(stream):
        for _ in range(5):
            torch.cuda._sleep(20_000_000)
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            step()
            a1.record(stream)
            stream.synchronize()
            pass_ms.append(a0.elapsed_time(a1))
    isolated_ms = statistics.median(pass_ms)

    # ---- per-launch durations of the dominant kernel (same stream) ----
    # Each launch is bracketed by timing events (which also keeps consecutive
    # launches from overlapping).  A fixed-length GPU delay is queued first so
    # that the host has enqueued the whole pass before the GPU reaches it: the
    # events then time kernels, not host launch latency.
    per = {}
    evs = []
    with torch.cuda.stream(stream):
        for rep in range(3):
            torch.cuda._sleep(40_000_000)
            evs = []
            for d in calls:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                launch(zt_q4, d, stream)
                b.record(stream)
                evs.append((d, a, b))
            stream.synchronize()
            for i, (d, a, b) in enumerate(evs):
                per.setdefault(i, []).append(a.elapsed_time(b))
    # dominant kernel: the pass kernel, one launch per step over all the bytes;
    # its duration = the mean event-bracketed call inside the timed region
    kb = total_bytes
    kms = statistics.mean(launch_ms)
    achieved = kb / (kms / 1e3) / 1e9
    per_kind = {}
    for i, (d, _, _) in enumerate(evs):
        per_kind.setdefault(d["p"].name, []).append(statistics.median(per[i]) * 1e3)
    per_kind_us = {k: round(sum(v) / len(v), 3) for k, v in per_kind.items()}

    # ---- end to end through the public API: every step copies its activations host -> device (pinned),
    # runs the pass and copies all its outputs device -> host.  Two buffer sets and a copy stream per
    # direction let the copies of neighbouring steps overlap the pass (step k's inputs go in while step
    # k - 1 computes; its outputs come back while step k + 1 computes); events order every reuse.  The
    # same steps run back to back on one stream are reported beside it (serial). ----
    x_host = xbuf.cpu().pin_memory()
    y_host = [torch.empty_like(ybuf, device="cpu").pin_memory() for _ in range(2)]
    h2d = x_host.numel()
    d2h = y_host[0].numel()
    xb2, yb2 = [xbuf, torch.empty_like(xbuf)], [ybuf, torch.empty_like(ybuf)]

    def retarget(cs, xs, ys):
        """the calls with x / y / argmax as views at the same offsets of other buffers"""
        out = []
        for d in cs:
            e = dict(d)
            for key, src, dst in (("x", xbuf, xs), ("y", ybuf, ys), ("am", ybuf, ys)):
                if key in d:
                    t = d[key]
                    off = t.data_ptr() - src.data_ptr()
                    nb = t.numel() * t.element_size()
                    e[key] = dst[off:off + nb].view(t.dtype).view(t.shape)
            out.append(e)
        return out

    passes = [zpass, make_pass(False, retarget(calls, xb2[1], yb2[1]))]
    h2d_s = torch.cuda.Stream(device=device)
    d2h_s = torch.cuda.Stream(device=device)

    def e2e_pipelined(n, e_start=None, e_end=None):
        done, out_done = [None, None], [None, None]
        if e_start is not None:
            e_start.record(h2d_s)
        for k in range(n):
            j = k & 1
            with torch.cuda.stream(h2d_s):
                if done[j] is not None:
                    h2d_s.wait_event(done[j])          # the pass that read this x set has finished
                xb2[j].copy_(x_host, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(h2d_s)
            stream.wait_event(ev_in)
            if out_done[j] is not None:
                stream.wait_event(out_done[j])         # this output set has been copied out
            passes[j].run(stream)
            ev_p = torch.cuda.Event()
            ev_p.record(stream)
            done[j] = ev_p
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_p)
                y_host[j].copy_(yb2[j], non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(d2h_s)
                out_done[j] = ev_o
        if e_end is not None:
            e_end.record(d2h_s)

    e2e_steps = max(1, min(args.steps, 200))
    e2e_pipelined(3)
    torch.cuda.synchronize()
    dist_barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_pipelined(e2e_steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = dist_max(e0.elapsed_time(e1), world, device)
    e2e_value = total_bytes * world * e2e_steps / (e2e_ms / 1e3) / 1e9
    assert all(p.errors() == 0 for p in passes), "a bounded wait of the pass kernel expired"

    def e2e_serial_step():
        xbuf.copy_(x_host, non_blocking=True)
        step()
        y_host[0].copy_(ybuf, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            e2e_serial_step()
        stream.synchronize()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(e2e_steps):
            e2e_serial_step()
        s1.record(stream)
        stream.synchronize()
    e2e_serial_value = total_bytes * e2e_steps / (s0.elapsed_time(s1) / 1e3) / 1e9

    # ---- a read-only stream probe of this GPU, beside the driver's copy peak:
    # torch.sum over 2 GiB of fp16 (a library kernel), best of 5 -- context for
    # the percentages only; any failure leaves it null ----
    read_probe = None
    try:
        buf = torch.ones((1 << 30,), dtype=torch.float16, device=device)
        best = float("inf")
        with torch.cuda.stream(stream):
            for _ in range(6):
                p0 = torch.cuda.Event(enable_timing=True)
                p1 = torch.cuda.Event(enable_timing=True)
                p0.record(stream)
                torch.sum(buf, dtype=torch.float32)
                p1.record(stream)
                stream.synchronize()
                best = min(best, p0.elapsed_time(p1))
        read_probe = round(buf.numel() * 2 / (best / 1e3) / 1e9, 1)
        del buf
    except Exception:   # noqa: BLE001 -- a context figure must never break the line
        read_probe = None

    # ---- config 4: the Llama-7B decode weight pass (3.72 GB), independent
    # and chained, each call between its own events on the launching stream ----
    lcalls, _, _ = build_pass(args, device, "llama7b")
    lbytes = sum(alg_bytes(d["p"]) for d in lcalls)
    lpass, lchain = make_pass(False, lcalls), make_pass(True, lcalls)
    l_steps = max(20, min(args.steps, 200))

    def per_call_mean_us(zp, steps):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with torch.cuda.stream(stream):
            for _ in range(3):
                zp.run(stream)
            for e0_, e1_ in ev:
                e0_.record(stream)
                zp.run(stream)
                e1_.record(stream)
            stream.synchronize()
        return statistics.mean(e0_.elapsed_time(e1_) for e0_, e1_ in ev) * 1e3

    l_us = per_call_mean_us(lpass, l_steps)
    l_chain_us = per_call_mean_us(lchain, max(10, l_steps // 4))
    assert lpass.errors() == 0 and lchain.errors() == 0, "a bounded wait of the Llama pass expired"
    del lpass, lchain, lcalls
    torch.cuda.empty_cache()

    # ---- config 3 (small batch) and the batched prefill, at modest step counts ----
    sweep = sweep_m_results(args.seed, device, stream, max(64, min(args.steps, 200)), 3,
                            float(measured_peaks().get("hbm_gbs", 6650.0)))
    batched = batched_pass_results(args.seed, device, calls, stream, (2, 4, 8, 16), max(10, min(args.steps, 50)),
                                   float(measured_peaks().get("hbm_gbs", 6650.0)))
    pre_rows, _, _ = prefill_results(args.seed, device, stream, [512, 2048], max(16, min(args.steps, 100)), 3)
    torch.cuda.empty_cache()

    # ---- CPU oracle baseline (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1:
        cores = host_cores()
        nb, secs = cpu_oracle_sample(args.seed, 4, cores)
        # the same oracle on one thread, on the first layer's o projection (5.3 MB): bounded to ~1 s
        import oracle as _oracle
        o1 = _oracle.get()
        p_o = synth.phi3_mini_layer()[1]
        qo, so, xo = synth.proj_inputs(args.seed, 0, p_o)
        t0 = time.perf_counter()
        o1.gemv(qo, so, xo, threads=1)
        t1 = time.perf_counter() - t0
        cpu = {"value": round(nb / secs / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"layers 0-3 of the pass (16 projections, {nb / 1e6:.1f} MB), float64 oracle, "
                         f"OpenMP over rows, {secs:.1f} s",
               "single_thread": {"value": round(alg_bytes(p_o) / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                                 "sample": f"layer 0 o projection ({alg_bytes(p_o) / 1e6:.1f} MB), {t1:.2f} s"}}

    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            peaks = json.load(fh)
    except (OSError, ValueError):
        pass
    peak = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
    traffic = None
    try:
        with open(os.path.join(ROOT, "profiles", "q4_pass_traffic.json")) as fh:
            tr = json.load(fh)
        if tr.get("kernel_sources_sha") == kernel_sources_sha():
            traffic = round(tr["dram_bytes_per_algorithmic_byte"] * kb)
    except (OSError, ValueError, KeyError):
        pass

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16xf16->f32 (int4 codes, fp16 scales)",
            "data": "synthetic",
            "config": {"workload": workload(args.layers, args.seed), "M": 1, "layers": args.layers, "launches_per_step": 2,
                       "entry_point": "zt_q4_pass (one persistent kernel over independent projections) + argmax reduction",
                       "bytes_per_step": total_bytes, "l2": f"inputs larger than L2 ({total_bytes / 1e9:.2f} GB per step, L2 126 MB)",
                       "parallelism": f"replicas x{world}"},
            "us_per_pass": round(ms_per_step * 1e3, 2),
            "pct_of_nominal_8TBs": round(value / world / NOMINAL_HBM_GBS * 100, 2),
            "pct_of_measured_peak": round(value / world / peak * 100, 2),
            "read_stream_probe_gbs": read_probe,
            "pct_of_read_stream_probe": round(value / world / read_probe * 100, 2) if read_probe else None,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "kernel": f"q4_pass_kernel (one launch per step over the {len(calls)} projections)",
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                         else "fallback 6.65 TB/s",
                         "bytes_per_launch": round(kb), "us_per_launch": round(kms * 1e3, 3),
                         "us_per_launch_after_idle": round(isolated_ms * 1e3, 3),
                         "duration": "mean of the event-bracketed zt_q4_pass calls of the timed region "
                                     "(pass kernel + argmax reduction)"},
            "chained_us_per_pass": round(chained_us, 2),
            "group_128": {"us_per_pass": round(g128_us, 2), "plain_us_per_pass": round(plain_us_g, 2),
                          "GBps": round(g128_bytes / g128_us / 1e3, 1), "bytes_per_pass": g128_bytes,
                          "steps": fz_steps,
                          "what": "the same pass with 128 k per scale (scale bytes / 4); calls alternating with the "
                                  "group-32 pass"},
            "decode_fusions": {"us_per_pass": round(fused_us, 2), "plain_us_per_pass": round(plain_us_short, 2),
                               "steps": fz_steps, "projections": n_fused,
                               "what": "RoPE epilogue on every Q/K, residual add + RMSNorm prologues on Q/K, V and "
                                       "gate_up (96 norms, x computed while staging); calls alternating with "
                                       "the plain pass, each between its own events"},
            "per_call_graph_us_per_pass": round(per_call_us, 2),
            "llama7b_pass": {"workload": llama_workload(args.seed), "us_per_pass": round(l_us, 2),
                             "GBps": round(lbytes / l_us / 1e3, 1), "frac": round(lbytes / l_us / 1e3 / peak, 4),
                             "bytes_per_pass": lbytes, "chained_us_per_pass": round(l_chain_us, 2),
                             "steps": l_steps, "kernel": "q4_pass_kernel + argmax reduction, one zt_q4_pass call",
                             "duration": "mean of event-bracketed zt_q4_pass calls"},
            "small_batch": {**sweep_summary(sweep),
                            "pass": {"workload": "the Phi-3-mini decode weight pass (129 projections, one zt_q4_pass "
                                                 "call) with M tokens per projection",
                                     "M": [b["M"] for b in batched], "us_per_pass": [b["us"] for b in batched],
                                     "GBps": [b["GBps"] for b in batched], "frac": [b["frac"] for b in batched]}},
            "prefill": {"workload": "Phi-3-mini qkv 3072->9216 (dequant + tcgen05 GEMM) and gate_up 3072->2x8192 "
                                    "+SiLU (cached binary16 weights), q4 group-32",
                        "tokens": {str(r["M"]): {k: v for k, v in r.items() if k != "M"} for r in pre_rows},
                        "peak_source": "MEASURED_PEAKS.json bf16_tflops (burst) and hbm_gbs"},
            "per_projection_us_isolated": per_kind_us,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "serial_value": round(e2e_serial_value, 2),
                    "what": "per step: one pinned H2D copy of the pass's activations, the pass (zt_q4_pass), one "
                            "D2H copy of all its outputs; two buffer sets and a copy stream per direction overlap "
                            "neighbouring steps' copies with the pass (serial_value: the same steps on one stream)"},
            "gpu_launches": 2 * args.steps,
            "clocks": clock_info,
        }
        print(json.dumps(line), flush=True)


def _timed_calls(stream, fn, steps: int, warmup: int) -> float:
    """us per call of fn(i), i = 0 .. steps - 1, after `warmup` untimed calls;
    one CUDA-event pair on the launching stream around the timed calls."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(warmup):
            fn(i)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(steps):
            fn(i)
        b.record(stream)
        stream.synchronize()
    return a.elapsed_time(b) / steps * 1e3


SWEEP_MS = (1, 2, 4, 8, 16)


def sweep_m_results(seed: int, device, stream, steps: int, warmup: int, hbm_peak: float):
    """The small-batch configuration: gate_up (K 3072, 2 x 8192 rows,
    SiLU(g)*u) at M = 1, 2, 4, 8, 16 tokens through the decode entry point
    (codes unpacked in registers into tensor-core mma operands), beside the
    tcgen05 path of the batched prefill (weights dequantized to binary16 per
    call; and on cached binary16 weights).  Eight weight copies (8 x 28.3 MB,
    > L2) in turn, so every call streams its weights from HBM."""
    import torch
    from int4_group_quantized_q4f16_b200 import zt_q4
    K, N, copies = 3072, 8192, 8
    p = synth.Proj("gate_up", "gate_up", K, N, synth.PROJ_GATE_UP)
    w, w16 = [], []
    for c in range(copies):
        qw, s, _ = synth.proj_inputs(seed, c, p)
        qd, sd = torch.from_numpy(qw.view(np.int32)).to(device), torch.from_numpy(s).to(device)
        w.append((qd, sd))
        w16.append(zt_q4.dequant_f16(qd, sd, stream=stream))
    stream.synchronize()
    ws = torch.empty((zt_q4.gemm_gate_up_workspace_bytes(16, N, K),), dtype=torch.uint8, device=device)
    gws = torch.empty((256,), dtype=torch.uint8, device=device)
    out = []
    for M in SWEEP_MS:
        x = torch.randn((M, K), generator=torch.Generator(device=device).manual_seed(M), device=device).half()
        y = torch.empty((M, N), dtype=torch.float16, device=device)
        n = max(steps, 8 * copies)
        dec = _timed_calls(stream, lambda i: zt_q4.gate_up_silu(w[i % copies][0], w[i % copies][1], x, y,
                                                                stream=stream), n, warmup * copies)
        tcd = _timed_calls(stream, lambda i: zt_q4.gemm_gate_up_silu(w[i % copies][0], w[i % copies][1], x, y,
                                                                     workspace=ws, stream=stream), n, warmup * copies)
        tcc = _timed_calls(stream, lambda i: zt_q4.gemm_f16w_gate_up_silu(w16[i % copies], x, y, workspace=gws,
                                                                          stream=stream), n, warmup * copies)
        assert zt_q4.gemm_errors(ws, 2 * N, K) == 0 and zt_q4.gemm_f16w_errors(gws) == 0
        nbytes = alg_bytes(p, M)
        out.append({"M": M, "decode_us": round(dec, 3), "decode_GBps": round(nbytes / dec / 1e3, 1),
                    "decode_frac": round(nbytes / dec / 1e3 / hbm_peak, 4), "bytes_per_call": nbytes,
                    "tcgen05_dequant_per_call_us": round(tcd, 3), "tcgen05_cached_f16_us": round(tcc, 3),
                    "calls": n})
    del w16
    return out


def sweep_summary(rows) -> dict:
    cross = next((r["M"] for r in rows
                  if min(r["tcgen05_dequant_per_call_us"], r["tcgen05_cached_f16_us"]) < r["decode_us"]), None)
    return {"workload": "gate_up K=3072 N=2x8192 +SiLU*up, q4 group-32, single calls, 8 weight copies in turn",
            "M": [r["M"] for r in rows], "decode_us": [r["decode_us"] for r in rows],
            "decode_GBps": [r["decode_GBps"] for r in rows], "decode_frac": [r["decode_frac"] for r in rows],
            "tcgen05_dequant_per_call_us": [r["tcgen05_dequant_per_call_us"] for r in rows],
            "tcgen05_cached_f16_us": [r["tcgen05_cached_f16_us"] for r in rows],
            "crossover_M": cross,
            "crossover": "smallest M at which the tcgen05 prefill path beats the decode kernel; null: not up to 16"}


def run_sweep_m(args, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=device)
    rows = sweep_m_results(args.seed, device, stream, args.steps, max(args.warmup, 3),
                           float(measured_peaks().get("hbm_gbs", 6650.0)))
    for r in rows:
        print(json.dumps({"metric": "q4 gate_up GEMV effective HBM GB/s", "value": r["decode_GBps"], "unit": "GB/s",
                          **r, "config": {"workload": "gate_up K=3072 N=2x8192 +SiLU*up, q4 group-32, single calls"}}),
              flush=True)
    print(json.dumps({"small_batch": sweep_summary(rows)}), flush=True)


def measured_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh)
    except (OSError, ValueError):
        return {}


def prefill_results(seed: int, device, stream, Ms, steps: int, warmup: int):
    """Batched prefill (M > 16): zt_q4_gemm = dequant to binary16 (HBM-bound)
    + tcgen05 GEMM (tensor-bound) on the Phi-3-mini qkv projection, and the
    fused gate_up + SiLU on cached binary16 weights.  Four weight copies
    rotate so the dequant streams from HBM; each timed region is bracketed by
    CUDA events on the launching stream."""
    import torch
    from int4_group_quantized_q4f16_b200 import zt_q4
    K, N, copies = 3072, 9216, 4
    p = synth.Proj("qkv", "gemv", K, N, synth.PROJ_QKV)
    w = []
    for c in range(copies):
        qw, s, _ = synth.proj_inputs(seed, c, p)
        qd, sd = torch.from_numpy(qw.view(np.int32)).to(device), torch.from_numpy(s).to(device)
        w.append((qd, sd, torch.empty((N, K), dtype=torch.float16, device=device)))
    peaks = measured_peaks()
    tc_peak = peaks.get("bf16_tflops")
    hbm_peak = peaks.get("hbm_gbs")
    gp = synth.Proj("gate_up", "gate_up", K, 8192, synth.PROJ_GATE_UP)
    ffn = []
    for c in range(copies):
        gq, gs, _ = synth.proj_inputs(seed, c, gp)
        ffn.append(zt_q4.dequant_f16(torch.from_numpy(gq.view(np.int32)).to(device), torch.from_numpy(gs).to(device),
                                     stream=stream))
    stream.synchronize()
    out = []
    for M in Ms:
        x = torch.randn((M, K), generator=torch.Generator(device=device).manual_seed(M), device=device).half()
        y = torch.empty((M, N), dtype=torch.float16, device=device)
        n = max(steps, 4 * copies)
        ws = [torch.empty((zt_q4.gemm_workspace_bytes(M, N, K),), dtype=torch.uint8, device=device)
              for _ in range(copies)]
        gws = torch.empty((zt_q4.gemm_f16w_workspace_bytes(M, N, K),), dtype=torch.uint8, device=device)
        w_ = warmup * copies
        both = _timed_calls(stream, lambda i: zt_q4.gemm(w[i % copies][0], w[i % copies][1], x, y, ws[i % copies],
                                                         stream=stream), n, w_)
        gemm = _timed_calls(stream, lambda i: zt_q4.gemm_f16w(w[i % copies][2], x, y, gws, stream=stream), n, w_)
        deq = _timed_calls(stream, lambda i: zt_q4.dequant_f16(w[i % copies][0], w[i % copies][1], w[i % copies][2],
                                                               stream=stream), n, w_)
        assert zt_q4.gemm_f16w_errors(gws) == 0 and all(zt_q4.gemm_errors(c, N, K) == 0 for c in ws)
        yg = torch.empty((M, 8192), dtype=torch.float16, device=device)
        gu_ws = torch.empty((256,), dtype=torch.uint8, device=device)
        gu = _timed_calls(stream, lambda i: zt_q4.gemm_f16w_gate_up_silu(ffn[i % copies], x, yg, gu_ws,
                                                                         stream=stream), n, w_)
        assert zt_q4.gemm_f16w_errors(gu_ws) == 0
        flops = 2.0 * M * N * K
        deq_bytes = N * K // 2 + N * (K // 32) * 2 + N * K * 2
        g_tf = flops / gemm / 1e6
        gu_tf = 2.0 * M * 2 * 8192 * K / gu / 1e6
        out.append({"M": M, "us_per_call": round(both, 2), "TFLOPs_dequant_and_gemm": round(flops / both / 1e6, 1),
                    "gemm_us": round(gemm, 2), "gemm_TFLOPs": round(g_tf, 1),
                    "gemm_frac": round(g_tf / tc_peak, 4) if tc_peak else None,
                    "dequant_us": round(deq, 2), "dequant_GBps": round(deq_bytes / deq / 1e3, 1),
                    "dequant_frac": round(deq_bytes / deq / 1e3 / hbm_peak, 4) if hbm_peak else None,
                    "gate_up_silu_us": round(gu, 2), "gate_up_silu_TFLOPs": round(gu_tf, 1),
                    "gate_up_silu_frac": round(gu_tf / tc_peak, 4) if tc_peak else None, "calls": n})
    return out, tc_peak, hbm_peak


def run_prefill(args, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=device)
    rows, tc_peak, hbm_peak = prefill_results(args.seed, device, stream,
                                              [int(v) for v in args.prefill_m.split(",")],
                                              max(min(args.steps, 200), 16), max(args.warmup, 3))
    for r in rows:
        print(json.dumps({
            "metric": "q4 prefill GEMM TFLOP/s (dequant to binary16 + tcgen05 GEMM)",
            "value": r["TFLOPs_dequant_and_gemm"], "unit": "TFLOP/s", "higher_is_better": True,
            "dtype": "f16 x f16 -> f32", **r,
            "roofline": {"bound": "tensor", "achieved": r["gemm_TFLOPs"], "peak": tc_peak, "unit": "TFLOP/s",
                         "frac": r["gemm_frac"], "kernel": "q4_gemm_tc_kernel",
                         "peak_source": "MEASURED_PEAKS.json bf16_tflops (burst; fp16 runs at the bf16 rate)"},
            "dequant_roofline": {"bound": "hbm", "achieved": r["dequant_GBps"], "peak": hbm_peak, "unit": "GB/s",
                                 "frac": r["dequant_frac"]},
            "config": {"workload": f"Phi-3-mini qkv projection 3072->9216 for {r['M']} tokens, q4 group-32, "
                                   "weights dequantized per call; gate_up_silu: 3072 -> 2 x 8192 on cached binary16 "
                                   "weights"}}), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.sweep_m:
            run_sweep_m(args, local)
        elif args.prefill:
            run_prefill(args, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
