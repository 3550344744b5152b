#!/usr/bin/env python
"""Throughput of the B200 sparse MoE feed-forward layer (forward pass).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One JSON line on rank 0.  A *step* is one pass of the whole layer (routing,
dispatch, both expert GEMMs, combine) over one batch of every layer of the
workload.  The default workload is the largest configuration: the
fine-grained layer with d = 7168, 256 routed experts of d_ff = 2048, top-8
softmax routing and one always-on shared expert of d_ff = 2048, T = 8192
tokens ("MoE" (theaiera.top) sec. 10.5, the "1 shared + 8 of 256" remark);
22.6 GB of bf16 weights, far more than the 126 MB L2, so every step streams
its weights from HBM.  ``--workload sweep`` runs the fixed-total-parameter
granularity sweep of the "万亿 MoE 只激活 4.9%" page instead (T = 512, d = 512,
E * d_ff = 32768, six layers), and the other names the Mixtral-shaped prefill
and decode layers and the small layer.

Metric: MoE-layer tokens/s (tokens x layers per second) and active TFLOP/s.
Timing: K steps captured in one CUDA graph, bracketed by a barrier and device
synchronisation, max over ranks; a second pass of the same K steps, captured
with CUDA events at every kernel boundary, gives each kernel's duration; a
third pass replays a one-step graph K times between events for the median
step time.
Multi-GPU is weak scaling: every rank runs the same workload on its own seeded
batch with its own weights (data parallel replicas, no collective on the data
path).  ``--impl reference`` times the fp64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_histogram_b200 import accounting as acc  # noqa: E402
from sparse_mixture_experts_histogram_b200 import synth  # noqa: E402

METRIC = "MoE-layer tokens/s & active TFLOP/s, % of bf16 tensor / HBM roofline"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


# ----------------------------------------------------------------------------- workloads
def workload(name: str) -> list:
    if name == "sweep":
        return synth.sweep()
    if name == "small":
        return [synth.small()]
    if name.startswith("mixtral_prefill_T"):
        rest = name[len("mixtral_prefill_T"):]
        skew = rest.endswith("_skewed")
        return [synth.mixtral_prefill(int(rest.replace("_skewed", "")), skew)]
    if name.startswith("mixtral_decode_T") and name.endswith("_fp8"):
        wl = synth.mixtral_decode(int(name[len("mixtral_decode_T"):-len("_fp8")]))
        return [dataclasses.replace(wl, name=wl.name + "_fp8", extra={"fp8": True})]
    if name.startswith("mixtral_decode_T"):
        return [synth.mixtral_decode(int(name[len("mixtral_decode_T"):]))]
    if name.startswith("fine_grained_T"):
        rest = name[len("fine_grained_T"):]
        if "_E" in rest:
            T, E = rest.split("_E")
            return [synth.fine_grained(int(T), int(E))]
        return [synth.fine_grained(int(rest))]
    raise SystemExit(f"unknown workload {name}")


def is_fp8(wl) -> bool:
    return bool(wl.extra.get("fp8"))


def make_inputs(wl, seed, device):
    """The workload's seeded inputs: bf16 experts, or e4m3 experts with row
    scales for the FP8 workloads."""
    if is_fp8(wl):
        return synth.make_fp8_experts(wl, seed=seed, device=device)
    return synth.make_inputs(wl, seed=seed, device=device)


def describe(wls, name):
    return {
        "workload": ("granularity_sweep_T512_d512_Edff32768" if name == "sweep" else name),
        "layers": [{"T": w.T, "d": w.d, "E": w.E, "d_ff": w.d_ff, "k": w.k,
                    **({"d_ff_shared": w.d_ff_shared} if w.d_ff_shared else {}),
                    **({"router_bias": f"+{synth.SKEW_BIAS} on expert {synth.SKEW_EXPERT}"}
                       if w.skew else {}),
                    **({"experts": "e4m3 codes with fp32 row scales, bf16 router"}
                       if is_fp8(w) else {})} for w in wls],
        "global_batch_tokens": sum(w.T for w in wls),
    }


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in a thread."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.samples = []
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", uuid], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                self.samples.append((time.time(), parts))

    def mark(self):
        return time.time()

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=2)
        except Exception:
            self.proc.kill()
        win = [p for (t, p) in self.samples if t0 - 0.1 <= t <= t1 + 0.1] or \
            [p for (_, p) in self.samples]
        mhz = [float(p[0]) for p in win if p[0].replace(".", "").isdigit()]
        mx = [float(p[1]) for p in win if p[1].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for p in win for i in range(4) if p[3 + i] == "Active"})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(win)}


def clocks_bad(c) -> bool:
    if any(r in BAD_REASONS for r in c.get("reasons", [])):
        return True
    if c.get("sm_mhz") and c.get("sm_max_mhz"):
        if c["sm_mhz"] < 0.6 * c["sm_max_mhz"] and not c["reasons"]:
            return True
    return False


# ----------------------------------------------------------------------------- distributed
def dist_init(nccl: bool):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and nccl:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def dist_max(v: float, world: int) -> float:
    """Max of ``v`` over the ranks (the slowest rank's time)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, tokens_per_step: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank processes ``tokens_per_step`` per step."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- oracle arm
def oracle_host_inputs(wls, inps):
    """Raw bf16 bits (host numpy arrays) of every layer's inputs, copied once
    from wherever the inputs live."""
    from sparse_mixture_experts_histogram_b200.synth import bits
    data = []
    for wl, inp in zip(wls, inps):
        b = None if inp["bias"] is None else inp["bias"].double().cpu().numpy()
        shared = (bits(inp["Ws1"]), bits(inp["Ws3"]), bits(inp["Ws2"])) if wl.d_ff_shared else None
        if is_fp8(wl):
            arrs = [bits(inp["x"]), bits(inp["Wg"])] + [
                inp[n].cpu().numpy() if n.startswith("q") else inp[n].double().cpu().numpy()
                for n in ("q1", "s1", "q3", "s3", "q2", "s2")]
        else:
            arrs = [bits(inp[n]) for n in ("x", "Wg", "W1", "W3", "W2")]
        data.append((wl, arrs, b, shared))
    return data


def oracle_step_fn(data, seed, tokens_per_layer):
    """A bounded sample of one step on the host cores: the oracle's forward
    (routing over all E experts, the k selected experts, the shared expert) of
    ``tokens_per_layer`` seeded tokens of every layer."""
    import oracle
    g = np.random.default_rng(seed)
    toks = [np.sort(g.choice(wl.T, size=min(tokens_per_layer, wl.T), replace=False))
            for (wl, _, _, _) in data]

    def step():
        n = 0
        for (wl, arrs, b, shared), tok in zip(data, toks):
            if is_fp8(wl):
                oracle.forward_fp8(*arrs, wl.k, bias=b, tokens=tok)
            else:
                oracle.forward(*arrs, wl.k, bias=b, tokens=tok, shared=shared)
            n += len(tok)
        return n
    return step


def run_oracle(data, steps, warmup, target_s=2.0, seed=42):
    """Times the oracle: calibrate a per-layer token sample that takes about
    ``target_s`` per step, then run ``warmup`` + ``steps`` steps."""
    import oracle
    oracle.build()
    probe = oracle_step_fn(data, seed, oracle.num_threads())
    t0 = time.perf_counter()
    n = probe()
    dt = max(time.perf_counter() - t0, 1e-6)
    per_tok = dt / n
    tpl = int(max(1, min(max(d[0].T for d in data), target_s / per_tok / len(data))))
    step = oracle_step_fn(data, seed, tpl)
    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    tot = 0
    for _ in range(steps):
        tot += step()
    el = time.perf_counter() - t0
    return {"value": tot / el, "tokens_per_layer": tpl, "seconds": el, "steps": steps,
            "cores": oracle.num_threads()}


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    wls = workload(args.workload)
    # Inputs are drawn where the GPU arm draws them (the same bits); the
    # oracle itself only ever runs on the host cores.
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inps = [make_inputs(wl, seed=42 + i, device=dev) for i, wl in enumerate(wls)]
    data = oracle_host_inputs(wls, inps)
    del inps
    r = run_oracle(data, args.steps, args.warmup, target_s=args.oracle_step_s)
    sample = (f"{r['tokens_per_layer']} seeded tokens of each of the {len(wls)} layer(s) per step "
              f"(fp64 oracle, all routing and expert work of those tokens)")
    line = {
        "impl": "reference", "metric": METRIC, "value": r["value"], "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * r["seconds"] / r["steps"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": describe(wls, args.workload),
        "cpu_baseline": {"value": r["value"], "unit": UNIT, "cores": r["cores"], "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": r["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def traffic_record(kernel_key):
    """DRAM traffic per launch of the dominant kernel from a committed ncu
    capture, if the kernel sources have not changed since."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    r = rec.get(kernel_key)
    if not r:
        return None
    h = hashlib.sha256()
    for src in r.get("sources", []):
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != r.get("sources_sha256"):
        return None
    return r


def profile_arm(args):
    """``--profile``: run every layer of the workload ``--steps`` times through
    the public API (eager launches, nothing timed) and exit -- the program an
    ncu capture wraps."""
    import sparse_mixture_experts_histogram_b200 as moe
    dev = torch.device("cuda", 0)
    wls = workload(args.workload)
    inps = [make_inputs(wl, seed=42 + i, device=dev) for i, wl in enumerate(wls)]
    outs = [torch.empty(wl.T, wl.d, dtype=torch.float32, device=dev) for wl in wls]
    ws = torch.empty(max(moe.moe_workspace_size_ex(w.T, w.d, w.E, w.d_ff, w.k, w.d_ff_shared)
                         for w in wls), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)
    for _ in range(args.steps):
        for wl, inp, out in zip(wls, inps, outs):
            if is_fp8(wl):
                moe.moe_forward_fp8(wl.T, wl.d, wl.E, wl.d_ff, wl.k, inp["x"], inp["Wg"],
                                    inp["bias"], inp["q1"], inp["s1"], inp["q3"], inp["s3"],
                                    inp["q2"], inp["s2"], out, ws)
            else:
                moe.moe_forward_ex(wl.T, wl.d, wl.E, wl.d_ff, wl.k, inp["x"], inp["Wg"],
                                   inp["bias"], inp["W1"], inp["W3"], inp["W2"], wl.d_ff_shared,
                                   inp.get("Ws1"), inp.get("Ws3"), inp.get("Ws2"), out, ws)
    st, code = moe.moe_get_device_error(ws)
    print(json.dumps({"profile_run": args.workload, "launch_rounds": args.steps,
                      "status": st, "error_word": code}))
    return 0 if st == 0 else 1


def gpu_arm(args):
    import sparse_mixture_experts_histogram_b200 as moe
    rank, world, local = dist_init(nccl=True)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wls = workload(args.workload)
    seed = synth.rank_seed(42, rank)
    moe.load_library()

    # ---- resident inputs and buffers
    inps, outs = [], []
    for i, wl in enumerate(wls):
        inps.append(make_inputs(wl, seed=seed + i, device=dev))
        outs.append(torch.empty(wl.T, wl.d, dtype=torch.float32, device=dev))
    ws_bytes = max(moe.moe_workspace_size_ex(w.T, w.d, w.E, w.d_ff, w.k, w.d_ff_shared)
                   for w in wls)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    # The inputs were drawn on the default stream; everything below runs on
    # its own stream, so wait for them first.
    torch.cuda.synchronize(dev)
    stream = torch.cuda.Stream(device=dev)

    # ---- routing pre-pass: experts each batch hits (for the algorithmic bytes)
    hit = []
    with torch.cuda.stream(stream):
        for wl, inp in zip(wls, inps):
            idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device=dev)
            w = torch.empty(wl.T, wl.k, dtype=torch.float32, device=dev)
            cnt = torch.empty(wl.E, dtype=torch.int32, device=dev)
            moe.moe_route(wl.T, wl.d, wl.E, wl.k, inp["x"], inp["Wg"], inp["bias"], idx, w, cnt,
                          ws, stream=stream)
            stream.synchronize()
            hit.append(int((cnt > 0).sum().item()))

    def layer_call(i, events=None, x=None, out=None):
        wl, inp = wls[i], inps[i]
        x = inp["x"] if x is None else x
        out = outs[i] if out is None else out
        if is_fp8(wl):
            a = (wl.T, wl.d, wl.E, wl.d_ff, wl.k, x, inp["Wg"], inp["bias"], inp["q1"],
                 inp["s1"], inp["q3"], inp["s3"], inp["q2"], inp["s2"], out, ws)
            if events is None:
                moe.moe_forward_fp8(*a, stream=stream)
            else:
                moe.moe_forward_fp8_traced(*a, events, stream=stream)
            return
        a = (wl.T, wl.d, wl.E, wl.d_ff, wl.k, x, inp["Wg"], inp["bias"], inp["W1"],
             inp["W3"], inp["W2"], wl.d_ff_shared, inp.get("Ws1"), inp.get("Ws3"),
             inp.get("Ws2"), out, ws)
        if events is None:
            moe.moe_forward_ex(*a, stream=stream)
        else:
            moe.moe_forward_traced(*a, events, stream=stream)

    def make_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        with torch.cuda.stream(stream):
            for e in evs:
                e.record(stream)
        stream.synchronize()
        return evs

    # ---- eager warm-up (loads kernels, sets attributes)
    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup)):
            for i in range(len(wls)):
                layer_call(i)
    stream.synchronize()
    st, code = moe.moe_get_device_error(ws, stream)
    if st != 0:
        raise SystemExit(f"device error word {code:#x} after warm-up")

    # ---- L2: a step whose algorithmic bytes fit in L2 would find its weights
    # there on the next step; such workloads write a buffer of twice the L2
    # size between steps, outside every timed interval.
    bytes_per_step = sum(acc.algorithmic_bytes(w.T, w.d, w.E, w.d_ff, w.k, h, w.d_ff_shared,
                                               fp8=is_fp8(w))
                         for w, h in zip(wls, hit))
    flush = (torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
             if bytes_per_step <= L2_BYTES else None)

    # ---- graphs: one step (warm-up / soak) and K traced steps (timed)
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        for i in range(len(wls)):
            layer_call(i)
    trace = [[make_events(moe.binding.TRACE_EVENTS) for _ in wls] for _ in range(args.steps)]
    gK = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gK, stream=stream):
        for s in range(args.steps):
            if flush is not None:
                flush.zero_()  # before the step's first event: not in any kernel's interval
            for i in range(len(wls)):
                layer_call(i, trace[s][i])
    gK_plain = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gK_plain, stream=stream):
        for s in range(args.steps):
            for i in range(len(wls)):
                layer_call(i)

    def timed(graph_k, soak_s=1.0, per_step=False):
        sampler = ClockSampler(local)
        t_start = time.time()
        with torch.cuda.stream(stream):
            n = 0
            while n < args.warmup or time.time() - t_start < soak_s:
                g1.replay()
                n += 1
                if n % 50 == 0:
                    stream.synchronize()
        stream.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        if per_step:
            # K steps, each between its own events, the L2 flush between them.
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
            with torch.cuda.stream(stream):
                for i in range(args.steps):
                    flush.zero_()
                    evs[2 * i].record(stream)
                    g1.replay()
                    evs[2 * i + 1].record(stream)
            torch.cuda.synchronize()
            tw1 = time.time()
            barrier(world)
            ms = dist_max(sum(evs[2 * i].elapsed_time(evs[2 * i + 1])
                              for i in range(args.steps)), world)
            return ms, sampler.stop(t_start, tw1)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        tw0 = time.time()
        with torch.cuda.stream(stream):
            e0.record(stream)
            graph_k.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        tw1 = time.time()
        barrier(world)
        ms = dist_max(e0.elapsed_time(e1), world)
        return ms, sampler.stop(t_start, tw1)

    # Timed region: K steps of the plain graph.  A second pass of the same K
    # steps with events at every kernel boundary gives each kernel's duration
    # (event nodes add a few microseconds each, so they stay out of the
    # headline number).
    per_step = flush is not None
    ms, clocks = timed(gK_plain, per_step=per_step)
    if clocks_bad(clocks):
        ms, clocks = timed(gK_plain, per_step=per_step)
        clocks["remeasured"] = True
    # The traced graph holds its own flushes between steps (before each
    # step's first event), so its per-kernel intervals stay cold-L2 too.
    ms_traced, _ = timed(gK, soak_s=0.2)

    # Median step: the one-step graph replayed K more times, each replay
    # between its own pair of events (the median over >= 20 replays).
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    torch.cuda.synchronize()
    if flush is None:
        with torch.cuda.stream(stream):
            step_ev[0].record(stream)
            for i in range(args.steps):
                g1.replay()
                step_ev[i + 1].record(stream)
        torch.cuda.synchronize()
        step_ms = [step_ev[i].elapsed_time(step_ev[i + 1]) for i in range(args.steps)]
    else:
        ev2 = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                flush.zero_()
                ev2[2 * i].record(stream)
                g1.replay()
                ev2[2 * i + 1].record(stream)
        torch.cuda.synchronize()
        step_ms = [ev2[2 * i].elapsed_time(ev2[2 * i + 1]) for i in range(args.steps)]
    ms_median = dist_max(statistics.median(step_ms), world)
    st, code = moe.moe_get_device_error(ws, stream)
    if st != 0:
        raise SystemExit(f"device error word {code:#x} after the timed region")

    # ---- per-kernel durations from the trace events of the timed region
    stages = moe.binding.TRACE_STAGES
    dur = {s: [] for s in stages}        # ms per launch
    per_layer_up = [[] for _ in wls]
    per_layer = [{s: [] for s in stages} for _ in wls]
    for s in range(args.steps):
        for i, wl in enumerate(wls):
            ev = trace[s][i]
            for j, name in enumerate(stages):
                t = ev[j].elapsed_time(ev[j + 1])
                if name.startswith("shared") and not wl.d_ff_shared:
                    continue
                if name == "scatter" and wl.d <= 1024:
                    continue  # no scatter launch: the expert kernel gathers x itself
                dur[name].append(t)
                per_layer[i][name].append(t)
                if name == "expert_ffn":
                    per_layer_up[i].append(t)
    kernel_ms = {k: (sum(v) / len(v) if v else None) for k, v in dur.items()}
    kernel_share = {k: (sum(v) / max(1e-12, sum(sum(x) for x in dur.values())))
                    for k, v in dur.items() if v}

    # ---- throughput and roofline
    tokens_per_step = sum(w.T for w in wls)
    flops_per_step = sum(acc.active_flops(w.T, w.d, w.E, w.d_ff, w.k, w.d_ff_shared) for w in wls)
    sec = ms / 1e3
    value = weak_scaling_value(world, tokens_per_step, args.steps, ms)
    pk, pk_src = peaks()
    # dominant kernel: the expert feed-forward (both projections, one launch)
    up_bytes = [acc.ffn_bytes(w.T, w.d, w.d_ff, w.k, h, fp8=is_fp8(w)) for w, h in zip(wls, hit)]
    up_flops = [acc.ffn_flops(w.T, w.d, w.d_ff, w.k) for w in wls]
    up_time = [sum(t) / len(t) for t in per_layer_up]
    ai = sum(up_flops) / sum(up_bytes)
    ridge = pk["bf16_tflops_sustained"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    if ai >= ridge:
        achieved = sum(up_flops) / sum(up_time) / 1e9  # TFLOP/s (ms -> 1e-3)
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "peak_source": f"bf16_tflops_sustained ({pk_src})"}
    else:
        achieved = sum(up_bytes) / sum(up_time) / 1e6  # GB/s
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "peak_source": f"hbm_gbs ({pk_src})"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if roof["bound"] == "tensor":
        roof["frac_of_burst_peak"] = roof["achieved"] / pk["bf16_tflops"]
    # The same against the B200's nominal figures (dense bf16 tensor peak,
    # HBM3e bandwidth), on which the targets are stated.
    spec_peak = SPEC_PEAKS["bf16_tflops"] if roof["bound"] == "tensor" else SPEC_PEAKS["hbm_gbs"]
    roof["spec"] = {"peak": spec_peak, "frac": roof["achieved"] / spec_peak,
                    "source": "B200 nominal: 2.25 PFLOP/s dense bf16, 8 TB/s HBM3e"}
    tr = traffic_record(f"expert_ffn:{args.workload}")
    roof["traffic"] = None if tr is None else tr["bytes_per_launch"]
    kinds = []
    if any(w.d <= 1024 for w in wls):
        kinds.append("ffn_small_kernel (d <= 1024: x rows gathered through the experts' token "
                     "lists, W1|W3 + SwiGLU and W2 per hidden chunk, one persistent launch)")
    for w in wls:
        if w.d <= 1024:
            continue
        # the library's choice: CTA pairs once a segment is expected to hold
        # more than 64 rows (1.5x the mean), one CTA per SM below that
        if is_fp8(w):
            kinds.append("ffn_fp8_kernel (e4m3 weights widened in tensor memory, W1|W3 + "
                         "SwiGLU, then W2, one persistent launch)")
        elif 3 * w.T * w.k > 128 * w.E:
            kinds.append("ffn_pair_kernel (cta_group::2 MMAs on CTA pairs, W1|W3 + SwiGLU, then W2"
                         + (", gate-weighted rows added into out" if w.k <= 2 and not w.d_ff_shared
                            else "") + ", one persistent launch)")
        else:
            kinds.append("ffn_kernel (grouped W1|W3 + SwiGLU, then W2, one persistent launch)")
    roof["kernel"] = "; ".join(dict.fromkeys(kinds))
    roof["algorithmic_bytes_per_launch"] = sum(up_bytes) / len(up_bytes)
    roof["flops_per_launch"] = sum(up_flops) / len(up_flops)
    roof["launch_ms"] = sum(up_time) / len(up_time)
    step_roof = max(flops_per_step / (pk["bf16_tflops_sustained"] * 1e12),
                    bytes_per_step / (pk["hbm_gbs"] * 1e9))
    step_roof_spec = max(flops_per_step / (SPEC_PEAKS["bf16_tflops"] * 1e12),
                         bytes_per_step / (SPEC_PEAKS["hbm_gbs"] * 1e9))

    # ---- end to end through the public API with host buffers
    # Every step copies each layer's x in from pinned host memory and its out
    # back.  Three streams pipeline the layers the way a server would: layer
    # i+1's input copy and layer i-1's output copy run while layer i computes.
    # Two sets of device buffers, alternating by step, so that a step's copies
    # never wait for the previous step's compute of the same layer.
    NB = 2
    xs_host = [inp["x"].cpu().pin_memory() for inp in inps]
    out_host = [[torch.empty(w.T, w.d, dtype=torch.float32).pin_memory() for w in wls]
                for _ in range(NB)]
    x_dev = [[torch.empty_like(inp["x"]) for inp in inps] for _ in range(NB)]
    o_dev = [[torch.empty(w.T, w.d, dtype=torch.float32, device=dev) for w in wls]
             for _ in range(NB)]
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    nl = len(wls)
    ev_in = [[torch.cuda.Event() for _ in range(nl)] for _ in range(NB)]
    ev_cmp = [[torch.cuda.Event() for _ in range(nl)] for _ in range(NB)]
    ev_out = [[torch.cuda.Event() for _ in range(nl)] for _ in range(NB)]
    torch.cuda.synchronize(dev)
    for b in range(NB):  # "earlier step" events for the first steps: already complete
        for i in range(nl):
            ev_cmp[b][i].record(stream)
            ev_out[b][i].record(s_out)

    def e2e_step(b):
        for i in range(nl):
            wl, inp = wls[i], inps[i]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_cmp[b][i])         # the earlier step has read x_dev[b][i]
                x_dev[b][i].copy_(xs_host[i], non_blocking=True)
                ev_in[b][i].record(s_in)
            stream.wait_event(ev_in[b][i])
            stream.wait_event(ev_out[b][i])           # the earlier o_dev[b][i] is copied out
            if flush is not None and i == 0:
                with torch.cuda.stream(stream):
                    flush.zero_()  # inside the end-to-end time: it only makes it longer
            layer_call(i, x=x_dev[b][i], out=o_dev[b][i])
            ev_cmp[b][i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[b][i])
                out_host[b][i].copy_(o_dev[b][i], non_blocking=True)
                ev_out[b][i].record(s_out)

    for it in range(max(3, args.warmup)):
        e2e_step(it % NB)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    stream.wait_event(e0)
    s_out.wait_event(e0)
    for it in range(args.steps):
        e2e_step(it % NB)
    for b in range(NB):
        for ev in ev_out[b]:
            stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = dist_max(e0.elapsed_time(e1), world)
    e2e_value = weak_scaling_value(world, tokens_per_step, args.steps, e2e_ms)
    h2d = sum(w.T * w.d * 2 for w in wls)
    d2h = sum(w.T * w.d * 4 for w in wls)
    ok = all(torch.isfinite(o).all().item() for o in outs)

    # router, [scatter: only layers with d > 1024], expert FFN, [shared FFN], combine
    launches_per_layer = [(3 if w.d <= 1024 else 4) + (1 if w.d_ff_shared else 0) for w in wls]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("fp16 MMA on e4m3 experts (bf16 router)" if any(is_fp8(w) for w in wls)
                  else "bf16"),
        "data": "synthetic",
        "config": {**describe(wls, args.workload), "parallelism": f"dp{world} (replicas)",
                   "l2": ("no flush: the step's working set "
                          f"({bytes_per_step / 1e6:.0f} MB of algorithmic bytes) exceeds the "
                          "126 MB L2" if flush is None else
                          f"flushed: the step's {bytes_per_step / 1e6:.0f} MB fit in the 126 MB "
                          "L2, so a 252 MB buffer is written between steps, outside the timed "
                          "intervals")},
        "active_tflops": world * flops_per_step * args.steps / sec / 1e12,
        "step_roofline_frac": step_roof * args.steps / sec * 1.0,
        "step_roofline_frac_spec": step_roof_spec * args.steps / sec * 1.0,
        "ms_per_step_median": ms_median,
        "median_replays": args.steps,
        "roofline": roof,
        "kernel_ms": kernel_ms,
        "kernel_share": kernel_share,
        "kernel_ms_per_layer": [{k: round(sum(v) / len(v), 5) for k, v in pl.items() if v}
                                for pl in per_layer],
        "ms_per_step_traced": ms_traced / args.steps,
        "experts_hit": hit,
        "gpu_launches": sum(launches_per_layer) * args.steps,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
                "path": "pinned host x -> device copy (copy stream), moe_forward_ex (compute "
                        "stream), device -> pinned host out (second copy stream), eager launches, "
                        "two device buffer sets alternating by step: copies overlap compute"
                        + ("; the L2 flush before each step is inside this time"
                           if flush is not None else "")},
        "clocks": clocks,
        "outputs_finite": ok,
        "cpu_baseline": None,
    }
    del g1, gK, gK_plain
    if world == 1 and not args.no_cpu_baseline:
        r = run_oracle(oracle_host_inputs(wls, inps), steps=2, warmup=0,
                       target_s=args.oracle_step_s)
        line["cpu_baseline"] = {
            "value": r["value"], "unit": UNIT, "cores": r["cores"], "kind": "oracle",
            "sample": (f"{r['tokens_per_layer']} seeded tokens of each of the {len(wls)} layers, "
                       f"2 steps, {r['seconds']:.1f} s on the host cores (fp64 oracle)")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def ep_arm(args):
    """``--ep-emulate R``: the expert-parallel layer (experts split over R
    ranks) with its R ranks emulated on this one GPU: the same kernels and
    buffers as on R GPUs, the ranks one after another on one stream, stream
    order in place of the collectives, every transfer a local store.  Prints
    one JSON line (``"impl": "ep_emulated"``): the group's tokens/s on this
    GPU and, per rank, the device time of its own kernels (route, dispatch,
    its experts, combine with the rank's shared expert), which is what one
    GPU of an R-GPU group spends in kernels; the NVLink transfers and the
    collectives are not in it."""
    import sparse_mixture_experts_histogram_b200 as moe
    from sparse_mixture_experts_histogram_b200 import ep
    wls = workload(args.workload)
    if len(wls) != 1 or is_fp8(wls[0]):
        raise SystemExit("--ep-emulate takes one bf16 layer")
    wl, R = wls[0], args.ep_emulate
    T = wl.T
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    moe.load_library()
    inp = synth.make_inputs(dataclasses.replace(wl, T=R * T), seed=42, device=dev)
    xs = [inp["x"][r * T:(r + 1) * T] for r in range(R)]
    outs = [torch.empty(T, wl.d, dtype=torch.float32, device=dev) for _ in range(R)]
    shared = (inp["Ws1"], inp["Ws3"], inp["Ws2"]) if wl.d_ff_shared else None
    layer = ep.EmulatedExpertParallel(R, T, wl.d, wl.E, wl.d_ff, wl.k, wl.d_ff_shared, device=dev)
    p = layer.plan
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    phases = ("route", "dispatch", "expert_ffn", "combine")

    def step(mark=lambda key: None):
        rx = [b.recv_x for b in layer.ranks]
        ry = [b.recv_y for b in layer.ranks]
        for r in range(R):
            b = layer.ranks[r]
            mark(("route", r))
            ep._route(p, b, xs[r], inp["Wg"], inp["bias"], b.counts)
            layer.counts_all[r].copy_(b.counts)
        for r in range(R):
            mark(("dispatch", r))
            ep._dispatch(p, layer.ranks[r], r, xs[r], layer.counts_all, rx)
        for r in range(R):
            lo, hi = ep.expert_block(wl.E, R, r)
            mark(("expert_ffn", r))
            ep._ffn(p, layer.ranks[r], inp["W1"][lo:hi], inp["W3"][lo:hi], inp["W2"][lo:hi])
        for r in range(R):
            mark(("combine", r))
            sy = ep._shared(p, layer.ranks[r], xs[r], shared)
            ep._combine(p, layer.ranks[r], T, ry, sy, outs[r])
        mark(("end", 0))

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    errs = [moe.moe_get_device_error(b.ws, stream)[1] for b in layer.ranks]
    if any(errs):
        raise SystemExit(f"device error words {errs}")
    rows = [int(b.recv_offsets[-1].item()) for b in layer.ranks]
    hit = [int((b.recv_offsets[1:] > b.recv_offsets[:-1]).sum().item()) for b in layer.ranks]

    # Whole emulated step: K steps in one CUDA graph between events.
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(args.steps):
            step()
    sampler = ClockSampler(0)
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = sampler.mark()
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    stream.synchronize()
    t1 = sampler.mark()
    clocks = sampler.stop(t0, t1)
    ms = e0.elapsed_time(e1) / args.steps

    # Per rank and phase: a one-step graph with an event node at every
    # boundary, replayed K times.
    per = {ph: [[] for _ in range(R)] for ph in phases}
    order = [(ph, r) for ph in phases for r in range(R)] + [("end", 0)]
    ev = {key: torch.cuda.Event(enable_timing=True, external=True) for key in order}
    g_tr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_tr, stream=stream):
        step(lambda key: ev[key].record(stream))
    for _ in range(args.steps):
        with torch.cuda.stream(stream):
            g_tr.replay()
        stream.synchronize()
        for a, b in zip(order, order[1:]):
            per[a[0]][a[1]].append(ev[a].elapsed_time(ev[b]) * 1e3)
    med = {ph: [statistics.median(v) for v in per[ph]] for ph in phases}
    rank_us = [sum(med[ph][r] for ph in phases) for r in range(R)]

    pk, src = peaks()
    ffn = []
    for r in range(R):
        flops = acc.ffn_flops(rows[r], wl.d, wl.d_ff, 1)
        yb = 2 if p.y_bf16 else 4 * p.ksplit  # output bytes per element of a row
        byts = 2 * 3 * hit[r] * wl.d * wl.d_ff + 2 * rows[r] * wl.d + yb * rows[r] * wl.d
        t = med["expert_ffn"][r] * 1e-6
        ridge = pk["bf16_tflops_sustained"] * 1e12 / (pk["hbm_gbs"] * 1e9)
        if byts and flops / byts > ridge:
            a = flops / t / 1e12
            ffn.append({"rows": rows[r], "experts_hit": hit[r], "bound": "tensor",
                        "achieved": a, "unit": "TFLOP/s",
                        "frac": a / pk["bf16_tflops_sustained"]})
        else:
            a = byts / t / 1e9
            ffn.append({"rows": rows[r], "experts_hit": hit[r], "bound": "hbm", "bytes": byts,
                        "achieved": a, "unit": "GB/s", "frac": a / pk["hbm_gbs"]})
    line = {
        "impl": "ep_emulated", "metric": METRIC, "value": R * T / (ms * 1e-3), "unit": UNIT,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload}_ep{R}_emulated", "ep_ranks": R,
                   "tokens_per_rank": T, "layer": describe(wls, args.workload)["layers"][0],
                   "recv_rows_per_rank": p.recv_rows, "down_ksplit": p.ksplit,
                   "output_rows": "bf16" if p.y_bf16 else "fp32",
                   "l2": "weights larger than L2 stream from HBM every step"
                   if 2 * 3 * wl.E * wl.d * wl.d_ff > L2_BYTES else "may be L2-resident"},
        "ep": {"per_rank_us": med, "rank_kernels_us_max": max(rank_us),
               "rank_kernels_us": rank_us, "expert_ffn": ffn, "peaks": src,
               "note": "R ranks emulated on one GPU: per-rank times are this GPU's kernel time "
                       "for that rank's work; NVLink transfers and the three collectives per "
                       "step are not included"},
        "clocks": {k: v for k, v in clocks.items() if k != "samples"},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="fine_grained_T8192",
                    help="fine_grained_T8192 (default: the largest config, 256 experts top-8 "
                         "plus a shared expert), sweep, small, mixtral_prefill_T{2048,8192}"
                         "[_skewed], mixtral_decode_T{1,8,32,128}[_fp8]")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--oracle-step-s", type=float, default=4.0,
                    help="seconds of host work per oracle step (bounded sample)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ep-emulate", type=int, default=0, metavar="R",
                    help="time the expert-parallel layer with R ranks emulated on one GPU")
    ap.add_argument("--profile", action="store_true",
                    help="run the layers --steps times untimed and exit (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return reference_arm(args)
    if args.profile:
        return profile_arm(args)
    if args.ep_emulate:
        return ep_arm(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    return gpu_arm(args)


if __name__ == "__main__":
    sys.exit(main())
