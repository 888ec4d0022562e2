#!/usr/bin/env python
"""Throughput of the bidirectional frame-wise delta-rule memory (VDA) on B200.

One step = the whole hot path over one H3-shaped synthetic batch (B=1,
24 heads, 102 latent frames of 1008 tokens, d=128, 512 text tokens, bf16
inputs, fp32 state): text state, frame Grams, per-frame factor, chunk
composition, both scans and the chunk readout, each through its C-ABI entry
point. Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl vdn|reference]

Multi-GPU (torchrun, one rank per GPU): heads are independent, so every rank
runs its own full H3 problem with no collective on the data path (weak
scaling); `value` is all ranks' frames / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "VDA scan+readout frames/s (tokens/s) at H3 shape on 1 B200; % of roofline"
FALLBACK_HBM_GBS = 6650.0
# FP32 FMA peak: 148 SMs x 128 lanes x 2 flop x 1.965 GHz (max SM clock).
ALU_F32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# DRAM bytes of one launch (dram__bytes_read.sum + dram__bytes_write.sum) at
# the H3 shape, keyed by stage, with the sha256 prefix of the kernel source
# the counters were taken on; reported as None as soon as that source changes.
# Each was captured on one kernel of a 4-head case (408 frames) and scaled by
# the frames a full launch processes (x6): the traffic of these kernels grows
# in proportion to the frames they stream.
NCU_TRAFFIC = {
    "frame_grams": {"bytes": 6 * (212.71e6 + 21.12e6), "source": "frame_wise_delta_b200/csrc/gram_tc.cu",
                    "sha256_16": "73b57c89dc3adf04", "workload": "h3", "capture": "h3 with 4 heads, x6"},
    "chunk_readout": {"bytes": 6 * (118.99e6 + 56.81e6), "source": "frame_wise_delta_b200/csrc/readout_tc.cu",
                      "sha256_16": "a4185e26db062a56", "workload": "h3", "capture": "h3 with 4 heads, x6"},
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["vdn", "reference"], default="vdn")
    ap.add_argument("--workload", default="h3")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (small profiling cases)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the tokens per frame (profiling the chain stages at full head count)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--gated", action="store_true",
                    help="time the pass with the readout epilogue (RMSNorm + sigmoid gate, synthetic gates)")
    ap.add_argument("--groups", type=int, default=1,
                    help="head groups of vdn_forward_pipelined (tensor path); 0 = plain vdn_forward")
    ap.add_argument("--bridge", action="store_true",
                    help="read through the decay bridge (the window's decay carried onto both states)")
    ap.add_argument("--shard", choices=["none", "heads"], default="none",
                    help="heads: the ranks split one problem's (b, h) pairs (strong scaling) instead of each "
                         "running a whole problem (weak scaling)")
    ap.add_argument("--stream", type=int, default=0,
                    help="time the causal streaming call instead: the clip as a live stream in segments of "
                         "this many frames (a multiple of the chunk; >= T for one segment)")
    return ap.parse_args()


def event_ms(a, b) -> float:
    """Elapsed ms between two recorded CUDA events (recorded by the library on
    the launching stream), read through the driver API."""
    import ctypes

    global _CU
    if "_CU" not in globals():
        _CU = ctypes.CDLL("libcuda.so.1")
        _CU.cuEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p, ctypes.c_void_p]
    out = ctypes.c_float()
    r = _CU.cuEventElapsedTime(ctypes.byref(out), ctypes.c_void_p(a.cuda_event), ctypes.c_void_p(b.cuda_event))
    if r != 0:
        raise RuntimeError(f"cuEventElapsedTime failed ({r})")
    return float(out.value)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return FALLBACK_HBM_GBS, 1590.0, "fallback"


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 50 ms while the timed loop runs. Samples carry
    their host timestamps; the summary keeps those taken between mark_start()
    and mark_end() (the timed region), or the nearest one when the region is
    shorter than the sampling period."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 50

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms",
                 str(self.PERIOD_MS), "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    @staticmethod
    def _stamp(s):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(s.strip(), fmt).timestamp()
            except ValueError:
                continue
        return None

    def summary(self):
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append((self._stamp(parts[0]), float(parts[2]), float(parts[3]),
                             {n for n, v in zip(names, parts[6:10]) if v.lower().startswith("active")}))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        in_window = rows
        if self.t0 is not None and self.t1 is not None and all(r[0] is not None for r in rows):
            in_window = [r for r in rows if self.t0 <= r[0] <= self.t1]
            if not in_window:  # a region shorter than the period: the sample nearest its middle
                mid = 0.5 * (self.t0 + self.t1)
                in_window = [min(rows, key=lambda r: abs(r[0] - mid))]
        reasons = set().union(*(r[3] for r in in_window))
        return {"sm_mhz": statistics.median(r[1] for r in in_window), "sm_max_mhz": max(r[2] for r in in_window),
                "reasons": sorted(reasons), "samples": len(in_window), "period_ms": self.PERIOD_MS,
                "window_s": None if self.t0 is None or self.t1 is None else round(self.t1 - self.t0, 4)}


# ------------------------------------------------------------- oracle arm
def oracle_sample(w, full, seconds: float):
    """Run the fp64 oracle head by head until `seconds` have passed."""
    import oracle
    import threadpoolctl

    info = threadpoolctl.threadpool_info()
    cores = max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    t0 = time.perf_counter()
    heads = 0
    for b in range(w.B):
        for h in range(w.H):
            oracle.vda_head({k: full[k][b, h] for k in full}, w.chunk, w.anchors)
            heads += 1
            if time.perf_counter() - t0 >= seconds:
                break
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    frames = w.B * w.T * heads / (w.B * w.H)
    return {"value": frames / dt, "unit": "frames/s", "cores": cores, "kind": "oracle",
            "sample": f"{heads} of {w.B * w.H} (b,h) pairs of {w.name}, all {w.T} frames x {w.U} tokens each; "
                      f"{dt:.1f} s fp64 numpy",
            "tokens_per_s": frames * w.U / dt}


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from frame_wise_delta_b200 import synth

    import oracle

    # One (b,h) pair per step: a bounded sample of the same workload. The
    # pairs' inputs are drawn before the warm-up, so the timed steps run the
    # oracle and nothing else; every pair is a whole problem of the same size,
    # so a few distinct pairs in turn stand for all of them.
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)][:4]
    inputs = [synth.generate_head(w, b, h) for b, h in pairs]

    def step(i):
        oracle.vda_head(inputs[i % len(inputs)], w.chunk, w.anchors)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    frames = w.T * args.steps / w.H  # each step: one of H heads of one batch item
    import threadpoolctl

    cores = max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()
                 if i.get("user_api") == "blas"] or [1])
    value = frames / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "frames/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "frames/s", "cores": cores, "kind": "oracle",
                         "sample": f"one (b,h) pair of {w.name} per step (all {w.T} frames), {len(pairs)} "
                                   f"distinct pairs in turn, inputs drawn before the timed steps"},
        "e2e": {"value": value, "unit": "frames/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, gated=False, shard="none", world=1):
    gates = "per-token write gates" if w.beta_per_token else "per-frame write gates"
    if gated:
        gates += ", gated RMSNorm readout epilogue"
    if getattr(w, "decay_bridge", False):
        gates += ", decay-bridge readout"
    return {"workload": f"{w.name}: B={w.B} H={w.H} T={w.T} U={w.U} d_k=d_v={w.d} n_text={w.n_text} "
                        f"chunk={w.chunk} anchors={w.anchors} {w.dtype} inputs, fp32 state, {gates}",
            "global_batch": w.B, "frames": w.B * w.T, "tokens": w.B * w.T * w.U,
            "l2": "inputs larger than L2 (Q+K+V bf16 = %.2f GB > 126 MB)" % (3 * w.B * w.H * w.T * w.U * w.d * 2 / 1e9),
            "parallelism": (f"one problem's (b,h) pairs split over {world} ranks, no data-path collective"
                            if shard == "heads" else "heads independent; one full problem per rank")}


# ---------------------------------------------------------- the CUDA arm
def main():
    args = parse()
    from frame_wise_delta_b200 import synth

    w = synth.WORKLOADS[args.workload]
    import dataclasses
    if args.heads:
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_h{args.heads}")
    if args.tokens:
        w = dataclasses.replace(w, U=args.tokens, name=f"{w.name}_u{args.tokens}")
    if args.bridge:
        w = dataclasses.replace(w, decay_bridge=True, name=f"{w.name}_bridge")
    if args.impl == "reference":
        return run_reference(args, w)

    import numpy as np
    import torch
    import torch.distributed as dist

    from frame_wise_delta_b200 import build, vdn
    from frame_wise_delta_b200 import dist as vdist

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", torch.cuda.current_device())

    def barrier():
        if world > 1:
            dist.barrier()

    # --shard heads: this rank's contiguous share of one problem's (b, h)
    # pairs, laid out as one batch of that many heads (strong scaling);
    # otherwise a whole problem per rank (weak scaling)
    whole = w
    if args.shard == "heads":
        import dataclasses
        pairs = vdist.shard_pairs(w.B, w.H, rank, world)
        w = dataclasses.replace(w, B=1, H=len(pairs), name=f"{w.name}_pairs{len(pairs)}")
        full = synth.generate_pairs(whole, pairs)
    else:
        full = synth.generate_all(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    host = {}
    for k in ("Q", "K", "V", "Kx", "Vx"):
        host[k] = torch.from_numpy(full[k]).to(dt).pin_memory()
    for k in ("beta", "alpha", "beta_x"):
        host[k] = torch.from_numpy(np.ascontiguousarray(full[k])).pin_memory()
    if args.gated:
        # gate logits ~ N(0, 4) in the input dtype, RMSNorm weights ~ U(0.5, 1.5)
        grng = np.random.default_rng(w.seed + 1000 + rank)
        host["gate"] = torch.from_numpy(
            (2.0 * grng.standard_normal((w.B, w.H, w.T, w.U, w.d), dtype=np.float32))).to(dt).pin_memory()
        host["norm_w"] = torch.from_numpy(grng.uniform(0.5, 1.5, (w.H, w.d)).astype(np.float32)).pin_memory()
    d = {k: v.to(dev) for k, v in host.items()}
    og = vdn.out_gate(d["gate"], d["norm_w"], 1e-6) if args.gated else None
    s = vdn.shape_for(w)
    B, H, T, U, D, C = w.B, w.H, w.T, w.U, w.d, w.C
    f32 = dict(dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    if args.stream:
        return stream_bench(args, w, s, d, dev, stream, barrier, rank, world, local)

    stages = ["text_state", "frame_grams", "frame_factor", "chunk_compose", "scan_bidir", "chunk_readout"]
    tensor_path = w.dtype == "bf16" and D == 128
    G = min(args.groups, B * H) if tensor_path else 0

    def make_forward(keep_states=True):
        if G:
            return vdn.PipelinedForward(s, groups=G, device=dev, keep_states=keep_states)
        return vdn.Forward(s, device=dev, keep_states=keep_states)

    fwd_dev = make_forward()
    # our kernels per step: text (gram, invert, injection chain) + gram +
    # invert + compose (M and J chains) + scan + readout, per head group
    # tensor path: text (3) + Grams per group (they also sweep P) + inverse, compose, scan, readout
    launches_per_step = (7 + max(G, 1)) if tensor_path else 7
    n_ev = 8 + G if G else 7

    def step(ev=None):
        if G:
            fwd_dev.events = ev if ev is not None else warm_ev
        fwd_dev(d["Q"], d["K"], d["V"], d["beta"], d["alpha"], d["Kx"], d["Vx"], d["beta_x"],
                events=None if G else ev, og=og)
    warm_ev = fwd_dev.events if G else None
    info = fwd_dev.info

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert int(info.item()) == 0, f"device status {int(info.item())}"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for e in evs:  # torch creates the CUDA event on its first record
        for x in e:
            x.record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                      else local) as clk:
        clk.mark_start()
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
        clk.mark_end()
    barrier()
    assert int(info.item()) == 0, f"device status {int(info.item())}"
    first, last = 0, n_ev - 1
    step_ms = [event_ms(e[first], e[last]) for e in evs]
    if G:
        stage_ms = {name: statistics.mean(pipelined_stage_ms(e, G)[name] for e in evs) for name in stages}
    else:
        stage_ms = {name: statistics.mean(event_ms(e[j], e[j + 1]) for e in evs)
                    for j, name in enumerate(stages)}
    total_ms = event_ms(evs[0][first], evs[-1][last])
    total_ms = vdist.max_over_ranks(total_ms)  # the slowest rank's device time
    ms_per_step = total_ms / args.steps
    # whole-job frames: every rank's own problem, or the one sharded problem
    frames_all = whole.B * whole.T if args.shard == "heads" else world * B * T
    value = frames_all / (ms_per_step / 1e3)

    # ---- end to end: pinned host inputs -> device -> vdn_forward -> O to host
    e2e = (e2e_measure(args, host, d, make_forward, stream, barrier, world, frames_all, dt, og)
           if not args.no_e2e else None)

    if rank == 0:
        hbm_gbs, bf16_tflops, peak_src = load_peaks()
        roof = roofline(w, stage_ms, hbm_gbs, peak_src, bf16_tflops)
        line = {
            "metric": METRIC, "value": value, "unit": "frames/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None, "dtype": "bf16",
            "state_dtype": "f32", "data": "synthetic",
            "config": workload_config(whole, args.gated, shard=args.shard, world=world),
            "tokens_per_s": value * U,
            "hbm_frac_whole_pass": alg_bytes(w, args.gated) / (ms_per_step / 1e3) / (hbm_gbs * 1e9),
            "roofline_whole_pass": whole_pass_roofline(w, ms_per_step, world, hbm_gbs, peak_src, args.gated),
            "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "step_ms_min_max": [min(step_ms), max(step_ms)],
            "step_ms_median": statistics.median(step_ms),
            "step_ms_p90": sorted(step_ms)[int(0.9 * (len(step_ms) - 1))],
            "roofline": roof,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "head_groups": G,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_sample(w, full, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def pipelined_stage_ms(e, G):
    """Per-stage device time of one vdn_forward_pipelined step from its 8 + G
    events, each stage timed on its own stream. The text state runs on the
    auxiliary stream beside the Grams."""
    t = 3 + G
    return {"text_state": event_ms(e[1], e[2]), "frame_grams": event_ms(e[0], e[3 + G - 1]),
            "frame_factor": event_ms(e[t], e[t + 1]), "chunk_compose": event_ms(e[t + 1], e[t + 2]),
            "scan_bidir": event_ms(e[t + 2], e[t + 3]), "chunk_readout": event_ms(e[t + 3], e[t + 4])}


def e2e_measure(args, host, d, make_forward, stream, barrier, world, frames_all, dt, og=None):
    """Same metric through vdn_forward_pipelined with every step's inputs copied
    from pinned host memory and its O copied back, inside the timed region.
    Two sets of device buffers and two copy streams let step i + 1's upload
    and step i - 1's download run while step i computes (PCIe carries both
    directions at once); every step still moves all of its own bytes."""
    import torch

    from frame_wise_delta_b200 import dist as vdist
    from frame_wise_delta_b200 import vdn

    dev = stream.device
    fw = [make_forward(keep_states=False) for _ in range(2)]
    din = [d, {k: torch.empty_like(v) for k, v in d.items()}]
    # the readout epilogue's gate logits and weights travel with each buffer set
    ogs = [og, None if og is None else vdn.out_gate(din[1]["gate"], din[1]["norm_w"], og.eps)]
    O_host = [torch.empty(fw[0].O.shape, dtype=dt).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = O_host[0].numel() * O_host[0].element_size()
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("uploaded", "computed", "downloaded")}
    for evs in ev.values():  # created and recorded once, so that every wait below has an event
        for e in evs:
            e.record(stream)

    def e2e_step(i):
        b = i & 1
        up.wait_event(ev["computed"][b])  # step i - 2 has read buffer b
        with torch.cuda.stream(up):
            for k in host:
                din[b][k].copy_(host[k], non_blocking=True)
        ev["uploaded"][b].record(up)
        stream.wait_event(ev["uploaded"][b])
        stream.wait_event(ev["downloaded"][b])  # step i - 2's O has left buffer b
        x = din[b]
        fw[b](x["Q"], x["K"], x["V"], x["beta"], x["alpha"], x["Kx"], x["Vx"], x["beta_x"], og=ogs[b])
        ev["computed"][b].record(stream)
        down.wait_event(ev["computed"][b])
        with torch.cuda.stream(down):
            O_host[b].copy_(fw[b].O, non_blocking=True)
        ev["downloaded"][b].record(down)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e2e_steps = max(4, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    up.wait_stream(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    te = vdist.max_over_ranks(e0.elapsed_time(e1))
    assert int(fw[0].info.item()) == 0 and int(fw[1].info.item()) == 0
    return {"value": frames_all / (te / e2e_steps / 1e3), "unit": "frames/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
            "overlap": "two device buffer sets; uploads and downloads on their own streams beside the compute"}


def stream_bench(args, w, s, d, dev, stream, barrier, rank, world, local):
    """The clip as a live stream through vdn_stream_segment: each step computes
    the text state, then runs the segments in order, carrying the two forward
    states between them (the states' copies are torch copies, not counted as
    our launches). Each segment's inputs sit in their own buffers, as a
    stream delivers them."""
    import torch

    from frame_wise_delta_b200 import dist as vdist
    from frame_wise_delta_b200 import vdn

    seg = min(args.stream, w.T)
    if seg < w.T and seg % w.chunk:
        raise SystemExit(f"--stream {seg}: segments must hold whole chunks of {w.chunk} frames")
    cuts = [(t0, min(seg, w.T - t0)) for t0 in range(0, w.T, seg)]
    bridged = bool(getattr(w, "decay_bridge", False))
    shapes = {T: vdn.make_shape(w.B, w.H, T, w.U, w.d, w.n_text, w.chunk, w.anchors, w.dtype,
                                beta_per_token=w.beta_per_token, decay_bridge=bridged) for _, T in cuts}
    ws = vdn.workspace(max(vdn.vdn_stream_workspace_bytes(x) for x in shapes.values()), dev)
    tws = vdn.workspace(vdn.vdn_text_state_workspace_bytes(s), dev)
    info = torch.zeros(1, dtype=torch.int32, device=dev)
    parts = [{k: d[k][:, :, t0:t0 + T].contiguous() for k in ("Q", "K", "V", "beta", "alpha")} for t0, T in cuts]
    outs = [(torch.empty((w.B, w.H, T, w.U, w.d), dtype=d["Q"].dtype, device=dev),
             torch.empty((w.B, w.H, shapes[T].C + 1, w.d, w.d), dtype=torch.float32, device=dev)) for _, T in cuts]
    S_T, S_prev, S_in = (torch.empty((w.B, w.H, w.d, w.d), dtype=torch.float32, device=dev) for _ in range(3))
    # with the decay bridge: each segment's last-chunk decay product, carried
    tails = [torch.empty((w.B, w.H, w.d), dtype=torch.float32, device=dev) for _ in range(2)]

    def step():
        vdn.vdn_text_state(s, d["Kx"], d["Vx"], d["beta_x"], S_T, tws, info)
        sp, si, ap = S_T, S_T, None
        for i, ((t0, T), x, (O, F)) in enumerate(zip(cuts, parts, outs)):
            if bridged:
                vdn.vdn_stream_segment_bridged(shapes[T], x["Q"], x["K"], x["V"], x["beta"], x["alpha"], t0, sp, si,
                                               ap, O, F, tails[i & 1], ws, info)
                ap = tails[i & 1]
            else:
                vdn.vdn_stream_segment(shapes[T], x["Q"], x["K"], x["V"], x["beta"], x["alpha"], t0, sp, si, O, F,
                                       ws, info)
            C = shapes[T].C
            S_prev.copy_(F[:, :, C - 1])
            S_in.copy_(F[:, :, C])
            sp, si = S_prev, S_in

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert int(info.item()) == 0, f"device status {int(info.item())}"
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local) as clk:
        clk.mark_start()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    barrier()
    assert int(info.item()) == 0, f"device status {int(info.item())}"
    ms_per_step = vdist.max_over_ranks(e0.elapsed_time(e1)) / args.steps
    value = vdist.throughput(w.B * w.T, world, ms_per_step / 1e3)
    tensor_path = w.dtype == "bf16" and w.d == 128
    if rank == 0:
        hbm_gbs, _, peak_src = load_peaks()
        frac = alg_bytes(w) * world / (ms_per_step / 1e3) / (hbm_gbs * 1e9)
        cfg = workload_config(w)
        cfg["workload"] += f", causal stream in segments of {seg} frames"
        print(json.dumps({
            "metric": "stream frames/s", "value": value, "unit": "frames/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "state_dtype": "f32", "data": "synthetic", "config": cfg, "segments": len(cuts),
            "roofline": {"kernel": "whole stream step", "bound": "hbm", "achieved": frac * hbm_gbs,
                         "peak": hbm_gbs, "unit": "GB/s", "frac": frac, "traffic": None,
                         "peak_source": f"{peak_src} HBM copy bandwidth"},
            "gpu_launches": ((3 if tensor_path else 2) + (6 if bridged else 5) * len(cuts)) * args.steps,
            "clocks": clk.summary()}), flush=True)
    if world > 1:
        dist_destroy()


def dist_destroy():
    import torch.distributed as dist
    dist.barrier()
    dist.destroy_process_group()


def alg_bytes(w, gated=False):
    """Algorithmic HBM bytes of the whole pass: Q, K, V read, O written (bf16),
    text keys/values read, gates read (write gates per frame or per token)."""
    e = 2 if w.dtype == "bf16" else 4
    qkvo = 4 * w.B * w.H * w.T * w.U * w.d * e
    text = 2 * w.B * w.H * w.n_text * w.d * e
    tb = getattr(w, "beta_per_token", False)
    gates = w.B * w.H * (w.T * (w.d + (w.U if tb else 1)) + (w.n_text if tb else 1)) * 4
    if gated:  # gate logits read once (input dtype) + RMSNorm weights
        gates += w.B * w.H * w.T * w.U * w.d * e + w.H * w.d * 4
    return qkvo + text + gates


def stage_work(w):
    """Algorithmic work of one launch of each stage, with its bound:
    frame_grams: reads K and V (2 U d input elements per frame, plus U gates
      per frame with per-token write gates);
    chunk_readout: reads Q and writes O (2 U d elements per frame);
    frame_factor: on the tensor path the CUDA cores sweep two 64 x 64 blocks per
      non-anchor frame (d^3 / 4 flop; the block products run on the tensor
      cores), 4 d^3 on the CUDA-core path (Gauss-Jordan on [I+A; B]);
    chunk_compose: 4 d^3 flop per frame step (M and J chains), per direction;
    scan_bidir: 2 d^3 flop per chunk and direction."""
    B, H, T, U, d, C = w.B, w.H, w.T, w.U, w.d, w.C
    BH = B * H
    e = 2 if w.dtype == "bf16" else 4
    tensor_path = w.dtype == "bf16" and d == 128
    frames = BH * T
    live = BH * (T - (2 if w.anchors and T > 1 else (1 if w.anchors else 0)))
    steps = 0
    for c in range(C):
        fr = [t for t in range(5 * c, min(5 * c + 5, T)) if not (w.anchors and t in (0, T - 1))]
        steps += len(fr) if tensor_path else max(0, len(range(5 * c, min(5 * c + 5, T))) - 1)
    return {
        "frame_grams": ("hbm", frames * (2 * U * d * e + (U * 4 if w.beta_per_token else 0))),
        "chunk_readout": ("hbm", frames * 2 * U * d * e),
        "frame_factor": ("alu", live * (d ** 3 // 4 if tensor_path else 4 * d ** 3)),
        "chunk_compose": ("tensor" if tensor_path else "alu", BH * 2 * steps * 4 * d ** 3),
        "scan_bidir": ("tensor" if tensor_path else "alu", BH * 2 * C * 2 * d ** 3),
    }


def intermediate_bytes(w):
    """HBM bytes a streaming stage moves beyond its algorithmic operands, per
    launch: the Gram kernel writes B_t and (tensor path) the 64 x 64 block R
    of A_t plus what its sweep pairs form for the block inverse (P^{-1} and
    X^T, 64 x 64 fp32 each, and the 36 x 64 values of S); both A_t halves on
    the CUDA-core path; the readout reads two fp32 states per chunk."""
    BH, T, d, C = w.B * w.H, w.T, w.d, w.C
    tensor_path = w.dtype == "bf16" and d == 128
    gram = (d * d * 4 + 3 * 64 * 64 * 4 + 36 * 64 * 4) if tensor_path else 2 * d * d * 4
    return {"frame_grams": BH * T * gram, "chunk_readout": BH * C * 2 * d * d * 4}


def roofline(w, stage_ms, hbm_gbs, peak_src, bf16_tflops=1607.7):
    """Roofline of the stage with the largest event time: its algorithmic
    work per launch (stage_work) over its mean launch time, against the
    measured peak of its bound. Bytes the kernel moves beyond that work
    (intermediate_bytes) and its ncu DRAM traffic are reported beside it,
    with traffic / algorithmic bytes; neither enters `achieved`."""
    units = stage_work(w)
    name = max((k for k in units), key=lambda k: stage_ms.get(k, 0.0))
    bound, amount = units[name]
    sec = stage_ms[name] / 1e3
    if bound == "hbm":
        achieved = amount / sec / 1e9
        peak, unit = hbm_gbs, "GB/s"
        src = f"{peak_src} HBM copy bandwidth"
    elif bound == "tensor":
        achieved = amount / sec / 1e12
        peak, unit = bf16_tflops, "TFLOP/s"
        src = f"{peak_src} dense bf16 (burst); fp32 products issued as 3 bf16 MMAs"
    else:
        achieved = amount / sec / 1e12
        peak, unit = ALU_F32_TFLOPS, "TFLOP/s"
        src = "FP32 FMA: 148 SMs x 128 lanes x 2 flop x 1.965 GHz"
    tr = None
    rec = NCU_TRAFFIC.get(name)
    if rec and rec["workload"] == w.name:
        import hashlib
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] == rec["sha256_16"]:
                tr = rec["bytes"]
    out = {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
           "frac": achieved / peak, "traffic": tr, "peak_source": src,
           "per_stage_ms": {k: round(v, 4) for k, v in stage_ms.items()}}
    if bound == "hbm":
        out["algorithmic_bytes"] = amount
        out["intermediate_bytes"] = intermediate_bytes(w).get(name, 0)
        out["traffic_over_algorithmic"] = None if tr is None else tr / amount
    return out


def whole_pass_roofline(w, ms_per_step, world, hbm_gbs, peak_src, gated=False):
    """The whole pass against HBM bandwidth, per GPU: the algorithmic bytes of
    one rank's work (Q, K, V read, O written, gates and text) over the step
    time, against one GPU's peak; job_bytes is all ranks' bytes."""
    achieved = alg_bytes(w, gated) / (ms_per_step / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s", "frac": achieved / hbm_gbs,
            "algorithmic_bytes": alg_bytes(w, gated), "job_bytes": alg_bytes(w, gated) * world,
            "peak_source": f"{peak_src} HBM copy bandwidth, per GPU"}


if __name__ == "__main__":
    main()
