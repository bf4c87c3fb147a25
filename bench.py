#!/usr/bin/env python
"""Throughput of the B200 MoE FFN layer (tokens/s) with its roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
    python bench.py --impl reference ...     # the CPU oracle as the reference arm

One step = one forward of the whole layer (router GEMM, selection, dispatch,
gate/up GEMM + SwiGLU, down GEMM x weight, combine) over one batch of seeded
synthetic tokens, with every input already resident in HBM.  Under torchrun
each rank runs an independent replica (tokens are independent: no collective
on the data path); the timed region is bracketed by a barrier and device
synchronisation, and the max over ranks is reported.  The JSON line also
carries the roofline of the dominant kernel, the oracle's CPU throughput, an
end-to-end figure through the C ABI with host buffers, and SM clocks sampled
during the timed region.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and % roofline (HBM GB/s decode, TFLOP/s prefill), 1×B200"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU work of the oracle sample")
    ap.add_argument("--T", type=int, default=None, help="override the workload's tokens")
    ap.add_argument("--E", type=int, default=None,
                    help="override the routed expert count (small profiling cases)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="report the eager timed region; by default `value` comes from replays "
                         "of one captured CUDA graph of the step (stage times and the roofline "
                         "always come from the eager timed region before it)")
    ap.add_argument("--dsa-unsorted", action="store_true",
                    help="DSA workloads: indices by key order (no sort by score)")
    ap.add_argument("--block", action="store_true",
                    help="time the pre-norm block out = h + MoE(RMSNorm(h)) (moe_forward_block)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="default decode run: skip the prefill and backward objects (T=8192 "
                         "Zipf) in the line")
    ap.add_argument("--backward", action="store_true",
                    help="time the layer's backward pass (moe_backward) on the workload instead "
                         "of the forward")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- distributed

def dist_setup():
    """One process per GPU (RANK/LOCAL_RANK/WORLD_SIZE/MASTER_* from the
    launcher).  NCCL when CUDA is present, gloo otherwise; a short timeout
    so that ranks waiting for one another end with an error."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v: float) -> float:
    """The job's time: the slowest rank's."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region: an NVML
    polling thread (every 0.5 ms), or nvidia-smi at 50 ms where NVML is absent."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.max_mhz = None
        self.proc = None
        self.thread = None
        self.stop = False

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            def poll():
                while not self.stop:
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             int(get_reasons(h))))
                    except Exception:
                        pass
                    time.sleep(0.0005)

            import threading
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.dev), "--query-gpu=clocks.sm,clocks.max.sm,"
                     "clocks_event_reasons.active", "--format=csv,noheader,nounits", "-lms", "50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                time.sleep(0.2)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            for ln in out.splitlines():
                f = [x.strip() for x in ln.split(",")]
                try:
                    self.samples.append((float(f[0]), int(f[2], 16)))
                    self.max_mhz = float(f[1])
                except (ValueError, IndexError):
                    continue

    def summary(self):
        sm = [c for c, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for b, n in self.REASONS.items() if bits & b),
                "samples": len(sm)}


# ---------------------------------------------------------------- ncu traffic

KERNEL_SOURCES = {
    # the kernel's own sources; the shared headers (ptx.cuh: instruction
    # wrappers, kernels.cuh: parameter structs and launch declarations) only
    # gain entries for other kernels, and an edit to an existing entry there
    # calls for new captures of the kernels that use it
    "gate_up_decode": ["csrc/gemm.cu", "csrc/tiles.cuh"],
    "gate_up_prefill": ["csrc/gemm_pair.cu"],
    "gate_up_fp8": ["csrc/gemm_fp8.cu", "csrc/tiles.cuh"],
    "gate_up_fp8_tm": ["csrc/gemm_fp8_tm.cu", "csrc/tiles.cuh"],
    "dsa_scores": ["csrc/dsa_scores.cu", "csrc/dsa_kernels.cuh", "csrc/tiles.cuh"],
}


def source_hash(kind):
    import hashlib
    m = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "sigmoid_top_routing_warp_b200", f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def profile_traffic(kind, algorithmic, workload):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summaries under profiles/, or None when there is none for this kernel or
    the kernel's source changed since the counters were taken."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    ratio = None
    records = []
    for name in sorted(os.listdir(pdir)):
        # machine-read blocks: each starts with a "kernel:" line
        with open(os.path.join(pdir, name)) as f:
            for line in f:
                line = line.strip()
                if ":" in line and line.split(":", 1)[0] in (
                        "kernel", "traffic_over_algorithmic", "traffic_bytes_per_launch",
                        "source_hash", "workload"):
                    k, v = line.split(":", 1)
                    if k == "kernel":
                        records.append({})
                    if records:
                        records[-1][k] = v.strip()
    generic = None
    for fields in records:
        if fields.get("kernel") != kind or fields.get("source_hash") != source_hash(kind):
            continue
        # a capture of this exact workload wins over a ratio scaled from a smaller case
        if "traffic_bytes_per_launch" in fields and fields.get("workload") == workload:
            return float(fields["traffic_bytes_per_launch"])
        if "traffic_over_algorithmic" in fields:
            # a ratio taken for this workload's shape, else one that covers the kernel
            if fields.get("workload") == workload and ratio is None:
                ratio = float(fields["traffic_over_algorithmic"])
            elif "workload" not in fields and generic is None:
                generic = float(fields["traffic_over_algorithmic"])
    ratio = ratio if ratio is not None else generic
    return None if ratio is None or algorithmic is None else ratio * algorithmic


# ---------------------------------------------------------------- work model

def layer_work(wl, touched: int):
    """Algorithmic FLOPs and HBM bytes of one layer call and of the gate/up
    GEMM (the dominant kernel).  fp8 layers stream 1-byte weight codes (plus
    one fp32 scale per 128x128 block) and 1-byte activation codes."""
    T, H, E, k, I, Is = wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is
    el = 1 if wl.dtype == "fp8" else 2
    sc = 4.0 / (128 * 128) if wl.dtype == "fp8" else 0.0   # scale bytes per weight
    flops = T * (2 * k * 3 * H * I + 2 * 3 * H * Is + 2 * H * E)
    wbytes = (touched * 3 * H * I + 3 * H * Is) * (el + sc)
    bytes_ = wbytes + E * H * 2 + 2 * T * H * 2
    g1_flops = 2 * T * k * 2 * I * H + 2 * T * 2 * Is * H
    g1_bytes = ((touched * 2 * I * H + 2 * Is * H) * (el + sc)   # weights streamed
                + (T * k * H + T * H) * el                       # gathered + shared activations
                + (T * k * I + T * Is) * el)                      # SwiGLU outputs
    return {"flops": flops, "bytes": bytes_, "g1_flops": g1_flops, "g1_bytes": g1_bytes}


def layer_config(wl, args, world):
    """The workload's identity, the same in both arms' JSON lines."""
    el = 1 if wl.dtype == "fp8" else 2
    sc = 4.0 / (128 * 128) if wl.dtype == "fp8" else 0.0
    resident = (wl.E * 3 * wl.H * wl.I + 3 * wl.H * wl.Is) * (el + sc)
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I,
            "n_shared": wl.n_shared, "n_group": wl.n_group, "topk_group": wl.topk_group,
            "block": "h + MoE(RMSNorm(h))" if args.block else None,
            "parallelism": "replicas" if world > 1 else "single",
            "l2": "inputs larger than L2: %.1f GB of expert weights resident, each step streams "
                  "those of the experts it touches" % (resident / 1e9)}


def dsa_config(wl, args):
    return {"workload": wl.name, "Sq": wl.Sq, "Sk": wl.Sk, "n_heads": wl.n_heads,
            "head_dim": 128, "topk": wl.topk, "causal": wl.causal,
            "sorted": not args.dsa_unsorted, "q_offset": wl.q_offset,
            "l2": "inputs larger than L2: %.0f MB of keys and %.0f MB of scores per step"
                  % (wl.Sk * wl.n_heads * 256 / 1e6, wl.Sq * wl.Sk * 4 / 1e6)}


# ---------------------------------------------------------------- our arm

def workload_of(args):
    from dataclasses import replace
    from sigmoid_top_routing_warp_b200 import workloads as W
    wl = W.WORKLOADS[args.workload]
    if args.T is not None:
        wl = replace(wl, T=args.T)
    if args.E is not None:
        wl = replace(wl, E=args.E, bias="uniform")
    return wl


def cfg_of(B, wl):
    return B.MoeConfig(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                       n_group=wl.n_group, topk_group=wl.topk_group, group_topn=wl.group_topn,
                       norm_topk_prob=wl.norm_topk_prob,
                       routed_scaling_factor=wl.routed_scaling_factor,
                       dtype=B.MOE_DTYPE_FP8_E4M3_BLOCK128 if wl.dtype == "fp8" else
                       B.MOE_DTYPE_BF16)


def scales_of(inp):
    return {k: inp[k] for k in ("w13_scale", "w2_scale", "w13s_scale", "w2s_scale") if k in inp}


def launches_per_step(B, cfg, block=False):
    from sigmoid_top_routing_warp_b200 import build as _b  # noqa: F401
    permute = 1 if cfg.T * cfg.k <= 4096 else 3
    quant = 1 if cfg.dtype == B.MOE_DTYPE_FP8_E4M3_BLOCK128 else 0
    # (block: RMSNorm), router GEMM, selection, permute, (fp8: quantise x), gather,
    # gate/up GEMM, down GEMM, combine
    return int(block) + 2 + permute + quant + 1 + 2 + 1


def run_ours(args, world, rank, local):
    from sigmoid_top_routing_warp_b200 import binding as B
    from sigmoid_top_routing_warp_b200 import workloads as W

    wl = workload_of(args)
    dev = torch.device("cuda", local if world > 1 else 0)
    inp = W.make_inputs(wl, device=dev, seed=wl.seed + rank)
    cfg = cfg_of(B, wl)
    ws = B.alloc_workspace(cfg, device=dev)
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    sc = scales_of(inp)
    gamma = W.make_norm_weight(wl, device=dev, seed=wl.seed + rank) if args.block else None
    inp["gamma"] = gamma

    def forward(x, events=None, st=None, dst=None):
        st = stream if st is None else st
        dst = out if dst is None else dst
        if args.block:  # x is the residual stream h
            B.moe_forward_block(cfg, x, gamma, W.RMS_NORM_EPS, inp["w_router"], inp["bias"],
                                inp["w13"], inp["w2"], inp["w13s"], inp["w2s"], dst, ws,
                                stream=st, stage_events=events, **sc)
        else:
            B.moe_forward(cfg, x, inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                          inp["w13s"], inp["w2s"], dst, ws, stream=st, stage_events=events,
                          **sc)

    def step(events=None, st=None):
        forward(inp["x"], events, st)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    B.moe_check_device_status(ws)
    offs = B.ws_view(ws, cfg, "offsets").cpu().numpy()
    touched = int((np.diff(offs) > 0).sum())

    # timed region: K steps, stage events recorded on the launching stream
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(B.MOE_NUM_STAGES + 1)]
           for _ in range(K)]
    for row in evs:
        for e in row:
            e.record(stream)  # materialise the handles
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    barrier(world)
    with ClockSampler(dev.index) as clk:
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for i in range(K):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    B.moe_check_device_status(ws)
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(world, ms)
    stages = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(B.MOE_NUM_STAGES)]
                       for i in range(K)])
    stage_ms = stages.mean(0)

    graph_ms = None
    graph_clocks = None
    if not args.eager:
        # one step captured on a side stream, replayed K times on it
        gs = torch.cuda.Stream(dev)
        gs.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gs):
            with torch.cuda.graph(graph, stream=gs):
                step(st=gs)
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize(dev)
        barrier(world)
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev.index) as gclk:
            with torch.cuda.stream(gs):
                g0.record(gs)
                for _ in range(K):
                    graph.replay()
                g1.record(gs)
            torch.cuda.synchronize(dev)
        barrier(world)
        graph_ms = max_over_ranks(world, g0.elapsed_time(g1))
        graph_clocks = gclk.summary()
        B.moe_check_device_status(ws)
        del graph
    if args.no_e2e:
        return {"wl": wl, "cfg": cfg, "inp": inp, "touched": touched, "ms": ms_max,
                "stage_ms": stage_ms, "clocks": clk.summary(), "e2e_ms": None,
                "launches": launches_per_step(B, cfg, args.block) * K, "B": B,
                "graph_ms": graph_ms, "graph_clocks": graph_clocks, "ws": ws}
    # end to end through the C ABI with host buffers, as a serving loop runs it:
    # every step copies its x from pinned host memory and its out back, on copy
    # streams with two device buffers each, so that step i's copies overlap the
    # neighbouring steps' layer calls (events order every buffer reuse)
    x_host = inp["x"].cpu().pin_memory()
    out_host = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(inp["x"]) for _ in range(2)]
    out_dev = [torch.empty_like(out) for _ in range(2)]
    # one stream per direction: an upload never queues behind a read-back that
    # waits for a layer call
    up_st, down_st = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("h2d", "done", "d2h")}
    used = [False, False]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(up_st):
            if used[b]:
                up_st.wait_event(ev["done"][b])  # step i-2 has read x_dev[b]
            x_dev[b].copy_(x_host, non_blocking=True)
            ev["h2d"][b].record(up_st)
        stream.wait_event(ev["h2d"][b])
        if used[b]:
            stream.wait_event(ev["d2h"][b])  # step i-2's out_dev[b] has been read back
        forward(x_dev[b], dst=out_dev[b])
        ev["done"][b].record(stream)
        with torch.cuda.stream(down_st):
            down_st.wait_event(ev["done"][b])
            out_host[b].copy_(out_dev[b], non_blocking=True)
            ev["d2h"][b].record(down_st)
        used[b] = True

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up_st.wait_stream(stream)
    down_st.wait_stream(stream)
    for i in range(K):
        e2e_step(i)
    stream.wait_stream(down_st)  # the last read-back is inside the timed region
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(world, e0.elapsed_time(e1))
    barrier(world)
    return {"wl": wl, "cfg": cfg, "inp": inp, "touched": touched, "ms": ms_max,
            "stage_ms": stage_ms, "clocks": clk.summary(), "e2e_ms": e2e_ms,
            "launches": launches_per_step(B, cfg, args.block) * K, "B": B,
            "graph_ms": graph_ms, "graph_clocks": graph_clocks, "ws": ws}


# ---------------------------------------------------------------- oracle (CPU)

def oracle_sample(wl, inp, seconds: float):
    """Time the CPU oracle (router logits, selection and layer; with a norm
    weight in inp["gamma"], the pre-norm block around them) on a bounded
    sample of the workload's tokens; returns (tokens/s, threads, sample)."""
    from oracle import oracle as O

    def u16(t):
        return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    fp8 = wl.dtype == "fp8"

    def wcodes(t):  # expert weights as the oracle takes them: bf16 bits or e4m3 codes
        return t.contiguous().cpu().numpy().astype(np.uint8) if fp8 else u16(t)

    def wscale(name, sel=None):
        if not fp8:
            return None
        t = inp[name] if sel is None else inp[name][sel]
        return t.contiguous().cpu().float().numpy()

    threads = O.set_threads(os.cpu_count() or 1)
    wg = u16(inp["w_router"])
    bias = inp["bias"].cpu().numpy()
    w13s, w2s = wcodes(inp["w13s"]), wcodes(inp["w2s"])
    n = max(1, min(wl.T, threads))
    spent, done, rounds = 0.0, 0, 0
    rng = np.random.default_rng(1)
    while spent < seconds and rounds < 6:
        toks = rng.choice(wl.T, size=min(n, wl.T), replace=False)
        x = u16(inp["x"][torch.as_tensor(toks, device=inp["x"].device)])
        gamma = inp.get("gamma")
        t_norm = 0.0
        if gamma is not None:  # block: the layer runs on RMSNorm(h)
            from sigmoid_top_routing_warp_b200 import workloads as W
            h = x
            tn = time.perf_counter()
            x, _ = O.rmsnorm(h, u16(gamma), W.RMS_NORM_EPS)
            t_norm = time.perf_counter() - tn
        oc = O.Config(T=len(toks), H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                      n_group=wl.n_group, topk_group=wl.topk_group, group_topn=wl.group_topn,
                      norm_topk_prob=wl.norm_topk_prob,
                      routed_scaling_factor=wl.routed_scaling_factor, fp8=fp8)
        # routing needs only W_g; the layer needs the experts these tokens use
        t0 = time.perf_counter()
        L = O.router_logits(oc, x, wg).astype(np.float32)
        idx, w, _ = O.route(oc, L, bias)
        t_route = time.perf_counter() - t0
        used = np.unique(idx)
        sel = torch.as_tensor(used, device=inp["w13"].device)
        w13, w2 = wcodes(inp["w13"][sel]), wcodes(inp["w2"][sel])
        remap = np.full(wl.E, -1, np.int64)
        remap[used] = np.arange(used.size)
        oc2 = O.Config(**{**oc.__dict__, "E": int(used.size)})
        t1 = time.perf_counter()
        y = O.layer(oc2, x, remap[idx].astype(np.int32), w, w13, w2, w13s, w2s,
                    w13_scale=wscale("w13_scale", sel), w2_scale=wscale("w2_scale", sel),
                    w13s_scale=wscale("w13s_scale"), w2s_scale=wscale("w2s_scale"))
        if gamma is not None:  # residual add
            y += (h.astype(np.uint32) << 16).view(np.float32)
        spent += t_norm + t_route + time.perf_counter() - t1
        done += len(toks)
        rounds += 1
        n = min(wl.T, n * 2)
    return done / spent, threads, "%d tokens of workload %s (%d rounds, %.1f s)" % (
        done, wl.name, rounds, spent)


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle as it stands, on this host's cores."""
    if rank != 0:
        return None
    from sigmoid_top_routing_warp_b200 import workloads as W
    if args.workload.startswith("dsa_"):
        wl = W.DSA_WORKLOADS[args.workload]
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        inp = W.make_dsa_inputs(wl, device=dev)
        per_step = max(2.0, args.cpu_seconds / max(1, args.steps + args.warmup))
        rates = []
        for i in range(args.warmup + args.steps):
            r, threads, sample = dsa_oracle_sample(wl, inp, per_step)
            if i >= args.warmup:
                rates.append(r)
        value = float(statistics.median(rates))
        return {"impl": "reference", "metric": DSA_METRIC, "value": value, "unit": "queries/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": wl.Sq / value * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": dsa_config(wl, args),
                "cpu_baseline": {"value": value, "unit": "queries/s", "cores": threads,
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    wl = workload_of(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = W.make_inputs(wl, device=dev)
    if args.block:  # the pre-norm block: the oracle's RMSNorm, layer and residual add
        inp["gamma"] = W.make_norm_weight(wl, device=dev, seed=wl.seed)
    per_step = max(2.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    rates = []
    for i in range(args.warmup + args.steps):
        r, threads, sample = oracle_sample(wl, inp, per_step)
        if i >= args.warmup:
            rates.append(r)
    value = float(statistics.median(rates))
    ms = wl.T / value * 1e3
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": layer_config(wl, args, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- main

# ---------------------------------------------------------------- DSA indexer

DSA_METRIC = "DSA indexer queries/s (scores + top-k) and % roofline (bf16 TFLOP/s), 1×B200"


def dsa_work(wl):
    """Unmasked (query, key) pairs, their MMA FLOPs (2 * heads * 128 each) and
    the top-k kernel's HBM bytes (scores read once, indices written)."""
    if wl.causal:
        lim = np.minimum(wl.q_offset + np.arange(wl.Sq) + 1, wl.Sk)
        pairs = float(lim.sum())
    else:
        pairs = float(wl.Sq) * wl.Sk
    return {"pairs": pairs, "flops": 2.0 * wl.n_heads * 128 * pairs,
            "topk_bytes": 4.0 * wl.Sq * wl.Sk + 4.0 * wl.Sq * wl.topk}


def dsa_oracle_sample(wl, inp, seconds):
    from oracle import oracle as O

    def u16(t):
        return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    threads = O.set_threads(os.cpu_count() or 1)
    k = u16(inp["k"])
    rng = np.random.default_rng(3)
    spent, done, n = 0.0, 0, max(1, threads)
    while spent < seconds and done < wl.Sq:
        rows = rng.choice(wl.Sq, size=min(n, wl.Sq), replace=False)
        for r in rows:
            q = u16(inp["q"][int(r):int(r) + 1])
            w = u16(inp["w"][int(r):int(r) + 1])
            t0 = time.perf_counter()
            sc = O.dsa_scores(q, k, w, wl.causal, wl.q_offset + int(r))
            O.dsa_topk(sc.astype(np.float32), wl.topk)
            spent += time.perf_counter() - t0
            done += 1
            if spent >= seconds:
                break
        n *= 2
    return done / spent, threads, "%d query rows of workload %s (%.1f s)" % (done, wl.name, spent)


def run_dsa(args, world, rank, local):
    from sigmoid_top_routing_warp_b200 import binding as B
    from sigmoid_top_routing_warp_b200 import workloads as W

    wl = W.DSA_WORKLOADS[args.workload]
    dev = torch.device("cuda", local if world > 1 else 0)
    inp = W.make_dsa_inputs(wl, device=dev, seed=wl.seed + rank)
    cfg = B.DsaConfig(Sq=wl.Sq, Sk=wl.Sk, n_heads=wl.n_heads, topk=wl.topk, causal=wl.causal,
                      q_offset=wl.q_offset, sorted=not args.dsa_unsorted)
    ws = B.dsa_alloc_workspace(cfg, device=dev)
    scores = B.dsa_scores_view(ws, cfg)
    idx = torch.empty((wl.Sq, wl.topk), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        B.dsa_index_scores(cfg, inp["q"], inp["k"], inp["w"], scores, ws, stream=stream)
        if ev:
            ev[1].record(stream)
        B.dsa_index_topk(cfg, scores, idx, stream=stream)
        if ev:
            ev[2].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    B.moe_check_device_status(ws)
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    with ClockSampler(dev.index) as clk:
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for i in range(K):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    B.moe_check_device_status(ws)
    ms = max_over_ranks(world, t0.elapsed_time(t1))
    sc_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    tk_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    e2e_ms = None
    # first key row a step uploads: the earlier context's keys (rows before k0 when the
    # queries are the context's last Sq tokens) are a cache that stays on the device
    k0 = wl.q_offset if (wl.causal and wl.q_offset + wl.Sq == wl.Sk) else 0
    if not args.no_e2e:
        # the same pipelining as the layer's end-to-end loop: uploads and read-backs on
        # one copy stream per direction, two device buffers of each, events ordering
        # every reuse; the scores buffer in the workspace is only touched on `stream`.
        # A step uploads its queries' q and w and the keys of its own tokens, like
        # the layer's loop that keeps its weights resident.
        names = ("q", "k", "w")
        host = {n: inp[n].cpu().pin_memory() for n in names}
        dev_in = [{n: torch.empty_like(inp[n]) for n in names} for _ in range(2)]
        for b in range(2):
            dev_in[b]["k"][:k0].copy_(inp["k"][:k0])
        idx_dev = [torch.empty_like(idx) for _ in range(2)]
        idx_host = [torch.empty((wl.Sq, wl.topk), dtype=torch.int32).pin_memory()
                    for _ in range(2)]
        up_st, down_st = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("h2d", "done", "d2h")}
        used = [False, False]

        def e2e_step(i):
            b = i % 2
            with torch.cuda.stream(up_st):
                if used[b]:
                    up_st.wait_event(ev["done"][b])
                dev_in[b]["q"].copy_(host["q"], non_blocking=True)
                dev_in[b]["w"].copy_(host["w"], non_blocking=True)
                dev_in[b]["k"][k0:].copy_(host["k"][k0:], non_blocking=True)
                ev["h2d"][b].record(up_st)
            stream.wait_event(ev["h2d"][b])
            if used[b]:
                stream.wait_event(ev["d2h"][b])
            B.dsa_indexer(cfg, dev_in[b]["q"], dev_in[b]["k"], dev_in[b]["w"], idx_dev[b], ws,
                          stream=stream)
            ev["done"][b].record(stream)
            with torch.cuda.stream(down_st):
                down_st.wait_event(ev["done"][b])
                idx_host[b].copy_(idx_dev[b], non_blocking=True)
                ev["d2h"][b].record(down_st)
            used[b] = True

        for i in range(max(3, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up_st.wait_stream(stream)
        down_st.wait_stream(stream)
        for i in range(K):
            e2e_step(i)
        stream.wait_stream(down_st)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        B.moe_check_device_status(ws)
        e2e_ms = max_over_ranks(world, e0.elapsed_time(e1))
    h2d = int(inp["q"].numel() * 2 + inp["w"].numel() * 2 + (wl.Sk - k0) * wl.n_heads * 128 * 2)
    return {"wl": wl, "inp": inp, "ms": ms, "sc_ms": sc_ms, "tk_ms": tk_ms, "clocks": clk.summary(),
            "e2e_ms": e2e_ms, "h2d_bytes": h2d}


def dsa_main(args, world, rank, local):
    peaks, peak_src = load_peaks()
    r = run_dsa(args, world, rank, local)
    wl, K = r["wl"], args.steps
    work = dsa_work(wl)
    value = world * wl.Sq * K / (r["ms"] / 1e3)
    ach = work["flops"] / (r["sc_ms"] / 1e3) / 1e12
    # a K-step run of about a millisecond per step is a burst: the burst peak
    # is the denominator, the sustained one beside it
    pk = peaks["bf16_tflops"]
    pk_sus = peaks.get("bf16_tflops_sustained", pk)
    tk_gbs = work["topk_bytes"] / (r["tk_ms"] / 1e3) / 1e9
    line = {"metric": DSA_METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": r["ms"] / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dsa_config(wl, args),
            "roofline": {"bound": "tensor", "achieved": ach, "peak": pk, "unit": "TFLOP/s",
                         "frac": ach / pk, "traffic": profile_traffic("dsa_scores", None, wl.name),
                         "peak_kind": "bf16 burst",
                         "frac_of_sustained_peak": ach / pk_sus,
                         "kernel": "dsa_scores_kernel (w x ReLU(q.k) over heads)",
                         "algorithmic_per_launch": work["flops"], "launch_ms": r["sc_ms"],
                         "peak_source": peak_src},
            "topk_roofline": {"bound": "hbm", "achieved": tk_gbs, "peak": peaks["hbm_gbs"],
                              "unit": "GB/s", "frac": tk_gbs / peaks["hbm_gbs"],
                              "launch_ms": r["tk_ms"]},
            "stages_ms": {"scores": r["sc_ms"], "topk": r["tk_ms"]},
            "gpu_launches": 2 * K, "clocks": r["clocks"],
            "e2e": None if r["e2e_ms"] is None else {
                "value": world * wl.Sq * K / (r["e2e_ms"] / 1e3), "unit": "queries/s",
                "h2d_bytes_per_step": r["h2d_bytes"],
                "d2h_bytes_per_step": wl.Sq * wl.topk * 4}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, threads, sample = dsa_oracle_sample(wl, r["inp"], args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "queries/s", "cores": threads, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_teardown(world)


# ---------------------------------------------------------------- backward

BWD_METRIC = ("MoE-layer backward tokens/s (gradients of x, router, expert and shared weights) "
              "and % roofline (bf16 TFLOP/s), 1×B200")


def backward_work(wl):
    """Algorithmic FLOPs of one backward step and of each of its GEMM stages
    (routed rows T*k; padding rows are overhead, not work)."""
    T, H, E, k, I, Is = wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is
    R = T * k
    st = {"gate_up_recompute": 2 * R * 2 * I * H + 2 * T * 2 * Is * H,
          "down_backward": 2 * R * H * I + 2 * T * H * Is,
          "input_grads": 2 * R * 2 * I * H + 2 * T * 2 * Is * H + 2 * T * E * H,
          "weight_grads": 2 * R * 3 * I * H + 2 * T * 3 * Is * H + 2 * T * E * H}
    return {"flops": float(sum(st.values())), "stages": st,
            # weight-gradient outputs (fp32) the step must write
            "grad_bytes": 4.0 * (E * 3 * H * I + 3 * H * Is + E * H)}


def run_backward(args, world, rank, local, inp=None):
    """Time moe_backward (K steps after W warm-ups, CUDA events on the stream,
    stage events per launch) on the workload's inputs, routed once by the
    library's own router outside the timed region."""
    from sigmoid_top_routing_warp_b200 import binding as B
    from sigmoid_top_routing_warp_b200 import workloads as W
    wl = workload_of(args)
    dev = torch.device("cuda", local if world > 1 else 0)
    if inp is None:
        inp = W.make_inputs(wl, device=dev, seed=wl.seed + rank)
    cfg = cfg_of(B, wl)
    T, H, E, k, I, Is = wl.T, wl.H, wl.E, wl.k, wl.I, wl.Is
    stream = torch.cuda.current_stream(dev)
    ws = B.alloc_workspace(cfg, device=dev)
    logits = torch.empty((T, E), device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), device=dev)
    B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], logits, idx, w, ws)
    dout = W.make_grad_output(wl, device=dev, seed=wl.seed + rank)
    g = {"dx": torch.empty((T, H), dtype=torch.bfloat16, device=dev),
         "dwg": torch.empty((E, H), device=dev),
         "dw13": torch.empty((E, 2 * I, H), device=dev),
         "dw2": torch.empty((E, H, I), device=dev),
         "dw13s": torch.empty((2 * Is, H), device=dev) if Is else None,
         "dw2s": torch.empty((H, Is), device=dev) if Is else None}
    bws = B.alloc_backward_workspace(cfg, device=dev)

    def step(events=None):
        B.moe_backward(cfg, inp["x"], inp["w_router"], logits, idx, w, inp["w13"], inp["w2"],
                       inp["w13s"] if Is else None, inp["w2s"] if Is else None, dout, g["dx"],
                       g["dwg"], g["dw13"], g["dw2"], g["dw13s"], g["dw2s"], bws,
                       stream=stream, stage_events=events)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    B.moe_check_device_status(bws)
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(B.MOE_NUM_BWD_STAGES + 1)]
           for _ in range(K)]
    for row in evs:
        for e in row:
            e.record(stream)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    barrier(world)
    with ClockSampler(dev.index) as clk:
        t0.record(stream)
        for i in range(K):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    B.moe_check_device_status(bws)
    ms = max_over_ranks(world, t0.elapsed_time(t1))
    stages = np.array([[evs[i][j].elapsed_time(evs[i][j + 1])
                        for j in range(B.MOE_NUM_BWD_STAGES)] for i in range(K)]).mean(0)
    touched = int((torch.bincount(idx.flatten().long(), minlength=E) > 0).sum().item())
    # permute (1 or 3 kernels), plan, gather, 4 GEMMs, router, combine
    launches = (1 if T * k <= 4096 else 3) + 8
    return {"wl": wl, "ms": ms, "stage_ms": stages, "clocks": clk.summary(), "touched": touched,
            "names": B.BWD_STAGE_NAMES, "launches": launches * K}


def backward_object(args, rb, peaks, peak_src, world):
    wl, K = rb["wl"], args.steps
    work = backward_work(wl)
    step_ms = rb["ms"] / K
    stage_ms = {n: float(v) for n, v in zip(rb["names"], rb["stage_ms"])}
    gemm = {n: stage_ms[n] for n in work["stages"]}
    dom = max(gemm, key=gemm.get)
    ach = work["stages"][dom] / (gemm[dom] / 1e3) / 1e12
    burst = peaks["bf16_tflops"]
    return {"metric": BWD_METRIC, "value": world * wl.T * K / (rb["ms"] / 1e3), "unit": UNIT,
            "ms_per_step": step_ms, "tflops": work["flops"] / (step_ms / 1e3) / 1e12,
            "roofline": {"bound": "tensor", "achieved": ach, "peak": burst, "unit": "TFLOP/s",
                         "frac": ach / burst, "traffic": None,
                         "kernel": "bwd_pair_gemm_kernel (%s)" % dom,
                         "algorithmic_per_launch": work["stages"][dom], "launch_ms": gemm[dom],
                         "peak_kind": "bf16 burst", "peak_source": peak_src,
                         "frac_of_sustained_peak":
                             ach / peaks.get("bf16_tflops_sustained", burst)},
            "layer_roofline": {"flops": work["flops"],
                               "t_roof_ms": 1e3 * work["flops"] / (burst * 1e12),
                               "frac_of_roofline": 1e3 * work["flops"] / (burst * 1e12) / step_ms},
            "stages_ms": stage_ms, "clocks": rb["clocks"], "gpu_launches": rb["launches"],
            "experts_touched": rb["touched"], "dtype": "bf16",
            "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k,
                       "I": wl.I, "n_shared": wl.n_shared, "n_group": wl.n_group,
                       "topk_group": wl.topk_group, "pass": "backward"}}


def routing_check(r):
    """Near-tie count of the timed batch, with the oracle as the checker (part
    of the CPU-baseline leg, outside the timed region): the oracle routes the
    GPU's own fp32 logits; the indices and weights must equal the GPU's bit for
    bit, and tokens whose k-th and (k+1)-th biased scores lie closer than 1e-4
    are counted."""
    from oracle import oracle as O
    wl, B, cfg, ws = r["wl"], r["B"], r["cfg"], r["ws"]
    L = B.ws_view(ws, cfg, "logits").cpu().numpy()
    idx = B.ws_view(ws, cfg, "topk_idx").cpu().numpy()
    w = B.ws_view(ws, cfg, "topk_w").cpu().numpy()
    oc = O.Config(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                  n_group=wl.n_group, topk_group=wl.topk_group, group_topn=wl.group_topn,
                  norm_topk_prob=wl.norm_topk_prob,
                  routed_scaling_factor=wl.routed_scaling_factor)
    oidx, ow, gap = O.route(oc, L, r["inp"]["bias"].cpu().numpy())
    exact = bool((idx == oidx).all() and (w.view(np.uint32) == ow.view(np.uint32)).all())
    return {"near_ties": int((gap < 1e-4).sum()), "near_tie_gap": 1e-4, "tokens": wl.T,
            "bit_exact_vs_oracle": exact}


def layer_line(args, r, peaks, peak_src, world):
    """The JSON line of one timed layer workload (our arm)."""
    wl, K = r["wl"], args.steps
    work = layer_work(wl, r["touched"])
    step_ms_total = r["graph_ms"] if r["graph_ms"] is not None else r["ms"]
    value = world * wl.T * K / (step_ms_total / 1e3)
    stage_names = r["B"].STAGE_NAMES
    g1_ms = float(r["stage_ms"][3])
    pair = r["cfg"].T * r["cfg"].k / r["cfg"].E > 96.0 and wl.dtype != "fp8"
    fp8 = wl.dtype == "fp8"
    # token-major fp8 kernel: hidden and intermediate sizes multiples of 512
    tm = fp8 and wl.H % 512 == 0 and wl.I % 512 == 0
    kind = ("gate_up_fp8_tm" if tm else "gate_up_fp8" if fp8 else
            "gate_up_prefill" if pair else "gate_up_decode")
    traffic = profile_traffic(kind, work["g1_bytes"], wl.name + ("_block" if args.block else ""))
    if fp8:  # no fp8 peak is measured: the bf16 peaks x the nominal fp8/bf16 ratio 2
        peaks = dict(peaks)
        for key in ("bf16_tflops", "bf16_tflops_sustained"):
            if key in peaks:
                peaks[key] = 2.0 * peaks[key]
    burst = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained", burst)
    pk_name = "fp8 (assumed 2x the measured bf16 peak; no fp8 peak measured)" if fp8 else "bf16"
    hbm_bound = work["bytes"] / (peaks["hbm_gbs"] * 1e9) >= work["flops"] / (burst * 1e12)
    if hbm_bound:
        ach = work["g1_bytes"] / (g1_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": traffic}
    else:
        # K steps of a few ms are a short burst, not a seconds-long loop: the
        # burst tensor peak is the denominator; the sustained one is beside it
        ach = work["g1_flops"] / (g1_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": burst, "unit": "TFLOP/s",
                "frac": ach / burst, "traffic": traffic,
                "peak_kind": pk_name + " burst",
                "frac_of_sustained_peak": ach / sustained}
    kname = ("fp8_tm_gemm_kernel<SWIGLU>" if tm else "fp8_gemm_kernel<SWIGLU>" if fp8 else
             "pair_gemm_kernel<SWIGLU>" if pair else "grouped_gemm_kernel<SWIGLU,16>")
    roof.update({"kernel": kname + " (gate/up GEMM + SwiGLU)",
                 "algorithmic_per_launch": work["g1_bytes"] if hbm_bound else work["g1_flops"],
                 "launch_ms": g1_ms, "peak_source": peak_src})
    layer_ms = step_ms_total / K
    layer = {"ms": layer_ms,
             "hbm_gbs": work["bytes"] / (layer_ms / 1e3) / 1e9,
             "tflops": work["flops"] / (layer_ms / 1e3) / 1e12,
             "t_roof_ms": 1e3 * max(work["bytes"] / (peaks["hbm_gbs"] * 1e9),
                                    work["flops"] / (burst * 1e12)),
             "tensor_peak_tflops": burst, "tensor_peak_kind": pk_name + " burst"}
    layer["frac_of_roofline"] = layer["t_roof_ms"] / layer_ms
    if not hbm_bound:
        layer["frac_of_sustained_roofline"] = 1e3 * max(
            work["bytes"] / (peaks["hbm_gbs"] * 1e9), work["flops"] / (sustained * 1e12)) / layer_ms
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": layer_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16",
            "data": "synthetic",
            "config": layer_config(wl, args, world),
            "routing": {"experts_touched": r["touched"],
                        "algorithmic_gb_per_step": work["bytes"] / 1e9},
            "roofline": roof, "layer_roofline": layer,
            "stages_ms": {n: float(v) for n, v in zip(stage_names, r["stage_ms"])},
            "gpu_launches": r["launches"],
            # the clocks of the region `value` comes from (graph replay by default)
            "clocks": r["graph_clocks"] if r["graph_clocks"] is not None else r["clocks"],
            "clocks_eager": r["clocks"],
            "graph": None if r["graph_ms"] is None else {
                "ms_per_step": r["graph_ms"] / K, "eager_ms_per_step": r["ms"] / K},
            "e2e": None if r["e2e_ms"] is None else {
                "value": world * wl.T * K / (r["e2e_ms"] / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": wl.T * wl.H * 2, "d2h_bytes_per_step": wl.T * wl.H * 2}}
    return line


def main():
    args = parse()
    world, rank, local = dist_setup()
    if args.workload.startswith("dsa_") and args.impl == "ours":
        dsa_main(args, world, rank, local)
        return
    if args.impl == "reference":
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        dist_teardown(world)
        return
    peaks, peak_src = load_peaks()
    if args.backward:
        rb = run_backward(args, world, rank, local)
        bo = backward_object(args, rb, peaks, peak_src, world)
        line = {"metric": bo.pop("metric"), "value": bo.pop("value"), "unit": UNIT,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": bo.pop("ms_per_step"), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": bo.pop("dtype"),
                "data": "synthetic", "config": bo.pop("config"), **bo}
        if rank == 0:
            print(json.dumps(line), flush=True)
        dist_teardown(world)
        return
    r = run_ours(args, world, rank, local)
    line = layer_line(args, r, peaks, peak_src, world)
    cpu_leg = rank == 0 and world == 1 and not args.no_cpu_baseline
    if cpu_leg:
        line["routing"].update(routing_check(r))
        v, threads, sample = oracle_sample(r["wl"], r["inp"], args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": sample}
    # The default run also times the prefill workload (T = 8192, Zipf loads),
    # the metric's tensor-bound configuration, with the same K and W; decode
    # stays the headline value.
    if (args.workload == "decode" and not args.no_prefill and not args.block
            and args.T is None and args.E is None):
        del r
        torch.cuda.empty_cache()
        pargs = argparse.Namespace(**{**vars(args), "workload": "prefill", "no_e2e": True})
        rp = run_ours(pargs, world, rank, local)
        pl = layer_line(pargs, rp, peaks, peak_src, world)
        line["prefill"] = {
            "workload": "prefill", "config": pl["config"], "value": pl["value"], "unit": UNIT,
            "ms_per_step": pl["ms_per_step"], "tflops": pl["layer_roofline"]["tflops"],
            "roofline": pl["roofline"], "layer_roofline": pl["layer_roofline"],
            "stages_ms": pl["stages_ms"], "clocks": pl["clocks"],
            "clocks_eager": pl["clocks_eager"], "graph": pl["graph"],
            "gpu_launches": pl["gpu_launches"], "routing": pl["routing"]}
        if cpu_leg:
            line["prefill"]["routing"].update(routing_check(rp))
        # the backward pass of the same prefill batch, on the same inputs
        inp_p = rp["inp"]
        del rp
        torch.cuda.empty_cache()
        rb = run_backward(pargs, world, rank, local, inp=inp_p)
        line["backward"] = backward_object(pargs, rb, peaks, peak_src, world)
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_teardown(world)


if __name__ == "__main__":
    main()
