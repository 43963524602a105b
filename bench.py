#!/usr/bin/env python
"""Benchmark of the routed-expert MoE layer on B200.

One step = one pass of the whole layer over one batch: route (top-k of fp32
router logits) -> permute + expert-hit histogram -> grouped gated FFN over the
routed experts (through the slot table) -> weighted combine, all in the
library's kernels, inputs already resident in HBM.

Default workload: one Gemma-shaped MoE layer, bf16 experts: 128 experts,
hidden 2816, expert intermediate 704 (11.34 MiB per expert), top-8, decode
batch of 64 tokens, router logits N(0,1), weights N(0,0.02), activations N(0,1).
To keep the expert weights out of L2 (126 MB), each step reads a different one
of 30 distinct layer copies (45.7 GB in HBM for bf16), so a layer's experts
come back only after 29 other layers' worth of traffic.  The batches of 1 and
8 tokens are measured in the same run and reported under "sweep".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--config decode-bf16|decode-int8|int4-decode|int4-prefill|tiny]
                  [--tokens T] [--parallel replicas|ep]

Multi-GPU (N > 1, launched by torchrun): by default every rank runs an
independent replica of the same workload (weak scaling, no collective on the
data path); the timing is the max over ranks.  --parallel ep splits the experts
over the ranks instead (each rank routes its own tokens; NCCL all-to-all
dispatch and return).

--impl reference times the CPU oracle (plain C, every host core) on a bounded
sample of the same workload on rank 0; it is the baseline, not the target.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

# Per-launch DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, summed
# over the gather and grouped-FFN launches of one layer call) from one-pass ncu
# captures of the kernels as they stand, keyed by (workload, --path):
# (bytes, algorithmic bytes of the captured call, what was captured).  The
# captured call is the first graph-replayed step of
#   bench.py --quick --headline-only --steps 10 --warmup 3 --layers 2
#            --no-cpu-baseline [--config C] [--tokens T]
# (batch 3 of seed 0; ncu -s skips the 8 distinct-expert probes and the 3 warm-up
# calls), whose distinct experts differ from the bench's 8-batch average, so the
# traffic is compared with that call's own algorithmic bytes.  A workload
# without an entry reports null.
_CAPTURE = ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
            "--clock-control none -k regex:'k_ffn|k_gather_rows', one layer call of bench.py --quick "
            "--headline-only --layers 2")
NCU_TRAFFIC_BYTES = {
    ("moe-layer-bf16-decode-T64", "auto"): (1506674944, 1499103232, _CAPTURE + " (gather + 2 tcgen05 launches)"),
    ("moe-layer-bf16-decode-T8", "auto"): (583954944, 582889472, _CAPTURE + " --tokens 8 (gather + 2 tcgen05 launches)"),
    ("moe-layer-bf16-decode-T1", "auto"): (95784192, 95163904, _CAPTURE + " --tokens 1 (2 one-token GEMV launches)"),
    ("moe-layer-int8-decode-T64", "auto"): (308761856, 304539136,
                                            _CAPTURE + " --config decode-int8 (gather + 2 tcgen05 launches)"),
    ("moe-layer-int8-decode-T8", "auto"): (144329472, 143187968,
                                           _CAPTURE + " --config decode-int8 --tokens 8 (gather + 2 tcgen05 launches)"),
    ("moe-layer-int8-decode-T1", "auto"): (47796224, 47719936,
                                           _CAPTURE + " --config decode-int8 --tokens 1 (2 one-token GEMV launches)"),
    ("moe-layer-int4-decode-T64", "auto"): (404659712, 398464000,
                                            _CAPTURE + " --config int4-decode (gather + 2 tcgen05 launches)"),
    ("moe-layer-int4-prefill-T1024", "auto"): (521776128, 410189824,
                                               _CAPTURE + " --config int4-prefill (gather + 2 tcgen05 launches)"),
}

# routes from which the library's AUTO path takes the tensor-core FFN (bf16, int8,
# int4), for counting launches: gather + 2 tensor-core launches, else 2 GEMV launches
TC_MIN_ROUTES = {0: 24, 1: 32, 2: 40}

CONFIGS = {
    # name: (weight format, logits kind, tokens, extra batches swept)
    "decode-bf16": ("bf16", "normal", 64, [1, 8]),
    "decode-int8": ("int8", "biased", 64, [1, 8]),
    "int4-decode": ("int4", "normal", 64, []),
    "int4-prefill": ("int4", "normal", 1024, []),
    "tiny": ("bf16", "normal", 16, []),
    # 30-layer stack, slot table, Zipf(1.1) routing, refresh every 8 steps
    "stack30": ("int4", "zipf", 64, [1, 8]),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=30)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="decode-bf16", choices=sorted(CONFIGS))
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--layers", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--quick", action="store_true", help="main batch only: no sweep, no e2e, no CPU baseline")
    ap.add_argument("--headline-only", action="store_true",
                    help="decode-bf16: skip the int8 / int4 / stack workloads reported under 'configs'")
    ap.add_argument("--stack-refresh", default="device", choices=["device", "host"],
                    help="stack30: placement refresh on the device (graph-captured, copies overlapped) or on the host")
    ap.add_argument("--path", default="auto", choices=["auto", "gemv", "tc"],
                    help="grouped-FFN kernels: AUTO picks by routes per call")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "ep"],
                    help="N > 1: independent replicas (default), or expert parallelism (each rank holds E/N "
                         "experts, NCCL all-to-all dispatch and return)")
    return ap.parse_args()


# --------------------------------------------------------------- multi-rank

def max_over_ranks(dist, value: float, device=None) -> float:
    """The slowest rank's time: every rank passes its own elapsed ms and gets the
    maximum (replicas run the same workload; the job is as fast as its slowest)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units all ranks processed per second, timed by the slowest rank."""
    return world * units_per_rank / (ms / 1e3)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- workload

def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def build_layers(moe, torch, fmt_name, E, H, I, n_layers, dev, seed=0):
    """n_layers distinct copies of the layer's expert blobs in HBM."""
    import synthetic as syn

    fmt = moe.FMT[fmt_name]
    eb = moe.moe_expert_bytes(fmt, H, I)
    layers = []
    for l in range(n_layers):
        if fmt == moe.MOE_W_BF16:
            # a bf16 blob is W13 then W2, all bf16: draw it in place
            home = torch.empty(E * eb, dtype=torch.uint8, device=dev)
            hv = home.view(torch.bfloat16)
            g = torch.Generator(device=dev)
            g.manual_seed(1000 * seed + l)
            step = 1 << 26
            for i in range(0, hv.numel(), step):
                n = min(step, hv.numel() - i)
                hv[i:i + n] = (torch.randn(n, generator=g, device=dev) * syn.WEIGHT_STD).to(torch.bfloat16)
            layers.append(moe.MoeLayer(fmt, E, H, I, home, expert_bytes=eb))
        else:
            w13, w2 = syn.torch_expert_weights(E, H, I, seed=seed, layer=l, device=dev)
            layers.append(moe.make_layer(fmt, w13, w2))
            del w13, w2
    torch.cuda.synchronize(dev)
    return layers


def make_batches(torch, kind, T, E, H, n, dev, seed=0):
    import synthetic as syn

    out = []
    for b in range(n):
        lg = syn.router_logits(T, E, kind, seed=seed + 17, layer=b)
        x = syn.activations(T, H, seed=seed + 23, layer=b)
        out.append((lg, x, torch.from_numpy(lg).to(dev),
                    torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)))
    return out


class Runner:
    """Device buffers for one batch size; step(i) runs the layer on batch i
    (one_call: as one moe_layer_forward call, with no FFN events)."""

    def __init__(self, moe, torch, layers, batches, T, k, dev, path=0, one_call=False):
        self.moe, self.torch, self.layers, self.batches, self.T, self.k = moe, torch, layers, batches, T, k
        self.path = path
        self.one_call = one_call
        E, H = layers[0].E, layers[0].H
        R = T * k
        i32 = torch.int32
        self.ids = torch.empty((T, k), dtype=i32, device=dev)
        self.w = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.perm = (torch.empty(E, dtype=i32, device=dev), torch.empty(E + 1, dtype=i32, device=dev),
                     torch.empty(R, dtype=i32, device=dev), torch.empty(R, dtype=i32, device=dev))
        self.hits = torch.zeros((len(layers), E), dtype=i32, device=dev)
        self.rows = torch.empty((R, H), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(moe.moe_grouped_ffn_workspace(layers[0], T, k), 16), dtype=torch.uint8, device=dev)
        self.y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.fws = (torch.empty(moe.moe_layer_forward_workspace(layers[0], T, k), dtype=torch.uint8, device=dev)
                    if one_call else None)
        self.ev = None
        self.side = None

    def step(self, i, ffn_events=None):
        moe = self.moe
        li = i % len(self.layers)
        L = self.layers[li]
        _, _, lg, x = self.batches[i % len(self.batches)]
        if self.one_call:
            moe.moe_layer_forward(L, lg, x, self.k, y=self.y, hits=self.hits[li], ids_out=self.ids, w_out=self.w,
                                  ws=self.fws)
            return
        # the routing and the FFN as separate calls, so that the FFN's event pair
        # times the FFN alone (moe_route_ffn, which the stacks use, would run a
        # one-token step's routing inside the FFN's first launch)
        _, _, counts, offsets, sr, rp = moe.moe_route_permute(lg, self.k, hits=self.hits[li],
                                                              ids_w=(self.ids, self.w), out=self.perm)
        if ffn_events is not None:
            self._mark(ffn_events[0])
        moe.moe_grouped_ffn(L, x, self.k, counts, offsets, sr, rows=self.rows, ws=self.ws, path=self.path)
        if ffn_events is not None:
            self._mark(ffn_events[1])
        moe.moe_combine(self.rows, rp, self.w, self.y)

    def _mark(self, ev):
        """Record a timing event on a side stream forked from the current one:
        inside a graph capture the event node then hangs off the last kernel
        (it fires when that kernel completes) without sitting between two
        kernels, so the programmatic-launch edges of the main chain stay."""
        torch = self.torch
        if self.side is None:
            self.side = torch.cuda.Stream()
        self.side.wait_stream(torch.cuda.current_stream())
        ev.record(self.side)

    def join(self):
        """Join the side stream back (the end of a capture that used _mark)."""
        if self.side is not None:
            self.torch.cuda.current_stream().wait_stream(self.side)

    def launches_per_step(self):
        """route + permute (one launch up to FUSED_MAX_T tokens, else two), FFN (2 GEMV
        launches, or gather + 2 tensor-core launches), combine"""
        return launches_per_layer(self.moe, self.T, self.k, self.layers[0].fmt, self.path)

    def distinct_experts(self):
        """Distinct routed experts of each batch (read back from our own routing)."""
        out = []
        for i in range(len(self.batches)):
            self.step(i)
            self.torch.cuda.synchronize()
            out.append(int((self.perm[0] > 0).sum().item()))
        return out


FFN_SAMPLE_EVERY = 1

# tokens up to which moe_route_permute is one launch
FUSED_MAX_T = 16
ROUTE_IN_FFN_MAX_E = 128  # moe_route_ffn routes inside the one-token FFN launches up to this E


def routes_in_ffn(moe, T, k, fmt, E, path):
    """Whether moe_route_ffn runs the routing inside the FFN's launches: one token,
    E <= ROUTE_IN_FFN_MAX_E, the AUTO path taking the GEMV kernels."""
    return T == 1 and E <= ROUTE_IN_FFN_MAX_E and path == moe.MOE_FFN_AUTO and T * k < TC_MIN_ROUTES[fmt]


def launches_per_layer(moe, T, k, fmt, path, E=None):
    """Our launches per layer step; E given: the step calls moe_layer_forward,
    whose one-token steps route inside the FFN's first launch and combine inside
    its second (no routing and no combine launch; the shared-memory fit of the
    fused combine holds at the bench's shapes)."""
    auto_tc = T * k >= TC_MIN_ROUTES[fmt]
    tc = path == moe.MOE_FFN_TC or (path == moe.MOE_FFN_AUTO and auto_tc)
    in_ffn = E is not None and routes_in_ffn(moe, T, k, fmt, E, path)
    route = 0 if in_ffn else (1 if T <= FUSED_MAX_T else 2)
    return route + (3 if tc else 2) + (0 if in_ffn else 1)


def _capture(torch, runner, first, n):
    """One CUDA graph of n consecutive steps, with an external event pair around
    the grouped-FFN launches of every FFN_SAMPLE_EVERY-th step (every step, so a
    20-step run gives 20 pairs).  The event nodes sit on a side stream: the first
    fires when the permute kernel completes, the second when the FFN's last
    launch does, and neither cuts the programmatic-launch edges of the kernel
    chain (an event node between two kernels would)."""
    g = torch.cuda.CUDAGraph()
    sampled = [] if runner.one_call else [j for j in range(n) if j % FFN_SAMPLE_EVERY == FFN_SAMPLE_EVERY // 2] or [0]
    evs = {j: (torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for j in sampled}
    with torch.cuda.graph(g):
        for j in range(n):
            runner.step(first + j, evs.get(j))
        runner.join()
    return g, list(evs.values())


def time_steps(torch, runner, steps, warmup, dist):
    """Exactly `steps` steps between two events, replayed from CUDA graphs of one
    rotation over the layers (so Python launch overhead is out of the timed
    region; each graph is launched once before it, untimed).  Returns (total ms,
    per-step FFN ms from the last replay of each graph)."""
    G = len(runner.layers)
    for i in range(warmup):
        runner.step(i)
    torch.cuda.synchronize()
    full, rem = steps // G, steps % G
    graphs = []
    if full:
        graphs.append(_capture(torch, runner, warmup, G))
    if rem:
        graphs.append(_capture(torch, runner, warmup, rem))
    for g, _ in graphs:  # a graph's first launch also uploads it: keep that out of the timed region
        g.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(full):
        graphs[0][0].replay()
    if rem:
        graphs[-1][0].replay()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    if dist is not None:
        dist.barrier()
    ffn_ms = [a.elapsed_time(b) for _, evs in graphs for a, b in evs]
    del graphs
    return ms, ffn_ms


def time_eager(torch, runner, steps, warmup):
    """The same steps launched one by one from Python (no CUDA graph), between
    two events: the eager counterpart of time_steps."""
    for i in range(warmup):
        runner.step(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        runner.step(warmup + i)
    t1.record()
    torch.cuda.synchronize()
    return t0.elapsed_time(t1)


def time_e2e(torch, moe, layers, batches, T, k, steps, warmup, dev):
    """End to end through moe_layer_forward with host buffers: every step copies
    its logits and x from pinned host memory and reads y back to pinned host
    memory.  As a serving loop would, the copies run on their own streams and
    overlap the layer of the neighbouring step (double-buffered device buffers,
    ordered by events): H2D of step i+1 and D2H of step i-1 while step i runs."""
    E, H = layers[0].E, layers[0].H
    host_lg = [torch.from_numpy(b[0]).pin_memory() for b in batches]
    host_x = [torch.from_numpy(b[1].view(np.int16)).pin_memory() for b in batches]
    host_y = [torch.empty((T, H), dtype=torch.int16).pin_memory() for _ in range(2)]
    d_lg = [torch.empty((T, E), dtype=torch.float32, device=dev) for _ in range(2)]
    d_x = [torch.empty((T, H), dtype=torch.int16, device=dev) for _ in range(2)]
    d_y = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ws = torch.empty(moe.moe_layer_forward_workspace(layers[0], T, k), dtype=torch.uint8, device=dev)
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b landed
    ev_done = [torch.cuda.Event() for _ in range(2)]   # the layer using buffer b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # y of buffer b read back
    for b in range(2):
        ev_done[b].record(comp)
        ev_out[b].record(comp)

    def one(i):
        b, src = i & 1, i % len(batches)
        s_in.wait_event(ev_done[b])                    # the layer two steps back is done with these inputs
        with torch.cuda.stream(s_in):
            d_lg[b].copy_(host_lg[src], non_blocking=True)
            d_x[b].copy_(host_x[src], non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        comp.wait_event(ev_out[b])                     # y of two steps back has been read
        moe.moe_layer_forward(layers[i % len(layers)], d_lg[b], d_x[b].view(torch.bfloat16), k, y=d_y[b], ws=ws)
        ev_done[b].record(comp)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            host_y[b].copy_(d_y[b].view(torch.int16), non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    for i in range(steps):
        one(warmup + i)
    comp.wait_stream(s_in)
    comp.wait_stream(s_out)
    t1.record(comp)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    return ms, T * E * 4 + T * H * 2, T * H * 2


def time_router(torch, moe, T, E, H, k, dev, n=200):
    """The router projection fused with top-k (the step before the layer), one
    launch per call on a different copy of the fp32 router weights (enough copies
    to span twice the L2), n calls replayed from one CUDA graph."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(8, -(-2 * l2 // (E * H * 4)))
    g = torch.Generator(device=dev)
    g.manual_seed(17)
    wr = torch.randn((copies, E, H), generator=g, device=dev, dtype=torch.float32) * 0.02
    x = (torch.randn((T, H), generator=g, device=dev, dtype=torch.float32)).to(torch.bfloat16)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        moe.moe_router_topk(x, wr[0], k, ids=ids, w=w)
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(n):
                moe.moe_router_topk(x, wr[i % copies], k, ids=ids, w=w)
        graph.replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        stream.synchronize()
        a.record(stream)
        graph.replay()
        b.record(stream)
        b.synchronize()
    us = a.elapsed_time(b) * 1e3 / n
    alg = E * H * 4 + T * H * 2 + T * k * 8
    del graph, wr
    return {"us": round(us, 2), "tokens_per_s": round(T / (us / 1e6), 1), "alg_bytes": alg,
            "hbm_gbs": round(alg / (us / 1e6) / 1e9, 1), "router_copies": copies}


def time_kernels(torch, moe, layer, T, E, H, I, k, dev, n=100):
    """Each step of the path on its own, replayed n times from a CUDA graph on
    the decode batch's shapes: average us per call and algorithmic GB/s (inputs
    read + outputs written).  The quantisers run on one expert's w13 [2I, H]."""
    import synthetic as syn

    g = torch.Generator(device=dev)
    g.manual_seed(23)
    lg = torch.from_numpy(syn.router_logits(T, E, "normal", seed=23)).to(dev)
    ids, w = moe.moe_route_topk(lg, k)
    perm = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(T * k, dtype=torch.int32, device=dev), torch.empty(T * k, dtype=torch.int32, device=dev))
    moe.moe_permute(ids, E, out=perm)
    perm1 = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
             torch.empty(k, dtype=torch.int32, device=dev), torch.empty(k, dtype=torch.int32, device=dev))
    perm8 = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
             torch.empty(8 * k, dtype=torch.int32, device=dev), torch.empty(8 * k, dtype=torch.int32, device=dev))
    rows = torch.randn((T * k, H), generator=g, device=dev, dtype=torch.float32)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    hits = torch.zeros(E, dtype=torch.int32, device=dev)
    ids2, w2 = ids.clone(), w.clone()
    table = torch.full((E,), -1, dtype=torch.int32, device=dev)
    table[:18] = torch.arange(18, dtype=torch.int32, device=dev)
    wq = (torch.randn((2 * I, H), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    q8, s8 = moe.moe_quantize_int8(wq)
    q4, s4 = moe.moe_quantize_int4(wq)
    thits = torch.randint(0, 9, (E,), generator=g, device=dev, dtype=torch.int32)
    rtable = table.clone()
    promo = torch.zeros((18, 2), dtype=torch.int32, device=dev)
    status = torch.zeros(3, dtype=torch.int32, device=dev)
    pool = torch.empty(18 * layer.expert_bytes, dtype=torch.uint8, device=dev)
    # a fixed promotion list for the copy timing: experts 18..35 into slots 0..17
    cpromo = torch.stack([torch.arange(18, 36, dtype=torch.int32, device=dev),
                          torch.arange(18, dtype=torch.int32, device=dev)], dim=1).contiguous()
    cstatus = torch.tensor([18, 18, 0], dtype=torch.int32, device=dev)
    R = T * k
    cases = [
        ("route_topk", lambda: moe.moe_route_topk(lg, k, ids=ids, w=w), T * E * 4 + R * 8),
        ("route_min_weight (0.6)", lambda: moe.moe_route_min_weight(ids2, w2, E, 0.6, slot_table=table), R * 16 + E * 4),
        ("permute + hits", lambda: moe.moe_permute(ids, E, hits=hits, out=perm), R * 4 + R * 8 + E * 12),
        ("route_permute (T=8, one launch)", lambda: moe.moe_route_permute(lg[:8], k, hits=hits,
                                                                          ids_w=(ids[:8], w[:8]), out=perm8),
         8 * E * 4 + 8 * k * 8 + 8 * k * 16 + E * 12),
        ("route_permute (T=1, one launch)", lambda: moe.moe_route_permute(lg[:1], k, hits=hits, ids_w=(ids[:1], w[:1]),
                                                                          out=perm1), E * 4 + k * 8 + k * 16 + E * 12),
        ("combine", lambda: moe.moe_combine(rows, perm[3], w, y), R * H * 4 + R * 8 + T * H * 2),
        ("quantize_int8 (one w13)", lambda: moe.moe_quantize_int8(wq, q8, s8), 2 * I * H * 3 + 2 * I * 4),
        ("quantize_int4 (one w13)", lambda: moe.moe_quantize_int4(wq, q4, s4), 2 * I * H * 2 + I * H + 2 * I * (H // 64) * 2),
        ("refresh_device (18 slots)", lambda: moe.moe_refresh_device(thits, 18, rtable, 18, promo=promo, status=status),
         E * 8),
        ("promote_copies (18 blobs)", lambda: moe.moe_promote_copies(layer.home, pool, layer.expert_bytes, cpromo,
                                                                   cstatus, 18), 2 * 18 * layer.expert_bytes),
    ]
    out = {}
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for name, fn, nbytes in cases:
            fn()
            stream.synchronize()
            if name.startswith("refresh_device"):
                rtable.copy_(table)  # the first call above changed it; replays refresh from the same table
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for _ in range(n):
                    fn()
            graph.replay()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            stream.synchronize()
            a.record(stream)
            graph.replay()
            b.record(stream)
            b.synchronize()
            us = a.elapsed_time(b) * 1e3 / n
            out[name] = {"us": round(us, 2), "alg_bytes": int(nbytes), "gbs": round(nbytes / (us / 1e6) / 1e9, 1)}
            del graph
    return out


def cpu_baseline(moe, torch, cfg_fmt, layers, batches, T, k, seconds, first_token_only=False):
    """The oracle (as it stands) on a bounded sample: whole tokens of batch 0 of
    layer 0, one at a time, until `seconds` have passed."""
    import oracle

    L = layers[0]
    E, H, I = L.E, L.H, L.I
    fmt = L.fmt
    lg, x = batches[0][0], batches[0][1]
    ids, _ = oracle.route_topk(lg, k)
    # host copies of the experts the sample can touch (input bytes, drawn by the
    # seeded generator); the oracle quantises bf16 weights itself for int8/int4
    need = sorted(set(ids.ravel().tolist()))
    eb = oracle.expert_bytes(fmt, H, I)
    slot = np.full(E, -1, np.int32)
    pool = np.zeros(len(need) * eb, np.uint8)
    home_host = None
    if fmt == 0:
        for i, e in enumerate(need):
            slot[e] = i
            pool[i * eb:(i + 1) * eb] = L.home[e * eb:(e + 1) * eb].cpu().numpy()
    else:
        return None  # the quantised formats need the source bf16 weights; bf16 is the benchmarked config
    OL = oracle.Layer(fmt, E, H, I, np.zeros(eb, np.uint8), pool=pool, slot_table=slot)
    # one thread first (a short sample), then every host thread
    oracle.set_threads(1)
    n1, t1 = 0, time.perf_counter()
    while True:
        oracle.moe_layer(OL, lg[n1 % T:n1 % T + 1], x[n1 % T:n1 % T + 1], k)
        n1 += 1
        e1 = time.perf_counter() - t1
        if e1 >= min(seconds / 3, 5.0) or first_token_only:
            break
    oracle.set_threads(os.cpu_count() or 1)
    threads = oracle.get_threads()
    n, t0 = 0, time.perf_counter()
    while True:
        t = n % T  # cycle through the batch's tokens until the time budget is spent
        oracle.moe_layer(OL, lg[t:t + 1], x[t:t + 1], k)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds or first_token_only:
            break
    del home_host
    return {"value": n / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} token evaluations cycling through the {T} tokens of one batch ({n * k} routes), "
                      f"whole layer (route, per-route fp64 FFN, combine), {el:.1f} s",
            "single_thread": {"value": round(n1 / e1, 3), "unit": "tokens/s", "cores": 1,
                              "sample": f"{n1} token evaluations, {e1:.1f} s"}}


def ffn_roofline(T, k, H, I, eb, distinct, ffn_ms, peaks, traffic):
    """Roofline object of the grouped FFN (the dominant kernel) for one workload:
    algorithmic bytes = distinct routed experts x expert_bytes + T*H*2 (x); flops
    = 2*T*k*3*H*I.  Decode batches (T <= 64) are bound by HBM, the prefill batch
    by the tensor pipe (against the sustained bf16 peak; its HBM fraction is
    reported beside it).  `ffn_ms` is the average of the live event pairs."""
    hbm_peak, _, tf_sust, src = peaks
    alg_bytes = distinct * eb + T * H * 2
    gbs = alg_bytes / (ffn_ms / 1e3) / 1e9
    flops = 2.0 * T * k * 3 * H * I
    tflops = flops / (ffn_ms / 1e3) / 1e12
    tr, tr_alg, tr_src = (None, None, None) if traffic is None else traffic
    if T > 64:
        return {"bound": "tensor", "achieved": round(tflops, 1), "peak": tf_sust, "unit": "TFLOP/s",
                "frac": round(tflops / tf_sust, 4), "traffic": tr, "traffic_alg_bytes": tr_alg,
                "traffic_capture": tr_src,
                "peak_source": f"{src} sustained bf16 (bf16_tflops_sustained)",
                "alg_flops_per_launch": flops,
                "hbm": {"achieved_gbs": round(gbs, 1), "peak": hbm_peak, "frac": round(gbs / hbm_peak, 4),
                        "alg_bytes_per_launch": int(alg_bytes)},
                "avg_launch_us": round(ffn_ms * 1e3, 2)}
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(gbs / hbm_peak, 4), "traffic": tr, "traffic_alg_bytes": tr_alg,
            "traffic_capture": tr_src,
            "peak_source": f"{src} (hbm_gbs)", "alg_bytes_per_launch": int(alg_bytes),
            "avg_launch_us": round(ffn_ms * 1e3, 2)}


def run_layer_config(ctx, layers, kind, T, name, seed=0):
    """One layer workload: T tokens per step over the rotated layer copies, steps
    replayed from CUDA graphs with an event pair around every grouped-FFN call.
    Returns (summary dict, runner, step ms list)."""
    moe, torch, args, dev, dist, world = ctx["moe"], ctx["torch"], ctx["args"], ctx["dev"], ctx["dist"], ctx["world"]
    L0 = layers[0]
    E, H, I, k = L0.E, L0.H, L0.I, ctx["k"]
    batches = make_batches(torch, kind, T, E, H, 8, dev, seed=seed)
    runner = Runner(moe, torch, layers, batches, T, k, dev, ctx["path"])
    distinct = runner.distinct_experts()
    ms, ffn_ms = time_steps(torch, runner, args.steps, args.warmup, dist)
    ms = max_over_ranks(dist, ms, dev)
    eb = L0.expert_bytes
    d_avg = sum(distinct[(args.warmup + i) % len(distinct)] for i in range(args.steps)) / args.steps
    f_avg = sum(ffn_ms) / len(ffn_ms)
    fmt_name = {0: "bf16", 1: "int8", 2: "int4"}[L0.fmt]
    workload = f"moe-layer-{fmt_name}-{'prefill' if T > 64 else 'decode'}-T{T}"
    traffic = NCU_TRAFFIC_BYTES.get((workload, args.path))
    out = {
        "workload": workload, "logits": kind,
        "tokens_per_s": round(world * T * args.steps / (ms / 1e3), 1),
        "us_per_step": round(ms / args.steps * 1e3, 2),
        "ffn_us": round(f_avg * 1e3, 2), "ffn_event_pairs": len(ffn_ms),
        "distinct_experts": round(d_avg, 2),
        "layer_hbm_gbs": round((d_avg * eb + T * H * 4 + T * E * 4) / (ms / args.steps / 1e3) / 1e9, 1),
        "roofline": ffn_roofline(T, k, H, I, eb, d_avg, f_avg, ctx["peaks"], traffic),
        "gpu_launches": runner.launches_per_step() * args.steps,
    }
    if T == 1 and ctx["path"] == moe.MOE_FFN_AUTO:
        # the same steps as one moe_layer_forward call each (for one token the
        # routing runs inside the FFN's first launch and the combine inside its
        # second): what a caller of the one-call entry point gets per layer
        r1 = Runner(moe, torch, layers, batches, T, k, dev, ctx["path"], one_call=True)
        ms1, _ = time_steps(torch, r1, args.steps, args.warmup, dist)
        ms1 = max_over_ranks(dist, ms1, dev)
        out["one_call"] = {"tokens_per_s": round(world * T * args.steps / (ms1 / 1e3), 1),
                           "us_per_step": round(ms1 / args.steps * 1e3, 2),
                           "gpu_launches": launches_per_layer(moe, T, k, L0.fmt, ctx["path"], E) * args.steps,
                           "call": "moe_layer_forward"}
        del r1
    return out, runner, ms, batches


def main():
    args = parse()
    fmt_name, kind, T0, sweep = CONFIGS[args.config]
    T = args.tokens or T0
    E, H, I, k = (8, 256, 128, 2) if args.config == "tiny" else (128, 2816, 704, 8)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, fmt_name, kind, T, E, H, I, k, world, rank)
    if args.config == "stack30":
        return stack_main(args, T, E, H, I, k, world, rank, local)
    if args.parallel == "ep":
        return ep_main(args, fmt_name, kind, T, E, H, I, k, world, rank, local)

    import torch

    import moe_router_softmax_b200 as moe

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        dist = tdist

    n_layers = args.layers if args.config != "tiny" else 2
    path = {"auto": moe.MOE_FFN_AUTO, "gemv": moe.MOE_FFN_GEMV, "tc": moe.MOE_FFN_TC}[args.path]
    peaks = measured_peaks()
    ctx = {"moe": moe, "torch": torch, "args": args, "dev": dev, "dist": dist, "world": world, "k": k,
           "path": path, "peaks": peaks}
    layers = build_layers(moe, torch, fmt_name, E, H, I, n_layers, dev)

    clocks = ClockSampler(local)
    clocks.start()
    head, runner, ms, batches = run_layer_config(ctx, layers, kind, T, "headline")
    clk = clocks.stop()
    ms_step = ms / args.steps
    value = whole_job_rate(T * args.steps, world, ms)
    eb = moe.moe_expert_bytes(moe.FMT[fmt_name], H, I)

    sweep_out = {}
    for Ts in ([] if args.quick else sweep):
        s_out, _, _, _ = run_layer_config(ctx, layers, kind, Ts, f"T{Ts}", seed=Ts)
        sweep_out[f"T{Ts}"] = s_out

    kernels = None
    if not args.quick and args.config != "tiny":
        try:
            kernels = time_kernels(torch, moe, layers[0], T, E, H, I, k, dev)
        except Exception as exc:  # keep the headline line even if a side measurement fails
            kernels = {"error": f"{type(exc).__name__}: {exc}"}
    router = {}
    if args.config != "tiny":
        for Tr in ([T] if args.quick else sorted({1, T, 1024})):
            r = time_router(torch, moe, Tr, E, H, k, dev)
            r["frac_of_hbm"] = round(r["hbm_gbs"] / peaks[0], 4)
            router[f"T{Tr}"] = r

    eager_steps = min(args.steps, 500)
    eager_ms = float("nan") if args.quick else time_eager(torch, runner, eager_steps, args.warmup)
    eager_ms = max_over_ranks(dist, eager_ms, dev)
    e2e_ms, h2d, d2h = (float("nan"), 0, 0) if args.quick else time_e2e(torch, moe, layers, batches, T, k,
                                                                         args.steps, args.warmup, dev)
    e2e_ms = max_over_ranks(dist, e2e_ms, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.quick:
        cpu = cpu_baseline(moe, torch, fmt_name, layers, batches, T, k, args.cpu_seconds)

    # the other workloads of the same layer shape, each with its own roofline:
    # int8 decode with skewed routing, int4 decode and prefill, and the 30-layer
    # stacks behind cache slots (int4 and bf16 both resident)
    configs = None
    if args.config == "decode-bf16" and not args.quick and not args.headline_only:
        configs = other_configs(ctx, layers, E, H, I, k, n_layers)

    line = {
        "metric": "MoE layer tokens/s and expert-weight HBM GB/s (% of roofline) at decode/prefill",
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": fmt_name,
        "data": "synthetic (seeded; Gemma-4-26B-A4B-shaped layer, random weights)",
        "config": {
            "workload": head["workload"],
            "ffn_path": args.path,
            "experts": E, "hidden": H, "intermediate": I, "top_k": k, "tokens": T,
            "weights": fmt_name, "logits": kind, "layers_rotated": n_layers,
            "l2": f"inputs larger than L2: each step reads a different one of {n_layers} layer copies "
                  f"({n_layers * E * eb / 1e9:.1f} GB of expert blobs)",
            "parallelism": f"replicas x{world}",
        },
        "layer_hbm_gbs": head["layer_hbm_gbs"],
        "roofline": dict(head["roofline"], kernel="grouped FFN (tcgen05: gather, w13+GELU gate, w2; "
                                                 "GEMV: w13+GELU gate, w2)",
                         ffn_event_pairs=head["ffn_event_pairs"]),
        "sweep": sweep_out,
        "configs": configs,
        "router_topk": router,
        "kernels": kernels,
        "eager": None if args.quick else {
            "tokens_per_s": round(world * T * eager_steps / (eager_ms / 1e3), 1),
            "ms_per_step": round(eager_ms / eager_steps, 5), "steps": eager_steps,
            "note": "the same steps launched from Python one by one (no CUDA graph)"},
        "e2e": {"value": round(world * T * args.steps / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": head["gpu_launches"],
        **({"one_call": head["one_call"]} if "one_call" in head else {}),
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def other_configs(ctx, bf16_layers, E, H, I, k, n_layers):
    """int8 decode (skewed logits) at T = 1, 8, 64; int4 decode T = 64 and prefill
    T = 1024; the 30-layer int4 and bf16 stacks at T = 1, 8, 64.  Each layer
    workload runs the same --steps/--warmup with its own live FFN events."""
    moe, torch, dev = ctx["moe"], ctx["torch"], ctx["dev"]
    out = {}
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    clocks.start()
    l8 = build_layers(moe, torch, "int8", E, H, I, n_layers, dev)
    for Ts in (64, 8, 1):
        out[f"int8-decode-T{Ts}"] = run_layer_config(ctx, l8, "biased", Ts, f"int8-T{Ts}", seed=100 + Ts)[0]
    del l8
    torch.cuda.empty_cache()
    l4 = build_layers(moe, torch, "int4", E, H, I, n_layers, dev)
    out["int4-decode-T64"] = run_layer_config(ctx, l4, "normal", 64, "int4-T64", seed=200)[0]
    out["int4-prefill-T1024"] = run_layer_config(ctx, l4, "normal", 1024, "int4-T1024", seed=300)[0]
    out["stack30"] = stack_configs(ctx, l4, bf16_layers, E, H, I, k)
    del l4
    torch.cuda.empty_cache()
    out["clocks"] = clocks.stop()
    return out


def stack_configs(ctx, l4, l16, E, H, I, k):
    """The 30-layer stacks of the layers already in HBM (int4 and bf16 both
    resident), 18 cache slots per layer, Zipf(1.1) routing, device placement
    refresh every 8 steps, 256 decode steps at T = 1, 8, 64."""
    moe, torch, dev = ctx["moe"], ctx["torch"], ctx["dev"]
    L, slots, steps = min(30, len(l4), len(l16)), 18, 256
    s4 = Stack(moe, torch, "int4", E, H, I, L, slots, dev, homes=l4[:L])
    s16 = Stack(moe, torch, "bf16", E, H, I, L, slots, dev, homes=l16[:L])
    hbm = ctx["peaks"][0]
    out = {"layers": L, "slots_per_layer": slots, "refresh_every": 8, "steps": steps,
           "refresh": "on the device, promotion copies on a second stream; one CUDA graph per 8-step window"}
    for name, st in (("int4", s4), ("bf16", s16)):
        for Ts in (1, 8, 64):
            ms, n, alg = stack_steps_device(torch, moe, st, Ts, k, steps, 8, seed=11 + Ts, path=ctx["path"])
            ms = max_over_ranks(ctx["dist"], ms, dev)
            ms_step = ms / n
            share = st.stats["resident_route_share"]
            out[f"{name}-T{Ts}"] = {
                "tokens_per_s": round(ctx["world"] * Ts * n / (ms / 1e3), 1), "ms_per_step": round(ms_step, 4),
                "roofline": {"bound": "hbm", "unit": "GB/s", "peak": hbm,
                             "achieved": round(alg / (ms_step / 1e3) / 1e9, 1),
                             "frac": round(alg / (ms_step / 1e3) / 1e9 / hbm, 4),
                             "alg_bytes_per_step": int(alg),
                             "note": "whole step of 30 layers (route, permute, FFN, combine, refresh, copies) "
                                     "against the distinct routed experts' bytes"},
                "placement": {"refreshes": st.stats["refreshes"], "promotions": st.stats["promotions"],
                              "demotions": st.stats["demotions"],
                              "routes_on_resident_slots": round(sum(share) / len(share), 4) if share else None},
            }
    del s4, s16
    return out


# ------------------------------------------------------ expert parallelism

def ep_main(args, fmt_name, kind, T, E, H, I, k, world, rank, local):
    """Expert parallelism: rank d holds experts [d*E/N, (d+1)*E/N) of each of the
    rotated layer copies and routes its own T tokens per step; routed rows go to
    their owners and back by NCCL all-to-all.  Eager steps (the split sizes are read
    on the host every step); timed on the device, max over ranks."""
    import datetime
    import socket

    import torch
    import torch.distributed as tdist

    import moe_router_softmax_b200 as moe
    from moe_router_softmax_b200.ep import ExpertParallelLayer, TorchExchange

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if "MASTER_ADDR" not in os.environ:          # one process without torchrun
        sock = socket.socket()
        sock.bind(("127.0.0.1", 0))
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(sock.getsockname()[1]), RANK="0",
                          WORLD_SIZE="1")
        sock.close()
    tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if E % world:
        raise SystemExit(f"E={E} is not a multiple of {world} ranks")
    El = E // world
    n_layers = args.layers if args.config != "tiny" else 2
    layers = build_layers(moe, torch, fmt_name, El, H, I, n_layers, dev, seed=rank)
    eps = [ExpertParallelLayer(L, E, rank, world, TorchExchange()) for L in layers]
    batches = make_batches(torch, kind, T, E, H, 8, dev, seed=rank)
    steps, warmup = args.steps, max(args.warmup, 3)

    def step(i):
        b = batches[i % len(batches)]
        return eps[i % n_layers].forward(b[2], b[3], k)

    for i in range(warmup):
        step(i)
    clocks = ClockSampler(local)
    clocks.start()
    tdist.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        step(warmup + i)
    t1.record()
    torch.cuda.synchronize(dev)
    tdist.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(tdist, t0.elapsed_time(t1), dev)
    line = {
        "metric": "MoE layer tokens/s and expert-weight HBM GB/s (% of roofline) at decode/prefill",
        "value": round(whole_job_rate(T * steps, world, ms), 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": round(ms / steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": fmt_name,
        "data": "synthetic (seeded; Gemma-4-26B-A4B-shaped layer, random weights)",
        "config": {
            "workload": f"moe-layer-{fmt_name}-{'prefill' if T > 64 else 'decode'}-T{T}",
            "experts": E, "hidden": H, "intermediate": I, "top_k": k, "tokens_per_rank": T,
            "weights": fmt_name, "logits": kind, "layers_rotated": n_layers,
            "l2": f"inputs larger than L2: each step reads a different one of {n_layers} layer copies "
                  f"({n_layers * El * moe.moe_expert_bytes(moe.FMT[fmt_name], H, I) / 1e9:.1f} GB per rank)",
            "parallelism": f"expert parallel x{world} ({El} experts per rank, NCCL all-to-all)",
        },
        "roofline": None,
        "gpu_launches": None,
        "clocks": clk,
        "note": "eager steps with one device-to-host read of the split sizes per step",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    tdist.barrier()
    tdist.destroy_process_group()


# ----------------------------------------------------------- the layer stack

class Stack:
    """A stack of MoE layers whose experts are read through per-layer cache slots.

    Every layer has its E home blobs and a pool of `slots` blobs; slot_of[l] (host)
    mirrors the device slot table.  Initial residents are experts 0..slots-1
    (expert_pool.rs, ExpertPool::new)."""

    def __init__(self, moe, torch, fmt_name, E, H, I, L, slots, dev, seed=0, homes=None):
        self.moe, self.torch = moe, torch
        self.homes = homes if homes is not None else build_layers(moe, torch, fmt_name, E, H, I, L, dev, seed=seed)
        self.fmt = moe.FMT[fmt_name]
        self.E, self.H, self.I, self.L, self.slots = E, H, I, L, slots
        self.eb = self.homes[0].expert_bytes
        self.slot_of = []
        self.layers = []
        self.pools = []
        self.tables = torch.empty((L, E), dtype=torch.int32, device=dev)  # row l = layer l's slot table
        for l in range(L):
            so = np.full(E, -1, np.int32)
            so[:slots] = np.arange(slots)
            pool = torch.empty(slots * self.eb, dtype=torch.uint8, device=dev)
            moe.moe_copy_to_slots(self.homes[l].home, pool, self.eb, np.arange(slots), np.arange(slots))
            table = self.tables[l]
            table.copy_(torch.from_numpy(so))
            self.layers.append(moe.MoeLayer(self.fmt, E, H, I, self.homes[l].home, pool=pool, slot_table=table,
                                            expert_bytes=self.eb))
            self.slot_of.append(so)
            self.pools.append(pool)
        self.stats = {"refreshes": 0, "promotions": 0, "demotions": 0, "resident_route_share": []}
        torch.cuda.synchronize(dev)

    def refresh(self, hits_host):
        """Placement refresh of every layer from one step's hit histogram
        (expert_pool.rs: target_gpu_from_counts, then apply_target_placement),
        promotion copies into the freed slots, slot tables uploaded."""
        moe = self.moe
        for l in range(self.L):
            h = hits_host[l]
            tot = int(h.sum())
            if tot:
                self.stats["resident_route_share"].append(float(h[self.slot_of[l] >= 0].sum()) / tot)
            target = moe.moe_refresh_target(h, self.slots)
            so, promote, demote = moe.moe_apply_placement(self.slot_of[l], self.slots, target)
            if len(promote):
                moe.moe_copy_to_slots(self.layers[l].home, self.pools[l], self.eb, promote, so[promote])
                self.layers[l].slot_table.copy_(self.torch.from_numpy(so), non_blocking=False)
            self.slot_of[l] = so
            self.stats["promotions"] += len(promote)
            self.stats["demotions"] += len(demote)
        self.stats["refreshes"] += 1


def stack_steps(torch, moe, stack, T, k, steps, warmup, seed, refresh_every=8, path=0):
    """`steps` decode steps through the whole stack; a placement refresh from the
    hits of every step that is a multiple of `refresh_every`.  Returns total ms."""
    import synthetic as syn

    dev = stack.layers[0].home.device
    E, H, L = stack.E, stack.H, stack.L
    W = refresh_every
    n = steps + warmup
    # inputs of every step, resident in HBM: Zipf(1.1) logits per (step, layer), x per step
    lg_all = torch.empty((n, L, T, E), dtype=torch.float32, device=dev)
    x_all = torch.empty((n, T, H), dtype=torch.bfloat16, device=dev)
    for st in range(n):
        lg_all[st] = torch.from_numpy(np.stack([syn.router_logits(T, E, "zipf", seed=seed, layer=l, step=st)
                                                for l in range(L)])).to(dev)
        x_all[st] = torch.from_numpy(syn.activations(T, H, seed=seed, layer=st).view(np.int16)).to(dev).view(torch.bfloat16)
    lg_stage = torch.empty((W, L, T, E), dtype=torch.float32, device=dev)
    x_stage = torch.empty((W, T, H), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(moe.moe_grouped_ffn_workspace(stack.layers[0], T, k), dtype=torch.uint8, device=dev)
    R = T * k
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    perm = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(R, dtype=torch.int32, device=dev), torch.empty(R, dtype=torch.int32, device=dev))
    rows = torch.empty((R, H), dtype=torch.float32, device=dev)
    ybuf = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    hits = torch.zeros((L, E), dtype=torch.int32, device=dev)

    fws = torch.empty(moe.moe_layer_forward_workspace(stack.layers[0], T, k), dtype=torch.uint8, device=dev)

    def one_step(j, with_hits):
        x = x_stage[j]
        for l in range(L):
            lay = stack.layers[l]
            y = ybuf[l & 1]
            if path == moe.MOE_FFN_AUTO:
                # the whole layer in one call: for one token the routing runs inside
                # the FFN's launches and the combine inside its second one
                moe.moe_layer_forward(lay, lg_stage[j, l], x, k, y=y, hits=hits[l] if with_hits else None,
                                      ids_out=ids, w_out=w, ws=fws)
            else:
                moe.moe_route_permute(lg_stage[j, l], k, hits=hits[l] if with_hits else None, ids_w=(ids, w),
                                      out=perm)
                moe.moe_grouped_ffn(lay, x, k, perm[0], perm[1], perm[2], rows=rows, ws=ws, path=path)
                moe.moe_combine(rows, perm[3], w, y)
            x = y

    def window_inputs(first):
        m = min(W, n - first)
        lg_stage[:m].copy_(lg_all[first:first + m])
        x_stage[:m].copy_(x_all[first:first + m])

    # prime one-time set-up, then capture: graph A = the refresh step (with hits),
    # graph B = the W-1 steps after it
    window_inputs(0)
    one_step(0, True)
    torch.cuda.synchronize()
    hits.zero_()
    ga, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(ga):
        one_step(0, True)
    with torch.cuda.graph(gb):
        for j in range(1, W):
            one_step(j, False)
    torch.cuda.synchronize()

    def run(first, count):
        st = first
        while st < first + count:
            window_inputs(st)
            hits.zero_()
            ga.replay()                                # step st (a multiple of W): counts hits
            stack.refresh(hits.cpu().numpy().view(np.uint32))  # syncs on the hit histogram
            rest = min(W - 1, first + count - st - 1)
            if rest == W - 1:
                gb.replay()
            else:
                for j in range(1, 1 + rest):
                    one_step(j, False)
            st += 1 + rest

    run(0, warmup)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    run(warmup, steps)
    t1.record()
    torch.cuda.synchronize()
    return t0.elapsed_time(t1)


def stack_steps_device(torch, moe, stack, T, k, steps, warmup, seed, refresh_every=8, path=0):
    """The same decode steps with the placement refresh done on the device
    (moe_refresh_device after each layer's forward at the refresh step, its
    promotion copies on a second stream, joined before that layer's next
    forward), so that a window of `refresh_every` steps is one CUDA graph with
    no host round trip and the copies overlap the following layers' compute.
    `steps` and `warmup` are rounded up to whole windows.  Returns (total ms,
    steps timed, algorithmic bytes per timed step: the distinct routed experts'
    blobs of every layer plus each layer's x, y and logits).  The distinct
    experts come from a host top-k of the same logits (continuous draws: no
    ties)."""
    import synthetic as syn

    dev = stack.layers[0].home.device
    E, H, L, S = stack.E, stack.H, stack.L, stack.slots
    W = refresh_every
    steps = -(-steps // W) * W
    warmup = max(1, -(-warmup // W)) * W
    n = steps + warmup
    lg_all = torch.empty((n, L, T, E), dtype=torch.float32, device=dev)
    x_all = torch.empty((n, T, H), dtype=torch.bfloat16, device=dev)
    distinct = 0
    for st in range(n):
        lg_h = np.stack([syn.router_logits(T, E, "zipf", seed=seed, layer=l, step=st) for l in range(L)])
        if st >= warmup:
            top = np.argpartition(-lg_h, k - 1, axis=2)[:, :, :k].reshape(L, -1)
            distinct += sum(np.unique(top[l]).size for l in range(L))
        lg_all[st] = torch.from_numpy(lg_h).to(dev)
        x_all[st] = torch.from_numpy(syn.activations(T, H, seed=seed, layer=st).view(np.int16)).to(dev).view(torch.bfloat16)
    alg_step = distinct / steps * stack.eb + L * (T * H * 4 + T * E * 4)
    lg_stage = torch.empty((W, L, T, E), dtype=torch.float32, device=dev)
    x_stage = torch.empty((W, T, H), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(moe.moe_grouped_ffn_workspace(stack.layers[0], T, k), dtype=torch.uint8, device=dev)
    R = T * k
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    perm = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(R, dtype=torch.int32, device=dev), torch.empty(R, dtype=torch.int32, device=dev))
    rows = torch.empty((R, H), dtype=torch.float32, device=dev)
    ybuf = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    hits = torch.zeros((L, E), dtype=torch.int32, device=dev)
    promo = torch.zeros((L, S, 2), dtype=torch.int32, device=dev)
    status = torch.zeros((L, 3), dtype=torch.int32, device=dev)
    snap = torch.empty((L, E), dtype=torch.int32, device=dev)
    acc = torch.zeros(4, dtype=torch.int64, device=dev)  # promotions, demotions, resident routes, routes
    side = torch.cuda.Stream(dev)

    fws = torch.empty(moe.moe_layer_forward_workspace(stack.layers[0], T, k), dtype=torch.uint8, device=dev)

    def layer(j, l, x):
        y = ybuf[l & 1]
        if path == moe.MOE_FFN_AUTO:
            # the whole layer in one call: for one token the routing runs inside
            # the FFN's launches and the combine inside its second one
            moe.moe_layer_forward(stack.layers[l], lg_stage[j, l], x, k, y=y, hits=hits[l] if j == 0 else None,
                                  ids_out=ids, w_out=w, ws=fws)
        else:
            moe.moe_route_permute(lg_stage[j, l], k, hits=hits[l] if j == 0 else None, ids_w=(ids, w), out=perm)
            moe.moe_grouped_ffn(stack.layers[l], x, k, perm[0], perm[1], perm[2], rows=rows, ws=ws, path=path)
            moe.moe_combine(rows, perm[3], w, y)
        return y

    def window():
        main = torch.cuda.current_stream()
        hits.zero_()
        snap.copy_(stack.tables)
        done = []
        x = x_stage[0]
        for l in range(L):
            x = layer(0, l, x)
            moe.moe_refresh_device(hits[l], S, stack.tables[l], S, promo=promo[l], status=status[l])
            ev = torch.cuda.Event()
            ev.record(main)
            side.wait_event(ev)
            with torch.cuda.stream(side):
                moe.moe_promote_copies(stack.homes[l].home, stack.pools[l], stack.eb, promo[l], status[l], S)
                ev2 = torch.cuda.Event()
                ev2.record(side)
            done.append(ev2)
        acc[0] += status[:, 0].sum()
        acc[1] += status[:, 1].sum()
        acc[2] += (hits * (snap >= 0)).sum()
        acc[3] += hits.sum()
        for j in range(1, W):
            x = x_stage[j]
            for l in range(L):
                if j == 1:
                    main.wait_event(done[l])  # layer l's promoted blobs and table are in place
                x = layer(j, l, x)
        main.wait_stream(side)

    def window_inputs(first):
        lg_stage.copy_(lg_all[first:first + W])
        x_stage.copy_(x_all[first:first + W])

    window_inputs(0)
    window()  # one-time set-up outside the capture (it also performs a refresh)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        window()
    torch.cuda.synchronize()
    acc.zero_()

    def run(first, count):
        for st in range(first, first + count, W):
            window_inputs(st)
            g.replay()

    run(0, warmup)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    run(warmup, steps)
    t1.record()
    torch.cuda.synchronize()
    a = acc.cpu().numpy()
    windows = (warmup + steps) // W
    stack.stats = {"refreshes": windows, "promotions": int(a[0]), "demotions": int(a[1]),
                   "resident_route_share": [float(a[2]) / float(a[3])] if a[3] else []}
    del g
    return t0.elapsed_time(t1), steps, alg_step


def stack_main(args, T, E, H, I, k, world, rank, local):
    """30-layer stacks (int4 and bf16, both resident), 18 cache slots per layer,
    Zipf(1.1) routing, placement refresh every 8 steps; tokens/s through the stack."""
    import torch

    import moe_router_softmax_b200 as moe

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    L, slots = (args.layers if args.layers != 30 else 30), 18
    steps = args.steps if args.steps != 3000 else 256
    warmup = max(args.warmup if args.warmup != 30 else 8, 3)
    path = {"auto": moe.MOE_FFN_AUTO, "gemv": moe.MOE_FFN_GEMV, "tc": moe.MOE_FFN_TC}[args.path]
    s4 = Stack(moe, torch, "int4", E, H, I, L, slots, dev, seed=1)
    s16 = Stack(moe, torch, "bf16", E, H, I, L, slots, dev, seed=2)
    device_refresh = args.stack_refresh == "device"

    def run_stack(st, Ts, seed):
        if device_refresh:
            return stack_steps_device(torch, moe, st, Ts, k, steps, warmup, seed=seed, path=path)[:2]
        return stack_steps(torch, moe, st, Ts, k, steps, warmup, seed=seed, path=path), steps

    resident_gb = (sum(h.home.numel() for h in s4.homes) + sum(h.home.numel() for h in s16.homes) +
                   sum(p.numel() for p in s4.pools) + sum(p.numel() for p in s16.pools)) / 1e9
    clocks = ClockSampler(local)
    clocks.start()
    ms, steps_done = run_stack(s4, T, 11)
    clk = clocks.stop()
    value = world * T * steps_done / (ms / 1e3)
    sweep = {}
    for name, st, Ts in [("bf16", s16, T)] + ([] if args.quick else [("int4", s4, t) for t in (1, 8) if t != T]):
        ms2, n2 = run_stack(st, Ts, 12 + Ts)
        sweep[f"{name}_T{Ts}"] = {"tokens_per_s": round(world * Ts * n2 / (ms2 / 1e3), 1),
                                  "ms_per_step": round(ms2 / n2, 4)}
    share = s4.stats["resident_route_share"]
    hbm_peak = measured_peaks()[0]
    line = {
        "metric": "MoE layer tokens/s and expert-weight HBM GB/s (% of roofline) at decode/prefill",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": steps_done, "warmup": warmup,
        "ms_per_step": round(ms / steps_done, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4", "data": "synthetic (seeded; Zipf(1.1) routing; random weights)",
        "config": {"workload": f"moe-stack{L}-int4-decode-T{T}", "layers": L, "experts": E, "hidden": H,
                   "intermediate": I, "top_k": k, "tokens": T, "slots_per_layer": slots, "refresh_every": 8,
                   "refresh": ("on the device, promotion copies on a second stream overlapping compute; one CUDA "
                               "graph per 8-step window" if device_refresh else
                               "on the host (hit histogram read back, placement, copies, table upload)"),
                   "logits": "zipf(1.1)", "resident_gb": round(resident_gb, 1), "ffn_path": args.path,
                   "l2": "inputs larger than L2: each step reads 30 layers' routed experts"},
        "placement": {"refreshes": s4.stats["refreshes"], "promotions": s4.stats["promotions"],
                      "demotions": s4.stats["demotions"],
                      "routes_on_resident_slots": round(sum(share) / len(share), 4) if share else None},
        "sweep": sweep,
        "hbm_peak_gbs": hbm_peak,
        "gpu_launches": steps_done * L * launches_per_layer(moe, T, k, s4.fmt, path, s4.E)
                        + (steps_done // 8) * L * (2 if device_refresh else 0),
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def reference_arm(args, fmt_name, kind, T, E, H, I, k, world, rank):
    """The CPU oracle on the same workload: each step is one token of the batch
    (k routes through the fp64 per-route FFN), on every host core; rank 0 only."""
    if rank != 0:
        return
    import oracle
    import synthetic as syn

    if fmt_name != "bf16":
        print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the bf16 layer only"}))
        return
    eb = oracle.expert_bytes(0, H, I)
    lg = syn.router_logits(T, E, kind, seed=17, layer=0)
    x = syn.activations(T, H, seed=23, layer=0)
    ids, _ = oracle.route_topk(lg, k)
    need = sorted(set(ids.ravel().tolist()))
    w13, w2 = {}, {}
    for e in need:  # the experts of this batch, drawn by the seeded host generator
        a = syn.normal_bf16((1, 2 * I, H), syn.WEIGHT_STD, 0, syn.S_W13, 0, e)
        b = syn.normal_bf16((1, H, I), syn.WEIGHT_STD, 0, syn.S_W2, 0, e)
        w13[e], w2[e] = a[0], b[0]
    slot = np.full(E, -1, np.int32)
    pool = np.zeros(len(need) * eb, np.uint8)
    for i, e in enumerate(need):
        slot[e] = i
        pool[i * eb:(i + 1) * eb] = oracle.pack_expert(0, H, I, w13[e], None, w2[e], None)
    OL = oracle.Layer(0, E, H, I, np.zeros(eb, np.uint8), pool=pool, slot_table=slot)
    oracle.set_threads(os.cpu_count() or 1)
    for i in range(args.warmup):
        t = i % T
        oracle.moe_layer(OL, lg[t:t + 1], x[t:t + 1], k)
    t0 = time.perf_counter()
    for i in range(args.steps):
        t = (args.warmup + i) % T
        oracle.moe_layer(OL, lg[t:t + 1], x[t:t + 1], k)
    el = time.perf_counter() - t0
    value = args.steps / el
    cores = oracle.get_threads()
    print(json.dumps({
        "impl": "reference",
        "metric": "MoE layer tokens/s and expert-weight HBM GB/s (% of roofline) at decode/prefill",
        "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"moe-layer-{fmt_name}-decode-T{T}", "experts": E, "hidden": H,
                   "intermediate": I, "top_k": k, "tokens": T, "weights": fmt_name, "logits": kind},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step one token of the {T}-token batch ({k} routes), "
                                   f"{args.steps} steps"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    main()
