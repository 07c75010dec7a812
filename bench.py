#!/usr/bin/env python
"""Benchmark of the MoE-layer forward (tokens/s) on 1..N B200s.

A step is one full layer forward (router -> top-k -> permute -> grouped SwiGLU
FFN -> combine) over one batch of synthetic tokens. Default workload: the
decode-shaped layer (H=2048, E=128, top-8, I=768, MXFP4 experts, bf16
activations, uniform routing) at T=64 tokens; T=1, T=8 and the prefill-shaped
NVFP4 layer (T=4096, Zipf-skewed routing) are reported alongside under "extra".

Timing: W warm-up steps, then K steps bracketed by a barrier and a device
synchronise, timed with CUDA events on the launching stream, max over ranks.
Every step replays a CUDA graph of the layer on one of NSETS copies of the
expert weights (and one of NSETS activation batches), so consecutive steps
read weights that are not in L2 ("inputs larger than L2").
Multi-GPU: replicas only (the layer has no exchange step); value = tokens of
all ranks / max time.

--impl reference times the CPU oracle (the plain C reference of the same math)
on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

NSETS = 16
L2_BYTES = 126 * 2**20


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------------------------------- clocks


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every 20 ms
    during the timed region (read-only queries; no setting is changed)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None

    def _handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(self.device)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def _run(self):
        import pynvml

        while not self._stop.is_set():
            try:
                self.samples.append(pynvml.nvmlDeviceGetClockInfo(self._h, pynvml.NVML_CLOCK_SM))
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.02)

    def __enter__(self):
        try:
            import pynvml

            self._h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self._h = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join(timeout=2)

    def summary(self):
        sm = self.samples
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------- workload


def active_expert_bytes(idx: torch.Tensor, layer) -> int:
    """Bytes of the experts that received at least one token (codes + scales)."""
    E = layer.E
    used = torch.bincount(idx.reshape(-1).long(), minlength=E) > 0
    per = synthetic.expert_bytes(layer.fmt, layer.H, layer.I)
    return int(used.sum().item()) * per


class LayerBench:
    """One layer configuration: NSETS weight copies, NSETS token batches, a graph per pair, and
    one graph of all NSETS calls in order (consecutive layer calls in one graph, as a serving
    engine captures a whole decode step: no graph launch between the layers)."""

    def __init__(self, moe, cfg: str, T: int, device, seed: int = 0, nsets: int = NSETS, act: str = "a16"):
        self.moe, self.cfg, self.T, self.dev, self.act = moe, cfg, T, device, act
        c = synthetic.CONFIGS[cfg]
        self.k, self.y32 = c["k"], c["y_fp32"]
        base = synthetic.make_layer(cfg, seed, device=device)
        self.layer = base
        # weights are prepacked once into the tiled layout (model-load work, not timed)
        tiled = moe.moe_prepack(moe.Experts.from_layer(base))
        del base.w13, base.w2, base.w13_scale, base.w2_scale
        self.sets = [base] * nsets
        self.experts = [tiled] + [self._clone(moe, tiled) for _ in range(nsets - 1)]
        self.xs = [synthetic.make_tokens(T, base.H, seed=100 + i, device=device) for i in range(nsets)]
        self.ws = torch.empty(moe.moe_workspace_size(T, base.H, base.I, base.E, self.k, self.y32),
                              dtype=torch.uint8, device=device)
        self.out = torch.empty(T, base.H, dtype=torch.bfloat16, device=device)
        self.idx = [torch.empty(T, self.k, dtype=torch.int32, device=device) for _ in range(nsets)]
        self.w = [torch.empty(T, self.k, dtype=torch.float32, device=device) for _ in range(nsets)]
        self.graphs = None

    @staticmethod
    def _clone(moe, ex):
        """The same tiled weights at another address (defeats L2 reuse across steps)."""
        return moe.Experts(ex.fmt, ex.E, ex.H, ex.I, ex.w13.clone(), ex.w2.clone(), None, None, ex.w13_tscale,
                           ex.w2_tscale, layout=ex.layout)

    def call(self, i: int):
        j = i % len(self.sets)
        s = self.sets[j]
        self.moe.moe_layer_forward(self.xs[j], s.wr, self.k, self.experts[j], bias=s.bias, y_fp32=self.y32,
                                   ws=self.ws, out=self.out, idx_out=self.idx[j], w_out=self.w[j], act=self.act)

    def capture(self):
        self.graphs = []
        st = torch.cuda.Stream(self.dev)
        st.wait_stream(torch.cuda.current_stream(self.dev))
        n0 = self.moe.moe_kernel_launch_count()
        with torch.cuda.stream(st):
            for j in range(len(self.sets)):   # warm the launch paths before capture
                self.call(j)
        # kernels one layer call enqueues (the captured graphs replay exactly these)
        self.launches_per_call = (self.moe.moe_kernel_launch_count() - n0) / len(self.sets)
        torch.cuda.current_stream(self.dev).wait_stream(st)
        torch.cuda.synchronize(self.dev)
        for j in range(len(self.sets)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.call(j)
            self.graphs.append(g)
        self.seq = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.seq):
            for j in range(len(self.sets)):
                self.call(j)
        torch.cuda.synchronize(self.dev)

    def step(self, i: int):
        self.graphs[i % len(self.graphs)].replay()

    def run(self, i0: int, n: int):
        """Steps i0 .. i0 + n - 1: whole replays of the sequence graph where a block of NSETS
        steps starts at a multiple of NSETS, single-call graphs for the rest."""
        ns = len(self.graphs)
        i, end = i0, i0 + n
        while i < end:
            if i % ns == 0 and end - i >= ns:
                self.seq.replay()
                i += ns
            else:
                self.graphs[i % ns].replay()
                i += 1

    def algorithmic_bytes(self, i: int) -> int:
        """Algorithmic bytes of one layer: router weights + experts with >= 1 token + x in + out."""
        j = i % len(self.sets)
        s = self.sets[j]
        router = s.wr.numel() * s.wr.element_size()
        return router + active_expert_bytes(self.idx[j], s) + 2 * self.T * s.H * 2

    def flops(self) -> float:
        s = self.layer
        return 2.0 * self.T * s.H * s.E + self.T * self.k * 6.0 * s.H * s.I


def time_steps(fn, K: int, W: int, device, barrier=None, run=None):
    """W untimed steps, then exactly K timed steps (fn(i) runs step i; run(i0, n), when
    given, runs steps i0 .. i0 + n - 1 instead)."""
    if run:
        run(0, W)
    else:
        for i in range(W):
            fn(i)
    torch.cuda.synchronize(device)
    if barrier:
        barrier()
    st = torch.cuda.current_stream(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    if run:
        run(W, K)
    else:
        for i in range(K):
            fn(W + i)
    e1.record(st)
    torch.cuda.synchronize(device)
    if barrier:
        barrier()
    return e0.elapsed_time(e1) / 1e3


def time_passes(fn, K: int, W: int, device, barrier, world, min_s: float = 0.5, max_passes: int = 400, run=None):
    """Timed regions of exactly K steps each (barrier + synchronise on both sides, CUDA
    events on the launching stream, max over ranks), repeated until together they span
    min_s, so the clock sampler sees the load; returns the per-pass seconds. Every rank
    runs the same number of passes (decided from the slowest rank's first pass)."""
    first = max_over_ranks(time_steps(fn, K, W, device, barrier, run), world, device)
    n = int(max(1, min(max_passes, math.ceil(min_s / max(first, 1e-9)))))
    out = [first]
    for p in range(1, n):
        out.append(max_over_ranks(time_steps(fn, K, 0, device, barrier, run), world, device))
    return out


def time_ffn_only(moe, lb: LayerBench, K: int, W: int, device):
    """Average duration of the grouped FFN call (gate/up + down launches) on the same data."""
    T, k = lb.T, lb.k
    P = T * k
    # permuted operands per set, prepared once (untimed)
    prep = []
    for j in range(len(lb.sets)):
        off, _, _, xp = moe.moe_permute(lb.idx[j], lb.layer.E, lb.xs[j])
        prep.append((xp, off))
    ws = torch.empty(moe.moe_workspace_size(P, lb.layer.H, lb.layer.I, lb.layer.E, 1, lb.y32), dtype=torch.uint8,
                     device=device)

    def fn(i):
        j = i % len(prep)
        moe.moe_grouped_ffn(prep[j][0], prep[j][1], lb.experts[j], y_fp32=lb.y32, ws=ws)

    sec = time_steps(fn, K, W, device)
    nbytes = []
    for j in range(len(lb.sets)):
        nbytes.append(active_expert_bytes(lb.idx[j], lb.sets[j]) + 2 * P * lb.layer.H * 2)
    # average algorithmic bytes over the rotation, weighted like the timed calls
    avg_bytes = sum(nbytes[(W + i) % len(nbytes)] for i in range(K)) / K
    return sec / K, avg_bytes


def source_sha():
    h = hashlib.sha256()
    for f in ("ffn_tc.cu", "ffn_mx.cu", "mx_codec.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "expert_ffn_layer_top_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(key: str):
    p = os.path.join(ROOT, "profiles", "ffn_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("src_sha") != source_sha():
            return None
        return d.get(key)
    except Exception:
        return None


# ------------------------------------------------------------------------------------------- arms


def tensor_peaks(moe) -> dict:
    """Dense tensor-core peaks of this GPU for the FFN's MMA kinds, from the library's own
    MMA loop (tcgen05, operands resident in shared memory, no memory traffic): TFLOP/s."""
    out = {}
    fn = getattr(moe, "moe_tensor_peak_tflops", None)
    if fn is None:
        return out
    for kind in ("bf16", "fp8", "mxfp4", "nvfp4"):
        try:
            out[f"{kind}_tflops"] = fn(kind)
        except Exception as exc:   # report, do not fail the bench
            out[f"{kind}_error"] = str(exc)[:120]
    return out


def cpu_oracle_tokens_per_s(cfg: str, T: int, budget_s: float = 12.0):
    import oracle

    L = synthetic.make_layer(cfg, 0)
    xs = [synthetic.make_tokens(T, L.H, seed=100 + i) for i in range(4)]
    n = 0
    t0 = time.time()
    while True:
        oracle.layer_forward(xs[n % len(xs)], L)
        n += 1
        if time.time() - t0 > budget_s:
            break
    dt = time.time() - t0
    return n * T / dt, oracle.threads(), f"{n} full {cfg} layer forward(s) at T={T} ({dt:.1f} s)"


HEADLINE_CONFIG = {"workload": "decode-shaped MoE layer, MXFP4 experts, T=64", "H": 2048, "E": 128, "k": 8,
                   "I": 768, "T": 64}


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (the job's time); a no-op at world size 1."""
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, rank, world):
    """The oracle (C, OpenMP on the host cores) on the headline workload.

    A step is the oracle's layer forward on S tokens of a T = 64 decode batch
    (rotating through the batch and four batches), S = 64 when the whole
    warm-up + timed run fits in about two minutes, else the largest S that
    does (at least 1). Under torchrun only rank 0 runs."""
    if rank != 0:
        return
    import oracle

    L = synthetic.make_layer("decode", 0)
    xs = [synthetic.make_tokens(64, L.H, seed=100 + i) for i in range(4)]
    t0 = time.time()
    oracle.layer_forward(xs[0], L)
    t64 = time.time() - t0
    n = args.warmup + args.steps
    budget = 120.0
    S = 64 if n * t64 <= budget else max(1, int(64 * budget / (n * t64)))
    if S < 64:   # small batches reuse fewer dequantised experts: re-check the cost at S
        while True:
            t0 = time.time()
            oracle.layer_forward(xs[1][:S], L)
            if S == 1 or n * (time.time() - t0) <= budget:
                break
            S = max(1, S // 2)

    def step(i):
        x = xs[(i * S // 64) % len(xs)]
        o = (i * S) % 64
        oracle.layer_forward(x[o:o + S] if o + S <= 64 else torch.cat([x[o:], x[:o + S - 64]]), L)

    for i in range(args.warmup):
        step(i)
    t0 = time.time()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.time() - t0
    tps = args.steps * S / dt
    sample = (f"{args.steps} timed steps, each one oracle layer forward of {S} of the 64 tokens of a decode batch "
              f"({dt:.1f} s)")
    line = {
        "impl": "reference", "metric": "moe_layer_tokens_per_s", "value": tps, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; weights N(0,0.02) quantised, x N(0,1))",
        "config": dict(HEADLINE_CONFIG, parallelism="host cores (oracle)"),
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_stack(moe, device, steps: int) -> dict:
    """The streaming stack: 43 FP8 layers whose experts live in pinned host memory (prepacked), a
    24 GB device LRU cache in front of them, T = 4 decode steps chained through the layers with a
    residual, routing popularity alternating between two Zipf(1.2) permutations per layer every
    128 steps. Reports tokens/s, the cache hit rate and the H2D bandwidth of its copies."""
    c = synthetic.CONFIGS["stack"]
    L_, E_, H_, k_, T_ = c["layers"], c["E"], c["H"], c["k"], c["T"][0]
    host, shapes, routers = [], [], []
    try:
        for l in range(L_):
            lay = synthetic.make_layer("stack", 0, device=device, layer=l)
            ex = moe.Experts.from_layer(lay)
            packed = moe.moe_prepack(ex)
            w13 = torch.empty(packed.w13.shape, dtype=torch.uint8, pin_memory=True)
            w2 = torch.empty(packed.w2.shape, dtype=torch.uint8, pin_memory=True)
            w13.copy_(packed.w13)
            w2.copy_(packed.w2)
            host.append(moe.Experts(packed.fmt, packed.E, packed.H, packed.I, w13, w2, layout=moe.LAYOUT_TILED))
            shapes.append(host[-1])   # with a cache only the format and sizes of the shape are read
            g = torch.Generator().manual_seed(9000 + l)
            perms = (torch.randperm(E_, generator=g), torch.randperm(E_, generator=g))
            biases = [synthetic.zipf_bias(E_, c["zipf"], H_, 0, perm=pm).to(device) for pm in perms]
            routers.append((lay.wr, biases))
            del lay, ex, packed
        torch.cuda.empty_cache()
    except RuntimeError as exc:   # host memory for the pool
        return {"unavailable": f"could not build the pinned expert pool: {exc}"[:200]}
    cache = moe.ExpertCache(int(c["cache_bytes"]), host, device=device.index)
    ws = torch.empty(moe.moe_workspace_size(T_, H_, c["I"], E_, k_), dtype=torch.uint8, device=device)
    drift = c["drift_every"]
    torch.cuda.synchronize(device)
    t0 = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for step in range(steps):
        x = synthetic.make_tokens(T_, H_, seed=50000 + step, device=device)
        for l in range(L_):
            wr, biases = routers[l]
            out = moe.moe_layer_forward(x, wr, k_, shapes[l], bias=biases[(step // drift) % 2], cache=cache,
                                        layer=l, ws=ws)
            x = (x.float() + out.float()).to(torch.bfloat16)
    e1.record()
    torch.cuda.synchronize(device)
    sec = e0.elapsed_time(e1) / 1e3
    st = cache.stats()
    rep = cache.report()
    cache.close()
    refs = st["hits"] + st["misses"]
    return {"tokens_per_s": T_ * steps / sec, "seconds": sec, "steps": steps, "layers": L_, "T": T_,
            "cache_bytes": int(c["cache_bytes"]), "hit_rate": st["hits"] / refs if refs else None,
            "hits": st["hits"], "misses": st["misses"], "h2d_bytes": st["bytes_h2d"],
            "h2d_gbs": st["bytes_h2d"] / st["copy_s"] / 1e9 if st["copy_s"] > 0 else None,
            # share of the timed region in which the copy stream was copying (the copies overlap the layers)
            "copy_s": st["copy_s"], "copy_busy_frac": st["copy_s"] / sec if sec > 0 else None,
            **_cache_breakdown(rep, sec), "wall_s": time.time() - t0}


def _cache_breakdown(rep: dict, sec: float) -> dict:
    """Where a cached run's time went, from the cache's own event and host timers."""
    per = 1e6 / max(rep["calls"], 1)
    return {"overlap_pct": 100.0 * rep["overlap_s"] / rep["copy_s"] if rep["copy_s"] > 0 else None,
            "us_per_call": {"total": sec * per, "table_update": rep["table_s"] * per,
                            "host_wait": rep["host_wait_s"] * per, "copy_issue": rep["issue_s"] * per,
                            "ffn_and_combine": rep["compute_s"] * per, "copy": rep["copy_s"] * per},
            "prefetched_experts": rep["prefetched"]}


def run_prefill_stack(moe, device, n_layers: int = 6, passes: int = 2, T: int = 4096) -> dict:
    """Full-layer double-buffered prefill streaming: n_layers FP8 layers of the streaming-stack
    shape in pinned host memory behind a device cache of three layers' slots, prefill batches of
    T = 4096 tokens (Zipf(1.2) routing reaches nearly every expert), with the whole next layer
    streamed in while each layer computes. Reports tokens/s per layer pass, the host-to-device
    rate and how much of the copying the layers' compute overlapped."""
    c = synthetic.CONFIGS["stack"]
    E_, H_, k_ = c["E"], c["H"], c["k"]
    host, routers = [], []
    try:
        for l in range(n_layers):
            lay = synthetic.make_layer("stack", 1, device=device, layer=l)
            packed = moe.moe_prepack(moe.Experts.from_layer(lay))
            w13 = torch.empty(packed.w13.shape, dtype=torch.uint8, pin_memory=True)
            w2 = torch.empty(packed.w2.shape, dtype=torch.uint8, pin_memory=True)
            w13.copy_(packed.w13)
            w2.copy_(packed.w2)
            host.append(moe.Experts(packed.fmt, packed.E, packed.H, packed.I, w13, w2, layout=moe.LAYOUT_TILED))
            routers.append((lay.wr, lay.bias))
            del lay, packed
        torch.cuda.empty_cache()
    except RuntimeError as exc:
        return {"unavailable": f"could not build the pinned expert pool: {exc}"[:200]}
    slot = moe.moe_prepacked_expert_bytes("fp8", H_, c["I"], 0) + moe.moe_prepacked_expert_bytes("fp8", H_, c["I"], 1)
    cache = moe.ExpertCache(3 * E_ * slot, host, device=device.index)
    cache.set_prefetch("full_layer")
    ws = torch.empty(moe.moe_workspace_size(T, H_, c["I"], E_, k_), dtype=torch.uint8, device=device)
    out = torch.empty(T, H_, dtype=torch.bfloat16, device=device)
    x0 = synthetic.make_tokens(T, H_, seed=60000, device=device)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for p in range(passes):
        x = x0
        for l in range(n_layers):
            wr, bias = routers[l]
            moe.moe_layer_forward(x, wr, k_, host[l], bias=bias, cache=cache, layer=l, ws=ws, out=out)
            x = (x.float() + out.float()).to(torch.bfloat16)
    e1.record()
    torch.cuda.synchronize(device)
    sec = e0.elapsed_time(e1) / 1e3
    st = cache.stats()
    rep = cache.report()
    cache.close()
    calls = passes * n_layers
    return {"tokens_per_s_per_layer": T * calls / sec, "ms_per_layer": sec / calls * 1e3, "layers": n_layers,
            "passes": passes, "T": T, "policy": "full_layer", "cache_slots": rep["n_slots"],
            "hits": st["hits"], "misses": st["misses"], "h2d_bytes": st["bytes_h2d"],
            "h2d_gbs": st["bytes_h2d"] / st["copy_s"] / 1e9 if st["copy_s"] > 0 else None,
            "copy_busy_frac": st["copy_s"] / sec if sec > 0 else None, **_cache_breakdown(rep, sec)}


def run_ours(args, rank, world, device):
    import expert_ffn_layer_top_b200 as moe

    barrier = None
    if world > 1:
        import torch.distributed as dist

        def barrier():
            dist.barrier(device_ids=[device.index])

    hbm, bf16_tf, peak_kind = _peaks()
    lb = LayerBench(moe, "decode", 64, device)
    lb.capture()
    extra = {}
    launches_per_step = lb.launches_per_call
    with ClockSampler(device) as clk:
        passes = time_passes(lb.step, args.steps, args.warmup, device, barrier, world, run=lb.run)
    clocks = clk.summary()
    sec = statistics.median(passes)
    tokens = lb.T * args.steps * world
    value = tokens / sec
    ms = sec / args.steps * 1e3
    # layer roofline context (algorithmic bytes of the steps just timed)
    alg = [lb.algorithmic_bytes(args.warmup + i) for i in range(min(args.steps, NSETS))]
    layer_gbs = (sum(alg) / len(alg)) / (ms * 1e-3) / 1e9

    # dominant kernel: the grouped FFN call, timed alone with events on the same rotation
    ffn_s, ffn_bytes = time_ffn_only(moe, lb, max(args.steps, 20), args.warmup, device)
    achieved = ffn_bytes / ffn_s / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": traffic_for("decode64_bytes_per_call"), "kernel": "grouped SwiGLU FFN call (MXFP4 block-scaled: mx_quant_kernel + ffn_mx_kernel up + down)",
                "peak_kind": peak_kind, "layer_achieved_gbs": layer_gbs,
                "frac_of_nominal_8000_gbs": achieved / 8000.0}

    # end to end through the C ABI with host buffers: every step copies its x in from pinned host memory and
    # its output back to pinned host memory. As in a serving loop, the copies run on two more streams (one
    # per direction, so neither queues behind the other) with double buffers: step i+1's input and step
    # i-1's output move while step i computes. The timed region ends when the last output has reached the
    # host.
    xh = [x.cpu().pin_memory() for x in lb.xs]
    oh = [torch.empty(lb.T, lb.layer.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(lb.xs[0]) for _ in range(2)]
    od = [torch.empty_like(lb.out) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    cs = torch.cuda.current_stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):
        ev_done[b].record(cs)
        ev_out[b].record(cs)

    def e2e_step(i):
        j, b = i % NSETS, i & 1
        with torch.cuda.stream(h2d):
            h2d.wait_event(ev_done[b])         # the layer that last read xd[b] has finished
            xd[b].copy_(xh[j], non_blocking=True)
            ev_in[b].record(h2d)
        cs.wait_event(ev_in[b])
        cs.wait_event(ev_out[b])               # od[b]'s previous contents have reached the host
        s = lb.sets[j]
        moe.moe_layer_forward(xd[b], s.wr, lb.k, lb.experts[j], bias=s.bias, ws=lb.ws, out=od[b])
        ev_done[b].record(cs)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_done[b])
            oh[b].copy_(od[b], non_blocking=True)
            ev_out[b].record(d2h)

    def e2e_steps(K: int, W: int):
        for i in range(W):
            e2e_step(i)
        torch.cuda.synchronize(device)
        if barrier:
            barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cs)
        for i in range(K):
            e2e_step(W + i)
        cs.wait_stream(d2h)                    # the last output copy is inside the timed region
        e1.record(cs)
        torch.cuda.synchronize(device)
        if barrier:
            barrier()
        return e0.elapsed_time(e1) / 1e3

    e2e_sec = e2e_steps(args.steps, args.warmup)
    e2e_sec = max_over_ranks(e2e_sec, world, device)
    e2e = {"value": tokens / e2e_sec, "unit": "tokens/s", "h2d_bytes_per_step": lb.T * lb.layer.H * 2,
           "d2h_bytes_per_step": lb.T * lb.layer.H * 2,
           "how": "eager moe_layer_forward calls; each step's H2D and D2H copies on their own streams, "
                  "double-buffered, overlapping the layers"}

    # side measurements (not the headline): other batch sizes, the prefill-shaped and large layers,
    # and the streaming stack
    if not args.quick and world == 1:   # the side workloads run on one GPU only
        peaks = tensor_peaks(moe)
        extra["tensor_peaks"] = peaks
        outs = {}
        for cfg, T, act in (("decode", 1, "a16"), ("decode", 8, "a16"), ("prefill", 4096, "a16"),
                            ("prefill", 4096, "a4"), ("large", 32, "a16"), ("large", 32, "a4"),
                            ("large", 8192, "a16"), ("large", 8192, "a4")):
            nsets = NSETS if cfg == "decode" else (2 if cfg == "large" else 4)
            b = lb if (cfg == "decode" and T == 64) else LayerBench(moe, cfg, T, device, nsets=nsets, act=act)
            b.capture()
            nsteps = max(10, args.steps // 2) if T < 8192 else max(10, min(args.steps // 2, 40))
            s = time_steps(b.step, nsteps, args.warmup, device, barrier, run=b.run)
            ms_b = s / nsteps * 1e3
            n_alg = [b.algorithmic_bytes(args.warmup + i) for i in range(min(8, len(b.sets)))]
            gbs = sum(n_alg) / len(n_alg) / (ms_b * 1e-3) / 1e9
            tf = b.flops() / (ms_b * 1e-3) / 1e12
            key = f"{cfg}_T{T}" + ("_a4" if act == "a4" else "")
            extra[key] = {"tokens_per_s": T / (ms_b * 1e-3) * world, "ms_per_layer": ms_b, "act": act,
                          "layer_gbs": gbs, "frac_hbm": gbs / hbm, "tflops": tf, "frac_bf16_peak": tf / bf16_tf}
            if cfg != "decode":
                # the FP4-weight layers against the dense FP4 tensor peak measured above (the
                # format's own peak applies to A4, where both operands are FP4)
                if peaks.get("nvfp4_tflops"):
                    extra[key]["frac_fp4_peak"] = tf / peaks["nvfp4_tflops"]
                b.call(0)
                torch.cuda.synchronize(device)
                outs[(cfg, T, act)] = b.out.float().clone()
            del b
            torch.cuda.empty_cache()
        # the A4 form is a different computation: its distance from A16 on the same inputs
        # (GPU outputs of both) is quantisation error, reported beside the parity tests'
        # oracle comparison
        for cfg, T in (("prefill", 4096), ("large", 32), ("large", 8192)):
            a, q = outs.get((cfg, T, "a16")), outs.get((cfg, T, "a4"))
            if a is not None and q is not None:
                extra[f"{cfg}_T{T}_a4"]["a4_vs_a16_max_rel"] = float((q - a).abs().max() / a.abs().max())
        extra["stack"] = run_stack(moe, device, args.stack_steps)
        extra["prefill_stack"] = run_prefill_stack(moe, device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        tps, cores, sample = cpu_oracle_tokens_per_s("decode", 64)
        cpu = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}

    line = {
        "metric": "moe_layer_tokens_per_s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "MXFP4 weights x bf16 activations carried as four E2M1 planes (tcgen05 kind::mxf4), fp32 accumulate",
        "data": "synthetic (seeded; weights N(0,0.02) quantised, x N(0,1))",
        "config": dict(HEADLINE_CONFIG, parallelism=f"replicas x{world}",
                       l2=f"{NSETS} rotating weight copies + activation batches (weights touched per step > L2)",
                       timing=f"median of {len(passes)} timed regions of exactly {args.steps} steps each "
                              f"(repeated until they span 0.5 s); a CUDA graph holds {NSETS} consecutive layer "
                              f"calls, one per weight copy, as a serving engine captures a decode step"),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(round(launches_per_step * args.steps)),
        "clocks": clocks, "extra": extra,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_profile(args, device):
    """W + K plain (non-graph) layer forwards of one workload; for ncu launch lists."""
    import expert_ffn_layer_top_b200 as moe

    cfg, T, *rest = args.profile.split(":")
    lb = LayerBench(moe, cfg, int(T), device, nsets=4, act=rest[0] if rest else "a16")
    for i in range(args.warmup + args.steps):
        lb.call(i)
    torch.cuda.synchronize(device)
    print(json.dumps({"profile": args.profile, "steps": args.steps, "warmup": args.warmup}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--quick", action="store_true", help="headline workload only")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--stack-steps", type=int, default=512, help="decode steps of the streaming-stack run")
    ap.add_argument("--profile", default=None, help="plain launches of one workload (cfg:T[:act], e.g. decode:64 or prefill:4096:a4) for ncu")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.profile:
        run_profile(args, device)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    try:
        run_ours(args, rank, world, device)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
