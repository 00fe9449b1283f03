"""Benchmark of the Split-KV hot path on B200: useful block-sparse attention TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = the whole hot path over one batch of synthetic input, through the C ABI:
realized-cost pass -> LPT plan onto one queue per SM -> chunk-partial forward (tcgen05) ->
exact LSE merge (+ backward for the training workload). Inputs are resident in HBM when timing
starts; each timed step is bracketed by CUDA events on the launching stream and preceded (outside
the events) by a 256 MB write that flushes the 126 MB L2.

Useful FLOPs count only unmasked (query, key) pairs: each of the block rows of an anchor a sees
a + block keys, per query head; forward 4*d per pair, backward 10*d per pair.

With N > 1 (torchrun) every rank runs an independent replica of the workload on its own GPU
(the hot path is single-GPU; there is no data-path collective); value = all ranks' useful FLOPs /
the slowest rank's time. `--impl reference` times the float64 CPU oracle instead, on a bounded
sample of the same workload, on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def useful_flops(inp, backward):
    w = inp.workload
    # (query, key) pairs: each query of a block sees the a context keys and the block's own keys;
    # the forward kernel computes both (context items and self items).
    pairs = sum(w.block * (int(a) + w.block) for a in inp.anchors.tolist())
    per_pair = 4 * w.head_dim * w.n_q_heads
    fwd = per_pair * pairs
    bwd = (10 * w.head_dim * w.n_q_heads * pairs) if backward else 0
    return fwd + bwd, fwd


def timed_step_count(step_ms: float, min_steps: int = 20, min_timed_ms: float = 1000.0) -> int:
    """Steps to time when the caller gives none: enough for `min_timed_ms` of timed work at `step_ms` per
    step, and at least `min_steps`."""
    return max(min_steps, int(math.ceil(min_timed_ms / max(step_ms, 1e-3))))


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary of `kernel` on `workload`, or None when
    the summary is missing, the kernel's sources changed since it was captured, or the workload's
    definition (its `workload:` line) is no longer the registered one."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}.{workload}.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    traffic = None
    for ln in lines:
        if ln.startswith("traffic_bytes_per_launch:"):
            traffic = int(ln.split(":")[1])
        elif ln.startswith("source_sha256 "):
            rel, digest = ln[len("source_sha256 "):].split(": ")
            try:
                cur = hashlib.sha256(open(os.path.join(ROOT, rel), "rb").read()).hexdigest()
            except OSError:
                return None
            if cur != digest.strip():
                return None
        elif ln.startswith("workload: "):
            if ln[len("workload: "):].strip() != repr(W.get(workload)):
                return None
    return traffic


def library_provenance():
    """The loaded library's build id against the sources beside it: a stale build runs other code."""
    try:
        from split_kv_lse_splitkv_b200 import binding, build
        got, want = binding.library_build_id(), build.source_digest()
    except Exception as e:  # provenance is a report: it never ends the run
        return {"build_id": None, "matches_sources": None, "error": repr(e)}
    return {"build_id": got[:16], "matches_sources": got == want}


def traffic_applies(w, plan):
    """The committed ncu summaries hold the registered workloads under the LPT plan: another run length,
    cost tile, packing or plan moves other bytes, so its line reports no traffic."""
    return w.dtype == "bf16" and plan == "lpt" and w == W.get(w.name)


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every millisecond while the
    timed region runs, plus one sample as it ends. Without NVML (or without a GPU) it records nothing
    and the summary says so ("source": "none")."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, device_index):
        self.device_index = device_index
        self.samples = []  # (sm_mhz, max_mhz, reason bits)
        self.stop = threading.Event()
        self.nvml = None
        self.handle = None
        self.max_mhz = None

    def _open(self):
        import pynvml
        pynvml.nvmlInit()
        self.nvml = pynvml
        props = torch.cuda.get_device_properties(self.device_index)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
                return
            except Exception:
                pass
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom, dev = getattr(props, "pci_domain_id", 0), getattr(props, "pci_device_id", 0)
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId_v2(f"{dom:08x}:{bus:02x}:{dev:02x}.0")
            return
        self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def _sample(self):
        # Two NVML queries per sample (the maximum clock is read once): each query takes a few
        # milliseconds, so fewer queries give more samples of a short timed region.
        n = self.nvml
        if self.max_mhz is None:
            self.max_mhz = float(n.nvmlDeviceGetMaxClockInfo(self.handle, n.NVML_CLOCK_SM))
        sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
        try:
            bits = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        except AttributeError:
            bits = n.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
        self.samples.append((float(sm), self.max_mhz, int(bits)))

    def _loop(self):
        while not self.stop.wait(0.001):
            try:
                self._sample()
            except Exception:
                return

    def __enter__(self):
        try:
            self._open()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
        except Exception:
            self.handle = None
        return self

    def __exit__(self, *a):
        if self.handle is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "none"}
        reasons = sorted({name for _, _, bits in self.samples for name, bit in self.REASONS if bits & bit})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples), "reasons": reasons, "samples": len(self.samples),
                "source": "nvml"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_oracle_plan(inp, n_workers):
    """The oracle's cost pass and LPT plan (pure Python, one thread) over the whole workload, timed once."""
    from oracle import schedule as OS
    w = inp.workload
    per_sample = [inp.anchors_of(s) for s in range(len(w.seq_lens))]
    t0 = time.perf_counter()
    _, costs, _ = OS.costs_closed_form(per_sample, w.seq_lens, w.chunk, w.key_tile, w.n_kv_heads,
                                       pack=w.blocks_per_item, runs=w.chunks_per_item, overhead=w.item_overhead)
    t1 = time.perf_counter()
    OS.lpt(costs.tolist(), n_workers)
    t2 = time.perf_counter()
    return {"cost_ms": (t1 - t0) * 1e3, "lpt_ms": (t2 - t1) * 1e3, "items": int(len(costs)),
            "workers": int(n_workers), "threads": 1}


def cpu_oracle_sample(inp, budget_s, backward):
    """Time the float64 oracle on whole blocks of the workload until ~budget_s of CPU work."""
    import numpy as np

    from oracle import attention as OA
    w = inp.workload

    def f64(t):
        return t.detach().to("cpu", torch.float64).numpy()

    p = OA.Problem(inp.anchors.numpy(), inp.anchor_off.numpy(), inp.key_off.numpy(), f64(inp.q), f64(inp.k),
                   f64(inp.v), f64(inp.kb), f64(inp.vb), block=w.block, scale=w.scale)
    n = int(inp.anchor_off[-1])
    order = np.random.default_rng(0).permutation(n)
    flops = 0
    t0 = time.perf_counter()
    done = []
    for j in order:
        a = int(inp.anchors[j])
        O, L = OA.forward(p, blocks=[j])
        flops += 4 * w.head_dim * w.n_q_heads * w.block * (a + w.block)
        if backward:  # from this forward's O and LSE, as a training step would
            OA.backward(p, f64(inp.do), O=O, LSE=L, blocks=[j])
            flops += 10 * w.head_dim * w.n_q_heads * w.block * (a + w.block)
        done.append(int(j))
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    what = "fwd+bwd" if backward else "fwd"
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": int(cores), "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"{len(done)} of {n} draft blocks (all {w.n_q_heads} heads, {what}), "
                      f"{dt:.1f} s float64 NumPy on the host"}


def workload_of(args):
    """The chosen workload, with --blocks-per-item, --chunks-per-item, --key-tile and --item-overhead
    overriding its query-tile packing, run length, cost tile and per-item cost constant when given."""
    import dataclasses
    w = W.get(args.workload)
    if args.blocks_per_item:
        w = dataclasses.replace(w, blocks_per_item=args.blocks_per_item)
    if args.chunks_per_item:
        w = dataclasses.replace(w, chunks_per_item=args.chunks_per_item)
    if args.key_tile:
        w = dataclasses.replace(w, key_tile=args.key_tile)
    if args.item_overhead >= 0:
        w = dataclasses.replace(w, item_overhead=args.item_overhead)
    return w


def workload_config(w, counts, n_workers, world, plan):
    """The `config` object of the JSON line: the same dict for both arms (how the steps are launched
    is reported beside it, under "launch")."""
    return {"workload": w.name, "seq_lens": list(w.seq_lens), "anchors": counts,
            "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv", "head_dim": w.head_dim, "chunk": w.chunk,
            "blocks_per_item": w.blocks_per_item, "chunks_per_item": w.chunks_per_item,
            "key_tile": w.key_tile, "item_overhead": w.item_overhead, "queues": n_workers,
            "l2": "flushed (256 MB write) before every timed step",
            "parallelism": f"replicas x{world}", "plan": plan}


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    w = workload_of(args)
    inp = W.make_inputs(w)
    vals = []
    steps = args.steps if args.steps is not None else 20
    budget = args.ref_budget if args.ref_budget else max(1.0, 150.0 / (args.warmup + steps))
    for i in range(args.warmup + steps):
        r = cpu_oracle_sample(inp, budget, w.backward)
        if i >= args.warmup:
            vals.append(r["value"])
    value = statistics.mean(vals)
    r["value"] = value
    workers = w.n_workers or (torch.cuda.get_device_properties(0).multi_processor_count
                              if torch.cuda.is_available() else 148)
    r["plan"] = cpu_oracle_plan(inp, workers)
    flops, _ = useful_flops(inp, w.backward)
    line = {"impl": "reference", "metric": "useful block-sparse attention TFLOP/s (fwd+bwd)" if w.backward else
            "useful block-sparse attention TFLOP/s (fwd)", "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup,
            # each timed step is a bounded sample of the workload: the whole step at the sampled rate
            "ms_per_step": flops / (value * 1e12) * 1e3, "ms_per_step_kind": "extrapolated from the sampled rate",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, [int(inp.anchor_off[i + 1] - inp.anchor_off[i])
                                          for i in range(len(w.seq_lens))], workers, args.gpus, args.plan),
            "launch": "host: float64 NumPy oracle", "cpu_baseline": r,
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def run_ours(args):
    from split_kv_lse_splitkv_b200 import SplitKV

    world, rank, local = dist_setup(args)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = workload_of(args)
    inp = W.make_inputs(w)
    counts = [int(inp.anchor_off[i + 1] - inp.anchor_off[i]) for i in range(len(w.seq_lens))]
    skv = SplitKV(w.seq_lens, counts, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.chunk, w.key_tile, w.scale,
                  w.torch_dtype, n_workers=w.n_workers, device=device, blocks_per_item=w.blocks_per_item,
                  chunks_per_item=w.chunks_per_item, item_overhead=w.item_overhead)
    host = {k: getattr(inp, k) for k in ("q", "k", "v", "kb", "vb", "anchors")}
    if w.backward:
        host["do"] = inp.do
    dev = {k: t.to(device) for k, t in host.items()}
    Nq, Hq, d = inp.q.shape
    o = torch.empty(Nq, Hq, d, dtype=w.torch_dtype, device=device)
    lse = torch.empty(Nq, Hq, dtype=torch.float32, device=device)
    grads = None
    if w.backward:
        f = dict(dtype=torch.float32, device=device)
        grads = (torch.empty(inp.q.shape, **f), torch.empty(inp.k.shape, **f), torch.empty(inp.v.shape, **f),
                 torch.empty(inp.kb.shape, **f), torch.empty(inp.vb.shape, **f))
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    # One non-default stream for every launch and copy (a CUDA graph is captured on a non-default stream).
    torch.cuda.synchronize(device)
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)
    phases = {"cost": [], "plan": [], "fwd": [], "merge": [], "bwd": []}

    def timed(name, fn, on):
        if not on:
            fn()
            return
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        phases[name].append((e0, e1))

    naive_load = None
    if args.plan == "naive":
        # Cost-blind equal-count split of the item list (index order) into contiguous queues, for the
        # comparison with LPT; built once (the anchors do not change), so each step runs the cost
        # pass and then the same kernels with these queues.
        skv.cost(dev["anchors"], stream)
        torch.cuda.synchronize(device)
        n, mq = int(skv.n_items.item()), skv.n_workers
        bounds = torch.tensor([(x * n) // mq for x in range(mq + 1)], dtype=torch.int64)
        skv.queue_off = bounds.to(torch.int32).to(device)
        skv.queue_items = torch.arange(max(1, n), dtype=torch.int32, device=device)
        csum = torch.cat([torch.zeros(1, dtype=torch.int64), skv.item_cost[:n].cpu().to(torch.int64).cumsum(0)])
        naive_load = (csum[bounds[1:]] - csum[bounds[:-1]]).double()

    def step(d, time_phases=False):
        timed("cost", lambda: skv.cost(d["anchors"], stream), time_phases)
        if args.plan != "naive":  # the naive split's queues were built once, above
            timed("plan", lambda: skv.plan_lpt(stream), time_phases)
        timed("fwd", lambda: skv.attn_fwd(d["q"], d["k"], d["v"], d["kb"], d["vb"], d["anchors"], stream=stream),
              time_phases)
        timed("merge", lambda: skv.lse_merge(d["anchors"], o, lse, stream=stream), time_phases)
        if w.backward:
            timed("bwd", lambda: skv.backward(d["q"], d["k"], d["v"], d["kb"], d["vb"], o, lse, d["do"], d["anchors"],
                                              grads, stream=stream), time_phases)

    # cost 3, LPT plan 3 (not with the naive split), fwd 1, merge 1; bwd: rows, one-pass backward
    launches_per_step = 3 + (0 if args.plan == "naive" else 3) + 1 + 1 + (2 if w.backward else 0)
    for _ in range(args.warmup):
        step(dev)
    torch.cuda.synchronize(device)
    skv.check_status()

    # The step's launches (cost, plan, forward, merge[, backward]) captured once as a CUDA graph and
    # replayed: the same kernels on the same buffers, without the host launch gaps between them.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
            step(dev)
        torch.cuda.synchronize(device)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize(device)
        skv.check_status()

    def timed_steps(n, run, time_phases):
        evs = []
        for _ in range(n):
            flush.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run(time_phases)
            e1.record(stream)
            evs.append((e0, e1))
        return evs

    replay = (lambda _: graph.replay()) if graph is not None else (lambda tp: step(dev, time_phases=tp))
    if args.steps is not None:
        steps = args.steps
    else:
        # Enough steps for at least 1 s of timed work (so that the clock record has hundreds of samples),
        # at least 20; the same count on every rank.
        probe = timed_steps(3, replay, False)
        torch.cuda.synchronize(device)
        t_step = max_over_ranks(sum(a.elapsed_time(b) for a, b in probe) / len(probe), world, device)
        steps = timed_step_count(t_step)
    aux_steps = min(steps, 50)  # per-phase and end-to-end timings

    # ---- device-timed region
    barrier(world)
    torch.cuda.synchronize(device)
    wall0 = time.perf_counter()
    with ClockSampler(local) as clocks:
        evs = timed_steps(steps, replay, graph is None)
        torch.cuda.synchronize(device)
    barrier(world)
    wall = time.perf_counter() - wall0
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    if graph is not None:
        # Per-phase times (for the roofline of the forward kernel) from as many eager steps, timed
        # the same way, after the graph-timed region.
        timed_steps(aux_steps, lambda tp: step(dev, time_phases=tp), True)
        torch.cuda.synchronize(device)
    phase_ms = {k: (sum(a.elapsed_time(b) for a, b in v) / len(v)) for k, v in phases.items() if v}
    fwd_ms = phase_ms["fwd"]
    merge_ms = phase_ms["merge"]
    ms_max = max_over_ranks(ms, world, device)
    skv.check_status()

    # ---- end to end through the public API with host buffers
    pinned = {k: t.pin_memory() for k, t in host.items()}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = o_host.numel() * o_host.element_size() + lse_host.numel() * lse_host.element_size()
    if w.backward:
        d2h = sum(g.numel() * g.element_size() for g in grads)
    dev2 = {k: torch.empty_like(t) for k, t in dev.items()}
    grads_host = [torch.empty(g.shape, dtype=g.dtype).pin_memory() for g in grads] if w.backward else []

    def e2e_step():
        for k, t in pinned.items():
            dev2[k].copy_(t, non_blocking=True)
        step(dev2)
        if w.backward:
            for gh, g in zip(grads_host, grads):
                gh.copy_(g, non_blocking=True)
        else:
            o_host.copy_(o, non_blocking=True)
            lse_host.copy_(lse, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(device)
    barrier(world)
    e_evs = []
    for _ in range(aux_steps):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_step()
        e1.record(stream)
        e_evs.append((e0, e1))
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e_evs) / len(e_evs), world, device)

    flops, fwd_kernel_flops = useful_flops(inp, w.backward)
    value = world * flops / (ms_max * 1e-3) / 1e12
    pk, src = peaks()
    fwd_kernel = "fwd_tc2_kernel" if int(skv.sizes.ctas_per_worker) == 2 else "fwd_tc_kernel"
    if w.dtype == "bf16":
        roof = {"bound": "tensor", "kernel": fwd_kernel, "peak": float(pk["bf16_tflops"]),
                "peak_source": f"{src} bf16 dense (burst)",
                "frac_of_sustained_peak": None}
    else:
        # fp32 CUDA-core kernel: 148 SMs x 128 FMA lanes x 2 FLOP x 1.965 GHz.
        roof = {"bound": "alu", "kernel": "fwd_simt_kernel<float>", "peak": 148 * 128 * 2 * 1.965e9 / 1e12,
                "peak_source": "derived fp32 FFMA peak at max SM clock"}
    achieved = fwd_kernel_flops / (fwd_ms * 1e-3) / 1e12
    peak = roof["peak"]
    if w.dtype == "bf16":
        # The same kernel against the measured sustained GEMM figure (clocks under the power cap), for
        # launches long enough to run in that regime.
        roof["frac_of_sustained_peak"] = achieved / float(pk.get("bf16_tflops_sustained", peak))
    load = naive_load if naive_load is not None else skv.load.cpu().double()
    predicted_imb = float(load.max() / load.mean() - 1.0) if load.sum() > 0 else 0.0
    csum = clocks.summary()

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_oracle_sample(inp, args.ref_budget or 10.0, w.backward)
            cpu["plan"] = cpu_oracle_plan(inp, skv.n_workers)
        line = {
            "metric": "useful block-sparse attention TFLOP/s (fwd+bwd)" if w.backward else
                      "useful block-sparse attention TFLOP/s (fwd)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": workload_config(w, counts, skv.n_workers, world, args.plan),
            "launch": "eager" if graph is None else "cuda graph of the step",
            "roofline": dict(roof, achieved=achieved, unit="TFLOP/s", frac=achieved / peak,
                             traffic=profiled_traffic(fwd_kernel, w.name) if traffic_applies(w, args.plan) else None,
                             kernel_ms=fwd_ms, algorithmic_flop=fwd_kernel_flops,
                             # useful TFLOP/s over the forward plus the merge, against the same peak
                             frac_fwd_merge=fwd_kernel_flops / ((fwd_ms + merge_ms) * 1e-3) / 1e12 / peak,
                             fwd_merge_ms=fwd_ms + merge_ms),
            "phase_ms": phase_ms,
            "imbalance": {f"predicted_{args.plan}": predicted_imb},
            **({"backward_roofline": {"kernels": "rows_kernel + bwd_tc_kernel",
                                      "algorithmic_flop": flops - fwd_kernel_flops,
                                      "achieved": (flops - fwd_kernel_flops) / (phase_ms["bwd"] * 1e-3) / 1e12,
                                      "peak": peak, "unit": "TFLOP/s",
                                      "frac": (flops - fwd_kernel_flops) / (phase_ms["bwd"] * 1e-3) / 1e12 / peak}}
               if w.backward and "bwd" in phase_ms and w.dtype == "bf16" else {}),
            "clocks": csum,
            "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * steps,
            "wall_s": wall,
            "cpu_baseline": cpu,
            "library": library_provenance(),
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for at least 1 s of timed work, at least 20)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="skewed_s256k", choices=sorted(W.WORKLOADS),
                    help="default: the largest single-GPU forward workload (S = 262144, ~4080 queries)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-budget", type=float, default=0.0,
                    help="seconds of CPU work per oracle sample (default: ~150 s spread over all reference steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eagerly launched steps instead of replaying one captured CUDA graph of the step")
    ap.add_argument("--blocks-per-item", type=int, default=0,
                    help="query-tile packing P (blocks per item) instead of the workload's: 256-row items "
                         "(P * 16 * G = 256) run on pairs of SMs, smaller ones on one SM")
    ap.add_argument("--chunks-per-item", type=int, default=0,
                    help="runs of L chunks per item (one partial per run) instead of the workload's L")
    ap.add_argument("--key-tile", type=int, default=0,
                    help="key tile of the planner's cost (Tk, a divisor of the chunk) instead of the workload's")
    ap.add_argument("--item-overhead", type=int, default=-1,
                    help="per-item constant of the planner's cost in key tiles instead of the workload's")
    ap.add_argument("--plan", default="lpt", choices=["lpt", "naive"],
                    help="naive: the cost-blind equal-count split instead of the LPT plan (for comparison)")
    args = ap.parse_args()
    try:
        if args.impl == "reference":
            run_reference(args)
        else:
            run_ours(args)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
