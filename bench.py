#!/usr/bin/env python
"""Benchmark of the pack -> attend -> unpack call on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5:1.0:512] [--impl ours|reference]

One step = one whole pack -> attend -> unpack call for every pruning stage of the workload,
replayed from a CUDA graph over inputs resident in HBM.  The default workload is the largest
single-GPU configuration: DeiT-B head shape (H=12, d=64, N=197), keep ratio 1.0, B=512 images
(100,864 tokens per call).  The call runs either as the single
launch rra_pack_attend_unpack (--path fused, the default: identical bytes out) or as the three
launches rra_pack, rra_attend, rra_unpack (--path three); the other path is timed afterwards
and reported beside it.  L2 is flushed (a 256 MiB write, untimed) before every timed step, and
each step is bracketed by CUDA events on the launching stream; per-kernel events recorded
inside the graph give the per-kernel times.

Prints ONE JSON line on rank 0: packed tokens/s (whole job), us per call, the roofline of the
dominant kernel, end-to-end throughput through the public API with pinned host buffers,
the float64 CPU oracle on a bounded sample (one core and all of the host's cores), clocks
sampled during the timed region, how many of this library's kernels ran in the timed region,
and (N = 1, unless --no-sweep) a `sweep` over every configured cell: config 5's keep ratio x
batch grid and three-stage rows, configs 1-4 -- per cell the graph-replayed us per call with L2
cold and warm, eager us per call, packed tokens/s, attention TFLOP/s, the kernel's fraction of
the HBM roofline, and the same for the three-call path.

With torchrun (N > 1) every rank runs an independent replica of the workload on its own GPU
(images are independent, so the path shards with no exchange): weak scaling, timings reduced
as the max over ranks.

--impl reference times the float64 CPU oracle itself (rank 0 only, all host cores, one thread
per image) on the same workload, metric and unit, one bounded sample of images per step.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ragged_varlen_attention_rra_b200 import rra, workloads  # noqa: E402

METRIC = "packed tokens/s & us per pack-attend-unpack call (1 B200, graph); % roofline"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# ex2 results per clock per SM of the special-function unit (the documented throughput of the base-2
# exponential on this architecture; the attention kernel's XU-pipe utilisation under ncu agrees with it)
EX2_PER_CLK_PER_SM = 16
L2_FLUSH_BYTES = 256 << 20
KERNELS = {"three": ("pack", "attend", "unpack"), "fused": ("pack_attend_unpack",)}
KERNEL_SOURCES = {
    "pack": "ragged_varlen_attention_rra_b200/csrc/pack_unpack.cu",
    "unpack": "ragged_varlen_attention_rra_b200/csrc/pack_unpack.cu",
    "attend": "ragged_varlen_attention_rra_b200/csrc/attend.cu",
    "pack_attend_unpack": "ragged_varlen_attention_rra_b200/csrc/attend.cu",
}


# ------------------------------------------------------------------------------------ helpers

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(x: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world_size: int, steps: int, tokens_per_call: int, max_total_ms: float) -> float:
    """Whole-job tokens/s: every rank runs `steps` calls of `tokens_per_call` tokens (independent
    replicas), and the job takes as long as its slowest rank."""
    return world_size * steps * tokens_per_call / (max_total_ms * 1e-3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s: the measured burst figure (a kernel timed alone), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def measure_ex2_rate(stream, num_sms, iters=2048, reps=5):
    """Exponentials per second of the whole GPU (ex2.approx.ftz.f32): the microbenchmark in
    libmicrobench.so, 8 blocks of 256 threads per SM, each thread 8 independent chains, timed with
    CUDA events on `stream` (best of `reps` launches).  None when the library is missing."""
    path = os.path.join(ROOT, "ragged_varlen_attention_rra_b200", "libmicrobench.so")
    if not os.path.exists(path):
        return None
    mb = ctypes.CDLL(path)
    mb.rra_mb_ex2_launch.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    mb.rra_mb_ex2_launch.restype = ctypes.c_int
    per = int(mb.rra_mb_ex2_per_block_iter())
    blocks = num_sms * 8
    out = torch.empty(blocks * 256, dtype=torch.float32, device="cuda")
    with torch.cuda.stream(stream):
        for _ in range(2):
            if mb.rra_mb_ex2_launch(out.data_ptr(), blocks, iters, ctypes.c_void_p(stream.cuda_stream)) != 0:
                return None
        best = None
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            mb.rra_mb_ex2_launch(out.data_ptr(), blocks, iters, ctypes.c_void_p(stream.cuda_stream))
            e1.record(stream)
            e1.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
    return blocks * per * iters / (best * 1e-3)


def attention_bounds_us(bytes_, flops, exps, hbm_gbs, ex2_per_s):
    """Lower bounds (us) on one attention launch from each resource: HBM bytes, tensor-core FLOPs
    at the bf16 peak, and exponentials at the measured (or nominal) exponential-unit rate."""
    tf, _ = tensor_peak()
    return {"hbm": bytes_ / (hbm_gbs * 1e3), "tensor": flops / (tf * 1e6), "exp": exps / ex2_per_s * 1e6}


def source_hash(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


E2E_CHUNK = 64  # images per chunk of the end-to-end (host memory in and out) measurement


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source still matches."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_sha") != source_hash(KERNEL_SOURCES[kernel]):
        return None
    return e.get("dram_bytes_per_launch")


def algorithmic_bytes(B, N, lengths, row_bytes, out_row_bytes):
    """Per-stage algorithmic HBM bytes of each kernel (the minimal reads + writes)."""
    T = int(lengths.sum())
    return {
        "pack": B * N + 2 * 3 * T * row_bytes + 4 * (B + 1),
        "attend": 3 * T * row_bytes + T * out_row_bytes + 4 * (B + 1),
        "unpack": T * out_row_bytes + B * N * out_row_bytes + B * N + 4 * (B + 1),
        # single launch: mask, the kept rows of Q/K/V, the padded output, cu_seqlens
        "pack_attend_unpack": B * N + 3 * T * row_bytes + B * N * out_row_bytes + 4 * (B + 1),
    }


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every ~0.5 ms by a
    background thread while the timed region runs (nvidia-smi's 200 ms loop is too coarse
    for a timed region of milliseconds)."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, torch_index, period_s=0.0005):
        self.torch_index = torch_index
        self.period = period_s
        self.samples = []
        self.error = None
        self.max_mhz = None

    def __enter__(self):
        import threading
        try:
            import pynvml as N
            N.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.torch_index).uuid)
            h = N.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            masks = {k: getattr(N, v) for k, v in self.REASONS.items()}
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.error = repr(e)
            self.thread = None
            return self
        self.stop = threading.Event()

        def run():
            while not self.stop.is_set():
                try:
                    mhz = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                    bits = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((mhz, [k for k, m in masks.items() if bits & m]))
                except Exception as e:
                    self.error = repr(e)
                    return
                time.sleep(self.period)
        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "error": self.error}
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


# ------------------------------------------------------------------------------------ CPU oracle

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_call(q, k, v, H, dtype, stage_masks, images):
    """One oracle pack-attend-unpack over the given images of every stage; returns tokens done.
    The oracle's C calls release the GIL, so threads running this on disjoint images run on
    separate cores."""
    from oracle import oracle as O
    sel = torch.as_tensor(images, dtype=torch.long)
    qs, ks, vs = q[sel], k[sel], v[sel]
    tokens = 0
    for m in stage_masks:
        ms = m[sel]
        qp, cu = O.pack(ms, qs)
        kp, _ = O.pack(ms, ks)
        vp, _ = O.pack(ms, vs)
        o = O.attend(qp, kp, vp, cu, H, 64, dtype=dtype)
        O.unpack(o, cu, ms)
        tokens += int(cu[-1])
    return tokens


def oracle_images(w, images, threads):
    """The oracle over `images` (every stage), one image per task on `threads` threads; tokens."""
    if threads <= 1:
        return sum(oracle_call(w.q, w.k, w.v, w.H, w.dtype, w.masks, [i]) for i in images)
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return sum(ex.map(lambda i: oracle_call(w.q, w.k, w.v, w.H, w.dtype, w.masks, [i]), images))


def cpu_baseline(w, budget_s=10.0):
    """The oracle, as it stands, on a bounded sample of the workload's images: first on one core
    for about budget_s / 3, then on all host cores (one thread per image) for about the rest."""
    from oracle import oracle as O
    O.load()
    cores = host_cores()
    out = {}
    for leg, threads, budget in (("single", 1, budget_s / 3), ("multi", cores, 2 * budget_s / 3)):
        t0 = time.perf_counter()
        tokens, done = 0, 0
        while time.perf_counter() - t0 < budget and done < 4 * w.B:
            batch = [(done + j) % w.B for j in range(threads)]
            tokens += oracle_images(w, batch, threads)
            done += len(batch)
        dt = time.perf_counter() - t0
        out[leg] = {"value": tokens / dt, "images": done, "seconds": dt, "threads": threads}
    m = out["multi"]
    return {"value": m["value"], "unit": UNIT, "cores": m["threads"], "kind": "oracle",
            "sample": f"{m['images']} image(s) of {w.name} (every stage) on {m['threads']} threads, one image "
                      f"per thread, float64 C, {m['seconds']:.1f} s; host has {cores} usable cores",
            "single_core": {"value": out["single"]["value"], "unit": UNIT, "cores": 1,
                            "sample": f"{out['single']['images']} image(s), {out['single']['seconds']:.1f} s"}}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = workloads.by_name(args.workload)
    from oracle import oracle as O
    O.load()
    cores = host_cores()
    per_step = max(1, min(w.B, args.ref_images if args.ref_images > 0 else cores))
    step_tokens, step_times = [], []
    for i in range(args.warmup + args.steps):
        imgs = [(i * per_step + j) % w.B for j in range(per_step)]
        t0 = time.perf_counter()
        tok = oracle_images(w, imgs, min(cores, per_step))
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            step_tokens.append(tok)
            step_times.append(dt)
    total_t = sum(step_times)
    value = sum(step_tokens) / total_t
    threads = min(cores, per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d": 64, "stages": len(w.masks),
                   "seed": w.seed, "recipe": w.recipe, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{per_step} image(s) of {w.name} per step, every stage, {threads} threads "
                                   f"(one image each); host has {cores} usable cores"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------ GPU arm

class Pipeline:
    """Device buffers + CUDA graphs of the whole call (all stages) on device-resident inputs:
    `graph` holds the kernels alone (the timed one: kernels that follow one another may overlap
    their start-up through programmatic dependent launch), `graph_ev` the same kernels with an
    event between each pair (for the per-kernel breakdown; the events serialise the kernels)."""

    def __init__(self, q, k, v, masks, out_dtype, stream, path):
        self.path = path
        self.q, self.k, self.v = q, k, v
        self.masks = masks
        self.B, self.N, self.H = q.shape[0], q.shape[1], q.shape[2]
        self.bufs = rra.Buffers(self.B, self.N, self.H, q.dtype, out_dtype=out_dtype)
        if path == "fused":  # the single launch uses no packed buffers
            self.bufs.packed = [t[:1] for t in self.bufs.packed]
            self.bufs.o = self.bufs.o[:1]
        self.ys = [torch.empty(self.B, self.N, self.H, 64, dtype=self.bufs.y.dtype, device="cuda") for _ in masks]
        self.stream = stream
        self.graph = None
        self.graph_ev = None
        self.events = None

    @property
    def kernels(self):
        return KERNELS[self.path]

    def enqueue(self, events=None):
        b = self.bufs
        s = self.stream
        nk = len(self.kernels)
        for i, m in enumerate(self.masks):
            if events:
                events[nk * i].record(s)
            if self.path == "fused":
                rra.rra_pack_attend_unpack(m, self.q, self.k, self.v, self.ys[i], b.cu, dev_error=b.err, stream=s)
                continue
            rra.rra_pack(m, [self.q, self.k, self.v], b.packed, b.cu, dev_error=b.err, stream=s)
            if events:
                events[nk * i + 1].record(s)
            rra.rra_attend(b.packed[0], b.packed[1], b.packed[2], b.o, b.cu, max_seqlen=self.N,
                           dev_error=b.err, stream=s)
            if events:
                events[nk * i + 2].record(s)
            rra.rra_unpack(b.o, b.cu, m, self.ys[i], fill_mode=0, dev_error=b.err, stream=s)
        if events:
            events[nk * len(self.masks)].record(s)

    def capture(self):
        with torch.cuda.stream(self.stream):
            self.enqueue()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self.enqueue()
        self.graph = g
        n_ev = len(self.kernels) * len(self.masks) + 1
        events = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_ev)]
        ge = torch.cuda.CUDAGraph()
        try:
            with torch.cuda.graph(ge, stream=self.stream):
                self.enqueue(events)
            self.graph_ev, self.events = ge, events
        except Exception:  # event-record nodes unavailable: no per-kernel breakdown
            self.graph_ev, self.events = None, None
        torch.cuda.synchronize()

    def kernel_times(self):
        """Per-launch ms of each kernel of the last replay, from the in-graph events."""
        if self.events is None:
            return None
        ev, nk = self.events, len(self.kernels)
        out = {k: [] for k in self.kernels}
        for s in range(len(self.masks)):
            for j, k in enumerate(self.kernels):
                out[k].append(ev[nk * s + j].elapsed_time(ev[nk * s + j + 1]))
        return out


def time_path(pipe, flush, steps, warmup, stream):
    """Warm-up, then `steps` timed replays of the kernels-only graph, each after an untimed L2
    flush (per-step ms); then as many replays of the graph with per-kernel events, same protocol
    (per-kernel per-launch ms)."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(warmup):
        with torch.cuda.stream(stream):
            flush.fill_(i & 0xFF)
            pipe.graph.replay()
    torch.cuda.synchronize()
    step_ms, kern = [], {k: [] for k in pipe.kernels}
    for i in range(steps):
        with torch.cuda.stream(stream):
            flush.fill_((i + 7) & 0xFF)
            start.record(stream)
            pipe.graph.replay()
            end.record(stream)
        stream.synchronize()
        step_ms.append(start.elapsed_time(end))
    if pipe.graph_ev is not None:
        for i in range(steps):
            with torch.cuda.stream(stream):
                flush.fill_((i + 11) & 0xFF)
                pipe.graph_ev.replay()
            stream.synchronize()
            for k, v in pipe.kernel_times().items():
                kern[k].extend(v)
    return step_ms, kern


def time_mask_producer(B, N, H, seed, flush, stream, steps, warmup, hbm_peak):
    """The token-selection step in front of the path (rra_l2_mask, top-k mode) on embeddings of
    the workload's width (C = 64 H, DeiT's embedding size) and keep counts from the configs'
    recipe: per-launch device time (L2 flushed before each launch), algorithmic bytes, GB/s."""
    C = 64 * H
    x = workloads.embeddings(B, N, C, "bf16", seed=seed).cuda()
    k = torch.from_numpy(workloads.keep_counts(B, N, seed=seed)).cuda()
    mask = torch.empty(B, N, dtype=torch.uint8, device="cuda")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for i in range(warmup + steps):
        with torch.cuda.stream(stream):
            flush.fill_((i + 3) & 0xFF)
            start.record(stream)
            rra.rra_l2_mask(x, mask, k_keep=k, stream=stream)
            end.record(stream)
        stream.synchronize()
        if i >= warmup:
            ms.append(start.elapsed_time(end))
    us = 1e3 * statistics.mean(ms)
    nbytes = B * N * C * 2 + B * N + 4 * B
    gbs = nbytes / (us * 1e3)
    return {"call": "rra_l2_mask (top-k)", "B": B, "N": N, "C": C, "us_per_launch": us,
            "alg_bytes_per_launch": nbytes, "gbs": gbs, "frac_of_hbm": gbs / hbm_peak}


def time_block(w, cu, flush, stream, steps, warmup):
    """The synthetic-weight DeiT block (NEXT 4) on the packed rows of the workload's first stage:
    LN1, QKV, the ragged attention, the output projection, LN2, FC1 + GELU, FC2 (rra.DeitBlock),
    with random N(0, 1) rows and seeded synthetic weights.  Whole-block time from a graph of the
    seven launches, per-stage time from a second graph with an event between stages (which
    serialises them), L2 flushed before each replay.  Reports the attention part (LN1, QKV,
    attention, projection) against the MLP part (LN2, FC1, FC2) and each GEMM's TFLOP/s."""
    H, B, N = w.H, w.B, w.N
    C = 64 * H
    if C % 128 != 0:
        return {"skipped": f"width C = {C} is not a multiple of 128, the GEMM kernel's narrowest output tile"}
    cap = B * N
    T = int(w.lengths[0].sum())
    g = torch.Generator(device="cuda").manual_seed(int(w.seed) + 5)
    x = torch.randn(cap, C, generator=g, device="cuda").to(torch.bfloat16)
    blk = rra.DeitBlock({k: v.cuda() for k, v in workloads.block_weights(C, seed=w.seed).items()}, cap, H)
    names = blk.STAGES
    with torch.cuda.stream(stream):
        blk(x, cu, B, N, stream=stream)
    stream.synchronize()
    graph, graph_ev = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(names) + 1)]
    with torch.cuda.graph(graph, stream=stream):
        blk(x, cu, B, N, stream=stream)
    with torch.cuda.graph(graph_ev, stream=stream):
        ev[0].record(stream)
        for i, name in enumerate(names):
            blk.stage(name, x, cu, B, N, stream)
            ev[i + 1].record(stream)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    whole, per = [], {n: [] for n in names}
    for i in range(warmup + steps):
        with torch.cuda.stream(stream):
            flush.fill_((i + 5) & 0xFF)
            start.record(stream)
            graph.replay()
            end.record(stream)
            flush.fill_((i + 6) & 0xFF)
            graph_ev.replay()
        stream.synchronize()
        if i >= warmup:
            whole.append(start.elapsed_time(end))
            for j, n in enumerate(names):
                per[n].append(ev[j].elapsed_time(ev[j + 1]))
    assert rra.rra_get_device_error(blk.err, stream) == 0
    us = {n: 1e3 * statistics.mean(v) for n, v in per.items()}
    gemm_flops = {"qkv": 2 * T * C * 3 * C, "proj": 2 * T * C * C, "fc1": 2 * T * C * 4 * C, "fc2": 2 * T * 4 * C * C}
    tf, tf_kind = tensor_peak()
    gemms = {n: {"us": us[n], "tflops": f / (us[n] * 1e-6) / 1e12, "frac_of_tensor_peak": f / (us[n] * 1e-6) / 1e12 / tf}
             for n, f in gemm_flops.items()}
    attn = sum(us[n] for n in ("ln1", "qkv", "attend", "proj"))
    mlp = sum(us[n] for n in ("ln2", "fc1", "fc2"))
    del graph, graph_ev
    return {"model": f"DeiT block, C = {C}, H = {H}, MLP {4 * C}, synthetic weights", "T": T,
            "us_per_block": 1e3 * statistics.mean(whole), "us_per_stage": us,
            "attention_part_us": attn, "mlp_part_us": mlp, "attention_share": attn / (attn + mlp),
            "gemms": gemms, "tensor_peak_tflops": tf, "tensor_peak_source": tf_kind,
            "note": "per-stage times come from a graph with events between stages (serialised)"}


def kernel_table(kms, alg, stages, hbm_peak):
    table = {}
    for k, v in kms.items():
        if not v:
            return None
        per_launch_us = 1e3 * statistics.mean(v)
        per_launch_bytes = alg[k] / stages
        gbs = per_launch_bytes / (per_launch_us * 1e3)
        table[k] = {"us_per_launch": per_launch_us, "gbs": gbs, "alg_bytes_per_launch": per_launch_bytes,
                    "frac_of_hbm": gbs / hbm_peak}
    return table


def attention_flops(lengths):
    return sum(4 * 64 * int(H_) * int((l.astype(np.int64) ** 2).sum()) for H_, l in lengths)


def empty_graph_floor(stream, reps=200):
    """Device time per replay of a graph holding one trivial kernel (a 4-byte fill): the floor
    that graph launch and kernel start-up put under any call."""
    x = torch.zeros(1, dtype=torch.int32, device="cuda")
    with torch.cuda.stream(stream):
        x.fill_(1)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        x.fill_(2)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(10):
            g.replay()
        start.record(stream)
        for _ in range(reps):
            g.replay()
        end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / reps * 1e3


def run_sweep(names, flush, stream, hbm_peak, cold_reps=10, warm_reps=100, eager_reps=30):
    """Every named cell on inputs drawn on the device (values of the largest batch of each shape,
    sliced for the smaller ones; masks from the cell's recipe).  Per cell: the single launch's
    graph replay us per call with L2 flushed before each replay (cold) and back to back (warm),
    eager us per call through the API, tokens/s, attention TFLOP/s, its HBM roofline fraction
    from in-graph events, and the three-call path's cold us per call with its output checked
    byte for byte against the single launch's."""
    shapes = {}
    for n in names:
        B, N, H, dt, std = workloads.shape_of(n)
        key = (N, H, dt, std)
        shapes[key] = max(shapes.get(key, 0), B)
    order = sorted(names, key=lambda n: workloads.shape_of(n)[1:])
    cells, cur_key, vals = {}, None, None
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for name in order:
        B, N, H, dt, std = workloads.shape_of(name)
        key = (N, H, dt, std)
        if key != cur_key:
            vals = None
            torch.cuda.empty_cache()
            vals = workloads.device_values(shapes[key], N, H, dt, seed=0, std=std)
            cur_key = key
        q, k, v = (t[:B] for t in vals)
        masks_np = workloads.sweep_masks(name)
        masks = [torch.from_numpy(np.ascontiguousarray(m)).cuda() for m in masks_np]
        lengths = [m.astype(bool).sum(axis=1) for m in masks_np]
        T_call = int(sum(int(l.sum()) for l in lengths))
        row_bytes = H * 64 * 2
        entry = {"B": B, "N": N, "H": H, "stages": len(masks), "tokens_per_call": T_call}
        res = {}
        for path in ("fused", "three"):
            pipe = Pipeline(q, k, v, masks, None, stream, path)
            pipe.capture()
            cold = []
            for i in range(cold_reps + 2):
                with torch.cuda.stream(stream):
                    flush.fill_(i & 0xFF)
                    start.record(stream)
                    pipe.graph.replay()
                    end.record(stream)
                stream.synchronize()
                if i >= 2:
                    cold.append(start.elapsed_time(end))
            kern = {kk: [] for kk in pipe.kernels}
            for i in range(cold_reps):
                with torch.cuda.stream(stream):
                    flush.fill_((i + 5) & 0xFF)
                    pipe.graph_ev.replay()
                stream.synchronize()
                for kk, vv in pipe.kernel_times().items():
                    kern[kk].extend(vv)
            res[path] = (pipe, 1e3 * statistics.mean(cold), kern)
            if path == "fused":
                with torch.cuda.stream(stream):
                    start.record(stream)
                    for _ in range(warm_reps):
                        pipe.graph.replay()
                    end.record(stream)
                torch.cuda.synchronize()
                entry["us_warm"] = start.elapsed_time(end) / warm_reps * 1e3
                with torch.cuda.stream(stream):
                    pipe.enqueue()
                    start.record(stream)
                    for _ in range(eager_reps):
                        pipe.enqueue()
                    end.record(stream)
                torch.cuda.synchronize()
                entry["us_eager"] = start.elapsed_time(end) / eager_reps * 1e3
        fused_pipe, us_cold, kern = res["fused"]
        three_pipe, us_cold3, kern3 = res["three"]
        for pipe in (fused_pipe, three_pipe):
            err = rra.rra_get_device_error(pipe.bufs.err, stream)
            if err != 0:
                raise RuntimeError(f"device error {rra.rra_status_string(err)} in sweep cell {name}")
        alg = {}
        for l in lengths:
            for kk, bb in algorithmic_bytes(B, N, l, row_bytes, row_bytes).items():
                alg[kk] = alg.get(kk, 0) + bb
        kt = kernel_table(kern, alg, len(masks), hbm_peak)
        kt3 = kernel_table(kern3, alg, len(masks), hbm_peak)
        flops = attention_flops([(H, l) for l in lengths])
        k_us = kt["pack_attend_unpack"]["us_per_launch"] * len(masks)
        entry.update({
            "us_cold": us_cold, "tokens_per_s": T_call / (us_cold * 1e-6),
            "kernel_us": kt["pack_attend_unpack"]["us_per_launch"],
            "frac_of_hbm": kt["pack_attend_unpack"]["frac_of_hbm"],
            "attention_tflops": flops / (k_us * 1e-6) / 1e12,
            "three_calls": {"us_cold": us_cold3, "kernels_us": {kk: vv["us_per_launch"] for kk, vv in kt3.items()},
                            "frac_of_hbm": {kk: vv["frac_of_hbm"] for kk, vv in kt3.items()},
                            "identical_output": all(torch.equal(a.view(torch.uint8), b.view(torch.uint8))
                                                    for a, b in zip(fused_pipe.ys, three_pipe.ys))},
        })
        cells[name] = entry
        del res, fused_pipe, three_pipe
    return {n: cells[n] for n in names}


def main_gpu(args):
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev_index = torch.cuda.current_device()
    w = workloads.by_name(args.workload)
    stream = torch.cuda.Stream()
    out_dtype = torch.float32 if args.out == "f32" else None
    dq, dk, dv = (t.cuda() for t in (w.q, w.k, w.v))
    dmasks = [m.cuda() for m in w.masks]
    pipe = Pipeline(dq, dk, dv, dmasks, out_dtype, stream, args.path)
    pipe.capture()
    stages = len(w.masks)
    lengths = w.lengths
    T_call = int(sum(int(l.sum()) for l in lengths))
    row_bytes = w.H * 64 * w.q.element_size()
    out_row_bytes = w.H * 64 * pipe.bufs.y.element_size()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev_index) as clk:
        step_ms, kern_ms = time_path(pipe, flush, args.steps, args.warmup, stream)
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    err = rra.rra_get_device_error(pipe.bufs.err, stream)
    if err != 0:
        raise RuntimeError(f"device error {rra.rra_status_string(err)} in the timed region")
    total_ms = reduce_max(float(sum(step_ms)), device="cuda")
    ms_per_step = total_ms / args.steps
    value = job_throughput(ws, args.steps, T_call, total_ms)

    # the other path, same workload, same protocol (reported beside the headline)
    other = Pipeline(dq, dk, dv, dmasks, out_dtype, stream, "three" if args.path == "fused" else "fused")
    other.capture()
    o_step_ms, o_kern_ms = time_path(other, flush, args.steps, args.warmup, stream)
    err = rra.rra_get_device_error(other.bufs.err, stream)
    if err != 0:
        raise RuntimeError(f"device error {rra.rra_status_string(err)} on the {other.path} path")
    same = all(torch.equal(a.view(torch.uint8), b.view(torch.uint8)) for a, b in zip(pipe.ys, other.ys))

    # dispatch floor: host time to enqueue one graph replay, and one eager call through the API
    torch.cuda.synchronize()
    n_disp = 0 if args.profile else 200
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0 = time.perf_counter()
        for _ in range(n_disp):
            pipe.graph.replay()
        host_graph_us = (time.perf_counter() - t0) / max(n_disp, 1) * 1e6
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(n_disp):
            pipe.enqueue()
        host_eager_us = (time.perf_counter() - t0) / max(n_disp, 1) * 1e6
        torch.cuda.synchronize()
    # back-to-back replays (warm L2): device time per call including graph launch gaps
    warm_us = None
    if n_disp:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(n_disp):
                pipe.graph.replay()
            end.record(stream)
        torch.cuda.synchronize()
        warm_us = start.elapsed_time(end) / n_disp * 1e3

    # ---- roofline of the dominant kernel
    hbm_peak, peak_kind = peaks()
    alg = {}
    for l in lengths:
        for k, b in algorithmic_bytes(w.B, w.N, l, row_bytes, out_row_bytes).items():
            alg[k] = alg.get(k, 0) + b
    per_kernel = kernel_table(kern_ms, alg, stages, hbm_peak)
    other_kernels = kernel_table(o_kern_ms, alg, stages, hbm_peak)
    roofline = None
    flops = attention_flops([(w.H, l) for l in lengths])
    exps = sum(w.H * int((l.astype(np.int64) ** 2).sum()) for l in lengths)
    if per_kernel:
        dom = max(per_kernel, key=lambda k: per_kernel[k]["us_per_launch"])
        ach = per_kernel[dom]["gbs"]
        clk_summary = clk.summary()
        sm_mhz = clk_summary["sm_mhz"] or clk_summary["sm_max_mhz"] or 1965
        bounds = None
        ex2 = None
        if dom in ("attend", "pack_attend_unpack"):
            n_sms = torch.cuda.get_device_properties(dev_index).multi_processor_count
            ex2_per_s = None if args.profile else measure_ex2_rate(stream, n_sms)
            ex2 = {"per_s": ex2_per_s, "source": "microbenchmark (libmicrobench.so, CUDA events)"}
            if ex2_per_s is None:
                ex2_per_s = EX2_PER_CLK_PER_SM * n_sms * sm_mhz * 1e6
                ex2 = {"per_s": ex2_per_s, "source": "nominal 16 per clock per SM"}
            ex2["per_clk_per_sm"] = ex2_per_s / (n_sms * sm_mhz * 1e6)
            bounds = attention_bounds_us(per_kernel[dom]["alg_bytes_per_launch"], flops / stages, exps / stages,
                                         hbm_peak, ex2_per_s)
        roofline = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                    "frac": ach / hbm_peak, "peak_source": peak_kind, "traffic": ncu_traffic(dom, w.name),
                    "alg_bytes_per_launch": per_kernel[dom]["alg_bytes_per_launch"],
                    "us_per_launch": per_kernel[dom]["us_per_launch"],
                    "lower_bounds_us": bounds, "ex2_rate": ex2,
                    "exps_per_launch": exps / stages, "flops_per_launch": flops / stages}
    attn_key = "pack_attend_unpack" if args.path == "fused" else "attend"
    attn_tflops = (flops / (per_kernel[attn_key]["us_per_launch"] * stages * 1e-6) / 1e12) if per_kernel else None

    # ---- end to end through the public API: pinned host inputs in, padded result out
    e2e = None
    if not args.no_e2e and not args.profile:
        host_in = [t.contiguous().pin_memory() for t in (w.q, w.k, w.v)]
        host_masks = [m.contiguous().pin_memory() for m in w.masks]
        host_out = [torch.empty(pipe.ys[0].shape, dtype=pipe.ys[0].dtype).pin_memory() for _ in w.masks]
        hs = rra.HostStream(w.B, w.N, w.H, w.q.dtype, stages=len(w.masks), chunk=E2E_CHUNK, out_dtype=out_dtype,
                            fused=args.path == "fused")
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def e2e_step():
            hs(host_masks, *host_in, host_out, stream=stream)
        for _ in range(max(3, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        e2e_ms = []
        for _ in range(args.steps):
            with torch.cuda.stream(stream):
                flush.fill_(1)
                e_start.record(stream)
            e2e_step()
            with torch.cuda.stream(stream):
                e_end.record(stream)
            stream.synchronize()
            e2e_ms.append(e_start.elapsed_time(e_end))
        tot = reduce_max(float(sum(e2e_ms)), device="cuda")
        h2d = 3 * w.q.numel() * w.q.element_size() + sum(m.numel() for m in w.masks)
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        e2e = {"value": job_throughput(ws, args.steps, T_call, tot), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": tot / args.steps,
               "api": f"rra.HostStream ({args.path} path, chunks of {min(E2E_CHUNK, w.B)} images: host-to-device copies, "
                      "kernels and device-to-host copies of successive chunks overlap)"}
        err2 = rra.rra_get_device_error(hs.err, stream)
        if err2 != 0:
            raise RuntimeError(f"device error {rra.rra_status_string(err2)} in the e2e region")
        del hs

    mask_producer = None if args.profile else time_mask_producer(w.B, w.N, w.H, w.seed, flush, stream, args.steps,
                                                                 args.warmup, hbm_peak)
    deit_block = None
    if not args.profile and not args.no_block and ws == 1:
        cu0 = torch.from_numpy(np.concatenate([[0], np.cumsum(w.lengths[0])]).astype(np.int32)).cuda()
        deit_block = time_block(w, cu0, flush, stream, args.steps, args.warmup)
    del pipe.graph_ev, other.graph_ev

    sweep = None
    if ws == 1 and not args.no_sweep and not args.profile:
        del other
        torch.cuda.empty_cache()
        with ClockSampler(dev_index, period_s=0.005) as sclk:
            floor = empty_graph_floor(stream)
            cells = run_sweep(workloads.sweep_names() if args.sweep == "all" else args.sweep.split(","), flush,
                              stream, hbm_peak)
        sweep = {"inputs": "Q/K/V drawn on the device (seeded, N(0, std^2) as each config), masks from each "
                           "config's recipe; L2 flushed (256 MiB write) before every cold replay",
                 "empty_graph_floor_us": floor, "clocks": sclk.summary(), "cells": cells}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and not args.profile:
        cpu = cpu_baseline(w, args.cpu_seconds)

    comparators = None
    if rank == 0 and ws == 1 and not args.profile and not args.no_comparators:
        comparators = {}
        for wl in dict.fromkeys(("c5:0.2:512", args.workload)):
            try:
                comparators[wl] = run_comparators(wl, min(args.steps, 10), 3)
                torch.cuda.empty_cache()
            except Exception as e:  # measurement context only: never lose the line for it
                comparators[wl] = {"error": f"{type(e).__name__}: {e}"[:200]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": {torch.bfloat16: "bf16", torch.float16: "f16"}[w.q.dtype],
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d": 64, "stages": stages,
                       "tokens_per_call": T_call, "seed": w.seed, "recipe": w.recipe, "path": args.path,
                       "out_dtype": str(pipe.bufs.y.dtype).replace("torch.", ""),
                       "l2": "flushed before every timed step (256 MiB write, untimed); inputs also exceed L2",
                       "parallelism": f"replicas x{ws}"},
            "us_per_call": ms_per_step * 1e3,
            "us_per_call_warm_back_to_back": warm_us,
            "host_dispatch_us": {"graph_replay": host_graph_us, "eager_call": host_eager_us},
            "kernels": per_kernel,
            "other_path": {"path": "three" if args.path == "fused" else "fused",
                           "us_per_call": 1e3 * statistics.mean(o_step_ms),
                           "tokens_per_s": T_call / (1e-3 * statistics.mean(o_step_ms)), "kernels": other_kernels,
                           "identical_output": bool(same)},
            "attention_tflops": attn_tflops,
            "mask_producer": mask_producer,
            "deit_block": deit_block,
            "roofline": roofline,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "clocks": clk.summary(),
            "gpu_launches": args.steps * len(pipe.kernels) * stages,
            "sweep": sweep,
            "comparators": comparators,
        }
        print(json.dumps(line), flush=True)
    del pipe
    if ws > 1:
        torch.distributed.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c5:1.0:512", help="c1 | c2 | c3:B | c4 | c5:r:B | c5s:B")
    ap.add_argument("--out", choices=["native", "f32"], default="native")
    ap.add_argument("--path", choices=["fused", "three"], default="fused",
                    help="single launch (default) or the three calls pack, attend, unpack")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-block", action="store_true", help="skip the synthetic-weight DeiT block timing")
    ap.add_argument("--sweep", default="all", help="'all' or a comma-separated list of workload names")
    ap.add_argument("--profile", action="store_true",
                    help="timed steps only (no dispatch loops, e2e, sweep or CPU leg): the command ncu captures")
    ap.add_argument("--mask-only", action="store_true",
                    help="time only the token-selection step (rra_l2_mask) on the workload's shape: the "
                         "command ncu captures for it")
    ap.add_argument("--block-only", action="store_true",
                    help="time only the synthetic-weight DeiT block on the workload's packed rows: the "
                         "command ncu captures for its kernels")
    ap.add_argument("--no-comparators", action="store_true",
                    help="skip the same-box comparator timing (torch's padded and NestedTensor SDPA)")
    ap.add_argument("--comparators", action="store_true",
                    help="time only torch's padded and NestedTensor SDPA against the single launch on "
                         "the workload's inputs (measurement context; library code)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-images", type=int, default=0,
                    help="images per step of the reference arm (default: one per host core)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.mask_only:
        return main_mask(args)
    if args.comparators:
        return main_comparators(args)
    if args.block_only:
        return main_block(args)
    return main_gpu(args)


def main_block(args):
    """One GPU: the synthetic-weight DeiT block alone on the workload's packed rows."""
    w = workloads.by_name(args.workload)
    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    cu0 = torch.from_numpy(np.concatenate([[0], np.cumsum(w.lengths[0])]).astype(np.int32)).cuda()
    print(json.dumps({"workload": w.name, "deit_block": time_block(w, cu0, flush, stream, args.steps, args.warmup)}),
          flush=True)
    return 0


def main_comparators(args):
    """One GPU: `run_comparators` on the workload, printed as one JSON line."""
    print(json.dumps({"comparators": run_comparators(args.workload, args.steps, args.warmup)}), flush=True)
    return 0


def run_comparators(workload, steps, warmup):
    """The same-box comparators on identical inputs, against the single launch --
    torch's padded SDPA (scaled_dot_product_attention over [B, H, N, 64] with a key-padding mask)
    and SDPA over a jagged NestedTensor of the kept tokens (values [T, H, 64] built once, outside
    the timed call).  Both are library code, called as they are.  Reports µs per call (events, L2
    flushed before each call) and the largest difference from the single launch's output on the
    kept rows."""
    import torch.nn.functional as F
    B, N, H, dt, std = workloads.shape_of(workload)
    q, k, v = workloads.device_values(B, N, H, dt, std=std)
    mask = torch.from_numpy(workloads.sweep_masks(workload)[0]).cuda()
    keep = mask.bool()
    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    y = torch.empty_like(q)
    cu = torch.empty(B + 1, dtype=torch.int32, device="cuda")
    qt, kt, vt = (t.transpose(1, 2) for t in (q, k, v))
    am = keep[:, None, None, :]
    with torch.cuda.stream(stream):
        rra.rra_pack_attend_unpack(mask, q, k, v, y, cu, stream=stream)
        offsets = cu.long()
        nq, nk, nv = (torch.nested.nested_tensor_from_jagged(t[keep], offsets).transpose(1, 2) for t in (q, k, v))
    stream.synchronize()

    def ours():
        rra.rra_pack_attend_unpack(mask, q, k, v, y, cu, stream=stream)

    out = {}

    def padded():
        out["padded"] = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am)

    def nested():
        out["nested"] = F.scaled_dot_product_attention(nq, nk, nv)

    def timed(fn):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ms = []
        for i in range(warmup + steps):
            with torch.cuda.stream(stream):
                flush.fill_((i + 1) & 0xFF)
                start.record(stream)
                fn()
                end.record(stream)
            stream.synchronize()
            if i >= warmup:
                ms.append(start.elapsed_time(end))
        return 1e3 * statistics.mean(ms)

    res = {"workload": workload, "B": B, "N": N, "H": H, "T": int(keep.sum()), "ours_us": timed(ours)}
    ref = y[keep].float()
    for name, fn in (("padded_sdpa", padded), ("nested_sdpa", nested)):
        try:
            res[name + "_us"] = timed(fn)
            o = out["padded"].transpose(1, 2)[keep] if name == "padded_sdpa" else out["nested"].transpose(1, 2).values()
            res[name + "_max_abs_diff"] = float((o.float() - ref).abs().max())
            res[name + "_over_ours"] = res[name + "_us"] / res["ours_us"]
        except Exception as e:  # a library path this torch build does not offer
            res[name + "_unavailable"] = f"{type(e).__name__}: {e}"[:200]
    return res


def main_mask(args):
    """One GPU: rra_l2_mask alone on the workload's shape (L2 flushed before each launch)."""
    w = workloads.by_name(args.workload)
    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    hbm_peak, _ = peaks()
    r = time_mask_producer(w.B, w.N, w.H, w.seed, flush, stream, args.steps, args.warmup, hbm_peak)
    print(json.dumps({"workload": w.name, "mask_producer": r}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
