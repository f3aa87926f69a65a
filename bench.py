"""Benchmark: packed variable-length attention forward on B200.

One step = one call of the C-ABI forward (schedule kernel + attention
kernel) over one packed batch of the long causal GQA workload (16 sequences,
lengths U[2048, 8192], 32 query / 8 K/V heads, head_dim 128, causal), inputs
already resident in HBM. The batch is seeded and synthetic.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--config 1..5] [--flush-l2]

``--config`` times one of the other named workloads instead (the parity-test
configurations: tiny packed causal, GenRec prompts, graph batch with pair and
per-key biases, short-query GQA); ``--flush-l2`` writes a 256 MB scrub buffer
between timed steps and times each call with its own events.

Prints one JSON line (rank 0). Under torchrun every rank runs its own batch
(weak scaling: per-GPU work fixed, no data-path collective); the time is the
max over ranks and the value the sum of all ranks' useful FLOPs over it.
``--impl reference`` times the CPU oracle on bounded samples of the same
workload instead (rank 0 only).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "varlen attn fwd useful TFLOP/s & tokens/s on 1 B200; % of bf16 tensor peak"
WORKLOAD = 5            # the long causal GQA workload; --config picks another
# Per workload: what bounds the kernel, and how its inputs were drawn.
BOUND = {1: "tensor", 2: "tensor", 3: "hbm", 4: "hbm", 5: "tensor"}
LENGTHS = {1: "fixed {5, 17, 32, 64}", 2: "uniform [128, 2048]", 3: "uniform [1, 256]",
           4: "fixed Lq 112, Lk 262", 5: "uniform [2048, 8192]"}
BIAS = {3: "pair grid fp32 [512,1,256,256] N(0,1), strides (65536,0,256,1); "
           "per-key fp32 [Tk,8] N(0,0.5)"}
L2_SCRUB_BYTES = 256 << 20
KERNEL_SOURCES = ["attn_sm100.cuh", "ptx.cuh", "common.cuh"]
PROFILE_FILE = os.path.join(ROOT, "profiles", "attn_fwd_sm100_long_causal_gqa.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's datasheet dense BF16 tensor figure for one B200: the HGX B200
# datasheet lists 36 PFLOPS FP16/BF16 per 8 GPUs with 2:4 sparsity, i.e.
# 18 PFLOPS dense per 8 GPUs = 2.25 PFLOPS per GPU.
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_SOURCE = ("NVIDIA HGX B200 datasheet: 36 PFLOPS FP16/BF16 per 8 GPUs with 2:4 "
                    "sparsity = 2.25 PFLOPS dense per GPU")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "packed_variable_length_attn_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _profiled_traffic():
    """DRAM bytes per launch of the attention kernel on the full long
    workload, from the committed ncu capture record, if it was taken on the
    current kernel source; else None."""
    try:
        with open(PROFILE_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha") != kernel_source_hash():
        return None
    try:
        return float(rec["dram_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


class ClockSampler:
    """SM clock, power and clock-event reasons of the benchmark's GPU, sampled
    every 10 ms through NVML (read-only queries) while the timed region runs;
    falls back to `nvidia-smi -lms 200`. summary() keeps the samples taken
    between mark_start() and mark_stop() (host time around the region)."""

    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    # NVML clocks-event reason bits
    BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
            "sw_power_cap": 0x4}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.rows = []  # (host time, sm MHz, max MHz, power W, set of reasons)
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.t0 = None
        self.t1 = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.cuda_index)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            u = str(uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            busid = (f"{getattr(props, 'pci_domain_id', 0):08X}:{bus:02X}:"
                     f"{getattr(props, 'pci_device_id', 0):02X}.0")
            return pynvml.nvmlDeviceGetHandleByPciBusId(busid)
        return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        try:
            import pynvml
            h = self._nvml_handle()
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self.stop_flag.is_set():
                    try:
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                        bits = get_reasons(h)
                        rs = {n for n, b in self.BITS.items() if bits & b}
                        self.rows.append((time.perf_counter(), float(sm), float(mx), pw, rs))
                    except Exception:  # noqa: BLE001 - a failed sample is skipped
                        pass
                    self.stop_flag.wait(0.01)
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            self.source = "nvml 10 ms"
            return
        except Exception:  # noqa: BLE001 - no NVML: fall back to nvidia-smi
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.cuda_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi 200 ms"
        self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _read_smi(self):
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9 and num(parts[1]) is not None:
                rs = {self.NAMES[i] for i in range(4) if parts[5 + i].lower() == "active"}
                self.rows.append((time.perf_counter(), num(parts[1]), num(parts[2]),
                                  num(parts[3]), rs))

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_stop(self):
        self.t1 = time.perf_counter()

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        rows = self.rows
        if self.t0 is not None and self.t1 is not None:
            inside = [r for r in rows if self.t0 <= r[0] <= self.t1]
            if inside:
                rows = inside
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0,
                    "source": self.source}
        sm = [r[1] for r in rows if r[1] is not None]
        mx = [r[2] for r in rows if r[2] is not None]
        pw = [r[3] for r in rows if r[3] is not None]
        reasons = sorted(set().union(*[r[4] for r in rows]))
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "power_w": statistics.median(pw) if pw else None,
                "samples": len(rows), "source": self.source}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _workload(args, seed=None):
    from packed_variable_length_attn_b200 import workloads
    w = workloads.make(getattr(args, "config", WORKLOAD), seed=seed)
    if args.sequences and args.sequences < w.batch:
        n = args.sequences
        tq, tk = int(w.cu_q[n]), int(w.cu_k[n])
        w = workloads.Workload(f"{w.name}_first{n}", w.lengths_q[:n], w.lengths_k[:n],
                               w.cu_q[:n + 1].clone(), w.cu_k[:n + 1].clone(), w.q[:tq].clone(),
                               w.k[:tk].clone(), w.v[:tk].clone(), w.n_heads, w.n_kv_heads,
                               w.head_dim, w.causal, w.softmax_scale,
                               None if w.bias_key is None else w.bias_key[:tk].clone(),
                               w.bias_pair, w.bias_strides, meta=dict(w.meta))
    return w


def run_reference(args, world, rank):
    """The CPU oracle on bounded samples of the workload, on the host cores."""
    if rank != 0:
        return
    w = _workload(args)
    # size each step so that warm-up + timed steps take about args.ref_total_s
    per_step = max(0.2, min(args.cpu_budget, args.ref_total_s / (args.steps + args.warmup)))
    res = oracle_sample_rate(w, budget_s=per_step)
    steps = args.steps
    times = []
    for _ in range(args.warmup):
        oracle_sample_rate(w, budget_s=None, n_rows=res["n_rows"], seed=1)
    for k in range(steps):
        r = oracle_sample_rate(w, budget_s=None, n_rows=res["n_rows"], seed=2 + k)
        times.append(r)
    flops = sum(r["flops"] for r in times)
    secs = sum(r["seconds"] for r in times)
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": _config(w, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": res["cores"],
                         "kind": "oracle",
                         "sample": f"{res['n_rows']} random (sequence, head, query row) outputs "
                                   "of the workload per step, useful FLOPs of those rows"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def oracle_sample_rate(w, budget_s=None, n_rows=None, seed=0):
    """Time oracle.rows on random output rows; returns flops, seconds, rows."""
    import numpy as np
    import oracle
    cores = oracle.default_threads()
    rng = np.random.default_rng(seed)

    def pick(n):
        seq = rng.integers(0, w.batch, n)
        head = rng.integers(0, w.n_heads, n)
        row = np.array([rng.integers(0, w.lengths_q[s]) for s in seq])
        return seq, head, row

    def flops_of(seq, row):
        tot = 0
        for s, r in zip(seq, row):
            lq, lk = w.lengths_q[s], w.lengths_k[s]
            nv = min(max(r + lk - lq + 1, 0), lk) if w.causal else lk
            tot += 4 * w.head_dim * nv
        return tot

    def timed(n):
        seq, head, row = pick(n)
        t0 = time.perf_counter()
        oracle.rows(w.q, w.k, w.v, w.cu_q, w.cu_k, w.n_heads, w.n_kv_heads, w.softmax_scale,
                    w.causal, seq, head, row, bias_key=w.bias_key, bias_pair=w.bias_pair,
                    bias_strides=w.bias_strides if w.bias_pair is not None else None,
                    threads=cores)
        return flops_of(seq, row), time.perf_counter() - t0

    if n_rows is None:
        n = 4 * cores
        f, s = timed(n)
        while s < 0.5:
            n *= 4
            f, s = timed(n)
        n_rows = max(1, int(n * budget_s / max(s, 1e-6)))
    f, s = timed(n_rows)
    return {"flops": f, "seconds": s, "n_rows": n_rows, "cores": cores}


def _config(w, args=None):
    from packed_variable_length_attn_b200 import metrics
    cfg = getattr(args, "config", WORKLOAD)
    pairs = metrics.useful_pairs(w.lengths_q, w.lengths_k, w.causal)
    qkv_bytes = (w.q.numel() + w.k.numel() + w.v.numel()) * 2
    if getattr(args, "flush_l2", False):
        l2 = f"L2 flushed: {L2_SCRUB_BYTES >> 20} MB scrub write between timed steps"
    elif qkv_bytes > 126e6:
        l2 = f"inputs larger than L2 (Q+K+V {qkv_bytes / 1e9:.2f} GB > 126 MB); no flush"
    else:
        l2 = f"hot L2 (Q+K+V {qkv_bytes / 1e6:.1f} MB; no flush)"
    d = {"workload": w.name, "sequences": w.batch, "lengths": LENGTHS[cfg],
         "total_tokens": w.total_q, "n_heads": w.n_heads, "n_kv_heads": w.n_kv_heads,
         "head_dim": w.head_dim, "causal": w.causal, "bias": BIAS.get(cfg),
         "useful_pairs_per_head": pairs, "seed": w.meta.get("seed"), "l2": l2}
    if getattr(args, "graph", False):
        d["launch"] = "CUDA graph replay of the captured step"
    if w.batch <= 64:
        d["lengths_drawn"] = list(w.lengths_q)
    return d


def rank_seed(rank: int, config: int = WORKLOAD) -> int:
    """Each rank draws its own batch of the workload (weak scaling)."""
    from packed_variable_length_attn_b200 import workloads
    return workloads.SEED_BASE + config + 1000 * rank


def reduce_over_ranks(stats, totals, world, device=None):
    """MAX over ranks of the times [timed ms, end-to-end ms, kernel ms] (the
    job is as slow as its slowest rank) and SUM of the work [FLOPs, tokens].
    The only collectives of the benchmark; every rank calls this once."""
    import torch
    import torch.distributed as dist
    s = torch.tensor(list(stats), dtype=torch.float64, device=device)
    t = torch.tensor(list(totals), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(s, op=dist.ReduceOp.MAX)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return s.tolist(), t.tolist()


def throughput_tflops(all_flops: float, ms_per_step: float) -> float:
    """Whole-job useful TFLOP/s: the FLOPs of all ranks over the slowest rank's time."""
    return all_flops / (ms_per_step * 1e-3) / 1e12


def run_gpu(args, world, rank, local):
    import torch
    import torch.distributed as dist
    import packed_variable_length_attn_b200 as va
    from packed_variable_length_attn_b200 import metrics, workloads

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    w = _workload(args, seed=rank_seed(rank, args.config))
    flops = metrics.useful_flops(w.lengths_q, w.lengths_k, w.causal, w.n_heads, w.head_dim)
    dev = torch.device("cuda", local)
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    cu_q, cu_k = w.cu_q.to(dev), w.cu_k.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.n_heads, w.total_q), dtype=torch.float32, device=dev)
    bias_kw = dict(
        bias_per_key=None if w.bias_key is None else w.bias_key.to(dev),
        bias_pair=None if w.bias_pair is None else w.bias_pair.to(dev),
        bias_pair_strides=w.bias_strides if w.bias_pair is not None else None)
    stream = torch.cuda.current_stream()

    def step():
        va.varlen_attn_fwd(q, k, v, cu_q, cu_k, w.max_seqlen_q, w.max_seqlen_k,
                           softmax_scale=w.softmax_scale, causal=w.causal, out=out, lse=lse,
                           **bias_kw)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if va.get_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    graph = None
    if args.graph:
        # the step captured once in a CUDA graph (after a warm-up call on the
        # capture stream, which sizes the library's workspace there) and
        # replayed: no host work per step
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            step()
        stream.wait_stream(cap)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            step()
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        if va.get_device_error() != 0:
            raise RuntimeError("device error during graph warm-up")

    # ---- timed region: K steps, device events, per-launch kernel events
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in kev:  # torch creates the CUDA events on first record
        a.record(stream)
        b.record(stream)
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.1)  # let the sampler start before the timed region
    sampler.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if args.flush_l2:
        # each call timed on its own, a scrub write larger than L2 between calls
        scrub = torch.empty(L2_SCRUB_BYTES // 4, dtype=torch.float32, device=dev)
        cev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.steps):
            scrub.fill_(float(i))
            cev[i][0].record(stream)
            if graph is not None:
                kev[i][0].record(stream)
                graph.replay()
                kev[i][1].record(stream)
            else:
                va.set_profile_events(*kev[i])
                step()
                va.set_profile_events()
            cev[i][1].record(stream)
    else:
        # one pass: the step time over K calls and, in the same calls, the
        # attention kernel's own time from events the library records around
        # its launch. (Those events sit between the schedule and attention
        # launches, so during timing the attention kernel's set-up does not
        # overlap the schedule kernel as it does in an unprofiled call.)
        t0.record(stream)
        if graph is not None:
            # per-step events around each replay (schedule + attention kernel)
            for i in range(args.steps):
                kev[i][0].record(stream)
                graph.replay()
                kev[i][1].record(stream)
        else:
            for i in range(args.steps):
                va.set_profile_events(*kev[i])
                step()
            va.set_profile_events()
        t1.record(stream)
    torch.cuda.synchronize()
    sampler.mark_stop()
    sampler.stop()
    if world > 1:
        dist.barrier()
    if args.flush_l2:
        elapsed_ms = sum(a.elapsed_time(b) for a, b in cev)
    else:
        elapsed_ms = t0.elapsed_time(t1)
    kernel_ms = [a.elapsed_time(b) for a, b in kev]
    if va.get_device_error() != 0:
        raise RuntimeError("device error during the timed region")

    # ---- end to end through host buffers (pinned), copies inside the region.
    # Every step copies its inputs host -> device, runs the call and reads its
    # output and LSE back to the host. Steps are pipelined the way a serving
    # loop would run them: two sets of device buffers, the input copies on one
    # copy stream and the output copies on another, so step k + 1's inputs
    # travel while step k computes and step k - 1's results come back (each
    # direction of the host link busy on its own).
    hq, hk, hv = q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()
    hcq, hck = cu_q.cpu().pin_memory(), cu_k.cpu().pin_memory()
    hbias = {key: t.cpu().pin_memory() for key, t in
             (("bias_per_key", bias_kw["bias_per_key"]), ("bias_pair", bias_kw["bias_pair"]))
             if t is not None}
    n_buf = 2
    hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(n_buf)]
    hlse = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(n_buf)]
    dbuf = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                 cq=torch.empty_like(cu_q), ck=torch.empty_like(cu_k), out=torch.empty_like(out),
                 lse=torch.empty_like(lse),
                 **{key: torch.empty_like(bias_kw[key]) for key in hbias})
            for _ in range(n_buf)]
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    computed = [None] * n_buf   # event: the call of the buffer set's last step is done
    read_back = [None] * n_buf  # event: its output has been copied to the host

    def e2e_step(kstep):
        b = kstep % n_buf
        d = dbuf[b]
        with torch.cuda.stream(h2d_stream):
            if computed[b] is not None:
                h2d_stream.wait_event(computed[b])   # inputs of set b no longer read
            d["q"].copy_(hq, non_blocking=True)
            d["k"].copy_(hk, non_blocking=True)
            d["v"].copy_(hv, non_blocking=True)
            d["cq"].copy_(hcq, non_blocking=True)
            d["ck"].copy_(hck, non_blocking=True)
            for key, t in hbias.items():
                d[key].copy_(t, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(h2d_stream)
        stream.wait_event(loaded)
        if read_back[b] is not None:
            stream.wait_event(read_back[b])          # output of set b copied out
        va.varlen_attn_fwd(d["q"], d["k"], d["v"], d["cq"], d["ck"], w.max_seqlen_q,
                           w.max_seqlen_k, softmax_scale=w.softmax_scale, causal=w.causal,
                           out=d["out"], lse=d["lse"], stream=stream,
                           bias_per_key=d.get("bias_per_key"), bias_pair=d.get("bias_pair"),
                           bias_pair_strides=bias_kw["bias_pair_strides"])
        done = torch.cuda.Event()
        done.record(stream)
        computed[b] = done
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(done)
            hout[b].copy_(d["out"], non_blocking=True)
            hlse[b].copy_(d["lse"], non_blocking=True)
            rb = torch.cuda.Event()
            rb.record(d2h_stream)
        read_back[b] = rb

    e2e_step(0)
    torch.cuda.synchronize()
    if not (torch.equal(hout[0].view(torch.int16), out.cpu().view(torch.int16))):
        raise RuntimeError("end-to-end output differs from the device-timed output")
    e_steps = max(1, min(args.steps, args.e2e_steps))
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)
    computed = [None] * n_buf
    read_back = [None] * n_buf
    for kstep in range(e_steps):
        e2e_step(kstep)
    for ev in read_back:
        if ev is not None:
            stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcq, hck, *hbias.values()))
    d2h = hout[0].numel() * hout[0].element_size() + hlse[0].numel() * hlse[0].element_size()

    # ---- reduce over ranks
    (elapsed_ms, e2e_ms, kern_ms), (all_flops, all_tokens) = reduce_over_ranks(
        [elapsed_ms, e2e_ms, sum(kernel_ms) / len(kernel_ms)], [float(flops), float(w.total_q)],
        world, device=dev)

    if rank == 0:
        peaks, peak_src = _peaks()
        ms_per_step = elapsed_ms / args.steps
        value = throughput_tflops(all_flops, ms_per_step)
        achieved = flops / (kern_ms * 1e-3) / 1e12  # this rank's kernel, per launch
        peak = float(peaks["bf16_tflops"])
        # profiled on the full long workload only
        traffic = (_profiled_traffic()
                   if not args.sequences and args.config == WORKLOAD and not args.flush_l2
                   else None)
        bound = BOUND[args.config]
        if bound == "hbm":
            abytes = metrics.algorithmic_bytes(w)
            rl = {"bound": "hbm", "achieved": abytes / (kern_ms * 1e-3) / 1e9,
                  "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                  "algorithmic_bytes_per_launch": abytes,
                  "peak_source": f"{peak_src} hbm_gbs",
                  "tflops_per_launch": flops / (kern_ms * 1e-3) / 1e12}
        else:
            rl = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                  "peak_source": f"{peak_src} bf16_tflops (burst)",
                  "frac_of_sustained": achieved / float(peaks["bf16_tflops_sustained"])}
        rl["frac"] = rl["achieved"] / rl["peak"]
        clk = sampler.summary()
        rl["sm_mhz_median"] = clk["sm_mhz"]
        if bound == "tensor":
            rl["datasheet_peak"] = DATASHEET_BF16_TFLOPS
            rl["frac_of_datasheet"] = achieved / DATASHEET_BF16_TFLOPS
            rl["datasheet_source"] = DATASHEET_SOURCE
        rl["traffic"] = traffic
        rl["kernel"] = (f"attn_fwd_sm100<{w.head_dim},{str(w.bias_key is not None).lower()},"
                        f"{str(w.bias_pair is not None).lower()}>")
        rl["kernel_ms_per_launch"] = kern_ms
        if args.graph:
            rl["kernel_ms_covers"] = "one graph replay: schedule and attention kernels"
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": f"synthetic (seeded N(0,1) bf16 Q/K/V; lengths {LENGTHS[args.config]})",
            "config": _config(w, args),
            "tokens_per_s": all_tokens / (ms_per_step * 1e-3),
            "pct_of_bf16_peak": 100.0 * value / (peak * world),
            "roofline": rl,
            "e2e": {"value": throughput_tflops(all_flops, e2e_ms), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": e_steps},
            "gpu_launches": va.launches_per_call() * args.steps,
            "clocks": clk,
        }
        if not args.no_cpu_baseline:
            r = oracle_sample_rate(w, budget_s=args.cpu_budget)
            line["cpu_baseline"] = {
                "value": r["flops"] / r["seconds"] / 1e12, "unit": "TFLOP/s",
                "cores": r["cores"], "kind": "oracle",
                "sample": f"{r['n_rows']} random (sequence, head, query row) outputs of the "
                          f"workload, {r['seconds']:.1f} s, useful FLOPs of those rows"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_layout(args, world, rank, local):
    """Packed-layout helpers on the long workload's Q padded to [16, 8192, 32, 128]
    bf16 (1.07 GB): unpad = mask_to_seqlens + gather_rows, pad = scatter_rows
    (zero fill + scatter). HBM-bound copies, reported as GB/s of the bytes they
    must move against the measured HBM peak. One JSON line per helper."""
    import torch
    import packed_variable_length_attn_b200 as va
    if rank != 0:
        return
    torch.cuda.set_device(local)
    w = _workload(args, seed=rank_seed(0, WORKLOAD))
    B, S = w.batch, 8192
    H, D = w.n_heads, w.head_dim
    dev = torch.device("cuda", local)
    mask = torch.zeros(B, S, dtype=torch.uint8, device=dev)
    for b, L in enumerate(w.lengths_q):
        mask[b, :L] = 1
    x = torch.empty(B * S, H, D, dtype=torch.bfloat16, device=dev).normal_()
    T = w.total_q
    rb = H * D * 2
    packed = torch.empty(T, H, D, dtype=torch.bfloat16, device=dev)
    padded = torch.empty_like(x)
    peaks, src = _peaks()
    cu, idx, mx = va.mask_to_seqlens(mask)

    def unpad():
        c, i, _ = va.mask_to_seqlens(mask)
        va.gather_rows(x, i, c, packed)

    def pad():
        va.scatter_rows(packed, idx, cu, padded)

    ops = {"unpad": (unpad, B * S + 2 * T * rb + 4 * (B + 1) + 4 * T),
           "pad": (pad, B * S * rb + 2 * T * rb)}
    for name, (fn, nbytes) in ops.items():
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(args.steps):
            fn()
        t1.record()
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / args.steps
        gbs = nbytes / (ms * 1e-3) / 1e9
        if va.get_device_error() != 0:
            raise RuntimeError("device error in the layout helpers")
        print(json.dumps({
            "metric": f"{name} (packed-layout helper) GB/s on 1 B200", "value": gbs,
            "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (the long workload's lengths as prefix masks)",
            "config": {"workload": f"{name}_long_causal_gqa_q", "batch": B, "seqlen": S,
                       "heads": H, "head_dim": D, "packed_rows": T, "row_bytes": rb},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]),
                         "unit": "GB/s", "frac": gbs / float(peaks["hbm_gbs"]),
                         "algorithmic_bytes_per_step": nbytes, "traffic": None,
                         "peak_source": f"{src} hbm_gbs"}}), flush=True)


def run_decode(args, world, rank, local):
    """K/V-cache decode step: 64 sequences, one new query token each, cached
    lengths U[1024, 8192] in a [64, 8192, 8, 128] bf16 cache (32/8 heads, the
    long workload's head split). HBM-bound: reported as GB/s of the bytes a
    step must move (cached K and V of every sequence once, q, out, LSE)
    against the measured HBM peak. --sequences B keeps the first B sequences,
    --decode-cache-len S gives a [B, S, 8, 128] cache with lengths U[S/8, S],
    --decode-qlen the new tokens per sequence."""
    import torch
    import packed_variable_length_attn_b200 as va
    if rank != 0:
        return
    torch.cuda.set_device(local)
    g = torch.Generator("cpu").manual_seed(20261299)
    B, S, Hq, Hkv, D = 64, args.decode_cache_len, 32, 8, 128
    lens = torch.randint(S // 8, S + 1, (B,), generator=g).to(torch.int32)
    if args.sequences and args.sequences < B:  # small case for profiling
        B = args.sequences
        lens = lens[:B]
    dev = torch.device("cuda", local)
    kc = torch.randn(B, S, Hkv, D, generator=g).to(torch.bfloat16).to(dev)
    vc = torch.randn(B, S, Hkv, D, generator=g).to(torch.bfloat16).to(dev)
    QL = max(1, args.decode_qlen)  # new query tokens per sequence (speculative steps: > 1)
    q = torch.randn(B * QL, Hq, D, generator=g).to(torch.bfloat16).to(dev)
    cu_q = torch.arange(B + 1, dtype=torch.int32, device=dev) * QL
    cs = lens.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty(Hq, B * QL, dtype=torch.float32, device=dev)
    nbytes = int(lens.sum()) * Hkv * D * 2 * 2 + 2 * q.numel() * 2 + lse.numel() * 4

    def step():
        va.varlen_attn_decode(q, cu_q, QL, kc, vc, cs, num_splits=args.decode_splits,
                              out=out, lse=lse)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    # cache (8.6 GB) larger than L2: no flush needed between steps
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    if va.get_device_error() != 0:
        raise RuntimeError("device error in decode")
    peaks, src = _peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({
        "metric": "kv-cache decode step GB/s on 1 B200", "value": gbs, "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": f"synthetic (seeded N(0,1) bf16 cache and queries; cached lengths "
                f"U[{S // 8}, {S}])",
        "config": {"workload": "kv_cache_decode", "sequences": B, "q_len": QL, "cache_len": S,
                   "cached_tokens": int(lens.sum()), "n_heads": Hq, "n_kv_heads": Hkv,
                   "head_dim": D, "num_splits": args.decode_splits or "auto",
                   "l2": f"cached K/V read per step {nbytes / 1e6:.0f} MB vs 126 MB L2; "
                         f"no flush"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]),
                     "unit": "GB/s", "frac": gbs / float(peaks["hbm_gbs"]),
                     "algorithmic_bytes_per_step": nbytes, "traffic": None,
                     "peak_source": f"{src} hbm_gbs"}}), flush=True)


def run_backward(args, world, rank, local):
    """Backward pass of the named workload (default: the long causal GQA
    batch): dQ, dK, dV (and the bias gradients where the workload has biases)
    from the forward's output and LSE and a seeded dO. Useful FLOPs = 2.5x the
    forward's (five products of 2*D per visible pair and head: S, dP, dV, dK,
    dQ); the kernels' own recomputation of S and dP for dQ is not counted."""
    import torch
    import packed_variable_length_attn_b200 as va
    from packed_variable_length_attn_b200 import metrics
    if rank != 0:
        return
    torch.cuda.set_device(local)
    w = _workload(args)
    dev = torch.device("cuda", local)
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    cu_q, cu_k = w.cu_q.to(dev), w.cu_k.to(dev)
    bk = None if w.bias_key is None else w.bias_key.to(dev)
    bp = None if w.bias_pair is None else w.bias_pair.to(dev)
    kw = dict(softmax_scale=w.softmax_scale, causal=w.causal, bias_per_key=bk, bias_pair=bp,
              bias_pair_strides=w.bias_strides if bp is not None else None)
    out, lse = va.varlen_attn_fwd(q, k, v, cu_q, cu_k, w.max_seqlen_q, w.max_seqlen_k, **kw)
    g = torch.Generator("cpu").manual_seed(20261301)
    dout = torch.randn(w.q.shape, generator=g).to(torch.bfloat16).to(dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def step():
        va.varlen_attn_bwd(q, k, v, out, lse, dout, cu_q, cu_k, w.max_seqlen_q, w.max_seqlen_k,
                           need_dbias_per_key=bk is not None, need_dbias_pair=bp is not None,
                           dq=dq, dk=dk, dv=dv, **kw)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.1)
    clocks.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    clocks.mark_stop()
    clocks.stop()
    clk = clocks.summary()
    ms = t0.elapsed_time(t1) / args.steps
    if va.get_device_error() != 0:
        raise RuntimeError("device error in the backward pass")
    fwd_flops = metrics.useful_flops(w.lengths_q, w.lengths_k, w.causal, w.n_heads, w.head_dim)
    flops = 2.5 * fwd_flops
    tf = flops / (ms * 1e-3) / 1e12
    peaks, src = _peaks()
    peak = float(peaks["bf16_tflops"])
    cfg = _config(w, args)
    cfg["pass"] = "backward (dQ, dK, dV" + (", bias gradients)" if bk is not None or
                                            bp is not None else ")")
    print(json.dumps({
        "metric": "varlen attn bwd useful TFLOP/s on 1 B200", "value": tf, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V/dO)", "config": cfg,
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                     "frac": tf / peak, "traffic": None, "peak_source": f"{src} bf16_tflops",
                     "useful_flops_per_step": flops},
        "gpu_launches": 4 * args.steps, "clocks": clk}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle work for the CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-total-s", type=float, default=150.0,
                    help="--impl reference: seconds of oracle work over all steps")
    ap.add_argument("--config", type=int, default=WORKLOAD, choices=[1, 2, 3, 4, 5],
                    help="named workload (default: the long causal GQA workload)")
    ap.add_argument("--graph", action="store_true",
                    help="time CUDA-graph replays of the captured step (no host work per step); "
                         "the per-launch time then covers the schedule and attention kernels")
    ap.add_argument("--flush-l2", action="store_true",
                    help="256 MB scrub write between timed steps; each call timed alone")
    ap.add_argument("--decode", action="store_true",
                    help="time a K/V-cache decode step instead of the forward")
    ap.add_argument("--decode-qlen", type=int, default=1,
                    help="--decode: new query tokens per sequence in the step")
    ap.add_argument("--decode-splits", type=int, default=0,
                    help="--decode: 0 = automatic (tensor cores; key ranges of the cache "
                         "when the (sequence, K/V head) pairs are fewer than the SMs); "
                         "S > 0 = S key ranges on the CUDA cores")
    ap.add_argument("--decode-cache-len", type=int, default=8192,
                    help="--decode: cache rows per sequence S (cached lengths U[S/8, S])")
    ap.add_argument("--layout", action="store_true",
                    help="time the packed-layout helpers (unpad, pad) instead of the forward")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (dQ, dK, dV) instead of the forward")
    ap.add_argument("--sequences", type=int, default=0,
                    help="use only the first N sequences (small case for profiling)")
    args = ap.parse_args()
    world, rank, local = _dist()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    if args.layout:
        run_layout(args, world, rank, local)
        return
    if args.decode:
        run_decode(args, world, rank, local)
        return
    if args.backward:
        run_backward(args, world, rank, local)
        return
    run_gpu(args, world, rank, local)


if __name__ == "__main__":
    main()
