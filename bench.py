"""Throughput of the Inkling MoE feed-forward layer on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

A step is one full forward pass of the layer (router, permutation, routed and
shared expert GEMMs, recombination) over one batch of T tokens, through the
library's one-call entry point ``moe_forward``, inputs resident in HBM.  The
same steps are then run as the op chain (``moe_route``, ``moe_permute``,
``moe_expert_ffn``, ``moe_combine``) with CUDA events between the ops, for the
per-op breakdown and the expert GEMMs' roofline.  The default workload is the layer
at the pages' hidden size: T=8192, H=6144, E=128, k=8, S=1, I=2048, bf16.

N > 1 (launched by torch.distributed.run, or with ``--gpus N`` alone, which
starts the N ranks itself the same way): every rank runs an independent
replica on its own GPU with its own token batch; the layer has no exchange
step, so there is no collective on the data path (weak scaling).  Timing is
taken on the device with CUDA events and reduced as the max over ranks.

On one GPU the line also carries ``per_config``: the task's other
workloads (the H=2048 layer, one decode step, the Zipf-skewed layer) timed in
the same run, each with its expert-GEMM roofline and its whole-step HBM
fraction.

``--impl reference`` times the CPU fp64 oracle instead, on a bounded token
sample per step, on rank 0 only.

``--workload dense-...`` times the model's dense feed-forward layer
(InklingDenseMLP, ``moe_dense_mlp``) the same way: a step is one forward pass
of that layer over T tokens.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import moe_workloads as mw  # noqa: E402

METRIC = "Inkling MoE-layer tokens/s and TFLOP/s (% of B200 bf16 peak / % HBM BW), 1 GPU"
DEFAULT_WORKLOAD = "bf16-T8192-H6144-E128k8S1-I2048"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes of one moe_expert_ffn call (its four grouped-GEMM launches) on
# these workloads: ncu dram__bytes_read.sum + dram__bytes_write.sum, one pass,
# summed over the launches.  A capture constant, not a
# measurement of this run: each entry names its capture.  An entry is removed
# when the kernels change, until it is captured again.
NCU_TRAFFIC_BYTES = {
    "bf16-T8192-H6144-E128k8S1-I2048": (12736334592, "ncu capture of 2026-12-03 (the four launches of "
                                        "one moe_expert_ffn call of the op chain, fp16 down "
                                        "projections, gate_up pair tiles drawn from a counter, "
                                        "chained launches, branch-free fp16 packing), "
                                        "profiles/traffic_expert_gemms_bf16-T8192-H6144-E128k8S1-I2048.md"),
}
# The other workloads the benchmark spec states, timed in the same run as the default
# one (the "per_config" block of the JSON line).
PER_CONFIG = ["bf16-T4096-H2048-E64k6S2-I1024", "decode-bf16-T32-H6144-E128k8S1-I2048",
              "zipf-bf16-T16384-H6144-E256k8S1-I1024"]
# Tokens of the oracle's sample per step (reference arm and cpu_baseline
# alike, so that the two report the same rate): the oracle converts every
# touched expert's weights to float64 on each call, so a step of a few tokens
# would time that set-up alone.
ORACLE_TOKENS_PER_STEP = 2048


def traffic_of(name):
    t = NCU_TRAFFIC_BYTES.get(name)
    return (None, None) if t is None else t


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples, every 20 ms, kept when they fall
    inside the timed region (``mark_start`` / ``mark_end`` give its host-time
    bounds; each sample carries nvidia-smi's timestamp)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        if self.path is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                stamp, frac = (parts[0].split(".") + ["0"])[:2]
                t = time.mktime(time.strptime(stamp, "%Y/%m/%d %H:%M:%S")) + float("0." + frac)
                rows.append((t, float(parts[2]), float(parts[3]), parts[5:10]))
            except ValueError:
                continue
        os.unlink(self.path)
        inside = [r for r in rows if self.t0 is not None and self.t1 is not None
                  and self.t0 <= r[0] <= self.t1]
        window = "timed region"
        if not inside:   # a region shorter than the sampling gap: the samples nearest to it
            inside = sorted(rows, key=lambda r: abs(r[0] - ((self.t0 or 0) + (self.t1 or 0)) / 2))[:2]
            window = "nearest samples"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for _, _, _, flags in inside:
            for n, v in zip(names, flags[1:]):
                if v.lower() == "active":
                    seen.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(seen), "samples": len(inside), "window": window}


# ------------------------------------------------------------- distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def finish(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------- CPU (oracle) arm
def oracle_run(w, inputs, tokens_per_step: int, steps: int, warmup: int, threads: int,
               seed_offset: int = 0):
    import oracle
    torch.set_num_threads(threads)
    n_done = 0
    t_total = 0.0
    for i in range(warmup + steps):
        tok = mw.token_sample(w, tokens_per_step, seed_offset=1000 + seed_offset + i)
        t0 = time.perf_counter()
        oracle.moe_forward_workload(inputs, w, tokens=tok, threads=threads)
        dt = time.perf_counter() - t0
        if i >= warmup:
            n_done += tok.numel()
            t_total += dt
    return n_done / t_total, n_done, t_total


def cpu_baseline(w, inputs, min_s: float = 10.0):
    """The oracle as it stands on the host cores, on bounded token samples of
    ORACLE_TOKENS_PER_STEP tokens (the reference arm's step): seeded samples
    until the oracle has run for at least ``min_s`` seconds."""
    threads = len(os.sched_getaffinity(0))
    n = min(w.T, ORACLE_TOKENS_PER_STEP)
    done, secs, steps = 0, 0.0, 0
    while secs < min_s:
        _, d1, s1 = oracle_run(w, inputs, n, 1, 0, threads, seed_offset=steps)
        done, secs, steps = done + d1, secs + s1, steps + 1
        if n >= w.T and steps >= 1 and secs >= min_s / 4:
            break   # the whole batch once is enough of a sample
    return {"value": done / secs, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{steps} seeded samples of {n} tokens of {w.name} (oracle fp64, {secs:.1f} s)"}


def reference_arm(args, world, rank):
    """Rank 0 alone runs the oracle; other ranks exit at once (no process group)."""
    w = mw.by_name(args.workload)
    if rank != 0:
        return
    inputs = mw.generate(w)
    threads = len(os.sched_getaffinity(0))
    # the same bounded sample per step as cpu_baseline: a few seconds per step
    tokens_per_step = min(w.T, ORACLE_TOKENS_PER_STEP)
    tps, done, secs = oracle_run(w, inputs, tokens_per_step, args.steps, args.warmup, threads)
    fl = mw.flops(w, 1)["total"]
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "H": w.H, "E": w.E, "k": w.k, "S": w.S, "I": w.I,
                   "tokens_per_step": tokens_per_step},
        "tflops": tps * fl / 1e12,
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{tokens_per_step} seeded tokens per step of {w.name}"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- GPU arm
def expert_ffn_bytes(w, touched: int, yel: int = 4) -> int:
    """Algorithmic bytes of moe_expert_ffn: the weights of every group with
    rows (routed experts with a nonzero count, every shared expert) once, the
    routed A rows (x_perm) and shared A rows (x) read once, h written and read
    once (2 bytes), the down rows written once (``yel`` bytes: 4 fp32, 2 fp16)."""
    el = 2 if w.dtype == "bf16" else 4
    rows = w.T * (w.k + w.S)
    return touched * 3 * w.H * w.I * el + rows * (w.H * el + 2 * w.I * el + yel * w.H)


def step_bytes(w, touched: int, yel: int = 4) -> int:
    """Algorithmic bytes of one layer step: the expert call's bytes, plus the
    fp32 router bank and bias, x read by the router and the shared experts'
    row gather, x_perm written, the down rows read back by the combine and
    the output written."""
    el = 2 if w.dtype == "bf16" else 4
    router = 4 * (w.E + w.S) * w.H + 4 * w.E + w.T * w.H * el
    permute = w.T * w.k * w.H * el
    combine = yel * w.T * (w.k + w.S) * w.H + w.T * w.H * el
    return expert_ffn_bytes(w, touched, yel) + router + permute + combine


def groupwise_bound_ms(w, counts, peaks, yel: int = 4) -> float:
    """The expert GEMMs' floor group by group: each group (routed expert with
    rows, every shared expert) takes at least max(its flops / the burst bf16
    peak, its bytes / the measured HBM bandwidth), with bytes its weights
    once plus, per row, the A row, h written and read and the down row
    written.  Groups with few rows are bound by their weights' bytes, so this
    floor lies above the aggregate flop floor."""
    P = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * 1e12
    BW = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])) * 1e9
    el = 2 if w.dtype == "bf16" else 4
    t = 0.0
    for r in list(counts) + [w.T] * w.S:
        if r > 0:
            fl = 6.0 * r * w.H * w.I
            by = 3 * w.H * w.I * el + r * (w.H * el + 2 * w.I * el + yel * w.H)
            t += max(fl / P, by / BW)
    return t * 1e3


def gemm_roofline(w, ffn_ms: float, touched: int, peaks, peak_src: str, yel: int = 4,
                  counts=None):
    """Roofline of the expert GEMMs (the four launches of moe_expert_ffn):
    tensor-bound against the measured burst bf16 peak (the calls are timed in
    a region of well under a second), or HBM-bound against the measured copy
    bandwidth when their flops per algorithmic byte fall below the ridge."""
    fl = mw.flops(w)
    ffn_flops = fl["routed"] + fl["shared"]
    ffn_bytes = expert_ffn_bytes(w, touched, yel)
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    s = ffn_ms / 1e3
    if ffn_flops / ffn_bytes >= peak * 1e12 / (hbm_peak * 1e9):
        roof = {"bound": "tensor", "achieved": ffn_flops / s / 1e12, "peak": peak,
                "unit": "TFLOP/s", "peak_source": f"{peak_src} bf16_tflops (burst)"}
        roof["frac"] = roof["achieved"] / peak
        roof["frac_of_sustained"] = roof["achieved"] / peak_sus
    else:
        roof = {"bound": "hbm", "achieved": ffn_bytes / s / 1e9, "peak": hbm_peak,
                "unit": "GB/s", "peak_source": f"{peak_src} hbm_gbs"}
        roof["frac"] = roof["achieved"] / hbm_peak
    roof["algorithmic_bytes"] = ffn_bytes
    roof["algorithmic_flops"] = ffn_flops
    roof["touched_groups"] = touched
    if counts is not None:
        gb = groupwise_bound_ms(w, counts, peaks, yel)
        roof["groupwise_bound_ms"] = gb
        roof["frac_of_groupwise_bound"] = gb / ffn_ms
    return roof


def device_inputs(moe, inputs, dev, down_f16: bool):
    """Inputs on the device; with ``down_f16`` the down projections' weights
    are replaced by their exact fp16 copies (made once, as at model load)."""
    d = {k: v.to(dev).contiguous() for k, v in inputs.items()}
    if down_f16:
        for n in ("w_down", "ws_down"):
            if n in d and d[n].numel():
                d[n] = moe.prepare_down_weights(d[n])
    return d


def time_workload(moe, name: str, steps: int, warmup: int, dev, stream, peaks, peak_src,
                  down_bf16: bool = False):
    """One of the task's other workloads, timed in this run: its op chain
    (route, permute, expert GEMMs, combine) for ``warmup`` + ``steps`` steps
    on device-resident seeded inputs, CUDA events around every op."""
    w = mw.by_name(name)
    inputs = mw.generate(w)
    L = moe.Layer.from_workload(w, down_f16=w.dtype == "bf16" and not down_bf16)
    d = device_inputs(moe, inputs, dev, L.down_f16)
    del inputs
    ws = moe.new_workspace(L, device=dev)
    T, k, S, H, E = L.T, L.k, L.S, L.H, L.E
    tw = torch.empty(T, k, dtype=torch.float32, device=dev)
    ti = torch.empty(T, k, dtype=torch.int32, device=dev)
    sg = torch.empty(T, S, dtype=torch.float32, device=dev) if S else None
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ps = torch.empty(T * k, dtype=torch.int32, device=dev)
    ip = torch.empty(T * k, dtype=torch.int32, device=dev)
    xp = torch.empty(T * k, H, dtype=L.dtype, device=dev)
    yr = torch.empty(T * k, H, dtype=L.y_dtype, device=dev)
    ys = torch.empty(S * T, H, dtype=L.y_dtype, device=dev) if S else None
    out = torch.empty(T, H, dtype=L.dtype, device=dev)
    wsgu, wsd = (d["ws_gate_up"], d["ws_down"]) if S else (None, None)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        moe.moe_route(L, d["x"], d["w_router"], d["corr_bias"], tw, ti, sg, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        moe.moe_permute(L, ti, None, d["x"], off, ps, ip, xp, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        moe.moe_expert_ffn(L, d["x"], xp, off, ps, tw, sg, d["w_gate_up"], d["w_down"], wsgu,
                           wsd, yr, ys, ws, stream)
        if ev is not None:
            ev[3].record(stream)
        moe.moe_combine(L, yr, ys, ip, out, ws, stream)
        if ev is not None:
            ev[4].record(stream)

    def fwd():
        moe.moe_forward(L, d["x"], d["w_router"], d["corr_bias"], d["w_gate_up"], d["w_down"],
                        wsgu, wsd, out, ws, stream=stream)

    # the step through moe_forward (timed as a whole), then the op chain
    # with events between the ops (breakdown and the expert GEMMs' time)
    for _ in range(warmup):
        fwd()
    torch.cuda.synchronize(dev)
    moe.read_device_status(ws, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index or 0) as clk:
        torch.cuda.synchronize(dev)
        clk.mark_start()
        e0.record(stream)
        for i in range(steps):
            fwd()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
    ms = e0.elapsed_time(e1) / steps
    for _ in range(warmup):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    moe.read_device_status(ws, stream)
    op_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / steps for i in range(4)]
    counts = (off[1:] - off[:-1]).cpu()
    touched = int((counts > 0).sum()) + S
    yel = 2 if L.down_f16 else 4
    roof = gemm_roofline(w, op_ms[2], touched, peaks, peak_src, yel, counts.tolist())
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    sb = step_bytes(w, touched, yel)
    res = {"ms_per_step": ms, "tokens_per_s": T / (ms / 1e3),
           "tflops": mw.flops(w)["total"] / (ms / 1e3) / 1e12,
           "op_ms": {"route": op_ms[0], "permute": op_ms[1], "expert_ffn": op_ms[2],
                     "combine": op_ms[3],
                     "op_chain_step": evs[0][0].elapsed_time(evs[-1][4]) / steps},
           "expert_gemms": roof,
           "step_hbm": {"algorithmic_bytes": sb, "achieved_gbs": sb / (ms / 1e3) / 1e9,
                        "frac": sb / (ms / 1e3) / 1e9 / hbm_peak},
           "clocks": clk.summary()}
    del d, ws, xp, yr, ys
    torch.cuda.empty_cache()
    return res


def gpu_arm(args, world, rank, local):
    import mixture_experts_feed_b200 as moe

    w = mw.by_name(args.workload)
    # every replica gets its own token batch (x seed differs per rank); same weights
    wr = w.replace(seed=w.seed) if rank == 0 else w
    inputs = mw.generate(wr)
    if rank > 0:
        g = torch.Generator().manual_seed(10_000 + rank)
        inputs["x"] = torch.randn(w.T, w.H, generator=g).to(w.torch_dtype)
    # bf16 layers run their down projections in fp16 (the weights copied once
    # to fp16 here, as at model load; outside every timed region)
    L = moe.Layer.from_workload(w, down_f16=w.dtype == "bf16" and not args.down_bf16)
    dev = torch.device("cuda", local)
    d = device_inputs(moe, inputs, dev, L.down_f16)
    x_host = inputs["x"].pin_memory()
    stream = torch.cuda.current_stream(dev)
    ws = moe.new_workspace(L, device=dev)
    T, k, S, H, E = L.T, L.k, L.S, L.H, L.E
    tw = torch.empty(T, k, dtype=torch.float32, device=dev)
    ti = torch.empty(T, k, dtype=torch.int32, device=dev)
    sg = torch.empty(T, S, dtype=torch.float32, device=dev) if S else None
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ps = torch.empty(T * k, dtype=torch.int32, device=dev)
    ip = torch.empty(T * k, dtype=torch.int32, device=dev)
    # the permuted copy of x, as moe_forward makes it (--gather-rows: none;
    # the gate_up GEMM then gathers the routed rows of x itself)
    xp = None if args.gather_rows else torch.empty(T * k, H, dtype=L.dtype, device=dev)
    yr = torch.empty(T * k, H, dtype=L.y_dtype, device=dev)
    ys = torch.empty(S * T, H, dtype=L.y_dtype, device=dev) if S else None
    out = torch.empty(T, H, dtype=L.dtype, device=dev)
    out_host = torch.empty(T, H, dtype=L.dtype).pin_memory()
    wsgu = d.get("ws_gate_up") if S else None
    wsd = d.get("ws_down") if S else None

    # --prenorm: the block's RMSNorm first (its own timed op), the layer on its output
    nw = mw.norm_weight(H, seed=w.seed, dtype=L.dtype).to(dev) if args.prenorm else None
    xn = torch.empty_like(d["x"]) if args.prenorm else None
    xin = xn if args.prenorm else d["x"]

    def step(ev=None, st=None):
        st = stream if st is None else st      # the stream to launch on (a capture stream too)
        if args.prenorm:
            if ev is not None:
                ev[5].record(st)
            moe.moe_rmsnorm(d["x"], nw, xn, mw.RMS_NORM_EPS, st)
        if ev is not None:
            ev[0].record(st)
        moe.moe_route(L, xin, d["w_router"], d["corr_bias"], tw, ti, sg, ws, st)
        if ev is not None:
            ev[1].record(st)
        moe.moe_permute(L, ti, None, xin, off, ps, ip, xp, ws, st)
        if ev is not None:
            ev[2].record(st)
        moe.moe_expert_ffn(L, xin, xp, off, ps, tw, sg, d["w_gate_up"], d["w_down"], wsgu, wsd,
                           yr, ys, ws, st)
        if ev is not None:
            ev[3].record(st)
        moe.moe_combine(L, yr, ys, ip, out, ws, st)
        if ev is not None:
            ev[4].record(st)

    def fwd(st=None):
        """One step through the one-call API (moe_forward / moe_forward_prenorm),
        inputs resident on the device: the headline step."""
        st = stream if st is None else st
        if args.prenorm:
            moe.moe_forward_prenorm(L, d["x"], nw, mw.RMS_NORM_EPS, d["w_router"], d["corr_bias"],
                                    d["w_gate_up"], d["w_down"], wsgu, wsd, out, ws, stream=st)
        else:
            moe.moe_forward(L, d["x"], d["w_router"], d["corr_bias"], d["w_gate_up"], d["w_down"],
                            wsgu, wsd, out, ws, stream=st)

    # the headline step: moe_forward, or the op chain in the row-gathering
    # mode (which moe_forward does not use)
    headline = (lambda st=None: step(st=st)) if args.gather_rows else fwd
    for _ in range(args.warmup):
        headline()
    torch.cuda.synchronize(dev)
    moe.read_device_status(ws, stream)
    graph = None
    if args.graph:
        # one step captured once and replayed
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(graph, stream=cap):
            headline(st=cap)
        torch.cuda.synchronize(dev)
        # the replay must do the step's work: from a zeroed output it gives the
        # eager step's bits
        out.zero_()
        graph.replay()
        torch.cuda.synchronize(dev)
        replayed = out.clone()
        out.zero_()
        headline()
        torch.cuda.synchronize(dev)
        if not (torch.equal(replayed, out) and bool(replayed.abs().sum() > 0)):
            raise RuntimeError("the captured graph does not reproduce the eager step")

    # ---- timed region: K steps, inputs (weights 9.7 GB at the default
    # workload) far larger than the 126 MB L2, so no flush is needed between steps
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize(dev)
        clk.mark_start()
        e_start.record(stream)
        for i in range(args.steps):
            if graph is None:
                headline()
            else:
                graph.replay()
        e_end.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
        barrier(world)
    clocks = clk.summary()
    moe.read_device_status(ws, stream)
    ms_step = max_over_ranks(e_start.elapsed_time(e_end) / args.steps, world)

    # ---- the same steps as the op chain with CUDA events between the ops:
    # the per-op breakdown and the expert GEMMs' own time (for the roofline)
    for _ in range(args.warmup):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    barrier(world)
    moe.read_device_status(ws, stream)
    op_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i in range(4)]
    norm_ms = (sum(e[5].elapsed_time(e[0]) for e in evs) / args.steps) if args.prenorm else None
    first = 5 if args.prenorm else 0
    chain_ms = evs[0][first].elapsed_time(evs[-1][4]) / args.steps

    # ---- end to end through the public one-call API with host buffers: every
    # step copies its input from pinned host memory and its output back.  Two
    # device buffer sets and three streams let step i's upload and step i-1's
    # download overlap step i-1's / step i's compute; each step still pays for
    # its own copies, and the region ends when the last output is on the host.
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_dev = [d["x"], torch.empty_like(d["x"])]
    out_dev = [out, torch.empty_like(out)]
    out_host2 = [out_host, torch.empty_like(out_host).pin_memory()]
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("h2d", "comp", "d2h")}

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev["comp"][b])                   # x_dev[b] free again
                x_dev[b].copy_(x_host, non_blocking=True)
                ev["h2d"][b].record(h2d_s)
            stream.wait_event(ev["h2d"][b])
            if i >= 2:
                stream.wait_event(ev["d2h"][b])                       # out_dev[b] read back
            if args.prenorm:
                moe.moe_forward_prenorm(L, x_dev[b], nw, mw.RMS_NORM_EPS, d["w_router"],
                                        d["corr_bias"], d["w_gate_up"], d["w_down"], wsgu, wsd,
                                        out_dev[b], ws, stream=stream)
            else:
                moe.moe_forward(L, x_dev[b], d["w_router"], d["corr_bias"], d["w_gate_up"],
                                d["w_down"], wsgu, wsd, out_dev[b], ws, stream=stream)
            ev["comp"][b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev["comp"][b])
                out_host2[b].copy_(out_dev[b], non_blocking=True)
                ev["d2h"][b].record(d2h_s)

    e2e_steps(max(2, args.warmup // 2))
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    h2d_s.wait_event(e0)
    e2e_steps(args.steps)
    stream.wait_stream(d2h_s)
    stream.wait_stream(h2d_s)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    moe.read_device_status(ws, stream)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)

    if rank == 0:
        peaks, peak_src = load_peaks()
        fl = mw.flops(w)
        ffn_ms = op_ms[2]          # the expert GEMMs' own time (op chain)
        counts = (off[1:] - off[:-1]).cpu()
        touched = int((counts > 0).sum()) + S
        yel = 2 if L.down_f16 else 4
        roof = gemm_roofline(w, ffn_ms, touched, peaks, peak_src, yel, counts.tolist())
        # the captured bytes are those of the launches reading x_perm; the
        # row-gathering mode reads x instead and has no capture
        traffic, traffic_src = traffic_of(w.name)
        roof["traffic"] = None if args.gather_rows else traffic
        roof["traffic_source"] = None if args.gather_rows or traffic is None else traffic_src
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        sb = step_bytes(w, touched, yel)
        tokens_s = world * T / (ms_step / 1e3)
        line = {
            "metric": METRIC, "value": tokens_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02^2) weights, random init)",
            "config": {"workload": w.name, "T": T, "H": H, "E": E, "k": k, "S": S, "I": w.I,
                       "route_scale": w.route_scale, "parallelism": f"replicas x{world}",
                       "down_projection": ("fp16: weights copied once from bf16, activated rows "
                                           "and expert output rows in fp16" if L.down_f16 else w.dtype),
                       "l2": "inputs larger than L2 (expert weights %.1f GB)" % (mw.weight_bytes(w) / 1e9)},
            "tflops": world * fl["total"] / (ms_step / 1e3) / 1e12,
            "op_ms": {"route": op_ms[0], "permute": op_ms[1], "expert_ffn": op_ms[2], "combine": op_ms[3],
                      "op_chain_step": chain_ms},
            "step": ("moe_forward_prenorm" if args.prenorm else "moe_forward") if not args.gather_rows
                    else "op chain (moe_route, moe_permute, moe_expert_ffn, moe_combine)",
            "roofline": {"kernel": "grouped expert GEMMs (gate_up + down launches of moe_expert_ffn, "
                                   "timed in the op chain)",
                         **roof},
            "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
                    "d2h_bytes_per_step": out_host.numel() * out_host.element_size()},
            "step_hbm": {"algorithmic_bytes": sb, "achieved_gbs": sb / (ms_step / 1e3) / 1e9,
                         "frac": sb / (ms_step / 1e3) / 1e9 / hbm_peak},
            "gpu_launches": (moe.forward_prenorm_kernel_count(L) if args.prenorm
                             else moe.forward_kernel_count(L)) * args.steps,
            "clocks": clocks,
        }
        if graph is not None:
            line["config"]["graph"] = True
        if args.gather_rows:
            line["config"]["a_rows"] = "gathered from x by the gate_up GEMM (no x_perm copy)"
            # the op chain: no row-gather launch in the permute, and the shared
            # experts inside the expert call (no side-stream launches)
            side = 2 if (S and w.dtype == "bf16") else 0
            line["gpu_launches"] -= args.steps * (1 + side)
        if args.prenorm:
            # the block: post_attention_layernorm, then the layer
            el_x = 2 if w.dtype == "bf16" else 4
            nb = 2 * T * H * el_x
            line["config"]["block"] = "rmsnorm prologue + layer"
            line["op_ms"]["rmsnorm"] = norm_ms
            line["rmsnorm_roofline"] = {"bound": "hbm", "achieved": nb / (norm_ms / 1e3) / 1e9,
                                        "peak": hbm_peak, "unit": "GB/s",
                                        "frac": nb / (norm_ms / 1e3) / 1e9 / hbm_peak,
                                        "algorithmic_bytes": nb}
        if world == 1 and not args.no_per_config and w.name == DEFAULT_WORKLOAD and graph is None:
            # the task's other workloads, timed in this run with the same
            # step counts (one GPU only: the replicas time the default one)
            del d, xp, yr, ys, ws
            torch.cuda.empty_cache()
            line["per_config"] = {n: time_workload(moe, n, args.steps, args.warmup, dev, stream,
                                                   peaks, peak_src, args.down_bf16)
                                  for n in PER_CONFIG}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, inputs)
        print(json.dumps(line), flush=True)
    finish(world)


# ------------------------------------------------------------- dense layer
DENSE_METRIC = "Inkling dense-MLP layer tokens/s and TFLOP/s (% of B200 bf16 peak / % HBM BW), 1 GPU"


def dense_oracle_run(w, inputs, tokens_per_step: int, steps: int, warmup: int, threads: int):
    import oracle
    torch.set_num_threads(threads)
    n_done, t_total = 0, 0.0
    for i in range(warmup + steps):
        tok = mw.dense_token_sample(w, tokens_per_step, seed_offset=1000 + i)
        t0 = time.perf_counter()
        oracle.dense_mlp(inputs["x"], inputs["w_gate_up"], inputs["w_down"], w.global_scale,
                         tokens=tok)
        dt = time.perf_counter() - t0
        if i >= warmup:
            n_done += tok.numel()
            t_total += dt
    return n_done / t_total, n_done, t_total


def dense_reference_arm(args, world, rank):
    w = mw.dense_by_name(args.workload)
    if rank != 0:
        return
    inputs = mw.generate_dense(w)
    threads = len(os.sched_getaffinity(0))
    tokens_per_step = int(max(1, min(64, 480 // max(1, args.steps + args.warmup))))
    tps, done, secs = dense_oracle_run(w, inputs, tokens_per_step, args.steps, args.warmup, threads)
    line = {
        "impl": "reference", "metric": DENSE_METRIC, "value": tps, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "H": w.H, "I": w.I,
                   "tokens_per_step": tokens_per_step},
        "tflops": tps * mw.dense_flops(w, 1) / 1e12,
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{tokens_per_step} seeded tokens per step of {w.name}"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def dense_gpu_arm(args, world, rank, local):
    import mixture_experts_feed_b200 as moe

    w = mw.dense_by_name(args.workload)
    inputs = mw.generate_dense(w)
    if rank > 0:
        g = torch.Generator().manual_seed(10_000 + rank)
        inputs["x"] = torch.randn(w.T, w.H, generator=g).to(w.torch_dtype)
    L = moe.DenseLayer.from_workload(w, down_f16=w.dtype == "bf16" and not args.down_bf16)
    dev = torch.device("cuda", local)
    d = device_inputs(moe, inputs, dev, L.down_f16)
    stream = torch.cuda.current_stream(dev)
    ws = moe.new_dense_workspace(L, device=dev)
    out = torch.empty(w.T, w.H, dtype=w.torch_dtype, device=dev)

    def step():
        moe.moe_dense_mlp(L, d["x"], d["w_gate_up"], d["w_down"], out, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    moe.read_device_status(ws, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize(dev)
        clk.mark_start()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
        barrier(world)
    clocks = clk.summary()
    moe.read_device_status(ws, stream)
    ms_step = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)

    # end to end through the same call with host buffers (double-buffered as
    # in the MoE arm: each step uploads its x and downloads its output)
    x_host = inputs["x"].pin_memory()
    out_host = [torch.empty(w.T, w.H, dtype=w.torch_dtype).pin_memory() for _ in range(2)]
    x_dev = [d["x"], torch.empty_like(d["x"])]
    out_dev = [out, torch.empty_like(out)]
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("h2d", "comp", "d2h")}

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev["comp"][b])
                x_dev[b].copy_(x_host, non_blocking=True)
                ev["h2d"][b].record(h2d_s)
            stream.wait_event(ev["h2d"][b])
            if i >= 2:
                stream.wait_event(ev["d2h"][b])
            moe.moe_dense_mlp(L, x_dev[b], d["w_gate_up"], d["w_down"], out_dev[b], ws, stream)
            ev["comp"][b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev["comp"][b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                ev["d2h"][b].record(d2h_s)

    e2e_steps(max(2, args.warmup // 2))
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    h2d_s.wait_event(e0)
    e2e_steps(args.steps)
    stream.wait_stream(d2h_s)
    stream.wait_stream(h2d_s)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    moe.read_device_status(ws, stream)

    if rank == 0:
        peaks, peak_src = load_peaks()
        el = 2 if w.dtype == "bf16" else 4
        flops = mw.dense_flops(w)
        # weights once; x read, h written and read, y (fp32) written and read,
        # out written
        nbytes = 3 * w.H * w.I * el + w.T * (w.H * el + 2 * w.I * el + 8 * w.H + w.H * el)
        peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        s_step = ms_step / 1e3
        if flops / nbytes >= peak * 1e12 / (hbm_peak * 1e9):
            roof = {"bound": "tensor", "achieved": flops / s_step / 1e12, "peak": peak,
                    "unit": "TFLOP/s", "peak_source": f"{peak_src} bf16_tflops_sustained"}
        else:
            roof = {"bound": "hbm", "achieved": nbytes / s_step / 1e9, "peak": hbm_peak,
                    "unit": "GB/s", "peak_source": f"{peak_src} hbm_gbs"}
        roof["frac"] = roof["achieved"] / roof["peak"]
        roof["traffic"] = NCU_TRAFFIC_BYTES.get(w.name)
        roof["algorithmic_bytes"] = nbytes
        roof["algorithmic_flops"] = flops
        line = {
            "metric": DENSE_METRIC, "value": world * w.T / s_step, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02^2) weights, random init)",
            "config": {"workload": w.name, "T": w.T, "H": w.H, "I": w.I,
                       "global_scale": w.global_scale, "parallelism": f"replicas x{world}",
                       "down_projection": "fp16 (weights copied once from bf16)" if L.down_f16 else w.dtype,
                       "l2": "inputs larger than L2 (weights %.2f GB)" % (3 * w.H * w.I * el / 1e9)},
            "tflops": world * flops / s_step / 1e12,
            "roofline": {"kernel": "dense gate_up + down GEMM launches of moe_dense_mlp (whole call timed)",
                         **roof},
            "e2e": {"value": world * w.T / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
                    "d2h_bytes_per_step": out_host[0].numel() * out_host[0].element_size()},
            "gpu_launches": moe.dense_kernel_count(L) * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            threads = len(os.sched_getaffinity(0))
            n = int(max(4, min(w.T, 64)))
            tps, done, secs = dense_oracle_run(w, inputs, n, 1, 0, threads)
            line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": threads,
                                    "kind": "oracle",
                                    "sample": f"{done} seeded tokens of {w.name} (oracle fp64, {secs:.1f} s)"}
        print(json.dumps(line), flush=True)
    finish(world)


def relaunch_ranks(n: int) -> int:
    """Run this script again under torch.distributed.run with n ranks on this
    node (rendezvous on 127.0.0.1, a free port); returns its exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time the default workload only (no per_config block)")
    ap.add_argument("--prenorm", action="store_true",
                    help="time the feed-forward block: the RMSNorm prologue, then the MoE layer")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step's op chain as one captured CUDA graph")
    ap.add_argument("--gather-rows", action="store_true",
                    help="no permuted copy of x: the gate_up GEMM gathers the routed rows")
    ap.add_argument("--down-bf16", action="store_true",
                    help="bf16 down projections (bf16 activated rows) instead of fp16")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # N ranks requested without an outer launcher: start them here, one
        # process per GPU under torch.distributed.run, and exit with its status
        sys.exit(relaunch_ranks(args.gpus))
    args.warmup = max(3, args.warmup)   # at least three untimed warm-up steps
    dense = args.workload in mw.DENSE_WORKLOADS
    if args.impl == "reference":
        arm = dense_reference_arm if dense else reference_arm
        arm(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args)
    (dense_gpu_arm if dense else gpu_arm)(args, world, rank, local)


if __name__ == "__main__":
    main()
