"""Benchmark of the online INT8 W8A8 hot path on B200.

Default workload (one "step"): one decode step of the two dense W8A8 linears
of a Qwen3.6-27B-class MLP at M = 8 tokens -- gate_up (K=5120 -> N=34816) and
down (K=17408 -> N=5120) -- each a per-token activation quant followed by the
weight-streaming GEMV with the dequant epilogue.  The headline metric is the
weight bytes streamed per second.  Two independent weight sets alternate
from step to step, so that no step finds its weights in L2.  The same JSON
line carries, last, a compact "workloads" object: the prefill GEMM TOPS
(M = 512 / 4096), the routed-MoE layer tokens/s (T = 1 / 8 / 512 / 4096), the
FWHT128-domain, head, trunk, shared-expert and MLP-block workloads, each with
its time and roofline fractions against the measured and the nominal peaks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--quick]   (headline only, no extra workloads)
    python bench.py --case NAME (one small workload for a profiler capture)

Multi-GPU: the path has no exchange step; N ranks run independent replicas
(weak scaling), timed on the device, max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
METRIC = "W8A8 int8 TOPS (prefill), weight GB/s (decode), MoE layer tokens/s vs roofline"
# Nominal peaks of the part (HGX B200 datasheet, dense): HBM3e ~8 TB/s; int8
# tensor ~4.5 POPS.  Every fraction is also reported against these.
NOMINAL_HBM_GBS = 8000.0
NOMINAL_INT8_TOPS = 4500.0
DECODE_M = 8
WEIGHT_SETS = 2       # ceil(2 * 126 MB / 267 MB) + 1: no step finds its weights in L2


# --------------------------------------------------------------------------- peaks / clocks
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


# --------------------------------------------------------------------------- ncu traffic record
def kernel_source_hash():
    """Hash of the decode-GEMV sources; a committed ncu traffic figure is used
    only while it was taken on exactly these sources."""
    import hashlib
    h = hashlib.sha256()
    for f in ("gemv.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "moe_gemm_absmax_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(profile="gemv_decode_gateup_m8.md"):
    """dram read + write bytes per launch from profiles/<profile>, if it was
    captured on the current sources (line 'source_hash: ...'), else None."""
    p = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(p):
        return None
    rec = {}
    for ln in open(p):
        if ":" in ln and ln.strip().startswith(("source_hash", "traffic_bytes_per_launch")):
            k, v = ln.split(":", 1)
            rec[k.strip()] = v.strip().strip("`")
    if rec.get("source_hash") != kernel_source_hash():
        return None
    try:
        return int(rec["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# --------------------------------------------------------------------------- timing helpers
def max_over_ranks(torch, value, world, device):
    """The largest of the ranks' values, on every rank (the value itself when alone):
    a multi-GPU time is the slowest rank's."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, bytes_per_rank, ms):
    """Whole-job GB/s: every rank streams bytes_per_rank per step, in the slowest rank's ms."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


def time_events(torch, fn, iters, flush=None):
    """Mean device time of fn() per call in ms, CUDA events on the current stream,
    one event pair per call; optional L2 flush between calls (outside the events).
    A short device-side sleep before the start event keeps the GPU busy while
    the host enqueues fn(), so no launch gap is timed."""
    st = torch.cuda.current_stream()
    ts = []
    for _ in range(iters):
        if flush is not None:
            flush()
        torch.cuda._sleep(200000)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        fn()
        b.record(st)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return float(np.mean(ts)), float(np.median(ts))


def graph_events(torch, fn, iters, flush=None):
    """Mean device time in ms of one replay of a CUDA graph that holds fn()
    (captured after warm-up on a side stream), CUDA events around each replay."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    t, _ = time_events(torch, g.replay, iters, flush=flush)
    del g
    return t


def local_gpu_index(torch):
    """nvidia-smi index of this process's GPU (first entry of CUDA_VISIBLE_DEVICES if set)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        first = vis.split(",")[torch.cuda.current_device()].strip()
        if first.isdigit():
            return int(first)
    return torch.cuda.current_device()


def make_flush(torch, dev):
    """Evicts L2 by reading a buffer twice its size (a read leaves no dirty
    lines whose write-back would compete with the next timed kernel)."""
    buf = torch.ones(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def flush():
        buf.max()
    return flush


# --------------------------------------------------------------------------- workloads
def quantize_on_gpu(torch, w8a8, w_np, dev):
    q, s = w8a8.quant_rows_f32(torch.from_numpy(w_np).to(dev))
    torch.cuda.synchronize()
    return q, s


def dense_weights(torch, w8a8, inputs, dev, seed=0):
    rng = np.random.default_rng([seed, 7])
    out = {}
    for name, d in (("gate_up", inputs.GATE_UP), ("down", inputs.DOWN)):
        w = inputs.weights(rng, (d["N"], d["K"]))
        out[name] = quantize_on_gpu(torch, w8a8, w, dev)
        del w
    return out


def bf16_dev(torch, bits, dev):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def linear_bytes(M, N, K):
    """Algorithmic HBM bytes of one W8A8 linear: weights + scales + bf16 in + bf16 out."""
    return N * K + 4 * N + 2 * M * K + 2 * M * N


def headline_config(world):
    """The workload both arms measure (the reference arm on the host's cores)."""
    return {"workload": "decode-shaped dense W8A8 linears, M=8 tokens: gate_up K=5120->N=34816 then "
                        "down K=17408->N=5120 (per-token act quant + weight-streaming GEMV + dequant)",
            "arithmetic": "int8 x int8 -> int32, fp32 scales, bf16 in/out",
            "tokens": DECODE_M, "weight_bytes_per_step": 267546624, "algorithmic_bytes_per_step": 268546048,
            "l2": f"{WEIGHT_SETS} weight sets of 267 MB alternate step by step (L2 126 MB): no step finds "
                  "its weights in L2",
            "parallelism": f"replicas x{world}"}


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def host_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def sig(v, n=4):
    """v rounded to n significant digits (compact JSON)."""
    if v is None or not np.isfinite(v) or v == 0:
        return v
    return float(f"{v:.{n}g}")


def cnum(v):
    """Compact number for the workloads record: integers from 100 up, else 3 significant digits."""
    if v is None or not np.isfinite(v):
        return v
    return int(round(v)) if abs(v) >= 100 else sig(v, 3)


# --------------------------------------------------------------------------- reference arm (CPU oracle)
def decode_weights_np(inputs, oracle, seed=0):
    """The headline's first weight set, quantized by the oracle (same draws as the GPU arm's set 0)."""
    rng = np.random.default_rng([seed, 7])
    out = {}
    for name, d in (("gate_up", inputs.GATE_UP), ("down", inputs.DOWN)):
        w = inputs.weights(rng, (d["N"], d["K"]))
        out[name] = oracle.quant_rows_f32(w)
        del w
    return out


def run_reference(args, rank, world):
    """The CPU oracle, as it stands, on the whole decode step (both linears, all
    rows) at the host's thread count; rank 0 only."""
    if rank != 0:
        return None
    import oracle
    from moe_gemm_absmax_b200 import inputs
    oracle.build()
    oracle.set_threads(host_threads())
    cores = oracle.get_threads()
    mats = decode_weights_np(inputs, oracle)
    xs = {n: inputs.dense_linear(11, DECODE_M, d["K"], 16, with_weights=False)[0]
          for n, d in (("gate_up", inputs.GATE_UP), ("down", inputs.DOWN))}
    wbytes = sum(mats[n][0].size + 4 * mats[n][0].shape[0] for n in mats)

    def step():
        for n in ("gate_up", "down"):
            oracle.linear(xs[n], *mats[n])
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = wbytes / dt / 1e9
    sample = (f"the whole decode step (all 34816 gate_up and 5120 down rows, M=8) per step, "
              f"one weight set (caches play no part on the host); {cores} threads, {cpu_model()}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": headline_config(world),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


def _per_call(fn, min_s):
    """Seconds per call of fn, timed over at least min_s after one untimed call."""
    fn()
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            return dt / n


def cpu_baseline(min_s=1.0):
    """The oracle, as it stands, on a bounded sample of each of the five
    workloads, at one thread and at every thread of this process's affinity
    mask.  Rates (GB/s, TOPS, tokens/s) of the sampled work; the headline value
    is the decode step's GB/s at all threads."""
    import oracle
    from moe_gemm_absmax_b200 import inputs
    oracle.build()
    nthr = host_threads()
    rng = np.random.default_rng([0, 8])
    cases = {}
    # tiny: the whole config
    xb, w = inputs.tiny_linear(0)
    qw, sw = oracle.quant_rows_f32(w)
    cases["tiny"] = dict(unit="GOP/s", work=2.0 * 16 * 512 * 512 / 1e9, fn=lambda: oracle.linear(xb, qw, sw),
                         sample="whole config: 16 x 512 -> 512")
    # decode step: the whole step (both matrices, every row) at M = 8
    mats = decode_weights_np(inputs, oracle)
    dm = {n: (inputs.dense_linear(11, DECODE_M, d["K"], 16, with_weights=False)[0], *mats[n])
          for n, d in (("gate_up", inputs.GATE_UP), ("down", inputs.DOWN))}
    dbytes = sum(dm[n][1].size + 4 * dm[n][1].shape[0] for n in dm)
    cases["decode"] = dict(unit="GB/s", work=dbytes / 1e9,
                           fn=lambda: [oracle.linear(*dm[n]) for n in ("gate_up", "down")],
                           sample="the whole decode step at M=8 (all 34816 gate_up and 5120 down rows), one "
                                  "weight set; GB/s of its int8 weights and fp32 scales")
    # prefill: M = 512 tokens against a row sample of gate_up
    xp = inputs.dense_linear(3, 512, inputs.GATE_UP["K"], 16, with_weights=False)[0]
    qp, sp = oracle.quant_rows_f32(inputs.weights(rng, (64, inputs.GATE_UP["K"])))
    cases["prefill"] = dict(unit="TOPS", work=2.0 * 512 * 64 * inputs.GATE_UP["K"] / 1e12,
                            fn=lambda: oracle.linear(xp, qp, sp),
                            sample="prefill gate_up at M=512 on 64 of its 34816 weight rows")
    # MoE at T = 8: the routed experts' weights only (drawn for the experts the tokens touch)
    E, H, I, k = inputs.MOE["E"], inputs.MOE["H"], inputs.MOE["I"], inputs.MOE["topk"]
    xm, lm = inputs.moe_tokens(0, 8)
    ids, _ = oracle.route(lm, k)
    w13 = np.zeros((E, 2 * I, H), np.int8)
    w2 = np.zeros((E, H, I), np.int8)
    s13 = np.ones((E, 2 * I), np.float32)
    s2 = np.ones((E, H), np.float32)
    mrng = np.random.default_rng([0, 1])
    for e in np.unique(ids):
        w13[e], s13[e] = oracle.quant_rows_f32(inputs.weights(mrng, (2 * I, H)))
        w2[e], s2[e] = oracle.quant_rows_f32(inputs.weights(mrng, (H, I)))
    cases["moe"] = dict(unit="tokens/s", work=8.0, fn=lambda: oracle.moe_forward(xm, lm, w13, s13, w2, s2, k),
                        sample=f"routed MoE layer at T=8 ({len(np.unique(ids))} touched experts), whole layer")
    # Hadamard: M = 2048, the rotation and group quant of x plus the GEMM on a row sample
    xh, wh = inputs.hadamard_linear(2048, 2048)
    qwh, swh, _ = oracle.fwht128_quant(wh[:64])

    def had():
        qx, sx, _ = oracle.fwht128_quant(xh)
        oracle.gemm_g128(qx, sx, qwh, swh)
    cases["hadamard"] = dict(unit="TOPS", work=2.0 * 2048 * 64 * 2048 / 1e12, fn=had,
                             sample="FWHT128 linear at M=2048: rotation + group quant of x, GEMM on 64 of "
                                    "4096 weight rows")
    out = {}
    for name, c in cases.items():
        rec = {"unit": c["unit"], "sample": c["sample"]}
        for label, n in (("t1", 1), ("tall", nthr)):
            oracle.set_threads(n)
            dt = _per_call(c["fn"], min_s)
            rec[label] = sig(c["work"] / dt)
        out[name] = rec
    oracle.set_threads(nthr)
    dec = out["decode"]
    return {"value": dec["tall"], "unit": "GB/s", "cores": nthr, "kind": "oracle",
            "sample": dec["sample"] + f"; {nthr} threads (sched_getaffinity)",
            "cpu_model": cpu_model(), "threads_one": 1, "threads_all": nthr, "configs": out}


# --------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, torch, dev):
    from moe_gemm_absmax_b200 import inputs, w8a8
    w8a8.lib()       # fails loudly when the CUDA library is missing
    peaks = load_peaks()
    hbm = peaks["hbm_gbs"]
    int8_peak = 2.0 * peaks["bf16_tflops"]           # dense int8 = 2 x dense bf16 (nominal ratio)
    M = DECODE_M
    sets = [dense_weights(torch, w8a8, inputs, dev, seed=s) for s in range(WEIGHT_SETS)]
    W = sets[0]
    xs = {}
    for name, d in (("gate_up", inputs.GATE_UP), ("down", inputs.DOWN)):
        xs[name] = bf16_dev(torch, inputs.dense_linear(11, M, d["K"], 16, with_weights=False)[0], dev)
    ys = {n: torch.empty((M, W[n][0].shape[0]), dtype=torch.bfloat16, device=dev) for n in W}
    wss = {n: torch.empty(max(256, w8a8.linear_workspace_size(M, W[n][0].shape[0], xs[n].shape[1])),
                          dtype=torch.uint8, device=dev) for n in W}
    order = ("gate_up", "down")

    def step(i):
        Ws = sets[i % WEIGHT_SETS]
        for n in order:
            w8a8.linear(xs[n], Ws[n][0], Ws[n][1], y=ys[n], ws=wss[n])

    step_bytes = sum(linear_bytes(M, W[n][0].shape[0], W[n][0].shape[1]) for n in order)
    weight_bytes = sum(W[n][0].numel() + 4 * W[n][0].shape[0] for n in order)

    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    # nvidia-smi samples every 100 ms; the timed loop alone is a few ms, so the
    # sampler runs across the whole GPU part of the benchmark
    clk = ClockSampler(local_gpu_index(torch))
    clk.__enter__()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    # a device-side sleep ahead of the start event keeps the GPU busy while the
    # host enqueues the K steps, so no launch gap of the host falls inside the
    # timed region; the region itself is the K steps
    torch.cuda._sleep(int(min(2e8, 60e3 * args.steps + 2e6)))
    e0.record(st)
    for i in range(args.steps):
        step(i)
    e1.record(st)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks(torch, e0.elapsed_time(e1) / args.steps, world, dev)
    value = job_throughput(world, weight_bytes, ms)

    # ---- roofline of the dominant kernel: the gate_up GEMV alone (pre-quantized codes)
    qx, sx = w8a8.quant_act(xs["gate_up"])
    N, K = W["gate_up"][0].shape
    y_k = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = make_flush(torch, dev)
    kfn = lambda: w8a8.gemm_q(qx, sx, W["gate_up"][0], W["gate_up"][1], w8a8.PATH_GEMV, y=y_k)
    for _ in range(3):
        kfn()
    k_ms, _ = time_events(torch, kfn, 20, flush=flush)
    k_bytes = N * K + 4 * N + M * K + 4 * M + 2 * M * N
    achieved = k_bytes / (k_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": recorded_traffic(), "algorithmic_bytes": k_bytes,
                "kernel": "gemv_dense_kernel (gate_up K=5120 -> N=34816, M=8)",
                "timing": "kernel alone, CUDA events per launch, L2 evicted by a read between launches",
                "peak_source": peaks["source"] + " (burst copy)",
                "nominal_peak": NOMINAL_HBM_GBS, "nominal_frac": achieved / NOMINAL_HBM_GBS}

    # ---- the down-proj GEMV alone, and the whole step replayed from a CUDA graph
    qxd, sxd = w8a8.quant_act(xs["down"])
    Nd, Kd = W["down"][0].shape
    y_d = torch.empty((M, Nd), dtype=torch.bfloat16, device=dev)
    dfn = lambda: w8a8.gemm_q(qxd, sxd, W["down"][0], W["down"][1], w8a8.PATH_GEMV, y=y_d)
    for _ in range(3):
        dfn()
    d_ms, _ = time_events(torch, dfn, 20, flush=flush)
    d_bytes = Nd * Kd + 4 * Nd + M * Kd + 4 * M + 2 * M * Nd
    graph_ms = graph_events(torch, lambda: [step(i) for i in range(WEIGHT_SETS)], 20) / WEIGHT_SETS

    # ---- end to end through the C ABI with host buffers: every step's x comes
    # from pinned host memory and its y goes back to it, the copies on a second
    # stream one step ahead / behind the compute (a serving loop's pipeline),
    # both inputs in one host-to-device copy and both outputs in one back
    xbytes = {n: xs[n].numel() * 2 for n in order}
    ybytes = {n: ys[n].numel() * 2 for n in order}
    h2d = sum(xbytes.values())
    d2h = sum(ybytes.values())
    hx = [torch.empty(h2d, dtype=torch.uint8).pin_memory() for _ in range(2)]
    hy = [torch.empty(d2h, dtype=torch.uint8).pin_memory() for _ in range(2)]
    for slot in range(2):
        o = 0
        for n in order:
            hx[slot][o:o + xbytes[n]].copy_(xs[n].view(torch.uint8).reshape(-1).cpu())
            o += xbytes[n]
    dxb = [torch.empty(h2d, dtype=torch.uint8, device=dev) for _ in range(2)]
    dyb = [torch.empty(d2h, dtype=torch.uint8, device=dev) for _ in range(2)]

    def view_bf16(buf, sizes, shapes):
        out, o = {}, 0
        for n in order:
            out[n] = buf[o:o + sizes[n]].view(torch.bfloat16).view(shapes[n])
            o += sizes[n]
        return out
    dx = [view_bf16(dxb[k], xbytes, {n: xs[n].shape for n in order}) for k in range(2)]
    dy = [view_bf16(dyb[k], ybytes, {n: ys[n].shape for n in order}) for k in range(2)]
    cs = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(nsteps):
        cs.wait_stream(st)   # the copies start inside the timed region
        with torch.cuda.stream(cs):
            dxb[0].copy_(hx[0], non_blocking=True)
            ev_in[0].record(cs)
        for i in range(nsteps):
            k = i % 2
            if i + 1 < nsteps:
                with torch.cuda.stream(cs):   # next step's x, once step i - 1 is done with that slot
                    dxb[1 - k].copy_(hx[1 - k], non_blocking=True)
                    ev_in[1 - k].record(cs)
            st.wait_event(ev_in[k])
            if i >= 2:
                st.wait_event(ev_out[k])      # step i - 2's y has left that slot
            Ws = sets[i % WEIGHT_SETS]
            for n in order:
                w8a8.linear(dx[k][n], Ws[n][0], Ws[n][1], y=dy[k][n], ws=wss[n])
            ev_done[k].record(st)
            with torch.cuda.stream(cs):
                cs.wait_event(ev_done[k])
                hy[k].copy_(dyb[k], non_blocking=True)
                ev_out[k].record(cs)
        st.wait_stream(cs)

    e2e_run(3)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(int(min(2e8, 60e3 * args.steps + 2e6)))
    a.record(st)
    e2e_run(args.steps)
    b.record(st)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / args.steps

    def rec(ms_, val, peak, nominal, extra_ms=None):
        r = [cnum(ms_ * 1e3), cnum(val), cnum(val / peak), cnum(val / nominal)]
        return r if extra_ms is None else r + [cnum(extra_ms * 1e3)]

    wl = {"dec_step_graph": rec(graph_ms, weight_bytes / (graph_ms * 1e-3) / 1e9, hbm, NOMINAL_HBM_GBS),
          "dec_gu_gemv": rec(k_ms, achieved, hbm, NOMINAL_HBM_GBS),
          "dec_dn_gemv": rec(d_ms, d_bytes / (d_ms * 1e-3) / 1e9, hbm, NOMINAL_HBM_GBS)}
    if not args.quick:
        del sets
        wl.update(run_extra(torch, w8a8, inputs, dev, W, hbm, int8_peak, flush, rec))
    clk.__exit__(None, None, None)
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": headline_config(world),
            "gpu_name": torch.cuda.get_device_name(dev),
            "step_frac": {"measured": value / world / hbm, "nominal": value / world / NOMINAL_HBM_GBS,
                          "bytes": "int8 weights + fp32 scales per step"},
            "roofline": roofline, "clocks": dict(clk.summary(), window="whole GPU part of the run"),
            "e2e": {"value": world * weight_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "how": "pinned host x in and y out every step (one copy each way), on a copy stream "
                           "pipelined one step ahead of / behind the compute"},
            "gpu_launches": 4 * args.steps,
            "peaks": {"hbm_gbs": hbm, "int8_tops": int8_peak, "source": peaks["source"],
                      "nominal_hbm_gbs": NOMINAL_HBM_GBS, "nominal_int8_tops": NOMINAL_INT8_TOPS},
            "workloads_fields": ["us", "value", "frac_measured", "frac_nominal",
                                 "pf: us of a1 + GEMM; moe1/moe8: us of a CUDA-graph replay; had2048: us of "
                                 "fwht128_quant + GEMM (the first four: the GEMM alone)"],
            "workloads_units": {"dec": "GB/s", "pf": "TOPS", "mlp8": "GB/s", "mlp4096": "TOPS", "aq": "GB/s",
                                "moe/moeg": "tokens/s (fractions: HBM bytes of the touched experts)",
                                "had1/head/trunk1/shx1/shx8": "GB/s", "had2048/trunk2048/shx512/shx4096": "TOPS"},
            "workloads": wl}
    return line


def run_extra(torch, w8a8, inputs, dev, W, hbm, int8_peak, flush, rec):
    out = {}
    # ---- prefill GEMMs (tcgen05), and the full linear incl. activation quant
    for M in (512, 4096):
        for n, tag in (("gate_up", "gu"), ("down", "dn")):
            N, K = W[n][0].shape
            x = bf16_dev(torch, inputs.dense_linear(3, M, K, 16, with_weights=False)[0], dev)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(w8a8.linear_workspace_size(M, N, K), dtype=torch.uint8, device=dev)
            qx, sx = w8a8.quant_act(x)
            fn_lin = lambda: w8a8.linear(x, W[n][0], W[n][1], y=y, ws=ws)
            fn_gemm = lambda: w8a8.gemm_q(qx, sx, W[n][0], W[n][1], w8a8.PATH_TCGEN05, y=y)
            for _ in range(3):
                fn_lin()
                fn_gemm()
            t_lin, _ = time_events(torch, fn_lin, 10, flush=flush)
            t_gemm, _ = time_events(torch, fn_gemm, 10, flush=flush)
            ops = 2.0 * M * N * K
            out[f"pf_{tag}{M}"] = rec(t_gemm, ops / (t_gemm * 1e-3) / 1e12, int8_peak, NOMINAL_INT8_TOPS, t_lin)
            del x, y, ws, qx, sx
    # ---- dense gated MLP block: the same two matrices as gate_up (w13) and down (w2)
    q13, s13 = W["gate_up"]
    q2, s2 = W["down"]
    I = q13.shape[0] // 2
    H = q2.shape[0]
    for M in (8, 4096):
        x = bf16_dev(torch, inputs.dense_linear(9, M, H, 16, with_weights=False)[0], dev)
        y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8a8.mlp_workspace_size(M, H, I), dtype=torch.uint8, device=dev)
        fn = lambda: w8a8.mlp_forward(x, q13, s13, q2, s2, y=y, ws=ws)
        for _ in range(3):
            fn()
        t, _ = time_events(torch, fn, 10, flush=flush)
        wbytes = q13.numel() + q2.numel() + 4 * (q13.shape[0] + H)
        ops = 2.0 * M * (2 * I) * H + 2.0 * M * H * I
        if M == 8:
            out["mlp8"] = rec(t, wbytes / (t * 1e-3) / 1e9, hbm, NOMINAL_HBM_GBS)
        else:
            out["mlp4096"] = rec(t, ops / (t * 1e-3) / 1e12, int8_peak, NOMINAL_INT8_TOPS)
        del x, y, ws
    # ---- per-token activation quant alone (a1) at the prefill shape
    for K in (5120, 17408):
        xq_in = bf16_dev(torch, inputs.dense_linear(5, 4096, K, 16, with_weights=False)[0], dev)
        qfn = lambda: w8a8.quant_act(xq_in)
        for _ in range(3):
            qfn()
        tq, _ = time_events(torch, qfn, 10, flush=flush)
        qb = 4096 * K * 3 + 4096 * 4
        out[f"aq4096x{K}"] = rec(tq, qb / (tq * 1e-3) / 1e9, hbm, NOMINAL_HBM_GBS)
        del xq_in
    # ---- routed MoE layer
    w13, w2 = inputs.moe_weights(0)
    q13, s13 = quantize_on_gpu(torch, w8a8, w13, dev)
    q2, s2 = quantize_on_gpu(torch, w8a8, w2, dev)
    # the same experts on the FWHT128 grid (bf16 rows rotated along K, group codes)
    g13 = w8a8.fwht128_quant(bf16_dev(torch, inputs.to_bf16_bits(w13).reshape(-1, w13.shape[2]), dev))
    g2 = w8a8.fwht128_quant(bf16_dev(torch, inputs.to_bf16_bits(w2).reshape(-1, w2.shape[2]), dev))
    del w13, w2
    E, I2, H = q13.shape

    def moe_rec(t, T, touched, per_expert, tg=None):
        byts = touched * per_expert + 2 * T * H * 2 + 2 * T * E
        gbs = byts / (t * 1e-3) / 1e9
        r = [cnum(t * 1e3), cnum(T / (t * 1e-3)), cnum(gbs / hbm), cnum(gbs / NOMINAL_HBM_GBS)]
        return r if tg is None else r + [cnum(tg * 1e3)]

    per_expert = q13[0].numel() + q2[0].numel() + 4 * (I2 + H)
    for T in (1, 8, 512, 4096):
        xb, lb = inputs.moe_tokens(0, T)
        x, lg = bf16_dev(torch, xb, dev), bf16_dev(torch, lb, dev)
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8a8.moe_workspace_size(T, E, H, I2 // 2, 8), dtype=torch.uint8, device=dev)
        fn = lambda: w8a8.moe_forward(x, lg, q13, s13, q2, s2, 8, y=y, ws=ws)
        for _ in range(3):
            fn()
        t, _ = time_events(torch, fn, 10, flush=flush)
        _, dbg = w8a8.moe_forward(x, lg, q13, s13, q2, s2, 8, debug=True)
        touched = int((dbg["counts"] > 0).sum().item())
        tg = graph_events(torch, fn, 10, flush=flush) if T <= 8 else None
        out[f"moe{T}"] = moe_rec(t, T, touched, per_expert, tg)
        del x, lg, y, ws
    del q13, q2
    # ---- routed MoE layer on the FWHT128 grid
    gq13, gs13 = g13[0].view(E, I2, H), g13[1].view(E, I2, H // 128)
    gq2, gs2 = g2[0].view(E, H, I2 // 2), g2[1].view(E, H, I2 // 256)
    per_expert = gq13[0].numel() + gq2[0].numel() + 2 * (gs13[0].numel() + gs2[0].numel())
    for T in (1, 8, 512, 4096):
        xb, lb = inputs.moe_tokens(0, T)
        x, lg = bf16_dev(torch, xb, dev), bf16_dev(torch, lb, dev)
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8a8.moe_g128_workspace_size(T, E, H, I2 // 2, 8), dtype=torch.uint8, device=dev)
        fn = lambda: w8a8.moe_g128_forward(x, lg, gq13, gs13, gq2, gs2, 8, y=y, ws=ws)
        for _ in range(3):
            fn()
        t, _ = time_events(torch, fn, 10, flush=flush)
        _, dbg = w8a8.moe_g128_forward(x, lg, gq13, gs13, gq2, gs2, 8, debug=True)
        touched = int((dbg["counts"] > 0).sum().item())
        out[f"moeg{T}"] = moe_rec(t, T, touched, per_expert)
        del x, lg, y, ws
    del g13, g2, gq13, gs13, gq2, gs2
    # ---- FWHT128-domain linear
    _, wb = inputs.hadamard_linear(0, 1)
    qw, sw = w8a8.fwht128_quant(bf16_dev(torch, wb, dev))
    for M in (1, 2048):
        xb, _ = inputs.hadamard_linear(M, M)
        x = bf16_dev(torch, xb, dev)
        y = torch.empty((M, qw.shape[0]), dtype=torch.bfloat16, device=dev)

        def fn():
            q, s = w8a8.fwht128_quant(x)
            w8a8.linear_g128(q, s, qw, sw, y=y)
        for _ in range(3):
            fn()
        t, _ = time_events(torch, fn, 10, flush=flush)
        N, K = qw.shape
        ops = 2.0 * M * N * K
        byts = N * K + 2 * N * (K // 128) + 2 * M * K + 2 * M * N
        if M == 1:
            out["had1"] = rec(t, byts / (t * 1e-3) / 1e9, hbm, NOMINAL_HBM_GBS)
        else:
            q, s = w8a8.fwht128_quant(x)
            gfn = lambda: w8a8.linear_g128(q, s, qw, sw, y=y)
            for _ in range(3):
                gfn()
            tg, _ = time_events(torch, gfn, 10, flush=flush)
            out["had2048"] = rec(tg, ops / (tg * 1e-3) / 1e12, int8_peak, NOMINAL_INT8_TOPS, t)
    # ---- head-shaped group-128 GEMM on the unrotated grid (N = 131072 rows, K = 2048)
    del qw, sw
    HN, HK = HEAD["N"], HEAD["K"]
    hw = torch.randn(HN, HK, generator=torch.Generator(device=dev).manual_seed(5), device=dev) * 0.02
    qw, sw = w8a8.group128_quant(hw.to(torch.bfloat16))
    del hw
    for M in (1, 8):
        xb, _ = inputs.hadamard_linear(M, M, K=HK, N=16)
        x = bf16_dev(torch, xb, dev)
        y = torch.empty((M, HN), dtype=torch.bfloat16, device=dev)

        def fn():
            q, s = w8a8.group128_quant(x)
            w8a8.linear_group128(q, s, qw, sw, y=y)
        for _ in range(3):
            fn()
        t, _ = time_events(torch, fn, 10, flush=flush)
        byts = HN * HK + 2 * HN * (HK // 128) + 2 * M * HK + 2 * M * HN
        out[f"head{M}"] = rec(t, byts / (t * 1e-3) / 1e9, hbm, NOMINAL_HBM_GBS)
    del qw, sw
    # ---- trunk linear in the two-level format, on the Hadamard config's shapes (N = 4096, K = 2048)
    d = inputs.HADAMARD
    _, wb = inputs.hadamard_linear(0, 1)
    tq, tu8, ts2 = w8a8.trunk_weight_quant(bf16_dev(torch, wb, dev))
    for M in (1, 2048):
        xb, _ = inputs.hadamard_linear(M, M)
        x = bf16_dev(torch, xb, dev)
        y = torch.empty((M, d["N"]), dtype=torch.bfloat16, device=dev)

        def fn():
            q, s = w8a8.fwht128_quant(x)
            w8a8.linear_trunk(q, s, tq, tu8, ts2, y=y)
        for _ in range(3):
            fn()
        t, _ = time_events(torch, fn, 10, flush=flush)
        N, K = tq.shape
        ops = 2.0 * M * N * K
        byts = N * K + N * (K // 256) + 2 * N + 2 * M * K + 2 * M * N
        out[f"trunk{M}"] = (rec(t, byts / (t * 1e-3) / 1e9, hbm, NOMINAL_HBM_GBS) if M == 1 else
                            rec(t, ops / (t * 1e-3) / 1e12, int8_peak, NOMINAL_INT8_TOPS))
    del tq, tu8, ts2
    # ---- shared expert (gate_up in the trunk format, down on the group-128 grid), H = 2048, I = 512
    H, I = inputs.MOE["H"], inputs.MOE["I"]
    rng = np.random.default_rng([0, 3])
    w13b = inputs.to_bf16_bits(inputs.weights(rng, (2 * I, H)))
    w2b = inputs.to_bf16_bits(inputs.weights(rng, (H, I)))
    sq13, su13, sr13 = w8a8.trunk_weight_quant(bf16_dev(torch, w13b, dev))
    sq2, ss2 = w8a8.fwht128_quant(bf16_dev(torch, w2b, dev))
    wbytes = sq13.numel() + su13.numel() + 2 * sr13.numel() + sq2.numel() + 2 * ss2.numel()
    for M in (1, 8, 512, 4096):
        xb, _ = inputs.moe_tokens(0, M)
        x = bf16_dev(torch, xb, dev)
        y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8a8.shared_expert_workspace_size(M, H, I), dtype=torch.uint8, device=dev)
        fn = lambda: w8a8.shared_expert_forward(x, sq13, su13, sr13, sq2, ss2, y=y, ws=ws)
        for _ in range(3):
            fn()
        t, _ = time_events(torch, fn, 10, flush=flush)
        ops = 2.0 * M * 3 * H * I
        byts = wbytes + 2 * M * H * 2
        out[f"shx{M}"] = (rec(t, byts / (t * 1e-3) / 1e9, hbm, NOMINAL_HBM_GBS) if M <= 8 else
                          rec(t, ops / (t * 1e-3) / 1e12, int8_peak, NOMINAL_INT8_TOPS))
        del x, y, ws
    return out


# head-shaped GEMM on the unrotated group-128 grid: "Qwen3.6-35B-A3B IQ8R - radiance
# container" gives no vocabulary size, so 131072 (2^17) rows over the MoE layer's
# hidden size
HEAD = dict(N=131072, K=2048)


# --------------------------------------------------------------------------- profiling cases
CASES = ("gemv_gateup_m8", "gemv_down_m8", "prefill_gateup_m512", "prefill_down_m512", "prefill_gateup_m4096",
         "prefill_down_m4096", "quant_m4096_k17408", "quant_m4096_k5120", "moe_t1", "moe_t8", "moe_t512",
         "moe_t4096", "moe_g128_t1", "moe_g128_t8", "moe_g128_t512", "moe_g128_t4096", "head_m1", "head_m8", "shared_m1", "shared_m4096", "hadamard_m1",
         "hadamard_m200", "hadamard_m2048")


def run_case(name, torch, dev, reps=4):
    """One small named workload for an ncu capture: inputs drawn on the device
    (seeded), the kernel of interest launched `reps` times, no timing."""
    from moe_gemm_absmax_b200 import inputs, w8a8
    w8a8.lib()
    g = torch.Generator(device=dev)
    g.manual_seed(1234)

    def randn(*shape, std=1.0):
        return torch.randn(*shape, generator=g, device=dev) * std

    kind, _, rest = name.partition("_")
    if name.startswith("moe_g128_"):
        kind, rest = "moe_g128", name[len("moe_g128_"):]
    if kind in ("gemv", "prefill"):
        which, m = rest.split("_")
        d = inputs.GATE_UP if which == "gateup" else inputs.DOWN
        M = int(m[1:])
        qw, sw = w8a8.quant_rows_f32(randn(d["N"], d["K"], std=0.02))
        qx, sx = w8a8.quant_act(randn(M, d["K"]).to(torch.bfloat16))
        path = w8a8.PATH_GEMV if kind == "gemv" else w8a8.PATH_TCGEN05
        y = torch.empty((M, d["N"]), dtype=torch.bfloat16, device=dev)
        torch.cuda.empty_cache()      # only live buffers stay on the device during the capture
        for _ in range(reps):
            w8a8.gemm_q(qx, sx, qw, sw, path, y=y)
    elif kind == "quant":
        m, k = rest.split("_")
        x = randn(int(m[1:]), int(k[1:])).to(torch.bfloat16)
        for _ in range(reps):
            w8a8.quant_act(x)
    elif kind == "moe":
        T = int(rest[1:])
        E, H, I, k = inputs.MOE["E"], inputs.MOE["H"], inputs.MOE["I"], inputs.MOE["topk"]
        q13, s13 = w8a8.quant_rows_f32(randn(E, 2 * I, H, std=0.02))
        q2, s2 = w8a8.quant_rows_f32(randn(E, H, I, std=0.02))
        x = randn(T, H).to(torch.bfloat16)
        lg = randn(T, E).to(torch.bfloat16)
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8a8.moe_workspace_size(T, E, H, I, k), dtype=torch.uint8, device=dev)
        torch.cuda.empty_cache()
        for _ in range(reps):
            w8a8.moe_forward(x, lg, q13, s13, q2, s2, k, y=y, ws=ws)
    elif kind == "moe_g128":
        T = int(rest[1:])
        E, H, I, k = inputs.MOE["E"], inputs.MOE["H"], inputs.MOE["I"], inputs.MOE["topk"]
        q13, s13 = w8a8.fwht128_quant(randn(E * 2 * I, H, std=0.02).to(torch.bfloat16))
        q2, s2 = w8a8.fwht128_quant(randn(E * H, I, std=0.02).to(torch.bfloat16))
        q13, s13 = q13.view(E, 2 * I, H), s13.view(E, 2 * I, H // 128)
        q2, s2 = q2.view(E, H, I), s2.view(E, H, I // 128)
        x = randn(T, H).to(torch.bfloat16)
        lg = randn(T, E).to(torch.bfloat16)
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8a8.moe_g128_workspace_size(T, E, H, I, k), dtype=torch.uint8, device=dev)
        torch.cuda.empty_cache()
        for _ in range(reps):
            w8a8.moe_g128_forward(x, lg, q13, s13, q2, s2, k, y=y, ws=ws)
    elif kind == "shared":
        M = int(rest[1:])
        H, I = inputs.MOE["H"], inputs.MOE["I"]
        q13, u13, r13 = w8a8.trunk_weight_quant(randn(2 * I, H, std=0.02).to(torch.bfloat16))
        q2, s2 = w8a8.fwht128_quant(randn(H, I, std=0.02).to(torch.bfloat16))
        x = randn(M, H).to(torch.bfloat16)
        y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w8a8.shared_expert_workspace_size(M, H, I), dtype=torch.uint8, device=dev)
        torch.cuda.empty_cache()
        for _ in range(reps):
            w8a8.shared_expert_forward(x, q13, u13, r13, q2, s2, y=y, ws=ws)
    elif kind == "head":
        M = int(rest[1:])
        qw, sw = w8a8.group128_quant(randn(HEAD["N"], HEAD["K"], std=0.02).to(torch.bfloat16))
        x = randn(M, HEAD["K"]).to(torch.bfloat16)
        y = torch.empty((M, HEAD["N"]), dtype=torch.bfloat16, device=dev)
        torch.cuda.empty_cache()
        for _ in range(reps):
            q, s = w8a8.group128_quant(x)
            w8a8.linear_group128(q, s, qw, sw, y=y)
    elif kind == "hadamard":
        M = int(rest[1:])
        d = inputs.HADAMARD
        qw, sw = w8a8.fwht128_quant(randn(d["N"], d["K"], std=0.02).to(torch.bfloat16))
        x = randn(M, d["K"]).to(torch.bfloat16)
        y = torch.empty((M, d["N"]), dtype=torch.bfloat16, device=dev)
        torch.cuda.empty_cache()
        for _ in range(reps):
            q, s = w8a8.fwht128_quant(x)
            w8a8.linear_g128(q, s, qw, sw, y=y)
    else:
        raise SystemExit(f"unknown case {name}; one of {', '.join(CASES)}")
    torch.cuda.synchronize()
    print(f"case {name}: ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--quick", action="store_true")
    ap.add_argument("--case", choices=CASES, default=None,
                    help="run one small named workload for a profiler capture and exit")
    args = ap.parse_args()
    if args.case is not None:
        import torch
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        run_case(args.case, torch, dev)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line))
        return

    import torch
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    line = run_ours(args, rank, world, torch, dev)
    if rank == 0:
        if world == 1:
            line["cpu_baseline"] = cpu_baseline()
        line["workloads"] = line.pop("workloads")   # the compact record goes last
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
