"""Benchmark of the weight-only quantized linear on B200.

A step is one pass of the hot path over one batch: for the default workload
(the decode sweep, asymmetric INT4 g128, K = N = 4096) one ``wq_linear`` call
for each M in {1, 2, 4, 8, 16}, each on a different resident copy of the
packed weight so that no call finds its weight in L2 (the copies together are
more than three times the L2 size).  ``value`` is whole-job algorithmic
GB/s: packed weight + scales + zero-points + X + Y bytes of every call,
divided by the device time of the K timed steps (CUDA events, max over
ranks).  The timed steps are replayed from CUDA graphs so that host launch
overhead does not pad the device timeline.

With the default workload the line also carries ``prefill``: the other half
of the metric, the compute-bound INT8 g256 8192 x 8192 layer at
M in {1024, 2048, 4096}, timed by the same protocol (its own step count,
``--prefill-steps`` capped by ``--steps``) and reported in TFLOP/s with its
own roofline, e2e and CPU baseline.

``e2e`` repeats the K steps through the public Python API with host
activations: each call copies X from pinned host memory, runs the linear and
copies Y back (both copies inside the timed region).

``--impl reference`` times the CPU oracle (plain fp64 C, all host cores) on a
bounded sample of the same workload and prints the same line with
``"impl": "reference"``.

Multi-GPU (torchrun): replicas only -- every rank runs the same workload on
its own GPU, no data-path collective; the timing barrier and the max over
ranks use the process group.
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "quantized-linear GB/s (M≤16) and TFLOPS (M≥1024), % of roofline, 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_int4_asym_g128")
    ap.add_argument("--ms", default="", help="comma list overriding the workload's batch sizes")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-context", action="store_true",
                    help="skip the per-call percentiles and the cuBLAS bf16 context line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--no-prefill", action="store_true",
                    help="with the default decode workload, skip the prefill half of the metric")
    ap.add_argument("--prefill-steps", type=int, default=300,
                    help="timed steps of the prefill half (capped by --steps)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [l.strip().split(", ") for l in self.tmp.read().splitlines() if l.strip()]
        self.tmp.close()
        try:
            os.unlink(self.tmp.name)
        except OSError:
            pass
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                for i, nm in enumerate(names):
                    if r[5 + i].strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workload
def build_workload(wl, Ms, device, copies_min_bytes):
    """Packed weight copies (quantized on the GPU by the library), X per M, bias."""
    import torch

    import mixed_gemm_b200 as wq
    import synth.workloads as W

    Wd = torch.from_numpy(W.make_weight(wl)).to(device)
    pw = wq.quantize_and_pack(Wd, wl.fmt, wl.group_size)
    del Wd
    torch.cuda.synchronize()
    R = max(2, int(math.ceil(copies_min_bytes / pw.nbytes)))
    R = min(R, 256)
    weights = [pw] + [pw.clone() for _ in range(R - 1)]
    xs = {}
    xa = W.make_x(wl, max(Ms))
    for M in Ms:
        xs[M] = torch.from_numpy(xa[:M].view(np.int16).copy()).view(torch.bfloat16).to(device)
    b = W.make_bias(wl)
    bias = None if b is None else torch.from_numpy(b.view(np.int16).copy()).view(
        torch.bfloat16).to(device)
    outs = {M: torch.empty((M, wl.N), dtype=torch.bfloat16, device=device) for M in Ms}
    return weights, xs, bias, outs, xa


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when the kernel source changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e:
        return None
    src = [os.path.join(ROOT, "mixed_gemm_b200", "csrc", x) for x in e.get("sources", [])]
    if not src or not all(os.path.exists(s) for s in src) or source_hash(src) != e.get("hash"):
        return None
    return e.get("bytes_per_launch")


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest value over all ranks (timings are taken as the slowest rank's)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, steps: int, work_per_step: float, sec: float, scale: float):
    """Units all ranks processed / the (max-over-ranks) time: every rank runs
    the same step on its own replica."""
    return world * steps * work_per_step / sec / scale


def context_numbers(wl, Ms, weights, xs, bias, outs, stream, l2, device):
    """Per batch size: per-call time over 20 replays of a 50-call graph (p50,
    p95), one launch timed alone (median of 20), and, as a reference point
    only, torch's bf16 F.linear (cuBLAS) on the dequantized weight held as
    bf16, with enough copies to exceed L2."""
    import torch
    import torch.nn.functional as F

    import mixed_gemm_b200 as wq
    R = len(weights)
    out = {}
    pw0 = weights[0]
    w32 = torch.empty((wl.N, wl.K), dtype=torch.float32, device=device)
    wq.wq_dequant(wl.fmt, wl.N, wl.K, wl.group_size, pw0.w, pw0.scales, pw0.aux, w32, stream)
    torch.cuda.synchronize()
    wbf = w32.to(torch.bfloat16)
    del w32
    nb = wbf.numel() * 2
    copies = max(1, min(16, -(-3 * l2 // nb)))
    wcs = [wbf] + [wbf.clone() for _ in range(copies - 1)]
    bias_t = None
    if bias is not None:
        bias_t = bias
    call = linear_call(wl, Ms, device)
    for M in Ms:
        def graph_of(fn, n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                fn(3)
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=stream):
                fn(n)
            return g

        def ours(n, base=[0]):
            for i in range(n):
                pw = weights[(base[0] + i) % R]
                call(xs[M], pw, bias, M, outs[M], stream)
            base[0] += n

        def ref(n, base=[0]):
            for i in range(n):
                F.linear(xs[M], wcs[(base[0] + i) % copies], bias_t)
            base[0] += n

        def per_call(g, n, reps):
            ts = []
            for _ in range(reps):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3 / n)
            return ts

        n = 50
        t_ours = per_call(graph_of(ours, n), n, 20)
        singles = []
        for _ in range(20):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                ours(1)
                e1.record(stream)
            torch.cuda.synchronize()
            singles.append(e0.elapsed_time(e1) * 1e3)
        with torch.cuda.stream(stream):
            t_ref = per_call(graph_of(ref, n), n, 10)
        out[str(M)] = {"per_call_us_p50": float(np.percentile(t_ours, 50)),
                       "per_call_us_p95": float(np.percentile(t_ours, 95)),
                       "single_launch_us": float(np.median(singles)),
                       "cublas_bf16_linear_us": float(np.median(t_ref))}
    del wcs, wbf
    torch.cuda.empty_cache()
    return {"per_M": out, "note": "cublas_bf16_linear_us: torch F.linear on the dequantized "
                                  "weight in bf16 (a reference point, not the target)"}


def cpu_sample(wl, Ms, rows, data):
    """One bounded oracle pass: every token of every M against `rows` output rows."""
    orc, codes, scales, aux, xa, b = data
    t0 = time.perf_counter()
    if wl.act_int8:
        # the oracle's activation-quantized linear on the first `rows` rows
        nb = codes.nbytes // wl.N
        sb = scales.nbytes // wl.N
        c = np.ascontiguousarray(codes.reshape(-1).view(np.uint8)[: rows * nb])
        s = np.ascontiguousarray(scales.reshape(-1).view(np.uint8)[: rows * sb]).view(np.uint16)
        for M in Ms:
            orc.linear_a8(wl.fmt, c.view(np.int8), s, rows, wl.K, wl.group_size, xa[:M],
                          None if b is None else b[:rows])
        return time.perf_counter() - t0
    for M in Ms:
        ms = np.repeat(np.arange(M), rows)
        ns = np.tile(np.arange(rows) * (wl.N // rows), M)
        orc.linear_sampled(wl.fmt, codes, scales, aux, wl.N, wl.K, wl.group_size, xa[:M], b,
                           ms, ns)
    return time.perf_counter() - t0


def cpu_baseline(wl, Ms, seconds, calibrate_only=False):
    """The oracle, as it stands, on a bounded sample of the workload (dequant
    + fp64 dot products for a subset of output rows, every token), in the
    workload's unit: algorithmic GB/s (decode) or TFLOP/s (prefill), scaled by
    the fraction of rows computed."""
    import oracle
    import synth.workloads as W

    tflops_metric = min(Ms) >= 1024
    unit, scale = ("TFLOP/s", 1e12) if tflops_metric else ("GB/s", 1e9)
    if wl.act_int8:
        unit = "TOPS"
    orc = oracle.Oracle()
    Wd = W.make_weight(wl)
    tq0 = time.perf_counter()
    codes, scales, aux = orc.quantize(wl.fmt, Wd, wl.group_size)
    quantize_s = time.perf_counter() - tq0          # the offline phase, whole weight
    del Wd
    xa = W.make_x(wl, max(Ms))
    b = W.make_bias(wl)
    data = (orc, codes, scales, aux, xa, b)
    if tflops_metric:
        total_work = sum(W.flops(M, wl.N, wl.K) for M in Ms)
    else:
        total_work = sum(W.algorithmic_bytes(wl, M) for M in Ms)
    rows = 16
    t = cpu_sample(wl, Ms, rows, data)
    rows = int(min(wl.N, max(1, rows * seconds / max(t, 1e-4))))
    desc = (f"{rows} of {wl.N} output rows for every token of M in {list(Ms)}, "
            f"{orc.threads()} threads")
    work_per_sample = total_work * rows / wl.N
    if calibrate_only:
        return {"rows": rows, "data": data, "cores": orc.threads(), "sample_desc": desc,
                "work_per_sample": work_per_sample}, 0.0
    # repeat the pass (a whole-workload pass can be far shorter than the target)
    reps, t = 0, 0.0
    while reps == 0 or t < 0.8 * seconds:
        t += cpu_sample(wl, Ms, rows, data)
        reps += 1
    value = reps * work_per_sample / t / scale
    cores = orc.threads()
    # the same oracle on one thread, on a smaller sample (a few seconds)
    orc.set_threads(1)
    try:
        rows1 = max(1, rows // max(1, cores) // 2)
        t1 = cpu_sample(wl, Ms, rows1, data)
        single = (total_work * rows1 / wl.N) / t1 / scale
    finally:
        orc.set_threads(cores)
    return {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
            "sample": desc + f", {reps} pass(es), {t:.1f} s",
            "single_thread": {"value": single, "unit": unit,
                              "sample": f"{rows1} rows, 1 thread, {t1:.1f} s"},
            "quantize_s": quantize_s}, t / reps


# ------------------------------------------------------------------ timing
def linear_call(wl, Ms, device):
    """The library call one batch of `wl` makes: wq_linear, or for the
    activation-quantized workload wq_linear_a8 with a preallocated
    workspace per batch size."""
    import torch

    import mixed_gemm_b200 as wq
    if not wl.act_int8:
        def call(x, pw, bias, M, out, stream):
            wq.wq_linear(x, pw.w, pw.scales, pw.aux, bias, M, wl.N, wl.K, wl.fmt, wl.group_size,
                         out, stream)
        return call
    ws = {M: torch.empty((wq.wq_linear_a8_workspace_size(M, wl.K),), dtype=torch.uint8,
                         device=device) for M in Ms}

    def call(x, pw, bias, M, out, stream):
        wq.wq_linear_a8(x, pw.w, pw.scales, bias, M, wl.N, wl.K, wl.fmt, wl.group_size, ws[M],
                        ws[M].numel(), out, stream)
    return call


def time_workload(wl, Ms, steps, warmup, device, l2, world, local_rank, do_e2e):
    """Device time of exactly `steps` steps of `wl` (one wq_linear per M, each
    on the next resident weight copy), replayed from CUDA graphs, CUDA events
    on the launch stream, max over ranks; plus the end-to-end pass through
    the public API with host buffers.  Returns the numbers the JSON line
    reports for this workload."""
    import torch

    import mixed_gemm_b200 as wq
    import synth.workloads as W

    tflops_metric = min(Ms) >= 1024
    unit = ("TOPS" if wl.act_int8 else "TFLOP/s") if tflops_metric else "GB/s"
    weights, xs, bias, outs, xa = build_workload(wl, Ms, device, 3 * l2)
    R = len(weights)
    launches_per_step = len(Ms)
    step_bytes = sum(W.algorithmic_bytes(wl, M) for M in Ms)
    step_flops = sum(W.flops(M, wl.N, wl.K) for M in Ms)
    stream = torch.cuda.Stream(device)
    counter = [0]
    call = linear_call(wl, Ms, device)
    if wl.act_int8:
        launches_per_step *= 2        # the activation quantizer, then the linear

    def step():
        for M in Ms:
            pw = weights[counter[0] % R]
            counter[0] += 1
            call(xs[M], pw, bias, M, outs[M], stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local_rank])

    # graphs of C steps each (the weight copies rotate inside the graph)
    C = max(1, min(200, steps))
    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
    torch.cuda.synchronize()

    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(nsteps):
                step()
        return g

    g_main = capture(C)
    rem = steps % C
    g_rem = capture(rem) if rem else None
    reps = steps // C

    # every graph is replayed once, untimed, whatever the step counts (a
    # graph's first launch uploads it); then W untimed warm-up steps
    with torch.cuda.stream(stream):
        g_main.replay()
        if g_rem is not None:
            g_rem.replay()
        for _ in range(warmup // C):
            g_main.replay()
        for _ in range(warmup % C):
            step()
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(device)
    uuid = getattr(props, "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(device.index))
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):   # graphs replay on the current stream
        ev0.record(stream)
        for _ in range(reps):
            g_main.replay()
        if g_rem is not None:
            g_rem.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, device)
    sec = ms_total / 1e3
    if tflops_metric:
        value = whole_job_value(world, steps, step_flops, sec, 1e12)
    else:
        value = whole_job_value(world, steps, step_bytes, sec, 1e9)
    per_launch_s = sec / (steps * launches_per_step)

    # roofline of the dominant kernel (every launch in the step runs it; for
    # the activation-quantized linear a call is the quantizer plus the
    # tcgen05 kernel, both inside the time per call)
    pk, pk_kind = peaks()
    calls_per_step = len(Ms)
    per_call_s = sec / (steps * calls_per_step)
    peak_note = None
    if tflops_metric and wl.act_int8:
        achieved = step_flops / calls_per_step / per_call_s / 1e12
        # dense INT8 tensor peak: the measured bf16 peak x 2 (the nominal
        # 4.5 / 2.25 PFLOP/s ratio)
        peak = 2.0 * pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        bound, r_unit = "tensor", "TOPS"
        peak_note = "int8 dense = 2 x measured bf16 burst (nominal int8 / bf16 ratio)"
    elif tflops_metric:
        achieved = step_flops / launches_per_step / per_launch_s / 1e12
        peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        bound, r_unit = "tensor", "TFLOP/s"
    else:
        achieved = step_bytes / launches_per_step / per_launch_s / 1e9
        peak = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        bound, r_unit = "hbm", "GB/s"
    kern_src = ["wq_decode.cu", "wq_internal.cuh"] if max(Ms) <= 16 else ["wq_prefill.cu",
                                                                            "wq_internal.cuh"]
    traffic = recorded_traffic(kern_src[0], wl.name)

    # e2e through the public API with host activations
    e2e = None
    if do_e2e:
        xh = {M: torch.from_numpy(xa[:M].view(np.int16).copy()).view(torch.bfloat16).pin_memory()
              for M in Ms}
        yh = {M: torch.empty((M, wl.N), dtype=torch.bfloat16).pin_memory() for M in Ms}
        e2e_steps = max(3, min(steps, 2000))
        k = [0]
        e2e_ws = None
        if wl.act_int8:
            e2e_ws = torch.empty((wq.wq_linear_a8_workspace_size(max(Ms), wl.K),),
                                 dtype=torch.uint8, device=device)

        def e2e_step():
            # every batch of the step from pinned host memory, results copied
            # back; one wait per step (the host may read every result after it)
            for M in Ms:
                pw = weights[k[0] % R]
                k[0] += 1
                if wl.act_int8:
                    wq.linear_a8(xh[M], pw, bias, out=yh[M], workspace=e2e_ws, stream=stream,
                                 sync=False)
                else:
                    wq.linear(xh[M], pw, bias, out=yh[M], stream=stream, sync=False)
            stream.synchronize()

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        es = max_over_ranks(e0.elapsed_time(e1), world, device) / 1e3
        ev = whole_job_value(world, e2e_steps, step_flops if tflops_metric else step_bytes, es,
                             1e12 if tflops_metric else 1e9)
        e2e = {"value": ev, "unit": unit, "steps": e2e_steps,
               "h2d_bytes_per_step": sum(M * wl.K * 2 for M in Ms),
               "d2h_bytes_per_step": sum(M * wl.N * 2 for M in Ms)}
    del g_main, g_rem
    return {
        "value": value, "unit": unit, "steps": steps, "warmup": warmup,
        "ms_per_step": ms_total / steps,
        "config": {"workload": wl.name, "format": wl.fmt, "group_size": wl.group_size,
                   "N": wl.N, "K": wl.K, "Ms": list(Ms), "parallelism": f"replicas{world}",
                   "l2": f"rotating {R} packed-weight copies ({R * weights[0].nbytes / 2**20:.0f} "
                         f"MiB > 3x L2 {l2 / 2**20:.0f} MiB)",
                   "timing": f"CUDA graphs of {C} steps, each replayed once untimed before "
                             "the warm-up; CUDA events on the launch stream"},
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": r_unit,
                     "frac": achieved / peak, "traffic": traffic, "peak_source": pk_kind,
                     "kernel": "decode_kernel" if max(Ms) <= 16 else "prefill_kernel",
                     **({"peak_note": peak_note} if peak_note else {})},
        "gpu_launches": steps * launches_per_step,
        "clocks": clk,
        "e2e": e2e,
        "_state": (weights, xs, bias, outs, stream),
    }


# ------------------------------------------------------------------ MoE
def time_moe(mw, steps, warmup, device, l2, world, local_rank, do_e2e, do_cpu, cpu_seconds):
    """One step = one single-launch grouped linear (wq_linear_grouped_dev) over
    the layer's experts, with the routing offsets resident on the device;
    stacked expert copies rotate past L2.  Context: the same step as one
    wq_linear per non-empty expert (host offsets)."""
    import torch

    import mixed_gemm_b200 as wq
    import synth.workloads as W

    counts = W.moe_counts(mw)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    experts = []
    for e in range(mw.E):
        wd = torch.from_numpy(W.moe_weight(mw, e)).to(device)
        experts.append(wq.quantize_and_pack(wd, mw.fmt, mw.group_size))
        del wd
    stacked = wq.stack_experts(experts)
    R = max(2, int(math.ceil(3 * l2 / stacked.nbytes)))
    copies = [stacked] + [stacked.clone() for _ in range(R - 1)]
    xa = W.moe_x(mw)
    x = torch.from_numpy(xa.view(np.int16).copy()).view(torch.bfloat16).to(device)
    off_d = torch.from_numpy(offsets).to(device)
    y = torch.empty((mw.rows, mw.N), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.Stream(device)
    work_bytes = W.moe_bytes(mw, counts)
    flops = 2.0 * mw.rows * mw.N * mw.K
    prefill_like = mw.rows // mw.E > 64
    # the library's dispatch: the decode kernel while the mean rows per expert
    # (rounded up) is at most 16, the tcgen05 kernel above
    tc_path = -(-mw.rows // mw.E) > 16
    counter = [0]

    def step():
        c = copies[counter[0] % R]
        counter[0] += 1
        wq.wq_linear_grouped_dev(x, c.w, c.scales, c.aux, None, off_d, mw.E, mw.rows, mw.N, mw.K,
                                 mw.fmt, mw.group_size, y, stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local_rank])

    C = max(1, min(100, steps))
    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(C):
            step()
    rem = steps % C
    g_rem = None
    if rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem, stream=stream):
            for _ in range(rem):
                step()
    with torch.cuda.stream(stream):
        g.replay()
        if g_rem is not None:
            g_rem.replay()
        for _ in range(max(1, warmup // C)):
            g.replay()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(device)
    uuid = getattr(props, "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(device.index))
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(steps // C):
            g.replay()
        if g_rem is not None:
            g_rem.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, device)
    sec = ms / 1e3
    pk, pk_kind = peaks()
    if prefill_like:
        value = whole_job_value(world, steps, flops, sec, 1e12)
        unit, bound = "TFLOP/s", "tensor"
        achieved = flops / (sec / steps) / 1e12
        peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    else:
        value = whole_job_value(world, steps, work_bytes, sec, 1e9)
        unit, bound = "GB/s", "hbm"
        achieved = work_bytes / (sec / steps) / 1e9
        peak = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])

    # context: the host loop of one launch per non-empty expert
    loop_us = None
    if world == 1:
        def loop_step():
            c = copies[counter[0] % R]
            counter[0] += 1
            wq.linear_grouped(x, [c_e for c_e in per_expert(c)], offsets, out=y, stream=stream)

        wb, sb, ab = wq.wq_packed_sizes(mw.fmt, mw.N, mw.K, mw.group_size)

        def per_expert(c):
            return [wq.PackedWeight(mw.fmt, mw.N, mw.K, mw.group_size, c.w[e * wb:(e + 1) * wb],
                                    c.scales[e * sb:(e + 1) * sb],
                                    None if c.aux is None else c.aux[e * ab:(e + 1) * ab])
                    for e in range(mw.E)]

        views = [per_expert(c) for c in copies]
        k = [0]

        def loop_once():
            v = views[k[0] % R]
            k[0] += 1
            wq.linear_grouped(x, v, offsets, out=y, stream=stream)

        for _ in range(3):
            loop_once()
        torch.cuda.synchronize()
        gl = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gl, stream=stream):
            for _ in range(10):
                loop_once()
        with torch.cuda.stream(stream):
            gl.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            gl.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        loop_us = e0.elapsed_time(e1) * 1e3 / 10
        del gl

    e2e = None
    if do_e2e:
        xh = torch.from_numpy(xa.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
        oh = torch.from_numpy(offsets).pin_memory()
        yh = torch.empty((mw.rows, mw.N), dtype=torch.bfloat16).pin_memory()
        e2e_steps = max(3, min(steps, 200))

        def e2e_step():
            with torch.cuda.stream(stream):
                x.copy_(xh, non_blocking=True)
                off_d.copy_(oh, non_blocking=True)
                step()
                yh.copy_(y, non_blocking=True)
            stream.synchronize()

        for _ in range(3):
            e2e_step()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        es = max_over_ranks(e0.elapsed_time(e1), world, device) / 1e3
        ev = whole_job_value(world, e2e_steps, flops if prefill_like else work_bytes, es,
                             1e12 if prefill_like else 1e9)
        e2e = {"value": ev, "unit": unit, "steps": e2e_steps,
               "h2d_bytes_per_step": int(xa.nbytes + offsets.nbytes),
               "d2h_bytes_per_step": int(mw.rows * mw.N * 2)}

    cb = None
    if do_cpu:
        cb = moe_cpu_baseline(mw, counts, offsets, xa, prefill_like, cpu_seconds)
    del g, g_rem
    return {
        "value": value, "unit": unit, "steps": steps, "warmup": warmup, "ms_per_step": ms / steps,
        "config": {"workload": mw.name, "format": mw.fmt, "group_size": mw.group_size,
                   "experts": mw.E, "N": mw.N, "K": mw.K, "rows": mw.rows,
                   "tokens": mw.tokens, "topk": mw.topk,
                   "counts": {"min": int(counts.min()), "max": int(counts.max()),
                              "empty": int((counts == 0).sum())},
                   "parallelism": f"replicas{world}",
                   "l2": f"rotating {R} stacked-expert copies "
                         f"({R * stacked.nbytes / 2**20:.0f} MiB > 3x L2 {l2 / 2**20:.0f} MiB)",
                   "timing": f"CUDA graphs of {C} steps, each replayed once untimed; CUDA "
                             "events on the launch stream"},
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s" if prefill_like else "GB/s", "frac": achieved / peak,
                     "traffic": recorded_traffic("wq_prefill.cu" if tc_path else "wq_decode_kernel.cuh",
                                                 mw.name),
                     "peak_source": pk_kind,
                     "kernel": "prefill_kernel" if tc_path else "decode_kernel"},
        "gpu_launches": steps, "clocks": clk, "e2e": e2e, "cpu_baseline": cb,
        "context": {"host_loop_us_per_step": loop_us,
                    "single_launch_us_per_step": ms / steps * 1e3,
                    "note": "host loop: one wq_linear per non-empty expert from host offsets"},
    }


def moe_cpu_baseline(mw, counts, offsets, xa, prefill_like, seconds):
    """The oracle on a bounded sample of the MoE step: every row of each
    expert against a subset of that expert's output features."""
    import oracle
    import synth.workloads as W

    orc = oracle.Oracle()
    q = []
    for e in range(mw.E):
        q.append(orc.quantize(mw.fmt, W.moe_weight(mw, e), mw.group_size))

    def sample(cols):
        t0 = time.perf_counter()
        for e in range(mw.E):
            a, b = int(offsets[e]), int(offsets[e + 1])
            if a == b:
                continue
            codes, scales, aux = q[e]
            ms = np.repeat(np.arange(b - a), cols)
            ns = np.tile(np.arange(cols) * (mw.N // cols), b - a)
            orc.linear_sampled(mw.fmt, codes, scales, aux, mw.N, mw.K, mw.group_size, xa[a:b],
                               None, ms, ns)
        return time.perf_counter() - t0

    cols = 2
    t = sample(cols)
    cols = int(min(mw.N, max(1, cols * seconds / max(t, 1e-4))))
    reps, t = 0, 0.0
    while reps == 0 or t < 0.8 * seconds:
        t += sample(cols)
        reps += 1
    frac = cols / mw.N
    if prefill_like:
        value, unit = reps * 2.0 * mw.rows * mw.N * mw.K * frac / t / 1e12, "TFLOP/s"
    else:
        value, unit = reps * W.moe_bytes(mw, counts) * frac / t / 1e9, "GB/s"
    return {"value": value, "unit": unit, "cores": orc.threads(), "kind": "oracle",
            "sample": f"{cols} of {mw.N} output features of every routed row of every expert, "
                      f"{orc.threads()} threads, {reps} pass(es), {t:.1f} s"}


# ------------------------------------------------------------------ main
def main():
    args = parse()
    import synth.workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in W.MOE:
        return main_moe(args, W.MOE[args.workload], world, rank, local_rank)
    wl = W.BY_NAME[args.workload]
    Ms = tuple(int(m) for m in args.ms.split(",")) if args.ms else wl.Ms
    tflops_metric = min(Ms) >= 1024
    unit = ("TOPS" if wl.act_int8 else "TFLOP/s") if tflops_metric else "GB/s"

    if args.impl == "reference":
        if rank != 0:
            return
        # each step: the oracle on a bounded sample, sized so that warm-up and
        # timed steps together take about a minute of host time
        per_step = min(12.0, max(0.05, 60.0 / max(1, args.steps + args.warmup)))
        cb, _ = cpu_baseline(wl, Ms, per_step, calibrate_only=True)
        rows = cb["rows"]
        for _ in range(args.warmup):
            cpu_sample(wl, Ms, rows, cb["data"])
        times = [cpu_sample(wl, Ms, rows, cb["data"]) for _ in range(max(1, args.steps))]
        t = sum(times)
        scale = 1e12 if tflops_metric else 1e9
        value = len(times) * cb["work_per_sample"] / t / scale
        desc = {"value": value, "unit": unit, "cores": cb["cores"], "kind": "oracle",
                "sample": cb["sample_desc"]}
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit,
                "n_gpus": args.gpus, "steps": len(times), "warmup": args.warmup,
                "ms_per_step": t / len(times) * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": wl.name, "N": wl.N, "K": wl.K, "Ms": list(Ms),
                           "format": wl.fmt, "group_size": wl.group_size},
                "cpu_baseline": desc,
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch

    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())

    import mixed_gemm_b200  # noqa: F401  (fails loudly when the library is missing)

    props = torch.cuda.get_device_properties(device)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20)
    head = time_workload(wl, Ms, args.steps, args.warmup, device, l2, world, local_rank,
                         not args.no_e2e)
    ctx = None
    if rank == 0 and world == 1 and not args.no_context:
        ctx = context_numbers(wl, Ms, *head["_state"][:5], l2, device)
    del head["_state"]
    torch.cuda.empty_cache()

    # the other half of the metric: the compute-bound prefill sweep, timed by
    # the same protocol on its own step count (a prefill step is ~1.5 ms)
    second = None
    if not args.no_prefill and not tflops_metric and args.workload == W.DECODE.name:
        pwl = W.PREFILL
        psteps = max(1, min(args.steps, args.prefill_steps))
        second = time_workload(pwl, pwl.Ms, psteps, max(3, min(args.warmup, psteps)), device, l2,
                               world, local_rank, not args.no_e2e)
        pctx = None
        if rank == 0 and world == 1 and not args.no_context:
            pctx = context_numbers(pwl, pwl.Ms, *second["_state"][:5], l2, device)
        del second["_state"]
        second["context"] = pctx
        torch.cuda.empty_cache()

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb, _ = cpu_baseline(wl, Ms, args.cpu_seconds)
        if second is not None:
            second["cpu_baseline"], _ = cpu_baseline(W.PREFILL, W.PREFILL.Ms, args.cpu_seconds)

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": head["value"], "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": head["config"], "roofline": head["roofline"],
        "gpu_launches": head["gpu_launches"], "clocks": head["clocks"], "e2e": head["e2e"],
        "cpu_baseline": cb, "context": ctx,
    }
    if second is not None:
        line["prefill"] = second
    print(json.dumps(line), flush=True)


def main_moe(args, mw, world, rank, local_rank):
    """The grouped (mixture-of-experts) workloads: one JSON line, like main()."""
    if args.impl == "reference":
        if rank != 0:
            return
        import synth.workloads as W
        counts = W.moe_counts(mw)
        offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
        prefill_like = mw.rows // mw.E > 64
        per_step = min(12.0, max(0.05, 60.0 / max(1, args.steps + args.warmup)))
        vals = [moe_cpu_baseline(mw, counts, offsets, W.moe_x(mw), prefill_like, per_step)
                for _ in range(max(1, args.steps))]
        v = float(np.median([c["value"] for c in vals]))
        unit = vals[0]["unit"]
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": v, "unit": unit,
                          "n_gpus": args.gpus, "steps": len(vals), "warmup": args.warmup,
                          "ms_per_step": per_step * 1e3, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "config": {"workload": mw.name},
                          "cpu_baseline": vals[0],
                          "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}), flush=True)
        return
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    import mixed_gemm_b200  # noqa: F401
    props = torch.cuda.get_device_properties(device)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20)
    r = time_moe(mw, args.steps, args.warmup, device, l2, world, local_rank, not args.no_e2e,
                 rank == 0 and world == 1 and not args.no_cpu_baseline, args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": r["value"], "unit": r["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": r["config"], "roofline": r["roofline"],
            "gpu_launches": r["gpu_launches"], "clocks": r["clocks"], "e2e": r["e2e"],
            "cpu_baseline": r["cpu_baseline"], "context": r["context"]}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
