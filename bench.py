"""Benchmark of the GPTQ per-layer solve on B200.

One step = the whole hot path for one layer: H = 2 X^T X over the calibration set
(tcgen05), prepare (dead columns, act-order, damping, U = upper-Cholesky(H^-1)), and the
blocked column sweep with its trailing updates, emitting packed codes, scales, zeros,
perm and g_idx.  Default workload: the largest single-GPU layer, the 70B-shaped down_proj
(W 8192x28672 fp16 ~N(0, 0.01^2), X 65536 tokens x 28672 bf16 with 1 % outlier channels
x20, 4-bit asymmetric, group 128, damp 0.01, act-order), seeded synthetic data; the other
layers are selectable with --config.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--config NAME]

Under torchrun each rank quantizes its own independent layer (weak scaling; no collective
on the data path); the timed region is bracketed by barriers and the max over ranks is
reported.  After the timed region one more step runs with the library's per-kernel
instrumentation (CUDA events around every launch) to name the dominant kernel and its
achieved rate.  Prints one JSON line on rank 0.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from post_weight_quantization_16_b200 import synth  # noqa: E402

METRIC = "GPTQ layer quant: Gweights/s + Hessian TFLOP/s, % of roofline, 1×B200"
WORKLOAD = "down_proj_8192x28672"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal dense tensor rates relative to bf16 (2.25 PFLOP/s): tf32 1.1 PFLOP/s
TF32_OVER_BF16 = 1.1 / 2.25

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of a kernel from one ncu
# capture of a smaller case, valid only while the kernel's sources hash to the ones captured.
# "scale" says how the capture's bytes grow to a full launch of the benchmarked workload.
PROFILED_TRAFFIC = {
    "hessian_syrk_pair": {
        "sources": {"post_weight_quantization_16_b200/csrc/hessian_tc.cuh": "99d3e9d95b42960505710a519acfa15b724aa743",
                    "post_weight_quantization_16_b200/csrc/sm100_ptx.cuh": "4ec31015a518232159fb85f700fb1d56e4a57de1"},
        "n": 4096, "tokens": 65536, "dram_bytes": 975.479040e6 + 24.431360e6, "scale": "tokens",
    },
}


def _sha1(path):
    import hashlib
    with open(os.path.join(ROOT, path), "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()


def profiled_traffic(kernel: str, n: int, n_tok: int):
    """Bytes per launch of `kernel` at width n and n_tok tokens, from the ncu record, or None."""
    rec = PROFILED_TRAFFIC.get(kernel)
    if rec is None or rec["n"] != n:
        return None
    for path, sha in rec["sources"].items():
        if _sha1(path) != sha:
            return None
    return rec["dram_bytes"] * n_tok / rec["tokens"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def choose_peak(peaks, timed_s: float, clk):
    """The burst bf16 peak for a short timed region at full clocks; the sustained one when the
    region lasted seconds and the clocks show the power cap (or sat well below their maximum)."""
    capped = bool(clk) and ("sw_power_cap" in clk.get("reasons", []) or
                            clk.get("sm_mhz", 0) < 0.9 * clk.get("sm_max_mhz", 1))
    if timed_s >= 1.0 and capped and "bf16_tflops_sustained" in peaks:
        return peaks["bf16_tflops_sustained"], "sustained", (
            f"timed region {timed_s:.1f} s with the clocks under the power cap (median SM "
            f"{clk.get('sm_mhz')} of {clk.get('sm_max_mhz')} MHz)")
    return peaks["bf16_tflops"], "burst", (
        f"timed region {timed_s:.2f} s" + ("" if capped else " at full clocks"))


def dominant_kernel(prof: dict):
    """Fold the per-role profile into kernels (the part of a role name before ':') and return
    (name, totals) of the kernel with the largest total time."""
    kern = {}
    for role, v in prof.items():
        k = role.split(":")[0]
        a = kern.setdefault(k, {"launches": 0, "ms": 0.0, "flops": 0.0, "bytes": 0.0, "roles": []})
        for f in ("launches", "ms", "flops", "bytes"):
            a[f] += v[f]
        a["roles"].append(role)
    name = max(kern, key=lambda k: kern[k]["ms"])
    return name, kern[name]


# ----------------------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def rank_layer(layer, rank):
    """Rank r quantizes its own layer: same shape and recipe, seeds offset by r."""
    if rank == 0:
        return layer
    import dataclasses
    return dataclasses.replace(layer, name=f"{layer.name}_r{rank}", x_seed=layer.x_seed + 7919 * rank,
                               w_seed=layer.w_seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = "clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown," \
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
             "clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same workload)
# ----------------------------------------------------------------------------------------
def cpu_oracle_baseline(layer, qs, tok_sample=16384, row_sample=256, col_sample=4096, data=None):
    """The oracle timed on a bounded sample of the layer, scaled to the whole layer.  The sample
    is the leading col_sample columns (pn) of the layer: the Hessian of tok_sample tokens over
    those columns (time x (N / tokens) x (n / pn)^2), prepare of that pn x pn Hessian
    (time x (n / pn)^3) and the blocked sweep of row_sample rows over the pn columns
    (time x (m / rows) x (n / pn)).  `data` = (X sample, W) generated beforehand, outside
    the timing."""
    from oracle import gptq_oracle as O
    cores = len(os.sched_getaffinity(0))
    tok_sample = min(tok_sample, layer.n_tok)
    row_sample = min(row_sample, layer.m)
    pn = min(col_sample, layer.n)
    if data is None:
        data = (synth.bf16_bits_to_f32(synth.make_x_bf16(layer, 0, tok_sample)[:, :pn]),
                synth.make_w_fp16(layer)[:row_sample, :pn].astype(np.float64))
    X, W = data
    X, W = X[:, :pn], W[:row_sample, :pn]
    t0 = time.perf_counter()
    H = O.hessian(X)
    t_h = (time.perf_counter() - t0) * (layer.n_tok / X.shape[0]) * (layer.n / pn) ** 2
    t0 = time.perf_counter()
    prep = O.prepare(H, qs.damp, qs.desc_act)
    t_p = (time.perf_counter() - t0) * (layer.n / pn) ** 3
    g = qs.group_size if (qs.group_size != -1 and pn % qs.group_size == 0) else -1
    Wp = W[:, prep["perm"]]
    t0 = time.perf_counter()
    O.gptq_sweep(Wp, prep["U"], qs.bits, g, bool(qs.sym), block=128)
    t_s = (time.perf_counter() - t0) * (layer.m / W.shape[0]) * (layer.n / pn)
    t_layer = t_h + t_p + t_s
    return {
        "value": layer.m * layer.n / t_layer / 1e9, "unit": "Gweights/s", "cores": cores, "kind": "oracle",
        "sample": (f"the leading {pn} of {layer.n} columns: Hessian of {X.shape[0]} of {layer.n_tok} tokens "
                   f"(scaled by tokens and (n/{pn})^2), prepare (scaled by (n/{pn})^3), blocked sweep of "
                   f"{W.shape[0]} of {layer.m} rows (scaled by rows and n/{pn}); float64 numpy"),
        "seconds_per_layer": t_layer, "stage_seconds": {"hessian": t_h, "prepare": t_p, "sweep": t_s},
    }


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, timed as it stands, on bounded samples."""
    if rank != 0:
        return
    if args.config not in synth.WORKLOADS:
        print(json.dumps({"impl": "reference", "unavailable": f"the oracle arm times the layer solve; {args.config} "
                                                              "is measured on the GPU arm only"}), flush=True)
        return
    layer, qs = synth.WORKLOADS[args.config]
    # each step a sample small enough that all warm-up and timed steps end within a few minutes
    n_steps = args.warmup + args.steps
    if n_steps <= 4:
        tok, rows, pn = 4096, 64, 4096
    elif n_steps <= 20:
        tok, rows, pn = 2048, 32, 2048
    else:
        tok, rows, pn = 1024, 16, 2048
    pn = min(pn, layer.n)
    data = (synth.bf16_bits_to_f32(synth.make_x_bf16(layer, 0, min(tok, layer.n_tok))[:, :pn]),
            synth.make_w_fp16(layer)[:rows, :pn].astype(np.float64))
    times = []
    r = None
    for step in range(n_steps):
        r = cpu_oracle_baseline(layer, qs, tok_sample=tok, row_sample=rows, col_sample=pn, data=data)
        if step >= args.warmup:
            times.append(r["seconds_per_layer"])
    t = sum(times) / len(times)
    val = layer.m * layer.n / t / 1e9
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "Gweights/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.config, "m": layer.m, "n": layer.n, "n_tok": layer.n_tok, "bits": qs.bits,
                   "group_size": qs.group_size, "sym": qs.sym, "damp": qs.damp, "desc_act": qs.desc_act},
        "cpu_baseline": {"value": val, "unit": "Gweights/s", "cores": cores, "kind": "oracle",
                         "sample": "each step: " + r["sample"]},
        "e2e": {"value": val, "unit": "Gweights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------------------
def path_rooflines(layer, qs, peak_bf16, hbm_gbs):
    """Lower bounds on the step time: every contraction at the bf16 peak against the sweep's
    bytes at HBM bandwidth; and the same with the factorization and trailing products at the
    rate of the precision the path computes them in (three tf32 products per fp32 product)."""
    n, m, N = layer.n, layer.m, layer.n_tok
    f_h = N * n * (n + 1)
    f_fact = 2 * n ** 3 / 3
    f_trail = 2 * m * sum(128 * (n - i2) for i2 in range(128, n, 128))
    g = n if qs.group_size == -1 else qs.group_size
    b_sweep = 2 * m * n + 2 * n * (n + 1) + m * n * qs.bits / 8 + 8 * m * n / g + 8 * n
    t_bytes = b_sweep / (hbm_gbs * 1e9)
    t_bf16 = max((f_h + f_fact + f_trail) / (peak_bf16 * 1e12), t_bytes)
    fp32_rate = peak_bf16 * TF32_OVER_BF16 / 3
    t_prec = max(f_h / (peak_bf16 * 1e12) + (f_fact + f_trail) / (fp32_rate * 1e12), t_bytes)
    return t_bf16, t_prec, {"hessian": f_h, "factorization": f_fact, "trailing": f_trail, "sweep_bytes": b_sweep}


def run_gpu(args, rank, world, local_rank):
    import torch
    from post_weight_quantization_16_b200 import build as B
    from post_weight_quantization_16_b200 import gptq as G

    B.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    layer0, qs = synth.WORKLOADS[args.config]
    layer = rank_layer(layer0, rank)
    peaks, peaks_src = load_peaks()

    # inputs resident in HBM before timing
    X_host = synth.make_x_bf16(layer)
    W_host = synth.make_w_fp16(layer)
    X = torch.from_numpy(X_host.view(np.int16)).to(dev).view(torch.bfloat16)
    W = torch.from_numpy(W_host).to(dev)
    stream = torch.cuda.current_stream(dev)
    ctx = G.GPTQContext(layer.n, layer.m, local_rank, stream)
    out = None
    perm_holder = [None]

    def step(timing=None):
        nonlocal out
        ctx.reset()
        if timing is not None:
            timing[0].record(stream)
        ctx.accumulate_hessian(X)
        if timing is not None:
            timing[1].record(stream)
        perm_holder[0] = ctx.prepare(qs.damp, qs.desc_act)
        if timing is not None:
            timing[2].record(stream)
        out = ctx.quantize_layer(W, qs.bits, qs.group_size, bool(qs.sym), want_w_hat=False, out=out)
        if timing is not None:
            timing[3].record(stream)

    for _ in range(args.warmup):
        step()
    ctx.synchronize()
    launches0 = ctx.launch_count()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                          int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    start.record(stream)
    for k in range(args.steps):
        step(ev[k])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    ctx.synchronize()
    launches = ctx.launch_count() - launches0

    ms_total = start.elapsed_time(stop)
    ms_total = max_over_ranks(ms_total, world, dev)
    t_h = [e[0].elapsed_time(e[1]) for e in ev]
    t_p = [e[1].elapsed_time(e[2]) for e in ev]
    t_q = [e[2].elapsed_time(e[3]) for e in ev]
    ms_step = ms_total / args.steps
    weights = layer.m * layer.n
    value = world * weights * args.steps / (ms_total / 1e3) / 1e9
    peak, peak_kind, peak_why = choose_peak(peaks, ms_total / 1e3, clk)
    n, m = layer.n, layer.m

    # one instrumented step right after the timed region: CUDA events around every launch
    ctx.set_profiling(True)
    step()
    prof = ctx.get_profile()
    ctx.set_profiling(False)
    kname, k = dominant_kernel(prof)
    tensor_kernel = k["flops"] > 0
    if kname.startswith("gemm_"):
        # fp32-faithful products as three tf32 products: the peak of one algorithmic fp32 flop
        kpeak, kunit = peak * TF32_OVER_BF16 / 3, "TFLOP/s"
        kpeak_src = (f"{peaks_src} bf16 dense {peak_kind} peak x {TF32_OVER_BF16:.3f} (nominal tf32/bf16) / 3 "
                     f"(three tf32 products per fp32 product)")
    elif tensor_kernel:
        kpeak, kunit, kpeak_src = peak, "TFLOP/s", f"{peaks_src} bf16 dense {peak_kind} peak"
    else:
        kpeak, kunit, kpeak_src = peaks["hbm_gbs"], "GB/s", f"{peaks_src} HBM copy bandwidth"
    achieved = (k["flops"] / 1e12 if tensor_kernel else k["bytes"] / 1e9) / (k["ms"] / 1e3)
    traffic = profiled_traffic(kname, n, layer.n_tok)
    roofline = {"bound": "tensor" if tensor_kernel else "hbm", "kernel": kname, "roles": k["roles"],
                "achieved": achieved, "peak": kpeak, "unit": kunit, "frac": achieved / kpeak,
                "traffic": traffic, "peak_source": f"{kpeak_src}; {peak_why}",
                "algorithmic_flops_per_launch": k["flops"] / k["launches"] if tensor_kernel else None,
                "algorithmic_bytes_per_launch": None if tensor_kernel else k["bytes"] / k["launches"],
                "launches": k["launches"], "ms_per_launch": k["ms"] / k["launches"],
                "timing": "per-launch CUDA events on the context's stream, one instrumented step after the timed region"}
    h_ms = statistics.mean(t_h)
    h_flops = layer.n_tok * n * (n + 1)           # algorithmic: upper triangle incl. diagonal
    h_tflops = h_flops / (h_ms / 1e3) / 1e12
    hessian_roofline = {"bound": "tensor", "kernel": "hessian_syrk_pair", "achieved": h_tflops, "peak": peak,
                        "unit": "TFLOP/s", "frac": h_tflops / peak, "algorithmic_flops_per_launch": h_flops,
                        "traffic": profiled_traffic("hessian_syrk_pair", n, layer.n_tok),
                        "timing": "CUDA events around the launch inside the timed region",
                        "peak_source": f"{peaks_src} bf16 dense {peak_kind}"}
    t_roof, t_prec, work = path_rooflines(layer, qs, peak, peaks["hbm_gbs"])

    # the packed result's consumer on this layer's own output (W4A16 product)
    # (a kernel timed alone: the burst bf16 peak)
    w4a16 = None if args.no_w4a16 else w4a16_measure(G, out, perm_holder[0], layer, qs, dev, stream, peaks,
                                                     peaks["bf16_tflops"])

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e_ms = None
    G_ = n // (n if qs.group_size == -1 else qs.group_size)
    d2h = m * n * qs.bits // 8 + 2 * m * G_ * 4 + 2 * n * 4
    h2d = X_host.nbytes + W_host.nbytes
    if not args.no_e2e:
        Xh = torch.from_numpy(X_host.view(np.int16)).view(torch.bfloat16).pin_memory()
        Wh = torch.from_numpy(W_host).pin_memory()
        e2e_ms = e2e_run(ctx, Xh, Wh, qs, dev, stream, reps=max(1, min(3, args.steps)))
        e2e_ms = max_over_ranks(e2e_ms, world, dev)
        del Xh, Wh

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_baseline(layer, qs)

    ctx.close()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "Gweights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16->f32", "data": "synthetic",
            "config": {"workload": args.config, "m": m, "n": n, "n_tok": layer.n_tok, "bits": qs.bits,
                       "group_size": qs.group_size, "sym": qs.sym, "damp": qs.damp, "desc_act": qs.desc_act,
                       "l2": "inputs larger than L2 (X is %.2f GB)" % (X_host.nbytes / 1e9),
                       "parallelism": f"replicas x{world} (one independent layer per GPU)"},
            "hessian_tflops": h_tflops,
            "stage_ms": {"hessian": h_ms, "prepare": statistics.mean(t_p), "quantize": statistics.mean(t_q)},
            "gweights_per_s_solve": weights / ((statistics.mean(t_p) + statistics.mean(t_q)) / 1e3) / 1e9,
            "path_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_step,
                              "t_roof_ms_at_path_precision": t_prec * 1e3,
                              "frac_at_path_precision": t_prec * 1e3 / ms_step,
                              "algorithmic_work": work, "peak_bf16_tflops": peak, "peak_kind": peak_kind},
            "roofline": roofline,
            "hessian_roofline": hessian_roofline,
            "kernels": prof,
            "w4a16": w4a16,
            "e2e": None if e2e_ms is None else {
                "value": world * weights / (e2e_ms / 1e3) / 1e9, "unit": "Gweights/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def w4a16_measure(G, out, perm, layer, qs, dev, stream, peaks, peak_bf16, reps=8):
    """Y = X W16^T from the step's packed codes (gptq_dequant_matmul) for a decode-sized and a
    prefill-sized batch of fp16 activations; each launch timed alone with CUDA events, L2
    flushed (a 256 MB write) before every repetition."""
    import torch
    n, m = layer.n, layer.m
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    res = {}
    for T in (16, 4096):
        X = torch.randn((T, n), device=dev, dtype=torch.float32).to(torch.float16)
        Y = torch.empty((T, m), dtype=torch.float32, device=dev)
        ws = torch.empty(int(G.lib().gptq_dequant_matmul_workspace_bytes(T, m, n, 1)), dtype=torch.uint8, device=dev)
        cap = torch.cuda.Stream(dev)  # graphs are captured on a stream of their own
        call = lambda st: G.dequant_matmul(X, out["codes"], out["scales"], out["zeros"], perm, qs.bits,
                                           qs.group_size, out=Y, workspace=ws, stream=st)
        call(stream)  # first call: kernel attributes and tensor-map encoding outside the capture
        torch.cuda.synchronize(dev)
        # the call as a CUDA graph, so that its host-side setup does not sit inside the timed window
        graph = torch.cuda.CUDAGraph()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            graph.capture_begin(capture_error_mode="thread_local")
            call(cap)
            graph.capture_end()
        torch.cuda.synchronize(dev)
        ms = []
        for r in range(reps + 2):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            with torch.cuda.stream(stream):
                graph.replay()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if r >= 2:
                ms.append(e0.elapsed_time(e1))
        del graph
        t = statistics.median(ms)
        g = n if qs.group_size == -1 else qs.group_size
        byts = m * n * qs.bits / 8 + 8 * m * (n // g) + 2 * T * n + 4 * T * m + 4 * n
        flops = 2.0 * T * m * n
        if T <= 64:
            ach = byts / (t / 1e3) / 1e9
            res[f"T{T}"] = {"ms": t, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": ach / peaks["hbm_gbs"], "algorithmic_bytes": byts}
        else:
            ach = flops / (t / 1e3) / 1e12
            res[f"T{T}"] = {"ms": t, "bound": "tensor", "achieved": ach, "peak": peak_bf16, "unit": "TFLOP/s",
                            "frac": ach / peak_bf16, "algorithmic_flops": flops}
    res["note"] = ("fp16 activations x fp16-dequantized weights, fp32 accumulation; act-order gather included; "
                   "median of %d graph replays of the call, L2 flushed before each; burst bf16 peak" % reps)
    return res


def e2e_run(ctx, Xh, Wh, qs, dev, stream, reps=2, batch_tokens=16384):
    """Host X and W in, packed codes/scales/zeros/perm/g_idx out.  The calibration set is
    copied in batches on a side stream, double-buffered against the Hessian kernel.  Device
    and pinned host buffers are allocated once, before the timed repetitions."""
    import torch
    n = ctx.n
    N = Xh.shape[0]
    copy_stream = torch.cuda.Stream(dev)
    bufs = [torch.empty((batch_tokens, n), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    Wd = torch.empty(Wh.shape, dtype=Wh.dtype, device=dev)
    out = None
    host = None
    times = []
    for _ in range(reps + 1):
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        copy_stream.wait_event(t0)
        ctx.reset()
        with torch.cuda.stream(copy_stream):
            Wd.copy_(Wh, non_blocking=True)
        w_ready = torch.cuda.Event()
        w_ready.record(copy_stream)
        nb = (N + batch_tokens - 1) // batch_tokens
        for b in range(nb):
            j = b & 1
            rows = min(batch_tokens, N - b * batch_tokens)
            if b >= 2:
                copy_stream.wait_event(consumed[j])
            with torch.cuda.stream(copy_stream):
                bufs[j][:rows].copy_(Xh[b * batch_tokens:b * batch_tokens + rows], non_blocking=True)
            copied[j].record(copy_stream)
            stream.wait_event(copied[j])
            ctx.accumulate_hessian(bufs[j][:rows])
            consumed[j].record(stream)
        perm = ctx.prepare(qs.damp, qs.desc_act)
        stream.wait_event(w_ready)
        out = ctx.quantize_layer(Wd, qs.bits, qs.group_size, bool(qs.sym), want_w_hat=False, out=out)
        res = dict(out, perm=perm)
        if host is None:  # first (untimed) repetition: pinned host outputs, reused afterwards
            host = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in res.items() if v is not None}
        for k, v in res.items():
            if v is not None:
                host[k].copy_(v, non_blocking=True)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        times.append(t0.elapsed_time(t1))
    return statistics.mean(times[1:])


def run_block(args, rank, world, local_rank):
    """The 7B-shaped block sweep as one pipelined run per step: seven layers with their own
    calibration sets (65536 tokens each), each quantized under the 18 settings of bits x
    group_size x damp (126 quantize runs, 14 factorizations, 7 Hessians), on a pipeline whose
    contexts are created before the timing.  The same jobs run one layer at a time through the
    context calls (contexts also created before the timing) give the sequential time."""
    import torch
    from post_weight_quantization_16_b200 import build as B
    from post_weight_quantization_16_b200 import gptq as G
    B.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    layers = synth.block7b_layers()
    settings = synth.block7b_settings()
    Xs = [torch.from_numpy(synth.make_x_bf16(L).view(np.int16)).to(dev).view(torch.bfloat16) for L in layers]
    Ws = [torch.from_numpy(synth.make_w_fp16(L)).to(dev) for L in layers]
    jobs = [dict(X=X, W=W, bits=q.bits, group_size=q.group_size, sym=q.sym, damp=q.damp, desc_act=q.desc_act)
            for X, W in zip(Xs, Ws) for q in settings]
    weights = sum(j["W"].shape[0] * j["W"].shape[1] for j in jobs)
    widths = {}
    for W in Ws:
        widths[W.shape[1]] = max(widths.get(W.shape[1], 0), W.shape[0])
    # output buffers allocated once, outside the timing
    _, outs = G._jobs(jobs, dev)
    for j, o in zip(jobs, outs):
        j["out"] = o
    # contexts of both arms created before the timing
    pipe = G.Pipeline(widths, local_rank, stream)
    ctxs = {n_: G.GPTQContext(n_, m_, local_rank, stream) for n_, m_ in widths.items()}

    def sequential():
        for X, W in zip(Xs, Ws):
            ctx = ctxs[W.shape[1]]
            ctx.reset()
            ctx.accumulate_hessian(X)
            for damp in (0.01, 0.1):
                ctx.prepare(damp, True)
                for q in settings:
                    if q.damp == damp:
                        ctx.quantize_layer(W, q.bits, q.group_size, q.sym, want_w_hat=False)
        for c in ctxs.values():
            c.synchronize()

    def timed(fn, k, w):
        for _ in range(w):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / k

    clocks = ClockSampler(local_rank)
    clocks.start()
    ms = timed(lambda: pipe.run(jobs), args.steps, args.warmup)
    clk = clocks.stop()
    ms_seq = timed(sequential, max(1, args.steps // 2), 1)
    pipe.close()
    for c in ctxs.values():
        c.close()
    line = {
        "metric": METRIC, "value": weights / (ms / 1e3) / 1e9, "unit": "Gweights/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16->f32", "data": "synthetic",
        "config": {"workload": "block7b: q,k,v,o 4096x4096, gate,up 11008x4096, down 4096x11008; 65536 tokens "
                               "each; 18 settings (bits 2/3/4 x group 64/128/per-channel x damp 0.01/0.1)",
                   "jobs": len(jobs), "factorizations": 14, "hessians": 7},
        "sequential_ms_per_step": ms_seq, "pipeline_speedup": ms_seq / ms, "clocks": clk,
    }
    print(json.dumps(line), flush=True)


AWQ_CONFIG = "awq_q_proj_4096x4096"
SEQ_CONFIG = "sequential_mlp_4096_11008"


def _median_call_ms(fn, stream, dev, steps, warmup, flush):
    """Median of `steps` single calls of fn, each bracketed by CUDA events on the launching stream
    after `warmup` untimed calls, with L2 flushed (a 256 MB write) before every call."""
    import torch
    ms = []
    for r in range(warmup + steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if r >= warmup:
            ms.append(e0.elapsed_time(e1))
    return statistics.median(ms)


def run_awq(args, rank, world, local_rank):
    """AWQ channel scaling plus round-to-nearest on the q_proj recipe (W 4096 x 4096, 65536
    calibration tokens of X, 0.5 GB: larger than L2), 4-bit asymmetric groups of 128; and the
    round-to-nearest quantizer alone on the same W, with and without the clipped range (the
    page's INT8 per-channel symmetric quantizer with clip ratio 0.99, and 4-bit groups).  Each
    call is timed alone after an L2 flush; HBM-bound: algorithmic bytes over the call's time."""
    import torch
    from post_weight_quantization_16_b200 import build as B
    from post_weight_quantization_16_b200 import gptq as G
    B.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    layer0, qs = synth.WORKLOADS["q_proj_4096x4096"]
    layer = synth.scaled_layer(layer0, n_tok=65536, name=AWQ_CONFIG)
    peaks, _ = load_peaks()
    X = torch.from_numpy(synth.make_x_bf16(layer).view(np.int16)).to(dev).view(torch.bfloat16)
    W = torch.from_numpy(synth.make_w_fp16(layer)).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    m, n, N = layer.m, layer.n, layer.n_tok
    res = {}
    out = {}

    def awq():
        out["awq"] = G.awq_quantize(X, W, 2.0, qs.bits, qs.group_size, qs.sym, want_w_hat=False, stream=stream)

    clocks = ClockSampler(local_rank)
    clocks.start()
    t_awq = _median_call_ms(awq, stream, dev, args.steps, args.warmup, flush)
    # the same call without calibration tokens skips only the channel sums: the difference is their time
    t_awq_no_x = _median_call_ms(lambda: G.awq_quantize(None, W, 2.0, qs.bits, qs.group_size, qs.sym, want_w_hat=False,
                                                        stream=stream), stream, dev, args.steps, args.warmup, flush)
    G_ = n // qs.group_size
    b_awq = 2 * N * n + 2 * m * n + m * n * qs.bits / 8 + 8 * m * G_ + 4 * n
    scale = out["awq"]["channel_scale"]
    for name, bits, g, sym, clip, sc in (("rtn_awq_scaled_4bit_g128_asym", 4, 128, False, 1.0, scale),
                                         ("rtn_4bit_g128_asym_clip0.99", 4, 128, False, 0.99, None),
                                         ("rtn_8bit_per_channel_sym_clip0.99", 8, -1, True, 0.99, None),
                                         ("rtn_8bit_per_channel_sym", 8, -1, True, 1.0, None)):
        t = _median_call_ms(lambda: G.rtn_quantize(W, bits, g, sym, clip, channel_scale=sc, want_w_hat=False,
                                                   stream=stream), stream, dev, args.steps, args.warmup, flush)
        gg = n if g == -1 else g
        byts = 2 * m * n + m * n * bits / 8 + 8 * m * (n // gg) + (4 * n if sc is not None else 0)
        ach = byts / (t / 1e3) / 1e9
        res[name] = {"ms": t, "algorithmic_bytes": byts, "achieved_gbs": ach, "frac_hbm": ach / peaks["hbm_gbs"]}
    clk = clocks.stop()
    ach = b_awq / (t_awq / 1e3) / 1e9
    line = {
        "metric": "AWQ layer quant (channel scaling + round-to-nearest): Gweights/s, 1xB200",
        "value": m * n / (t_awq / 1e3) / 1e9, "unit": "Gweights/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_awq, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": AWQ_CONFIG + ", 65536 tokens", "m": m, "n": n, "n_tok": N, "bits": qs.bits,
                   "group_size": qs.group_size, "sym": qs.sym, "s_protect": 2.0,
                   "l2": "flushed before every call (256 MB write)"},
        "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": ach / peaks["hbm_gbs"], "algorithmic_bytes": b_awq, "traffic": None},
        "rtn": res, "clocks": clk,
        "split": {"ms_without_tokens": t_awq_no_x, "channel_sums_ms": t_awq - t_awq_no_x,
                  "channel_sums_gbs": 2 * N * n / ((t_awq - t_awq_no_x) / 1e3) / 1e9 if t_awq > t_awq_no_x else None},
    }
    print(json.dumps(line), flush=True)


def run_sequential(args, rank, world, local_rank):
    """Sequential quantization of the 7B-shaped MLP pair (up 11008 x 4096, ReLU, down 4096 x 11008)
    through gptq.quantize_sequential: layer 0 calibrated on 65536 tokens of the block recipe, layer
    1 on ReLU of layer 0's product with its own quantized weights; 4-bit asymmetric groups of 128,
    damp 0.01, act-order.  One step = the whole stack through the public call, with its contexts
    kept between steps; the same with contexts created and closed in every step is reported beside
    it.  Inputs resident before timing; the intermediate activations (1.4 GB) exceed L2."""
    import torch
    from post_weight_quantization_16_b200 import build as B
    from post_weight_quantization_16_b200 import gptq as G
    B.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    up, _ = synth.WORKLOADS["block7b_up_11008x4096"]
    down, _ = synth.WORKLOADS["block7b_down_4096x11008"]
    qs = synth.QuantSetting(4, 128, False, 0.01, True)
    peaks, _ = load_peaks()
    X0 = torch.from_numpy(synth.make_x_bf16(up).view(np.int16)).to(dev).view(torch.bfloat16)
    Ws = [torch.from_numpy(synth.make_w_fp16(L)).to(dev) for L in (up, down)]
    layers = [dict(W=W, bits=qs.bits, group_size=qs.group_size, sym=qs.sym, damp=qs.damp, desc_act=qs.desc_act)
              for W in Ws]

    ctxs = {}

    def step(keep):
        res = G.quantize_sequential(X0, layers, act=1, stream=stream, contexts=ctxs if keep else None)
        torch.cuda.synchronize(dev)
        return res

    def timed(keep):
        for _ in range(args.warmup):
            step(keep)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step(keep)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    clocks = ClockSampler(local_rank)
    clocks.start()
    ms = timed(True)              # contexts created in the warm-up and kept between steps
    clk = clocks.stop()
    ms_fresh = timed(False)       # every step creates and closes its contexts
    G.close_contexts(ctxs)
    N = up.n_tok
    # lower bound: every contraction at the bf16 peak (each layer's solve, and layer 0's product)
    peak = choose_peak(peaks, ms / 1e3 * args.steps, clk)[0]
    t_roof = 0.0
    flops = 0.0
    for L in (up, down):
        Lr = synth.scaled_layer(L, n_tok=N)
        t_bf16, _, parts = path_rooflines(Lr, qs, peak, peaks["hbm_gbs"])
        t_roof += t_bf16
        flops += parts["hessian"] + parts["factorization"] + parts["trailing"]
    f_prod = 2.0 * N * up.m * up.n
    t_roof += f_prod / (peak * 1e12)
    weights = sum(L.m * L.n for L in (up, down))
    line = {
        "metric": "Sequential quantization of an MLP pair: Gweights/s, 1xB200",
        "value": weights / (ms / 1e3) / 1e9, "unit": "Gweights/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16->f32", "data": "synthetic",
        "config": {"workload": SEQ_CONFIG + ": up 11008x4096 -> ReLU -> down 4096x11008, 65536 tokens",
                   "bits": qs.bits, "group_size": qs.group_size, "sym": qs.sym, "damp": qs.damp,
                   "desc_act": qs.desc_act, "l2": "inputs and activations larger than L2"},
        "path_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms, "peak_bf16_tflops": peak,
                          "flops": flops + f_prod},
        "contexts": "kept between steps (created during warm-up)",
        "ms_per_step_contexts_created_each_step": ms_fresh,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=WORKLOAD, choices=sorted(synth.WORKLOADS) + ["block7b", AWQ_CONFIG, SEQ_CONFIG])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the separate host-buffer end-to-end measurement")
    ap.add_argument("--no-w4a16", action="store_true", help="skip the dequantizing product on the layer's output")
    args = ap.parse_args()
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        if args.config == "block7b":
            args.config = "block7b_q_4096x4096"
        run_reference(args, rank, world)
        return
    if args.config == "block7b":
        run_block(args, rank, world, local_rank)
        return
    if args.config == AWQ_CONFIG:
        run_awq(args, rank, world, local_rank)
        return
    if args.config == SEQ_CONFIG:
        run_sequential(args, rank, world, local_rank)
        return
    run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
