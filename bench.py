"""Benchmark of the GPTQ per-layer solve on B200.

One step = the whole hot path for one layer: H = 2 X^T X over the calibration set
(tcgen05), prepare (dead columns, act-order, damping, U = upper-Cholesky(H^-1)), and the
blocked column sweep with its trailing updates, emitting packed codes, scales, zeros,
perm and g_idx.  Workload: the Llama-7B-shaped q_proj layer (W 4096x4096 fp16, X 262144
tokens x 4096 bf16 with 0.5 % outlier channels x30, 4-bit asymmetric, group 128,
damp 0.01, act-order), seeded synthetic data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun each rank quantizes its own independent layer (weak scaling; no collective
on the data path); the timed region is bracketed by barriers and the max over ranks is
reported.  Prints one JSON line on rank 0.
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
WORKLOAD = "q_proj_4096x4096"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernel from one
# ncu capture (profiles/hessian_syrk_pair_kernel__block7b_q_65536tok_x4096.md), valid only while the
# kernel's sources are the ones captured.  The capture ran 65536 tokens; X traffic grows in
# proportion to the tokens, so it is scaled per token to a full launch.
PROFILED_TRAFFIC = {
    "hessian_syrk_pair_kernel": {
        "sources": {"post_weight_quantization_16_b200/csrc/hessian_tc.cuh": "99d3e9d95b42960505710a519acfa15b724aa743",
                    "post_weight_quantization_16_b200/csrc/sm100_ptx.cuh": "fa523347e627c8a77d87a07310da3ca52cf8c71e"},
        "n": 4096, "tokens": 65536, "dram_bytes": 975.479040e6 + 24.431360e6,
    },
}


def profiled_traffic(kernel: str, n: int, n_tok: int):
    import hashlib
    rec = PROFILED_TRAFFIC.get(kernel)
    if rec is None or rec["n"] != n:
        return None
    for path, sha in rec["sources"].items():
        with open(os.path.join(ROOT, path), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != sha:
                return None
    return rec["dram_bytes"] * n_tok / rec["tokens"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


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
def cpu_oracle_baseline(layer, qs, tok_sample=16384, row_sample=256, prep_n=None, data=None):
    """The oracle timed on a bounded sample of the layer, scaled to the whole layer: the Hessian
    on tok_sample tokens (time x n_tok / tok_sample); prepare on the leading prep_n x prep_n
    block of H (time x (n / prep_n)^3; the whole H when prep_n is None) and the sweep of
    row_sample rows over those prep_n columns (time x (m / row_sample) x (n / prep_n)).
    `data` = (X sample, W) generated beforehand, outside the timing."""
    from oracle import gptq_oracle as O
    cores = len(os.sched_getaffinity(0))
    tok_sample = min(tok_sample, layer.n_tok)
    row_sample = min(row_sample, layer.m)
    if data is None:
        data = (synth.bf16_bits_to_f32(synth.make_x_bf16(layer, 0, tok_sample)),
                synth.make_w_fp16(layer).astype(np.float64))
    X, W = data
    t0 = time.perf_counter()
    H = O.hessian(X)
    t_h = (time.perf_counter() - t0) * (layer.n_tok / X.shape[0])
    pn = layer.n if prep_n is None else min(prep_n, layer.n)
    t0 = time.perf_counter()
    prep = O.prepare(H[:pn, :pn], qs.damp, qs.desc_act)
    t_p = (time.perf_counter() - t0) * (layer.n / pn) ** 3
    g = qs.group_size if (qs.group_size != -1 and pn % qs.group_size == 0) else -1
    Wp = W[:row_sample, :pn][:, prep["perm"]]
    t0 = time.perf_counter()
    O.gptq_sweep(Wp, prep["U"], qs.bits, g, bool(qs.sym), block=128)
    t_s = (time.perf_counter() - t0) * (layer.m / row_sample) * (layer.n / pn)
    t_layer = t_h + t_p + t_s
    return {
        "value": layer.m * layer.n / t_layer / 1e9, "unit": "Gweights/s", "cores": cores, "kind": "oracle",
        "sample": (f"Hessian on {X.shape[0]} of {layer.n_tok} tokens (scaled), prepare and sweep on the leading "
                   f"{pn} of {layer.n} columns (scaled by n^3 and n), sweep of {row_sample} of {layer.m} rows "
                   f"(scaled); float64 numpy"),
        "seconds_per_layer": t_layer, "stage_seconds": {"hessian": t_h, "prepare": t_p, "sweep": t_s},
    }


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, timed as it stands, on bounded samples."""
    if rank != 0:
        return
    layer, qs = synth.WORKLOADS[args.config]
    # each step a sample small enough that all warm-up and timed steps end within a few minutes
    n_steps = args.warmup + args.steps
    if n_steps <= 4:
        tok, rows, pn = 4096, 64, None
    elif n_steps <= 20:
        tok, rows, pn = 2048, 32, 2048
    else:
        tok, rows, pn = 1024, 16, 2048
    tok = min(layer.n_tok, max(64, int(tok * min(1.0, (4096 / layer.n) ** 2))))  # its cost grows as n^2
    data = (synth.bf16_bits_to_f32(synth.make_x_bf16(layer, 0, tok)), synth.make_w_fp16(layer).astype(np.float64))
    times = []
    r = None
    for step in range(n_steps):
        r = cpu_oracle_baseline(layer, qs, tok_sample=tok, row_sample=rows, prep_n=pn, data=data)
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

    def step(timing=None):
        nonlocal out
        ctx.reset()
        if timing is not None:
            timing[0].record(stream)
        ctx.accumulate_hessian(X)
        if timing is not None:
            timing[1].record(stream)
        ctx.prepare(qs.damp, qs.desc_act)
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

    # dominant kernel: the tcgen05 Hessian (one launch per step)
    h_ms = statistics.mean(t_h)
    h_flops = layer.n_tok * layer.n * (layer.n + 1)           # algorithmic: upper triangle incl. diagonal
    h_tflops = h_flops / (h_ms / 1e3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    n, m = layer.n, layer.m
    roofline = {"bound": "tensor", "kernel": "hessian_syrk_pair_kernel", "achieved": h_tflops, "peak": peak,
                "unit": "TFLOP/s", "frac": h_tflops / peak, "traffic": profiled_traffic("hessian_syrk_pair_kernel", n, layer.n_tok),
                "peak_source": f"{peaks_src} bf16 dense, sustained", "algorithmic_flops_per_launch": h_flops}

    # whole-path roofline: contraction flops at the bf16 peak vs the sweep's bytes at HBM bandwidth
    f_path = layer.n_tok * n * (n + 1) + 2 * n ** 3 / 3 + 2 * m * sum(128 * (n - i2) for i2 in range(128, n, 128))
    b_sweep = 2 * m * n + 2 * n * (n + 1) + m * n * qs.bits / 8 + 8 * m * n / qs.group_size + 8 * n
    t_roof = max(f_path / (peak * 1e12), b_sweep / (peaks["hbm_gbs"] * 1e9))

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e_ms = None
    if not args.no_e2e:
        Xh = torch.from_numpy(X_host.view(np.int16)).view(torch.bfloat16).pin_memory()
        Wh = torch.from_numpy(W_host).pin_memory()
        e2e_ms = e2e_run(ctx, Xh, Wh, qs, dev, stream, reps=max(1, min(3, args.steps)))
        e2e_ms = max_over_ranks(e2e_ms, world, dev)
    G_ = n // (n if qs.group_size == -1 else qs.group_size)
    d2h = m * n * qs.bits // 8 + 2 * m * G_ * 4 + 2 * n * 4
    h2d = X_host.nbytes + W_host.nbytes

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
            "path_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_step},
            "roofline": roofline,
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


def e2e_run(ctx, Xh, Wh, qs, dev, stream, reps=2, batch_tokens=16384):
    """Host X and W in, packed codes/scales/zeros/perm/g_idx out.  The calibration set is
    copied in batches on a side stream, double-buffered against the Hessian kernel."""
    import torch
    n = ctx.n
    N = Xh.shape[0]
    copy_stream = torch.cuda.Stream(dev)
    bufs = [torch.empty((batch_tokens, n), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    times = []
    for _ in range(reps + 1):
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        copy_stream.wait_event(t0)
        ctx.reset()
        Wd = torch.empty(Wh.shape, dtype=Wh.dtype, device=dev)
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
        out = ctx.quantize_layer(Wd, qs.bits, qs.group_size, bool(qs.sym), want_w_hat=False)
        out = dict(out, perm=perm)
        host = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in out.items() if v is not None}
        for k, v in out.items():
            if v is not None:
                host[k].copy_(v, non_blocking=True)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        times.append(t0.elapsed_time(t1))
    return statistics.mean(times[1:])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the separate host-buffer end-to-end measurement")
    args = ap.parse_args()
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
