"""Host-side pieces of bench.py on the CPU: the traffic record's source check, the clock
sampler's parsing, the oracle baseline and the reference arm's JSON line."""
import argparse
import json
import threading

import bench
from post_weight_quantization_16_b200 import synth


def test_profiled_traffic_gated_by_sources(monkeypatch):
    (kernel, rec), = bench.PROFILED_TRAFFIC.items()
    fresh = dict(rec, sources={p: bench._sha1(p) for p in rec["sources"]})   # as if captured from these sources
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, kernel, fresh)
    v = bench.profiled_traffic(kernel, rec["n"], rec["tokens"] * 4)
    assert v is not None and abs(v - 4 * rec["dram_bytes"]) < 1e-3 * v  # scaled per token
    assert bench.profiled_traffic("no_such_kernel", rec["n"], 1) is None
    assert bench.profiled_traffic(kernel, rec["n"] + 128, 1) is None
    stale = dict(rec, sources={p: "0" * 40 for p in rec["sources"]})
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, kernel, stale)
    assert bench.profiled_traffic(kernel, rec["n"], rec["tokens"]) is None  # edited kernel: no number


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_sampler_parses_reasons():
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.t = threading.Thread(target=lambda: None)
    s.t.start()
    s.lines = ["1965, 1965, 900.1, 0x0, Not Active, Not Active, Not Active, Not Active",
               "1890, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
               "garbage", "1900, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active"]
    out = s.stop()
    assert out == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_cpu_oracle_baseline_on_tiny_layer():
    layer, qs = synth.WORKLOADS["tiny_256x512"]
    r = bench.cpu_oracle_baseline(layer, qs, tok_sample=512, row_sample=32)
    assert r["value"] > 0 and r["kind"] == "oracle" and r["cores"] >= 1
    assert set(r["stage_seconds"]) == {"hessian", "prepare", "sweep"}
    r2 = bench.cpu_oracle_baseline(layer, qs, tok_sample=256, row_sample=16, col_sample=256)
    assert r2["value"] > 0 and "leading 256 of 512 columns" in r2["sample"]
    # a wide layer stays bounded: only the leading columns are generated and timed
    big, bq = synth.WORKLOADS["down_proj_8192x28672"]
    r3 = bench.cpu_oracle_baseline(big, bq, tok_sample=256, row_sample=8, col_sample=256)
    assert r3["value"] > 0 and r3["seconds_per_layer"] > r2["seconds_per_layer"]


def test_reference_arm_line(capsys):
    args = argparse.Namespace(config="tiny_256x512", steps=2, warmup=1, gpus=1)
    bench.run_reference(args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0 and line["config"]["workload"] == "tiny_256x512"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    bench.run_reference(args, 1, 2)  # other ranks do nothing
    assert capsys.readouterr().out == ""


def test_peak_choice_follows_the_clocks():
    peaks = {"bf16_tflops": 1644.2, "bf16_tflops_sustained": 1385.2, "hbm_gbs": 6468.0}
    capped = {"sm_mhz": 1440.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.choose_peak(peaks, 4.4, capped)[:2] == (1385.2, "sustained")
    assert bench.choose_peak(peaks, 0.15, capped)[:2] == (1644.2, "burst")     # too short
    assert bench.choose_peak(peaks, 4.4, full)[:2] == (1644.2, "burst")        # not capped
    assert bench.choose_peak(peaks, 4.4, None)[:2] == (1644.2, "burst")


def test_dominant_kernel_folds_roles():
    prof = {"gemm_tf32x3:factor": {"launches": 10, "ms": 50.0, "flops": 1e13, "bytes": 0.0},
            "gemm_tf32x3:trailing": {"launches": 20, "ms": 30.0, "flops": 5e12, "bytes": 0.0},
            "hessian_syrk_pair": {"launches": 1, "ms": 45.0, "flops": 5e13, "bytes": 4e9},
            "sweep_block": {"launches": 224, "ms": 10.0, "flops": 0.0, "bytes": 3e9}}
    name, k = bench.dominant_kernel(prof)
    assert name == "gemm_tf32x3" and k["ms"] == 80.0 and k["launches"] == 30 and k["flops"] == 1.5e13
    assert sorted(k["roles"]) == ["gemm_tf32x3:factor", "gemm_tf32x3:trailing"]


def test_path_rooflines_of_the_q_proj_layer():
    layer, qs = synth.WORKLOADS["q_proj_4096x4096"]
    t_bf16, t_prec, work = bench.path_rooflines(layer, qs, 1644.2, 6468.0)
    assert abs(work["hessian"] - 4.399e12) / 4.399e12 < 1e-3
    assert abs(t_bf16 * 1e3 - 2.74) < 0.01          # every product at the bf16 peak
    assert t_prec > t_bf16                            # fp32-faithful products at the tf32 rate / 3
