"""Host-side pieces of bench.py on the CPU: the traffic record's source check, the clock
sampler's parsing, the oracle baseline and the reference arm's JSON line."""
import argparse
import json
import threading

import bench
from post_weight_quantization_16_b200 import synth


def test_profiled_traffic_gated_by_sources(monkeypatch):
    (kernel, rec), = bench.PROFILED_TRAFFIC.items()
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
    r2 = bench.cpu_oracle_baseline(layer, qs, tok_sample=256, row_sample=16, prep_n=256)
    assert r2["value"] > 0 and "256 of 512 columns" in r2["sample"]


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
