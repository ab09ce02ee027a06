"""bench.py's default JSON line carries every key of the benchmark contract,
with the roofline and throughput figures derived as stated.  The GPU work is
replaced by fakes (the decode run returns a result of the shape it produces;
the secondary measurements and the oracle timing return fixed values), so
main() assembles and prints the line on the CPU."""
import json
import sys

import pytest

import bench

STACK_BYTES = 601_620_480.0          # 40 layers x 9 units x 1,671,168 B at batch 1


def fake_decode(args, world, rank):
    assert world == 1 and args.tokens in (1, 4) and args.format in ("mxfp4", "nvfp4", "bf16")
    us = 316.0
    return dict(ms=args.steps * 0.3238, tok_s=1e3 / 0.3238, hbm_gbs=1858.0, step_bytes=STACK_BYTES,
                launches=2 * args.steps, clocks={"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [], "samples": 40},
                kernels={"dec_stack": {"ms_total": us * args.steps / 1e3, "launches": args.steps, "us_avg": us},
                         "route": {"ms_total": 0.0109 * args.steps, "launches": args.steps, "us_avg": 10.9}},
                kernel_steps=args.steps, gate_up_bytes=0.0, down_bytes=0.0, stack_bytes=STACK_BYTES,
                e2e={"value": 2927.0, "unit": "tok/s", "h2d_bytes_per_step": 45056, "d2h_bytes_per_step": 4096})


@pytest.fixture
def line(monkeypatch, capsys):
    monkeypatch.setattr(bench, "dist_setup", lambda args: (1, 0, 0))
    monkeypatch.setattr(bench, "run_ours", fake_decode)
    monkeypatch.setattr(bench, "measure_prefill", lambda: {"workload": "prefill"})
    monkeypatch.setattr(bench, "measure_misses", lambda: {"workload": "miss"})
    monkeypatch.setattr(bench, "measure_glm", lambda: {"decode": {}, "prefill": {}})
    monkeypatch.setattr(bench, "measure_decode_dsv4", lambda pk: {"workload": "dsv4"})
    monkeypatch.setattr(bench, "oracle_tok_s", lambda T, threads: (0.22 if threads > 1 else 0.05, 12))
    monkeypatch.setattr(bench, "host_cores", lambda: 16)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "10", "--warmup", "3"])
    bench.main()
    out = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(out) == 1
    return json.loads(out[0])


def test_contract_keys(line):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["metric"] == bench.METRIC and line["unit"] == "tok/s" and line["higher_is_better"] is True
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 10, 3)
    assert line["scaling"] == "weak" and line["vs_baseline"] is None and line["data"] == "synthetic"
    assert "workload" in line["config"] and "model" not in line["config"]
    assert set(line["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    assert set(line["cpu_baseline"]) >= {"value", "unit", "cores", "kind", "sample"}
    assert set(line["e2e"]) == {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert set(line["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    assert line["prefill"] == {"workload": "prefill"} and line["miss"] == {"workload": "miss"}
    b4 = line["decode_batch4"]
    assert "batch 4" in b4["workload"] and b4["tok_s"] > 0 and 0 < b4["kernel_frac"] < 1.5
    fm = line["decode_formats"]
    assert set(fm) == {"nvfp4", "bf16"} and "NVFP4" in fm["nvfp4"]["workload"] and "BF16" in fm["bf16"]["workload"]
    assert "MXFP4" in line["config"]["workload"]


def test_derived_figures(line):
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["kernel"] == "dec_stack"
    assert r["achieved"] == pytest.approx(STACK_BYTES / 316e-6 / 1e9)       # algorithmic bytes / launch time
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert r["traffic"] == pytest.approx(bench.STACK_TRAFFIC_PER_BYTE * STACK_BYTES)
    assert line["ms_per_step"] == pytest.approx(0.3238)
    assert line["value"] == pytest.approx(1e3 / 0.3238)
    assert line["gpu_launches"] == 20
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 16
    assert line["cpu_baseline"]["value"] == 0.22 and line["cpu_baseline"]["single_thread"]["value"] == 0.05


def test_layerwise_line_reports_the_gate_up_kernel(monkeypatch, capsys):
    gu_bytes = 9 * 1_114_112.0                      # Wg + Wu codes and scales of 9 units

    def fake(args, world, rank):
        r = fake_decode(args, world, rank)
        r["kernels"] = {"gate_up": {"ms_total": 0.0136 * 40 * args.steps, "launches": 40 * args.steps, "us_avg": 13.6},
                        "down_combine": {"ms_total": 0.0136 * 40 * args.steps, "launches": 40 * args.steps,
                                         "us_avg": 13.6}}
        r["gate_up_bytes"], r["down_bytes"] = gu_bytes, gu_bytes / 2
        return r
    monkeypatch.setattr(bench, "dist_setup", lambda args: (1, 0, 0))
    monkeypatch.setattr(bench, "run_ours", fake)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "4", "--warmup", "3", "--layerwise", "--no-extra"])
    monkeypatch.setattr(bench, "oracle_tok_s", lambda T, threads: (0.22 if threads > 1 else 0.05, 12))
    bench.main()
    line = json.loads([ln for ln in capsys.readouterr().out.splitlines() if ln.strip()][0])
    r = line["roofline"]
    assert r["kernel"] == "gate_up" and r["traffic"] is None
    assert r["achieved"] == pytest.approx(gu_bytes / 13.6e-6 / 1e9)
    assert line["gate_up_gbs"] == pytest.approx(r["achieved"])
    assert "prefill" not in line and "miss" not in line
    assert line["config"]["decode_kernels"] == "two per layer"
