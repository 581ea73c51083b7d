"""bench.py on the CPU: the reference arm's JSON line (the oracle timed on the
host cores), what the other ranks of a multi-rank launch do there, the
argument guards, and the small helpers the GPU arm's line is built from."""

import json

import pytest

import bench


def _line(capsys, argv):
    assert bench.main(argv) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1, lines
    return json.loads(lines[0])


def test_reference_arm_prints_one_complete_line(capsys, monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    out = _line(capsys, ["--impl", "reference", "--workload", "cfg1", "--steps", "2", "--warmup", "3",
                         "--cpu-budget", "1"])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference" and out["metric"] == bench.METRIC and out["unit"] == bench.UNIT
    assert out["steps"] == 2 and out["warmup"] == 3 and out["n_gpus"] == 1
    assert out["value"] > 0 and out["higher_is_better"] is True
    assert out["config"]["workload"] == bench.workload_spec("cfg1").name
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == out["value"] and cb["cores"] >= 1 and cb["sample"]
    assert out["e2e"] == {"value": out["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3"]) == 0
    assert capsys.readouterr().out.strip() == ""


def test_argument_guards(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--warmup", "2"])  # fewer than 3 warm-up steps
    monkeypatch.setenv("WORLD_SIZE", "4")
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--gpus", "2", "--warmup", "3"])  # launch and flag disagree
    with pytest.raises(SystemExit):
        bench.workload_spec("no_such_workload")


def test_line_helpers():
    spec = bench.workload_spec("cfg2")
    fp4, lowrank = bench.layer_flops(spec, 32)
    assert fp4 == 2 * 4096 * 3072 * 3072
    assert lowrank == 2 * 4096 * 3072 * 32 * 2
    assert bench.aggregate(5.0, 4, 2.0) == 10.0
    assert bench.qkv_shape(9216) and not bench.qkv_shape(3072 + 64)
    assert bench.rank_seed(1, 0) == 1 and bench.rank_seed(1, 3) != bench.rank_seed(1, 2)
    peak, hbm, origin = bench.measured_peaks()
    assert peak > 0 and hbm > 0 and origin in ("measured", "fallback")
    # traffic is taken from a committed ncu summary only for the workload it was captured on
    assert bench.profiled_traffic("gemm_kernel", "some_other_workload") is None
    t = bench.profiled_traffic("gemm_kernel", "attn_proj_M4096_K3072_N3072_r32")
    assert t is None or t > 0


def test_measured_peaks_fall_back_per_value(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (1590.0, 6650.0, "fallback")  # no file
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6551.0, "bf16_tflops": 1666.4}')
    assert bench.measured_peaks() == (1666.4, 6551.0, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6551.0, "bf16_tflops": null}')
    assert bench.measured_peaks() == (1590.0, 6551.0, "measured, fallback for bf16_tflops")
    (tmp_path / "MEASURED_PEAKS.json").write_text("not json")
    assert bench.measured_peaks() == (1590.0, 6650.0, "fallback")


def test_sustained_peak_and_power_cap_rule(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.sustained_bf16_peak() == (1400.0, "fallback")  # no file
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"bf16_tflops": 1666.4, "bf16_tflops_sustained": 1363.8}')
    assert bench.sustained_bf16_peak() == (1363.8, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text("[]")
    assert bench.sustained_bf16_peak() == (1400.0, "fallback")
    # the sustained peak applies only when the power cap held the median clock below its maximum
    assert bench.power_capped({"sm_mhz": 1893.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    assert not bench.power_capped({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    assert not bench.power_capped({"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": []})
    assert not bench.power_capped({})


def test_clock_summary_keeps_the_benchmarked_gpu_under_load():
    c = bench.ClockSampler(uuid="GPU-bbbb")
    c.lines = [
        "GPU-aaaa, 1965, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, Active",
        "GPU-bbbb, 345, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active",  # idle: below the floor
        "GPU-bbbb, 1965, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "GPU-bbbb, 1905, 1965, 1000.0, 0x4, Not Active, Not Active, Not Active, Active",
        "GPU-bbbb, 1935, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1935.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 4 and s["samples_under_load"] == 3
    empty = bench.ClockSampler().summary()
    assert empty["sm_mhz"] is None and empty["samples"] == 0
