"""Host logic of bench.py that needs no GPU: the clock sampler keeps only the samples
stamped inside the timed region and reports their median SM clock and every throttle
reason seen there (nvidia-smi's CSV replaced by a written file)."""
import datetime
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _row(t, mhz, active):
    ts = t.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    reasons = ", ".join("Active" if a else "Not Active" for a in active)
    return f"{ts}, {mhz}, 1965, 700.00, 0x0000000000000000, {reasons}"


def test_clock_sampler_summarises_the_timed_region_only(tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    t = datetime.datetime(2026, 1, 1, 12, 0, 0)
    sec = lambda s: t + datetime.timedelta(seconds=s)
    rows = [
        _row(sec(0.0), 810, (0, 0, 0, 0)),       # before the timed region (idle clock)
        _row(sec(1.0), 1900, (0, 0, 0, 1)),      # inside: power cap active
        _row(sec(1.1), 1965, (0, 0, 0, 0)),
        _row(sec(1.2), 1950, (0, 0, 0, 0)),
        "garbled line",
        _row(sec(3.0), 600, (1, 0, 0, 0)),       # after: hw_slowdown, must not count
    ]
    cs = bench.ClockSampler(0)
    cs.path = str(tmp_path / "clocks.csv")
    with open(cs.path, "w") as f:
        f.write("\n".join(rows) + "\n")

    class Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0
    cs.proc = Proc()
    cs.t0, cs.t1 = sec(0.5), sec(2.0)
    out = cs.stop()
    assert out["samples_in_timed_region"] == 3
    assert out["sm_mhz"] == 1950.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(cs.path)


def test_clock_sampler_without_nvidia_smi_reports_nothing():
    sys.path.insert(0, ROOT)
    import bench
    cs = bench.ClockSampler(0)
    assert cs.stop() is None


def test_our_arm_prints_every_contract_key(monkeypatch, capsys):
    """bench.py's own line assembly, with the GPU measurements replaced by fixed numbers:
    the JSON line carries every key of the benchmark contract, value is the whole job's
    bytes over the timed milliseconds, and the roofline fraction is achieved / peak."""
    sys.path.insert(0, ROOT)
    import json
    import types
    import bench
    from bit_weight_only_w4_b200 import workloads

    wl = workloads.workload(bench.DECODE_CFG)
    projs = [{"bytes": 1_000_000} for _ in wl.layers]
    step_bytes = bench.N_LAYERS * 4_000_000
    monkeypatch.setattr(bench, "prepare_weights", lambda w4, torch: (wl, projs, step_bytes))
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    monkeypatch.setattr(bench, "time_chain_per_launch", lambda *a, **k: (100.0, clk))
    monkeypatch.setattr(bench, "time_chain_e2e", lambda *a, **k: (200.0, 32768, 98304))
    monkeypatch.setattr(bench, "time_chain", lambda *a, **k: (150.0, None, 10 * 4))
    monkeypatch.setattr(bench, "time_decode", lambda *a, **k: {
        "total_ms": 40.0, "launches": 3 * bench.N_LAYERS * len(projs), "clocks": None,
        "per_layer": {"qkv": 10.0}})
    monkeypatch.setattr(bench, "cpu_oracle_sample", lambda *a, **k: (0.04, 12.0, "stub"))
    monkeypatch.setattr(bench, "threaded_sample", lambda threads: [[None]] * threads)
    monkeypatch.setattr(bench, "cpu_oracle_threads", lambda parts, target_s=8.0: (0.04 * len(parts), 8.0))
    monkeypatch.setattr(bench, "threaded_desc", lambda parts, sec: "stub threads")
    monkeypatch.setattr(bench, "load_peaks", lambda: ({"hbm_gbs": 6000.0, "bf16_tflops": 1600.0}, "measured"))
    import bit_weight_only_w4_b200 as w4
    monkeypatch.setattr(w4, "LIB_PATH", __file__)       # "built": no build attempted
    args = types.SimpleNamespace(steps=10, warmup=3, quick=True, no_cpu=False, gpus=1)
    bench.our_arm(args, 1, 0, 0)
    line = json.loads(capsys.readouterr().out)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert key in line, key
    assert line["value"] == 10 * step_bytes / 0.1 / 1e9
    assert line["ms_per_step"] == 10.0
    r = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in r, key
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - r["achieved"] / 6000.0) < 1e-12
    e = line["e2e"]
    assert e["h2d_bytes_per_step"] == 32768 and e["d2h_bytes_per_step"] == 98304
    assert e["value"] == 10 * step_bytes / 0.2 / 1e9
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == 0.04 * cb["cores"]
    assert cb["single_thread"]["cores"] == 1 and "cpu_model" in cb and cb["nproc"] >= 1
    assert line["gpu_launches"] == 10 * bench.N_LAYERS * 4
    assert line["step_layer_sequence"]["ms_per_step"] == 15.0
    assert "workload" in line["config"]
