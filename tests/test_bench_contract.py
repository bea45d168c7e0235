"""The bench line's contract, checked on the CPU through the reference arm (the fp64
oracle on a bounded sample): one JSON line with every key of the bench contract, the same
metric and workload as the GPU arm, and the reference-arm extras (impl, cpu_baseline,
an e2e object with zero host<->device bytes)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line_has_the_contract_keys():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    sys.path.insert(0, ROOT)
    import bench
    assert d["metric"] == bench.METRIC and d["impl"] == "reference"
    assert d["config"]["workload"] == bench.DEFAULT_WORKLOAD
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["n_gpus"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_clock_summary_keeps_the_timed_window_only():
    """The bench's clock record: samples outside the timed region (the idle lead-in, the
    work after it) change neither the median clock nor the throttle reasons."""
    import datetime
    import bench

    base = datetime.datetime(2026, 12, 2, 12, 0, 0)

    def line(dt_ms, sm, power, hw="Not Active", cap="Not Active"):
        ts = (base + datetime.timedelta(milliseconds=dt_ms)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, 0, {sm}, 1965, {power}, 0x0, {hw}, Not Active, Not Active, {cap}\n"

    lines = [line(0, 345, 120.0, hw="Active"),         # idle lead-in, outside the window
             line(100, 1800, 700.0, cap="Active"),
             line(150, 1900, 720.0),
             line(200, 1850, 710.0),
             "garbage line\n",
             line(400, 1965, 150.0, hw="Active")]       # after the window
    t0 = (base + datetime.timedelta(milliseconds=90)).timestamp()
    t1 = (base + datetime.timedelta(milliseconds=210)).timestamp()
    c = bench.summarize_clocks(lines, t0, t1)
    assert c["samples"] == 3 and c["window"] == "timed region"
    assert c["sm_mhz"] == 1850.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert c["power_w_max"] == 720.0

    # a region shorter than the sampling interval: the nearest samples stand in, labelled
    t0 = (base + datetime.timedelta(milliseconds=120)).timestamp()
    t1 = (base + datetime.timedelta(milliseconds=130)).timestamp()
    c = bench.summarize_clocks(lines, t0, t1)
    assert c["samples"] == 2 and c["window"].startswith("nearest")
    assert bench.summarize_clocks(["nothing parseable\n"], t0, t1)["samples"] == 0


def test_traffic_record_follows_its_kernel_sources(tmp_path, monkeypatch):
    """A DRAM-traffic record is reported only while the sources its kernel is built from
    hash to the record's sha1; a change to another kernel's source leaves it valid."""
    import shutil
    import bench

    csrc = os.path.join(ROOT, "long_context_attention_fwd_b200", "csrc")
    root = tmp_path / "repo"
    (root / "long_context_attention_fwd_b200").mkdir(parents=True)
    shutil.copytree(csrc, root / "long_context_attention_fwd_b200" / "csrc")
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    wl = "some_workload"
    rec = {"workloads": {wl: {k: {"dram_bytes_per_launch": 1000 + i, "sources_sha1": bench.kernel_sources_sha1(k)}
                              for i, k in enumerate(bench.KERNEL_SOURCES)}}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.measured_traffic(wl, "attn_bwd_kernel") == 1001
    assert bench.measured_traffic(wl, "attn_fwd_kernel") == 1000
    assert bench.measured_traffic("other_workload", "attn_bwd_kernel") is None
    # edit the forward's own header: its record goes stale, the backward's stays
    fwd = root / "long_context_attention_fwd_b200" / "csrc" / "attn_fwd.cuh"
    fwd.write_text(fwd.read_text() + "\n// edited\n")
    assert bench.measured_traffic(wl, "attn_fwd_kernel") is None
    assert bench.measured_traffic(wl, "attn_bwd_kernel") == 1001
    # a shared header invalidates both
    ptx = root / "long_context_attention_fwd_b200" / "csrc" / "sm100_ptx.cuh"
    ptx.write_text(ptx.read_text() + "\n// edited\n")
    assert bench.measured_traffic(wl, "attn_bwd_kernel") is None

