"""bench.py's reference arm on CPU: one JSON line with the contract's keys.

`bench.py --impl reference` times the oracle on the host cores (it needs no
GPU), so the line it prints can be checked here: the same metric, unit and
direction as the GPU arm, a cpu_baseline block describing the sample, and an
e2e block with no host-device bytes.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    import bench
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert abs(d["value"] - 4 / (d["ms_per_step"] / 1000)) < 1e-6 * d["value"]  # tiny: T = 4
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] and d["config"]["T"] == 4
    assert d["vs_baseline"] is None and d["data"] == "synthetic"


def test_peaks_burst_and_sustained():
    """The roofline denominators come from the measured-peaks file: the burst
    bf16 figure by default, the sustained one for a run that met the power cap."""
    import bench
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    hbm, bf16, src = bench.peaks()
    hbm_s, bf16_s, src_s = bench.peaks(sustained=True)
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        assert (hbm, bf16, src) == (j["hbm_gbs"], j["bf16_tflops"], "measured")
        assert hbm_s == j["hbm_gbs"] and bf16_s == j["bf16_tflops_sustained"] and src_s == "measured sustained"
        assert bf16_s < bf16
    else:
        assert src == "fallback" and src_s == "fallback sustained"


def test_captured_traffic_only_for_its_workload_and_sources(monkeypatch):
    """A recorded DRAM figure is reported for its own workload while the kernel
    sources hash to the recorded value, and never for another workload or after
    a source change."""
    import bench
    import synth
    from dataclasses import replace
    rec = bench.TRAFFIC[0]
    cfg = synth.CONFIGS[rec["config"]]
    T = rec["T"]
    live = bench.sources_sha256(rec["sources"])
    monkeypatch.setitem(rec, "sources_sha256", live)
    assert bench.captured_traffic(replace(cfg, E=rec["E"]), T) == (rec["dram_bytes"], rec["kernels"])
    assert bench.captured_traffic(replace(cfg, E=rec["E"]), T + 1) == (None, None)     # other T
    assert bench.captured_traffic(replace(cfg, E=rec["E"] // 4), T) == (None, None)    # other E
    monkeypatch.setitem(rec, "sources_sha256", "0" * 64)                               # sources changed
    assert bench.captured_traffic(replace(cfg, E=rec["E"]), T) == (None, None)


def test_oracle_thread_count_is_settable():
    """The single-threaded CPU baseline runs the same oracle on one thread."""
    import oracle
    n = oracle.num_threads()
    try:
        assert oracle.set_num_threads(1) == 1 and oracle.num_threads() == 1
    finally:
        oracle.set_num_threads(n)
    assert oracle.num_threads() == n
