"""The benchmark's reference arm on CPU: the timed fp64 oracle on a bounded sample prints the one
JSON line of the contract (rank 0 only; any other rank exits 0 without work or output)."""
import hashlib
import json
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env):
    env = dict(os.environ, **extra_env)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "c1",
                           "--steps", "1", "--warmup", "3", "--cpu-seconds", "1"],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_one_contract_line():
    res = _run({"RANK": "0"})
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"].startswith("c1")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    res = _run({"RANK": "1"})
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == ""


def test_clock_summary_reports_median_max_and_active_reasons():
    sys.path.insert(0, ROOT)
    import bench
    lines = [
        "1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1800, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1700, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "[N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",   # unreadable sample
        "short line",
    ]
    s = bench.ClockSampler.summarize(lines)
    assert s == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    hot = lines[:1] + ["1200, 1965, 800, 0x8, Active, Not Active, Active, Not Active"]
    assert bench.ClockSampler.summarize(hot)["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.ClockSampler.summarize([]) is None


def test_traffic_figure_is_dropped_once_the_kernel_changes(monkeypatch):
    # the committed DRAM bytes per launch belong to one version of the forward kernel's source
    sys.path.insert(0, ROOT)
    import bench
    w = "c3_llama3_8b_gqa_L212992_N16"
    with open(os.path.join(ROOT, "profiles", "ring_fwd_kernel_traffic.json")) as f:
        rec = json.load(f)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["kernel_source_hash"])
    assert bench.traffic_from_profile(w) == rec["per_launch_bytes"][w]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.traffic_from_profile(w) is None


def _csrc_hash(files):
    """First 16 hex digits of sha256 over the kernel sources' bytes, in the order given."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "sequence_long_context_ring_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def test_every_profile_summary_matches_the_current_kernel_source():
    """Each ncu summary under profiles/ names the kernel sources it was captured from, with a
    hash of their bytes; once any of them changes, the summary is stale and must be captured
    again (and this test fails until it is)."""
    line = re.compile(r"^Source hash: ([0-9a-f]{16}) over (.+?)\s*$", re.M)
    pdir = os.path.join(ROOT, "profiles")
    names = sorted(f for f in os.listdir(pdir) if f.endswith(".md"))
    assert names, "no ncu summaries"
    for fn in names:
        with open(os.path.join(pdir, fn)) as fh:
            m = line.search(fh.read())
        assert m, f"{fn}: no 'Source hash: <hex> over <files>' line"
        files = [x.strip() for x in m.group(2).split(",")]
        assert _csrc_hash(files) == m.group(1), f"{fn}: captured from kernel sources that have changed since"
    with open(os.path.join(pdir, "ring_fwd_kernel_traffic.json")) as fh:
        d = json.load(fh)
    assert d["kernel_source_hash"] == _csrc_hash(["fwd_kernel.cuh", "sm100.cuh"]), "traffic figure is stale"
