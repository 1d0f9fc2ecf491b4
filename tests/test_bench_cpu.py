"""The reference arm of ``bench.py`` (the float64 oracle on the host cores): its JSON line
carries the fields the measurement contract names, and only rank 0 of a multi-rank launch
prints it (the other ranks exit 0 without work).  No GPU involved."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env, *args):
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env.update(extra_env)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def _line(out):
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out
    return json.loads(lines[0])


def test_reference_arm_line():
    p = _run({}, "--config", "1", "--steps", "1", "--warmup", "3")
    assert p.returncode == 0, p.stderr
    d = _line(p.stdout)
    assert d["impl"] == "reference" and d["value"] > 0 and d["ms_per_step"] > 0
    for k in ("metric", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "vs_baseline",
              "dtype", "data", "config"):
        assert k in d, k
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"].startswith("config 1")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_on_rank_zero_only():
    p1 = _run({"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}, "--config", "1", "--steps", "1",
              "--warmup", "3")
    assert p1.returncode == 0, p1.stderr
    assert not [l for l in p1.stdout.splitlines() if l.startswith("{")]
    p0 = _run({"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"}, "--config", "1", "--steps", "1",
              "--warmup", "3")
    assert p0.returncode == 0, p0.stderr
    assert _line(p0.stdout)["n_gpus"] == 2


def test_peak_choice_follows_the_sampled_clock():
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16": 1700.0, "bf16_sust": 1390.0, "sm_max_mhz": 1965.0}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    slow = {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.pick_tc_peak(peaks, at_max) == (1700.0, "burst")
    assert bench.pick_tc_peak(peaks, capped) == (1390.0, "sustained")
    assert bench.pick_tc_peak(peaks, slow) == (1390.0, "sustained")
    assert bench.pick_tc_peak(peaks, {"sm_mhz": None, "reasons": []}) == (1390.0, "sustained")


def test_level_kernel_bytes_by_hand():
    # one level step 8 -> 16 with 10 refined parents: mark reads 4*512 and writes 64 bytes;
    # scan/list read the 64-byte mask twice, write 12*(2^3) and 4*10; the fill reads 4*512 + 64
    # and writes 4*(8*512 - 80)
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    cfg = W.CONFIGS[3].with_(r0=8, n_levels=2)
    st = [{"active_parents": [0, 10]}]
    b = bench.level_kernel_bytes(cfg, st)
    assert b["mark"] == 2048 + 64
    assert b["scan_list"] == 128 + 96 + 40
    assert b["fill"] == 2048 + 64 + 4 * (4096 - 80)
