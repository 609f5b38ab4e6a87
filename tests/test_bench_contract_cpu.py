"""bench.py's reference arm (the fp64 CPU oracle, timed) runs on a machine without a GPU: its one
JSON line carries the keys and units the benchmark contract asks for."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def reference_line(*extra):
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--ref-seconds", "3", *extra], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("extra,workload", [
    ((), "relu_aux_bias_bf16_4096x4096x4096"),
    (("--workload", "gemm_bias_f16_1024x512x2048"), "gemm_bias_f16_1024x512x2048"),
    (("--shape", "256,256,512,bf16,drelu_bgrad,col,kn"), "custom_bf16_drelu_bgrad_256x256x512_kn"),
])
def test_reference_arm_json_line(extra, workload):
    d = reference_line(*extra)
    assert d["impl"] == "reference"
    assert d["metric"].startswith("fused GEMM+bias(+act) TFLOP/s")
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 2, 1)
    assert d["scaling"] == "weak" and d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"]["workload"] == workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert (e["value"], e["unit"]) == (d["value"], d["unit"])
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_clock_record_covers_the_window_after_a_short_timed_region():
    """A timed region shorter than the sampler's period: the clock block is read over the timed
    region plus the back-to-back window that follows it, and says how many samples each holds."""
    sys.path.insert(0, ROOT)
    import bench
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    # samples every 50 ms from t = 0 to 1 s: idle (1965 MHz) before t = 0.1, loaded (1400 MHz) after
    s.samples = [(0.05 * i, ["ts", "0", "1965" if 0.05 * i < 0.1 else "1400", "1965", "900", "0x4",
                             "Not Active", "Not Active", "Not Active", "Active"]) for i in range(21)]
    flops = 2.0 * 4096 ** 3
    rec = bench.clock_record(s, 0.21, 0.212, (300, 0.6, 0.8), flops * 20, 1500.0)
    assert rec["timed_region"] == {"samples": 0, "value": 1500.0}   # 2 ms between two samples
    assert rec["samples"] >= 10 and rec["sm_mhz"] == 1400.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    w = rec["window"]
    assert w["replays_of_timed_region"] == 300 and w["samples"] >= 10 and w["sm_mhz"] == 1400.0
    assert abs(w["value"] - flops * 20 * 300 / 0.6 / 1e12) < 1e-6
    assert abs(w["value_per_ghz"] - w["value"] / 1.4) < 1e-9
    # without a window the timed region alone is summarised
    assert "window" not in bench.clock_record(s, 0.2, 0.5, None, flops, 1500.0)
