"""bench.py's JSON line carries every key of the measurement contract with
values of the right kind (a short run on the GPU; both arms)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args):
    out = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=900)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_native_line():
    d = _run(["--steps", "100", "--warmup", "3", "--e2e-steps", "3", "--cpu-budget", "1.5"])
    assert d["metric"] and d["unit"] == "GB/s" and d["n_gpus"] == 1
    assert d["steps"] == 100 and d["warmup"] == 3 and d["ms_per_step"] > 0
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == "bf16" and d["data"] == "synthetic"
    assert d["config"]["workload"] == "h3_transport_step_T32768_W6"
    assert d["value"] > 1000.0
    n = d["pct_of_nominal_peak"]
    assert n["peak_gbs"] == 8000.0 and abs(n["value"] - 100.0 * d["value"] / 8000.0) < 0.01
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] > 0 and r["achieved"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    assert r["traffic"] is None or r["traffic"] > 0.9 * r["algorithmic_bytes_per_launch"]
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["sample"]
    assert c["unit"] == d["unit"]
    assert c["one_core"]["cores"] == 1 and c["one_core"]["value"] > 0
    assert isinstance(c["cpu_model"], str) and c["cpu_model"]
    e = d["e2e"]
    assert e["unit"] == d["unit"] and 0 < e["value"] < d["value"]
    assert e["h2d_bytes_per_step"] == 4_227_872_768 and e["d2h_bytes_per_step"] == 1_879_048_192
    assert e["round_trip_ok"] is True
    assert d["gpu_launches"] == 5 * d["steps"]
    k = d["clocks"]
    assert k["samples"] > 0 and k["sm_mhz"] > 0 and k["sm_max_mhz"] >= k["sm_mhz"]
    assert isinstance(k["reasons"], list)
    shares = sum(v["share"] for v in d["kernels"].values())
    assert abs(shares - 1.0) < 0.01


def test_reference_line():
    d = _run(["--impl", "reference", "--steps", "2", "--warmup", "3", "--reference-budget", "4"])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


@pytest.mark.parametrize("mode,launches", [
    ("seq_to_head", 2), ("head_to_seq", 6), ("reduce_scatter", 2), ("gated_reduce_scatter", 2),
    ("all_gather", 2), ("staged_seq_to_head", 12), ("rank_seq_to_head", 2)])
def test_profile_modes_run(mode, launches):
    """Every --profile mode (the commands of the ncu captures) runs its kernel."""
    out = subprocess.run([sys.executable, "bench.py", "--profile", mode, "--steps", "2",
                          "--profile-tokens", "4096"], cwd=ROOT, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    rec = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert rec["profile"] == mode and rec["tokens"] == 4096 and rec["launches"] == launches
