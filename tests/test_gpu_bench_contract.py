"""bench.py's JSON line carries every key of the measurement contract with
values of the right kind (a short run on the GPU; both arms)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


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
    assert d["dtype"] == "bf16" and d["accumulate_dtype"] == "f32" and d["data"] == "synthetic"
    assert d["config"]["workload"] == bench.WORKLOAD == \
        "qkvg_T250000_W4_chunked+reduce_scatter_T65536_C7168_W8"
    assert d["config"] == bench.step_config(1)  # the reference arm's config too
    assert d["config"]["relayout"]["window_bytes"] == 896_000_000
    assert d["config"]["bytes_per_step"] == 2 * 2 * 14_336_000_000 + 8_455_731_200
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
    # in: QKVG, 8 partials, bias; out: the QKVG round trip and the reduce rows
    assert e["h2d_bytes_per_step"] == 14_336_000_000 + 7_516_192_768 + 14_336
    assert e["d2h_bytes_per_step"] == 14_336_000_000 + 939_524_096
    assert e["round_trip_ok"] is True
    # the same copies alone bound the end-to-end step from below
    assert 0 < e["link_bound_ms_per_step"] and 0 < e["frac_of_link_bound"] <= 1.05
    # one batch plane per launch each way (4 + 4) and one reduce-scatter launch
    assert d["gpu_launches"] == 9 * d["steps"]
    assert {k: v["launches_per_step"] for k, v in d["kernels"].items()} == \
        {"seq_to_head": 4, "head_to_seq": 4, "ragged_reduce_scatter": 1}
    k = d["clocks"]
    assert k["samples"] > 0 and k["sm_mhz"] > 0 and k["sm_max_mhz"] >= k["sm_mhz"]
    assert isinstance(k["reasons"], list)
    shares = sum(v["share"] for v in d["kernels"].values())
    assert abs(shares - 1.0) < 0.01
    # the bar every kernel of the step must clear: 70 % of B200's ~8 TB/s,
    # by algorithmic bytes over CUDA-event time at full size
    for name, k in d["kernels"].items():
        assert k["gbs"] >= 0.70 * 8000.0, (name, k["gbs"])
    # beside the line: the same window cut into token ranges of all planes
    c = d["chunk_shapes"]
    assert c["window_bytes"] == 896_000_000
    r = c["token_ranges_all_planes"]
    assert r["round_trip_ok"] is True and r["tokens_per_launch"] == 15625
    for k in ("seq_to_head", "head_to_seq"):
        assert r[k]["launches_per_call"] == 4 and r[k]["planes_per_launch"] == 4
        assert r[k]["gbs"] >= 0.70 * 8000.0, (k, r[k]["gbs"])
        assert c["one_plane_per_launch"][k]["launches_per_call"] == 4


def test_reference_line():
    d = _run(["--impl", "reference", "--steps", "2", "--warmup", "3", "--reference-budget", "4"])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["config"] == bench.step_config(1)  # the native arm's config
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True
    assert d["cpu_baseline"]["sample_tokens"] > 0 and d["cpu_baseline"]["sample_rows"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


@pytest.mark.parametrize("mode,layout,window,launches", [
    ("seq_to_head", 0, -1, 8), ("head_to_seq", 0, -1, 8), ("seq_to_head", 3, -1, 8),
    ("head_to_seq", 2, -1, 8), ("seq_to_head", 0, 0, 2), ("reduce_scatter", 0, -1, 2),
    ("gated_reduce_scatter", 0, -1, 2), ("all_gather", 0, -1, 2),
    ("staged_seq_to_head", 0, -1, 16), ("rank_seq_to_head", 0, -1, 8),
    ("seq_to_head", 0, 14_680_064, 8), ("head_to_seq", 0, 14_680_064, 8)])
def test_profile_modes_run(mode, layout, window, launches):
    """Every --profile mode (the commands of the ncu captures) runs its kernel:
    the relayouts one batch plane per launch (4 planes, 2 calls), or in one
    launch with no window."""
    # a window of one plane of one rank of the 4096-token operand (1,024 tokens
    # x 56 x 128 x 2 B = 14,680,064 B) cut into token ranges of all four
    # planes: 256 tokens a launch, four per call (the token-range captures)
    tok = ["--profile-token-chunks"] if window == 14_680_064 else []
    out = subprocess.run([sys.executable, "bench.py", "--profile", mode, "--steps", "2",
                          "--profile-tokens", "4096", "--profile-rows", "4096",
                          "--profile-layout", str(layout), "--profile-window", str(window), *tok],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-2000:]
    rec = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert rec["profile"] == mode and rec["launches"] == launches
    assert rec["token_chunks"] == bool(tok)
    assert rec["tokens" if "reduce" not in mode and mode != "all_gather" else "rows"] == 4096
