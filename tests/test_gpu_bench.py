"""bench.py's JSON line on a small cache (2 layers of the Mistral-shaped
workload): every key the benchmark contract asks for is present and
consistent, and the optional blocks (attention, entropy, layer-by-layer
encode, parity against the oracle) run; a second run checks the per-workload
summaries (tiny and decode-append at full size)."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def line():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    res = subprocess.run([sys.executable, "bench.py", "--workload", "mistral7b_32k", "--layers",
                          "2", "--steps", "3", "--warmup", "3", "--e2e-steps", "1", "--cpu-tokens",
                          "4096", "--layerwise", "--configs", "none", "--parity-layers", "0,1"],
                         cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [x for x in res.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, res.stdout[-2000:]
    return json.loads(lines[0])


def test_contract_keys(line):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["steps"] == 3 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["config"]["workload"] == "mistral7b_32k" and line["config"]["layers"] == 2
    assert line["gpu_launches"] == 3 * 7


def test_roofline_and_baselines(line):
    r = line["roofline"]
    assert r["bound"] in ("hbm", "tensor", "alu") and r["unit"] == "GB/s"
    assert 0 < r["achieved"] and 0 < r["peak"]
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert r["traffic"] is None  # recorded for the full 32-layer launch only
    c = line["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["sample"]
    assert c["host_cores"] >= c["cores"] and c["single_thread"]["value"] > 0
    for stage in ("score", "select", "encode", "decode"):
        assert line["rooflines"][stage]["ms"] > 0
    e = line["e2e"]
    assert e["value"] > 0 and e["unit"] == line["unit"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert e["link"]["h2d_gbs"] > 0 and 0 < e["frac_of_h2d_bound"] <= 1.5
    assert line["clocks"]["sm_mhz"] > 0 and isinstance(line["clocks"]["reasons"], list)


def test_reconstruction_diagnostic(line):
    """The oracle's own reconstruction of this workload's layer 0 (4096-token
    sample) has mean cosine 0.981 / relative L2 error 0.195 for the 3-bit keys
    and 0.891 / 0.503 for the 2-bit values; the bounds sit around those."""
    r = line["reconstruction"]
    assert r["layers_sampled"] == [0]
    assert 0.95 < r["k"]["cosine_mean"] <= 1.0 and 0.0 < r["k"]["rel_l2_mean"] < 0.3
    assert 0.85 < r["v"]["cosine_mean"] <= 1.0 and 0.0 < r["v"]["rel_l2_mean"] < 0.6


def test_exact_layout_block(line):
    x = line["exact_layout"]
    assert x["encode_ms"] > 0 and x["decode_ms"] > 0
    assert x["bits_per_coordinate"] == {"k": 3.125, "v": 2.125}
    assert x["bits_per_elem"] < line["bits_per_elem"]
    assert x["rooflines"]["encode"]["frac"] > 0


def test_optional_blocks(line):
    a = line["decode_attention"]
    assert a["fused_ms"] > 0 and a["decode_then_sdpa_ms"] > 0
    for mode in ("delta", "plain"):
        s = line["entropy_stage"][mode]
        assert s["round_trip_exact"] is True
        assert 0 < s["codes_bits_per_elem_coded"] < 4
    c = line["entropy_correlated"]
    assert c["delta"]["round_trip_exact"] and c["plain"]["round_trip_exact"]
    # correlated tokens: the difference makes the codes cheaper to code
    assert c["delta"]["codes_ratio"] > c["plain"]["codes_ratio"]
    w = line["layerwise_encode"]
    assert w["all_layers_ms"] > 0 and w["layer_by_layer_ms"] > 0


def test_parity_block(line):
    p = line["parity"]
    assert p["layers_checked"] == [0, 1]
    assert p["unexcused"] == 0 and p["failures"] == [] and p["bf16_elements_differing"] == 0
    assert p["elements"] == 2 * 2 * 8 * line["config"]["kept_per_layer"] * 128


def test_config_summaries():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    res = subprocess.run([sys.executable, "bench.py", "--workload", "mistral7b_32k", "--layers",
                          "1", "--steps", "3", "--warmup", "3", "--no-e2e", "--no-attend",
                          "--no-entropy", "--cpu-tokens", "2048", "--configs",
                          "tiny,decode_append", "--config-steps", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads([x for x in res.stdout.splitlines() if x.startswith("{")][0])
    c = line["configs"]
    assert set(c) == {"tiny", "decode_append"}
    t = c["tiny"]
    assert t["value"] > 0 and abs(t["bits_per_elem"] - 2.75) < 1e-9
    assert t["rooflines"]["encode"]["frac"] > 0 and t["cpu_baseline"]["value"] > 0
    a = c["decode_append"]
    assert a["steps"] == 256 and a["stages_ms"]["append_encode"] > 0
    assert a["stages_ms"]["layer_decode"] > 0 and a["cpu_baseline"]["value"] > 0
