"""Host-side checks of bench.py (no GPU): the reference arm's JSON line keeps
the contract, the algorithmic byte and flop counts match their definitions,
and the ncu traffic figure is only used for the sources it was taken on."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from synth import CONFIGS  # noqa: E402


def test_reference_arm_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "0",
                        "--ref-tokens", "64"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["config"]["workload"] == "long_d128" and line["config"]["step_tokens"] == 64
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert cb["host_cpu_count"] == os.cpu_count()
    # the value is the measured rate of the sampled step itself: no scaling factor
    assert abs(line["value"] - 64 / (line["ms_per_step"] * 1e-3)) < 1e-6 * line["value"]


def test_algorithmic_bytes_and_flops():
    c = CONFIGS["llm_d64"]
    # q, k, v, o bf16 + per-token eta fp32 + the final fp32 state
    assert bench.algorithmic_bytes(c, c.B, c.H, c.T) == c.B * c.H * (c.T * (4 * 64 * 2 + 4) + 64 * 64 * 4)
    m = CONFIGS["momentum_d128"]
    assert bench.algorithmic_bytes(m, m.B, m.H, m.T) == m.B * m.H * (m.T * (4 * 128 * 2 + 4) + 2 * 128 * 128 * 4)
    assert bench.executed_flops(c, c.B, c.H, c.T, 64) == c.B * c.H * c.T * (4 * 64 * 64 + 4 * 64 * 64)


def test_traffic_figure_needs_matching_sources(tmp_path, monkeypatch):
    h = bench.src_hash()  # of the repository's kernel sources
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "llm_d64_c64.traffic.txt").write_text(f"src_hash={h}\ndram_bytes_per_call=123\n")
    (prof / "long_d128_c128.traffic.txt").write_text("src_hash=000000000000\ndram_bytes_per_call=456\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))  # profiles/ from the temporary tree
    monkeypatch.setattr(bench, "src_hash", lambda: h)   # sources still the repository's
    assert bench.read_traffic("llm_d64", 64) == 123.0
    assert bench.read_traffic("long_d128", 128) is None
    assert bench.read_traffic("momentum_d128", 128) is None


@pytest.mark.parametrize("name", sorted(bench.CHUNKED_SOURCES))
def test_hashed_sources_exist(name):
    assert os.path.exists(os.path.join(ROOT, "test_layers_causal_b200", "csrc", name))


def test_parity_helper_against_the_oracle_samples():
    """The bench's parity figure: fp32 rounding for the oracle's own output,
    the relative error of a known perturbation otherwise; a prefix of every
    sequence is compared with the oracle run on that prefix (causality)."""
    import torch
    c = CONFIGS["tiny_f32"]
    x = bench.make_case(c)
    _, _, o_full = bench.oracle_sample(c, c.T, x)
    o = torch.from_numpy(o_full).reshape(c.B, c.H, c.T, c.d_v)
    p = bench.parity(o, o_full)
    assert p["sequences"] == 2 and p["rel_frobenius_max"] < 1e-7 and p["pass"]  # fp32 rounding only
    p = bench.parity(1.03 * o, o_full)
    assert abs(p["rel_frobenius_max"] - 0.03) < 1e-6 and not p["pass"]
    _, _, o_pre = bench.oracle_sample(c, 100, x)
    p = bench.parity(o, o_pre)
    assert p["tokens_each"] == 100 and p["rel_frobenius_max"] < 1e-7


def test_cpu_baseline_returns_the_line_object_and_its_outputs():
    c = CONFIGS["tiny_f32"]
    x = bench.make_case(c)
    line, o_ref = bench.cpu_baseline(c, 128, x)
    assert line["kind"] == "oracle" and line["cores"] >= 1 and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["host_cpu_count"] == os.cpu_count()
    assert "first 128 of 256 tokens of all 2" in line["sample"]
    assert o_ref.shape == (2, 128, c.d_v)
