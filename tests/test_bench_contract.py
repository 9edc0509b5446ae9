"""The JSON line of bench.py carries every key the harness reads.

The reference arm runs on the host only, so it is run here for real (every
kind of workload, one step each); the CUDA arm's line is assembled by the
same helper the GPU runs use, from stand-in numbers."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

TOP = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
       "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


import pytest  # noqa: E402


@pytest.mark.parametrize("workload", ["small", "varlen", "sparse", "dropout", "fp8"])
def test_reference_arm_line(workload):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", workload, "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert TOP <= set(d) and d["impl"] == "reference"
    assert d["value"] > 0 and d["value"] == d["cpu_baseline"]["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_cuda_arm_line_keys():
    roof = bench._roof("fa_bwd_kernel", 2.7e12, 2.6, 1671.6, "measured", 1.3e9, 1407.4)
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(roof)
    assert abs(roof["frac"] - roof["achieved"] / 1671.6) < 1e-12
    cpu = {"value": 0.01, "unit": "TFLOP/s", "cores": 16, "kind": "oracle", "sample": "s"}
    e2e = {"value": 150.0, "unit": "TFLOP/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1}
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    line = bench._base_line(1000.0, 20, 3, 75.0, 1, "bf16", {"workload": "w"},
                            {"ms": 1.0}, {"ms": 2.6}, roof, roof, cpu, e2e, clk, 4)
    assert TOP <= set(line)
    assert {"roofline", "gpu_launches", "clocks"} <= set(line)
    assert line["gpu_launches"] == 80 and line["ms_per_step"] == 75.0 / 20
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    json.dumps(line)  # serialisable


@pytest.mark.parametrize("workload", ["mid", "varlen"])
def test_reference_arm_other_ranks_exit_without_work(workload):
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", workload, "--gpus", "2", "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    assert not [ln for ln in out.stdout.splitlines() if ln.startswith("{")]


def test_cpu_baseline_cuts_long_slices(monkeypatch):
    """Slices longer than max_rows are cut to their first max_rows queries and
    keys before the oracle sees them; shorter ones go whole."""
    import types
    import torch
    import oracle
    seen = []
    real = oracle.ref_fwd_slice

    def spy(q, k, v, *a, **kw):
        seen.append((q.shape, k.shape, v.shape))
        return real(q, k, v, *a, **kw)
    monkeypatch.setattr(oracle, "ref_fwd_slice", spy)
    B, H, N, d = 1, 2, 96, 16
    w = types.SimpleNamespace(B=B, H=H, N=N, d=d, scale=d ** -0.5, causal=True, name="cut")
    g = torch.Generator().manual_seed(0)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g) for _ in range(4))
    whole = bench.cpu_baseline_slices(w, q, k, v, do, None, budget_s=60.0)
    assert "whole" in whole["sample"] and seen == [((N, d),) * 3] * H
    seen.clear()
    cut = bench.cpu_baseline_slices(w, q, k, v, do, None, budget_s=60.0, max_rows=32)
    assert "cut to its first 32" in cut["sample"] and seen == [((32, d),) * 3] * H
    assert whole["kind"] == cut["kind"] == "oracle" and cut["value"] > 0 and cut["cores"] >= 1
