"""Host-side logic of bench.py, on CPU: the FLOP and byte counts the bench
line divides by, the per-kernel table, the order in which the end-to-end
step copies its inputs, the peak file fallback, and one short run of the
reference arm (the CPU oracle) with the fields the bench line promises."""

import json
import os
import subprocess
import sys
import types

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _gflop(shapes, M, r):
    return sum(bench.flops_fwd_bwd(M, n, k, r) for n, k in shapes) / 1e9


def test_fwd_bwd_flops_match_the_workload_totals():
    """4MNK + 6MKr + 6MNr per linear; the totals the workloads are quoted
    with (512x512 at 64 tokens r=16; 4096^2 at 4096 tokens; the MLP's three
    linears at 8192 tokens; the decoder layer's seven at 16384 tokens)."""
    assert _gflop([(512, 512)], 64, 16) == pytest.approx(0.0734, abs=5e-4)
    assert _gflop([(4096, 4096)], 4096, 64) == pytest.approx(287.8, abs=0.1)
    mlp = [(11008, 4096), (11008, 4096), (4096, 11008)]
    assert _gflop(mlp, 8192, 64) == pytest.approx(4575, abs=1)
    layer = [(4096, 4096)] * 4 + mlp
    assert _gflop(layer, 16384, 64) == pytest.approx(13754, abs=1)


def test_nf4_bytes_per_param():
    """2 B read, half a byte of codes, one FP8 constant per 64, one fp32 per
    16384 written: 2.5159 B per parameter."""
    assert bench.NF4_BYTES_PER_PARAM == pytest.approx(2.515869, abs=1e-6)
    assert 64.76e9 * (bench.NF4_BYTES_PER_PARAM - 2) / 1e9 == pytest.approx(33.41, abs=0.01)


def test_kernel_table_aggregates_per_step():
    recs = [("fused_fwd", 2.0), ("fused_dx", 1.0), ("fused_fwd", 2.0), ("adamw8", 0.5),
            ("fused_fwd", 2.0), ("fused_dx", 1.0), ("fused_fwd", 2.0), ("adamw8", 0.5)]
    k = bench.kernel_table(recs, steps=2)
    assert k["fused_fwd"]["launches"] == 4
    assert k["fused_fwd"]["ms_total"] == pytest.approx(8.0)
    assert k["fused_fwd"]["ms_per_step"] == pytest.approx(4.0)
    assert k["fused_fwd"]["ms_avg"] == pytest.approx(2.0)
    assert sum(v["share"] for v in k.values()) == pytest.approx(1.0)
    assert k["adamw8"]["share"] == pytest.approx(1.0 / 11.0)


def test_e2e_input_order_follows_first_use():
    """Forward reads the units' inputs in unit order, backward the upstream
    gradients in reverse; an input shared by several units is copied once."""
    grouped = types.SimpleNamespace(units=[{"x": "attn"}, {"x": "o"}, {"x": "mlp"}, {"x": "down"}])
    assert bench.LayerStep.input_order(grouped) == [
        "X_attn", "X_o", "X_mlp", "X_down", "dY_3", "dY_2", "dY_1", "dY_0"]
    flat = types.SimpleNamespace(units=[{"x": x} for x in ("attn", "attn", "attn", "o", "mlp", "mlp", "down")])
    order = bench.LayerStep.input_order(flat)
    assert order[:4] == ["X_attn", "X_o", "X_mlp", "X_down"]
    assert order[4:] == [f"dY_{i}" for i in range(6, -1, -1)]


def test_peaks_file_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == bench.FALLBACK_PEAKS["hbm_gbs"]
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6500.0, "bf16_tflops": 1600.0,
                                                              "bf16_tflops_sustained": 1390.0}))
    p = bench.load_peaks()
    assert p["source"] == "measured"
    assert (p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"]) == (6500.0, 1600.0, 1390.0)


def test_reference_arm_line():
    """`--impl reference` runs the CPU oracle on a bounded sample and prints
    one JSON line with the fields of the bench line."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["steps"] == 1
    assert line["warmup"] == 3 and line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
