"""Host-side pieces of bench.py that need no GPU: the peak table and the
roofline fractions reported beside the measured one."""
import json

import pytest

import bench


def test_load_peaks_reads_measured_file(tmp_path, monkeypatch):
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"bf16_tflops": 1647.8, "bf16_tflops_sustained": 1344.1, "hbm_gbs": 6543.4}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    pk = bench.load_peaks()
    assert pk == {"bf16_tflops": 1647.8, "bf16_tflops_sustained": 1344.1, "hbm_gbs": 6543.4,
                  "source": "measured"}


def test_load_peaks_falls_back_when_missing(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    pk = bench.load_peaks()
    assert pk["source"] == "fallback"
    assert pk["bf16_tflops"] == 1590.0 and pk["hbm_gbs"] == 6650.0
    # held under the power cap the same GEMM settles lower than its burst rate
    assert pk["bf16_tflops_sustained"] == 1400.0 < pk["bf16_tflops"]


def test_tensor_fracs():
    pk = {"bf16_tflops": 1647.8, "bf16_tflops_sustained": 1344.1, "hbm_gbs": 6543.4}
    fr = bench.tensor_fracs(672.05, pk)
    assert fr["frac_of_sustained"] == pytest.approx(0.5)
    assert fr["frac_of_datasheet"] == pytest.approx(672.05 / 2250.0)
    assert fr["peak_sustained"] == 1344.1 and fr["peak_datasheet"] == 2250.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun every rank but 0 leaves the reference arm at once,
    without work or output (and without touching a process group)."""
    monkeypatch.setattr(bench, "dist_env", lambda: (2, 1, 1))
    args = bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
