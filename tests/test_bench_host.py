"""Host-side logic of bench.py that decides what a bench line may claim (no GPU).

The roofline `traffic` figure comes from a committed ncu summary and is only valid for the
kernel source it was captured on; the peaks come from the measured file or the stated
fallback. Both rules are exercised on a scratch copy of the files they read."""
import os
import shutil

import bench


def _scratch_root(tmp_path):
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    (root / "decoder_only_transformer_layer_b200" / "csrc").mkdir(parents=True)
    shutil.copy(os.path.join(bench.ROOT, "profiles", "gemv_llama3-8b_decode_full.md"), root / "profiles")
    shutil.copy(os.path.join(bench.ROOT, "decoder_only_transformer_layer_b200", "csrc", "gemv.cu"),
                root / "decoder_only_transformer_layer_b200" / "csrc")
    return root


def test_traffic_is_reported_only_for_the_profiled_kernel_source(tmp_path, monkeypatch):
    root = _scratch_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    summary = (root / "profiles" / "gemv_llama3-8b_decode_full.md").read_text()
    assert "traffic_bytes_per_launch:" in summary and "kernel_sha256:" in summary
    expected = int(summary.split("traffic_bytes_per_launch:")[1].split()[0])
    got = bench.measured_traffic()
    # the committed summary was taken on the committed source, or the figure is withheld
    assert got in (expected, None)
    # a one-byte change of the kernel source withdraws the figure
    src = root / "decoder_only_transformer_layer_b200" / "csrc" / "gemv.cu"
    src.write_bytes(src.read_bytes() + b"\n")
    assert bench.measured_traffic() is None
    # as does a missing summary
    (root / "profiles" / "gemv_llama3-8b_decode_full.md").unlink()
    assert bench.measured_traffic() is None


def test_peaks_fall_back_to_the_stated_figures_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    P = bench.peaks()
    assert P["src"] == "fallback" and P["hbm"] == 6650.0 and P["tc"] == 1590.0


def test_peaks_read_the_measured_file(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(src):
        return  # written per pod by the driver; the fallback test covers its absence
    shutil.copy(src, tmp_path / "MEASURED_PEAKS.json")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    P = bench.peaks()
    assert P["src"] == "measured" and P["hbm"] > 1000 and P["tc"] > 100
