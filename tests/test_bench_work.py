"""Host-side checks of the benchmark's work model: the per-kernel algorithmic
FLOPs and bytes that the roofline fractions divide by (no GPU needed)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from gsa_inputs import CONFIGS  # noqa: E402


def test_compressed_and_special_flops_at_1000_frames():
    cfg = CONFIGS["pi3_f1000"]
    w = bench.algorithmic_work(cfg, cfg.topk)
    R = 1000 * 9 * 9                      # 36x36 grid, 4x4 regions
    assert cfg.num_regions == R
    assert w["comp_attn_topk"]["flops"] == pytest.approx(4 * 64 * R * R * 16)
    Ms, M = 1000 * 5, 1000 * 36 * 36
    assert w["special"]["flops"] == pytest.approx(4 * 64 * Ms * (Ms + M) * 16)
    # selection: each valid query attends the tokens of its k regions (k * s^2 = 512 keys)
    assert w["selection"]["flops"] == pytest.approx(4 * 64 * M * 512 * 16)
    assert "fixed_attn" not in w


def test_fixed_context_split_keeps_the_total():
    """With fixed frames (bf16) the fixed context is its own kernel: its FLOPs
    leave the selection's count, and the two together equal one selection over
    the union of the keys plus the gate."""
    cfg = CONFIGS["vggt_f256"]
    w = bench.algorithmic_work(cfg, cfg.topk)
    nfix = len(cfg.fixed_frames) * (cfg.num_special + cfg.grid_h * cfg.grid_w)
    assert nfix == 4122
    M = cfg.num_img_valid
    assert w["fixed_attn"]["flops"] == pytest.approx(4 * 64 * M * nfix * 16)
    assert w["selection_gate"]["flops"] + w["fixed_attn"]["flops"] == pytest.approx(
        w["selection"]["flops"] + w["epilogue"]["flops"])
    assert w["selection_gate"]["flops"] == pytest.approx(4 * 64 * M * 512 * 16 + w["epilogue"]["flops"])
    assert "fixed_attn" in bench.TENSOR_KERNELS


def test_fp32_contexts_keep_the_fixed_context_in_the_selection():
    cfg = CONFIGS["pi3_f32"].with_(dtype="fp32", fixed_frames=(0,))
    w = bench.algorithmic_work(cfg, cfg.topk)
    assert "fixed_attn" not in w


def test_traffic_record_is_tied_to_the_sources(tmp_path, monkeypatch):
    """A traffic figure is used only while the recorded source hash matches; a
    record of a smaller workload is scaled by the ratio of compulsory bytes."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = "abcdef123456"
    (prof / "ncu_traffic.txt").write_text(
        "# kernel workload bytes source_sha\n"
        f"comp_attn_topk pi3_f1000 123 {sha}\n"
        "comp_attn_topk pi3_f128 456 000000000000\n"
        f"pool pi3_f128 1000 {sha}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda kernel="": sha)
    assert bench.read_traffic("comp_attn_topk", "pi3_f1000")[0] == 123.0
    assert bench.read_traffic("comp_attn_topk", "pi3_f128")[0] is None
    assert bench.read_traffic("special", "pi3_f1000")[0] is None
    b, note = bench.read_traffic("pool", "pi3_f1000", {"pi3_f128": 10.0, "pi3_f1000": 78.0})
    assert b == pytest.approx(7800.0) and "scaled" in note
    assert bench.read_traffic("pool", "pi3_f1000")[0] is None


def test_each_kernel_hashes_its_own_sources():
    assert bench.kernel_source_sha("pool") != bench.kernel_source_sha("comp_attn_topk")
    assert bench.kernel_source_sha("special") == bench.kernel_source_sha("comp_attn_topk")
