"""The DRAM-traffic figure bench.py reports beside the roofline comes from a
committed ncu summary and must be dropped once the kernel's own sources
change (host-only edits elsewhere keep it)."""
import os

import bench


def _tree(tmp_path, line):
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    (root / "quantized_opt_decode_b200").mkdir()
    os.symlink(os.path.join(bench.ROOT, "quantized_opt_decode_b200", "csrc"),
               root / "quantized_opt_decode_b200" / "csrc")
    (root / "profiles" / "ncu_traffic.txt").write_text("# comment\n" + line + "\n")
    return str(root)


def test_every_kernel_kind_names_existing_sources():
    csrc = os.path.join(bench.ROOT, "quantized_opt_decode_b200", "csrc")
    for kind, files in bench.KERNEL_FILES.items():
        assert files, kind
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (kind, f)


def test_traffic_kept_while_the_kernel_sources_match(tmp_path, monkeypatch):
    h = bench.csrc_hash(bench.KERNEL_FILES["attn_decode"])
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path, f"attn_decode  123456  {h}  capture.md"))
    assert bench.ncu_traffic("attn_decode") == 123456.0
    assert bench.ncu_traffic("fc1") is None  # no line for it


def test_traffic_dropped_once_the_kernel_sources_differ(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path, "attn_decode  123456  0123456789abcdef  capture.md"))
    assert bench.ncu_traffic("attn_decode") is None


def test_kernel_hash_ignores_other_files():
    # the attention figure depends on its own files only, not on the GEMM's
    a = bench.csrc_hash(bench.KERNEL_FILES["attn_decode"])
    assert a == bench.csrc_hash(list(reversed(bench.KERNEL_FILES["attn_decode"])))
    assert "gemm_tc.cu" not in bench.KERNEL_FILES["attn_decode"]
    assert a != bench.csrc_hash(bench.KERNEL_FILES["fc1"])
