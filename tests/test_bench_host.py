"""Host logic of bench.py (no GPU): the DRAM traffic a bench line reports
comes from a committed ncu summary only while the summary's source hash
matches the kernel sources as they are; otherwise the line says null."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_traffic_is_read_only_for_the_current_sources(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.file_sha([str(src)])
    (prof / "k_w.md").write_text("# k\n\nkernel_sha256: %s\ndram_bytes_per_launch: 12345678\n" % sha)
    assert bench.profiled_traffic("k_w.md", [str(src)]) == 12345678.0
    src.write_text("kernel v2\n")                      # the kernel changed after the capture
    assert bench.profiled_traffic("k_w.md", [str(src)]) is None
    assert bench.profiled_traffic("missing.md", [str(src)]) is None


def test_committed_profiles_name_their_command_and_hash():
    """Every committed kernel summary carries the lines the bench reads and
    a command that runs committed files (bench.py) under ncu with
    --clock-control none."""
    pdir = os.path.join(ROOT, "profiles")
    for name in sorted(os.listdir(pdir)):
        text = open(os.path.join(pdir, name)).read()
        assert "ncu " in text and "--clock-control none" in text, name
        assert "python bench.py" in text, name
        assert "_work" not in text, name
        if not name.startswith("launches"):
            assert "kernel_sha256:" in text and "dram_bytes_per_launch:" in text, name
