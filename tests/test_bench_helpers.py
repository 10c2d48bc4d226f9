"""Host-side helpers of bench.py: the code-only source hash that decides
whether a committed ncu summary still describes a kernel, and the metric
bookkeeping of the roofline (CPU only)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_ignores_comments_and_layout():
    a = "int x = 1; // one\n/* block\ncomment */ int y=2;\n"
    b = "int x = 1;\nint y=2; // two\n"
    assert bench._code_only(a) == bench._code_only("int x = 1; int y=2;")
    assert bench._code_only(b) == bench._code_only("int x = 1; int y=2;")
    assert bench._code_only("int x = 1;") != bench._code_only("int x = 2;")


def test_kernel_hashes_cover_their_sources():
    from speculative_decoding_verification_86_b200 import build
    for kernel, files in bench.KERNEL_SOURCES.items():
        for name in files:
            assert os.path.exists(os.path.join(build.CSRC, name)), (kernel, name)
        h = bench.kernel_source_hash(kernel)
        assert len(h) == 16 and h == bench.kernel_source_hash(kernel)


def test_profiled_traffic_reads_a_matching_summary(tmp_path, monkeypatch):
    h = bench.kernel_source_hash("k_engine")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k_engine_x_y.md").write_text("# t\n\n- source_hash: `%s`\n- dram_bytes_per_launch: `123`\n" % h)
    (prof / "k_engine_x_z.md").write_text("# t\n\n- source_hash: `0000000000000000`\n- dram_bytes_per_launch: `9`\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k_engine", "x_y") == 123.0
    assert bench.profiled_traffic("k_engine", "x_z") is None   # another kernel's code
    assert bench.profiled_traffic("k_engine", "missing") is None
