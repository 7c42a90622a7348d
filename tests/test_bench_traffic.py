"""bench.py's `traffic` figure comes from profiles/traffic.txt only while the
kernel sources match the row's digest: a row of another digest, another
workload or another kernel gives None (no number measured on other code)."""
import os

import bench


def _write(tmp_path, lines):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.txt").write_text("\n".join(lines) + "\n")


def test_traffic_row_needs_the_current_digest(tmp_path, monkeypatch):
    # the digest is of the repository's kernel sources, so copy them beside the file
    digest = bench.source_digest(bench.KERNEL_SOURCES)
    for p in bench.KERNEL_SOURCES:
        dst = tmp_path / p
        dst.parent.mkdir(parents=True, exist_ok=True)
        with open(os.path.join(bench.ROOT, p), "rb") as f:
            dst.write_bytes(f.read())
    _write(tmp_path, ["# comment", f"k2_decode gemm_gate_up_swiglu 123 {digest}",
                      "k2_decode_w4a16 gemm_gate_up_swiglu 456 0000000000000000"])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k2_decode", "gemm_gate_up_swiglu") == 123.0
    assert bench.profiled_traffic("k2_decode_w4a16", "gemm_gate_up_swiglu") is None
    assert bench.profiled_traffic("k2_decode", "gemm_down") is None
    assert bench.profiled_traffic("v3", "gemm_gate_up_swiglu") is None
