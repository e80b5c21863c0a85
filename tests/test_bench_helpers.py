"""bench.py's roofline `traffic`: DRAM bytes of a kernel from the committed ncu table,
reported only while the kernel's sources hash as they did at capture time."""
import os

import bench


def _table(tmp_path, rows):
    p = tmp_path / "traffic.md"
    lines = ["| kernel | dram read (bytes) | dram write (bytes) | duration (ms) | source |", "|---|---:|---:|---:|---|"]
    lines += [f"| {k} | {r} | {w} | 1.0 | {h} |" for k, r, w, h in rows]
    p.write_text("\n".join(lines) + "\n")
    return str(p)


def test_traffic_only_for_matching_sources(tmp_path):
    d = bench.source_digest("k_bwd_dkdv")
    assert d is not None and len(d) == 16
    path = _table(tmp_path, [("k_bwd_dkdv", 100, 23, d), ("k_attn_fwd", 7, 8, "0" * 16)])
    assert bench.measured_traffic("k_bwd_dkdv", path) == 123.0
    assert bench.measured_traffic("k_attn_fwd", path) is None       # sources changed since the capture
    assert bench.measured_traffic("k_select", path) is None          # not a tracked kernel
    assert bench.measured_traffic("k_bwd_dkdv", str(tmp_path / "missing.md")) is None


def test_committed_table_parses():
    path = os.path.join(bench.ROOT, "profiles", "dram_traffic_grid72x88x160.md")
    for k in bench.KERNEL_TU:
        v = bench.measured_traffic(k, path)
        assert v is None or v > 0
