"""bench.py's roofline `traffic`: DRAM bytes of a kernel from the committed
small-grid ncu capture, scaled by selected pairs, reported only while the
kernel's sources hash as they did at capture time."""
import os

import bench


def _table(tmp_path, rows):
    p = tmp_path / "traffic.md"
    lines = ["| kernel | dram read (bytes) | dram write (bytes) | duration (ms) | selected pairs | source |",
             "|---|---:|---:|---:|---:|---|"]
    lines += [f"| {k} | {r} | {w} | 1.0 | {n} | {h} |" for k, r, w, n, h in rows]
    p.write_text("\n".join(lines) + "\n")
    return str(p)


def test_traffic_scaled_by_pairs_only_for_matching_sources(tmp_path):
    d = bench.source_digest("k_bwd_dkdv")
    assert d is not None and len(d) == 16
    path = _table(tmp_path, [("k_bwd_dkdv", 100, 23, 1000, d), ("k_attn_fwd", 7, 8, 10, "0" * 16)])
    assert bench.measured_traffic("k_bwd_dkdv", 1000, path) == 123.0
    assert bench.measured_traffic("k_bwd_dkdv", 4000, path) == 492.0          # four times the pairs
    assert bench.measured_traffic("k_attn_fwd", 10, path) is None            # sources changed since
    assert bench.measured_traffic("k_select", 10, path) is None              # not a tracked kernel
    assert bench.measured_traffic("k_bwd_dkdv", 1000, str(tmp_path / "missing.md")) is None


def test_committed_table_parses():
    path = os.path.join(bench.ROOT, "profiles", bench.TRAFFIC_PROFILE)
    if not os.path.exists(path):
        return
    for k in bench.KERNEL_TU:
        v = bench.measured_traffic(k, 1e12, path)
        assert v is None or v > 0
