"""Host-side pieces of bench.py that need no GPU: the ncu traffic table it
reads for the roofline and the source hash that invalidates it."""
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rows():
    with open(os.path.join(ROOT, "profiles", "gemm_dram_traffic.md")) as f:
        for line in f:
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) == 4 and cells[2].isdigit():
                yield cells


def test_traffic_table_parses_and_covers_default_workload():
    rows = list(_rows())
    assert rows, "no data rows"
    names = {r[0] for r in rows}
    assert "bert_fc1_wanda_3072x768_m4096" in names
    for wl, kernel, traffic, h in rows:
        assert int(traffic) > 0 and kernel.startswith("gemm_sp") and len(h) == 16


def test_traffic_lookup_follows_the_source_hash():
    cur = bench.gemm_src_hash()
    assert len(cur) == 16
    for wl, _, traffic, h in _rows():
        assert bench.gemm_traffic(wl) == (int(traffic) if h == cur else None)
    assert bench.gemm_traffic("no_such_workload") is None
