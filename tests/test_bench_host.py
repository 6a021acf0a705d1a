"""Host-side pieces of bench.py that need no GPU: the ncu traffic table it
reads for the roofline and the source hash that invalidates it."""
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rows():
    with open(os.path.join(ROOT, "profiles", "gemm_dram_traffic.md")) as f:
        for line in f:
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) == 5 and cells[3].isdigit():
                yield cells


def test_traffic_table_parses_and_covers_default_workload():
    rows = list(_rows())
    assert rows, "no data rows"
    names = {r[0] for r in rows}
    assert "bert_fc1_wanda_3072x768_m4096" in names
    for wl, plan, kernel, traffic, h in rows:
        assert int(traffic) > 0 and kernel.startswith("gemm_sp") and len(h) == 16
        assert bench.family_of(plan) in bench.FAMILY_SOURCES


def test_traffic_lookup_follows_plan_and_source_hash():
    for wl, plan, _, traffic, h in _rows():
        cur = bench.gemm_src_hash(bench.family_of(plan))
        assert len(cur) == 16
        assert bench.gemm_traffic(wl, plan) == (int(traffic) if h == cur else None)
        other = "single" if plan.startswith("pair") else "pair256"
        assert bench.gemm_traffic(wl, other) is None   # another kernel: no number
    assert bench.gemm_traffic("no_such_workload", "pair256") is None
