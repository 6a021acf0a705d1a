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


def _rank_main(rank, world, port, out):
    import os

    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank step times differ; every rank must see the slowest one
        t = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        v = bench.job_tflops(world, 100, 2e12, t)
        out.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_multi_rank_time_is_max_over_ranks_gloo():
    # the bench's N > 1 aggregation, as two gloo ranks on the CPU
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(2))
    for rank, t, v in got:
        assert t == 15.0
        assert abs(v - 2 * 100 * 2e12 / (15.0e-3) / 1e12) < 1e-9


def test_single_process_reduction_is_identity():
    import torch
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_tflops(1, 10, 1e12, 10.0) == 1000.0
