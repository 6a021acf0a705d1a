"""Host-side pieces of bench.py that need no GPU: the ncu traffic table it
reads for the roofline, the source hash that invalidates it, the peak
denominators and the bounded CPU-oracle sample."""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rows():
    with open(os.path.join(ROOT, "profiles", "gemm_dram_traffic.json")) as f:
        return json.load(f)["rows"]


def test_traffic_table_parses():
    rows = _rows()
    assert rows, "no data rows"
    for r in rows:
        assert int(r["traffic_bytes"]) > 0 and r["kernel"].startswith("gemm_sp")
        assert len(r["family_src_hash"]) == 16
        assert bench.family_of(r["plan"]) in bench.FAMILY_SOURCES


def test_traffic_lookup_follows_plan_and_source_hash(tmp_path):
    for r in _rows():
        cur = bench.gemm_src_hash(bench.family_of(r["plan"]))
        assert len(cur) == 16
        want = int(r["traffic_bytes"]) if r["family_src_hash"] == cur else None
        assert bench.gemm_traffic(r["workload"], r["plan"]) == want
        other = "single" if r["plan"].startswith("pair") else "pair256"
        assert bench.gemm_traffic(r["workload"], other) is None   # another kernel: no number
    assert bench.gemm_traffic("no_such_workload", "pair256") is None
    # a row recorded with the current hash is found; a stale hash is not
    cur = bench.gemm_src_hash("pair")
    p = tmp_path / "t.json"
    p.write_text(json.dumps({"rows": [
        {"workload": "w", "plan": "pair256", "kernel": "gemm_sp_pair", "traffic_bytes": 7,
         "family_src_hash": cur},
        {"workload": "v", "plan": "pair256", "kernel": "gemm_sp_pair", "traffic_bytes": 9,
         "family_src_hash": "0" * 16}]}))
    assert bench.gemm_traffic("w", "pair256", str(p)) == 7
    assert bench.gemm_traffic("v", "pair256", str(p)) is None


def test_peaks_and_bytes():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    assert bench.sparse_peak(peaks, False, False) == 3200.0
    assert bench.sparse_peak(peaks, False, True) == 2800.0
    assert bench.sparse_peak(peaks, True, False) == 6400.0
    # X + values + metadata + Y for bf16; int8 halves X and the values
    assert bench.gemm_bytes(16, 64, 128, False) == 2 * 16 * 128 + 64 * 128 + 64 * 16 + 2 * 16 * 64
    assert bench.gemm_bytes(16, 64, 128, True) == 16 * 128 + 64 * 64 + 64 * 16 + 2 * 16 * 64 + 256


def test_oracle_sample_is_bounded_and_extrapolates():
    # the CPU baseline on a slice of the largest configuration stays within
    # its budget and reports the flops of a whole step
    from structured_sparse_gemm_sp24_b200 import inputs as I
    wl = I.Workload("cut", W=I.normal_bf16((16384, 1024), 1.0, 0),
                    X=I.normal_bf16((16384, 1024), 1.0, 1))
    import time
    t0 = time.perf_counter()
    flops, secs, sample, cores = bench.oracle_sample(wl, 0.3)
    assert time.perf_counter() - t0 < 5.0
    assert flops == 2.0 * 16384 * 16384 * 1024 and secs > 0 and cores >= 1
    assert "extrapolated" in sample
    # a small problem is done whole
    small = I.Workload("tiny", W=I.normal_bf16((64, 128), 1.0, 0),
                       X=I.normal_bf16((16, 128), 1.0, 1))
    assert "whole step" in bench.oracle_sample(small, 5.0)[2]


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


def test_back_to_back_timings_run_the_step_work(monkeypatch):
    # the per-configuration "back to back" figures time prep_call() and
    # gemm_call(); together they must issue exactly the library calls of one
    # step, in order.  The launching entry points are replaced by recorders
    # (no GPU), the size queries stay the library's own.
    import torch
    from structured_sparse_gemm_sp24_b200 import build as sp24_build
    from structured_sparse_gemm_sp24_b200 import inputs as I
    from structured_sparse_gemm_sp24_b200 import sp24 as B
    sp24_build.build()
    B.lib()
    calls = []
    for name in ["sp24_prune", "sp24_prune_compress", "sp24_prune_progressive",
                 "sp24_prune_compress_int8", "sp24_act_scale", "sp24_quantize", "sp24_gemm"]:
        monkeypatch.setattr(B, name, (lambda n: lambda *a, **k: calls.append(n))(name))
    workloads = [I.tiny(), I.bert_fc1(), I.int8_long_tail(M=64, N=256, K=256)]
    for wl in workloads:
        r = bench.Runner(wl, torch.device("cpu"))
        calls.clear()
        r.step()
        step_calls = list(calls)
        calls.clear()
        r.prep_call()
        r.gemm_call()
        assert calls == step_calls, (wl.name, calls, step_calls)
        assert step_calls[-1] == "sp24_gemm"
        # the prep stage's bytes cover what its calls move
        assert r.prep_bytes() >= r.compress_bytes() > 0
