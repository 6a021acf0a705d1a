#!/usr/bin/env python
"""Benchmark of the 2:4 sparse path on B200 (one JSON line on rank 0).

A step is one pass of the whole path over one batch of synthetic input:
  bf16 workloads:  [Wanda: column norms] -> fused prune+compress 2:4 ->
                   sparse GEMM Y = X * W'^T; the progressive (BERT fc1)
                   workload forms the 3:4 mask, the 2:4 mask on its
                   survivors and the compressed operand in one pass
  int8 workload:   prune 2:4 -> per-channel scale -> compress to int8 ->
                   per-tensor activation scale -> quantise X -> int8 sparse
                   GEMM with bf16 dequantisation.
The default workload is the largest single-GPU configuration, the square
16384^3 problem (W, X, Y 512 MB each, all larger than the 126 MB L2).
`value` = dense-equivalent TFLOP/s of the GEMM (2*M*N*K per step) over the
whole step time; the roofline of the dominant kernel (the GEMM) is reported
beside it, and a `configs` block gives the GEMM and prune/compress figures of
every other configured workload (BERT fc1, LLM projections at M = 16, 128 and
2048, INT8, square 4096 / 8192, the 1x1 convolution).  Inputs are resident in
HBM; L2 is flushed between timed steps by writing a 512 MB buffer and reading
it back (so the flush's own write-back is not charged to the next kernel).

Multi-GPU: one process per GPU (torchrun), each rank runs an independent
replica of the workload (weak scaling); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from structured_sparse_gemm_sp24_b200 import inputs as I  # noqa: E402
from structured_sparse_gemm_sp24_b200 import sp24 as B  # noqa: E402

METRIC = "2:4 sparse GEMM dense-equiv TFLOP/s & % sparse TC peak; prune+compress GB/s"
DEFAULT_WORKLOAD = "square_16384"
# the other configured workloads, reported in the `configs` block
CONFIG_WORKLOADS = (
    "bert_fc1",
    "llm_11008x4096_m2048", "llm_4096x11008_m2048",
    "llm_11008x4096_m128", "llm_4096x11008_m128",
    "llm_11008x4096_m16", "llm_4096x11008_m16",
    "int8", "square_4096", "square_8192", "conv1x1",
)
SPARSE_RATIO = 2.0          # nominal sparse / dense bf16 tensor throughput (4.5 / 2.25 PF)
INT8_RATIO = 2.0            # nominal int8 / bf16 tensor throughput (9 / 4.5 POPS sparse)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_SUSTAINED = 1400.0
L2_FLUSH_BYTES = 512 << 20


def flush_l2(buf: torch.Tensor) -> None:
    """Evicts the workload's data from L2 (126 MB) before a timed step: writes
    the 512 MB buffer, then reads it back, so that the write-back of the
    flush's own dirty lines happens here and not inside the next timed
    kernel (a write-only flush leaves ~126 MB of dirty lines whose eviction
    the next HBM-bound kernel would pay for)."""
    buf.zero_()
    buf.view(torch.int32).sum()
TRAFFIC_TABLE = os.path.join(ROOT, "profiles", "gemm_dram_traffic.json")


# --------------------------------------------------------------------- peaks
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": FALLBACK_BF16_SUSTAINED, "source": "fallback"}


def sparse_peak(peaks, int8: bool, sustained: bool) -> float:
    """Dense-equivalent sparse tensor peak (TFLOP/s or TOPS): the measured dense
    bf16 figure times the nominal sparse (and int8) ratios."""
    base = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    return base * SPARSE_RATIO * (INT8_RATIO if int8 else 1.0)


# -------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML every ~20 ms (read only)."""

    REASONS = {
        0x0000000000000001: "gpu_idle", 0x0000000000000002: "applications_clocks_setting",
        0x0000000000000004: "sw_power_cap", 0x0000000000000008: "hw_slowdown",
        0x0000000000000010: "sync_boost", 0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown", 0x0000000000000080: "hw_power_brake_slowdown",
        0x0000000000000100: "display_clock_setting",
    }

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------- workload
class Runner:
    """Device buffers for one workload and the calls of one step."""

    def __init__(self, wl: I.Workload, device):
        self.wl = wl
        self.dev = device
        self.N, self.K, self.M = wl.N, wl.K, wl.M
        d = device
        self.W = wl.W.to(d)
        self.X = wl.X.to(d)
        self.Xc = wl.Xc.to(d) if wl.Xc is not None else None
        N, K, M = self.N, self.K, self.M
        self.mask1 = torch.empty((N, K // 8), dtype=torch.uint8, device=d)
        self.mask2 = torch.empty((N, K // 8), dtype=torch.uint8, device=d)
        self.ws = torch.empty(max(B.sp24_prune_workspace_bytes(K, B.SP24_WANDA), 16),
                              dtype=torch.uint8, device=d)
        vdt = torch.int8 if wl.int8 else torch.bfloat16
        self.vals = torch.empty((N, K // 2), dtype=vdt, device=d)
        self.meta = torch.empty(B.sp24_meta_bytes(N, K), dtype=torch.uint8, device=d)
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=d)
        if wl.int8:
            self.s_w = torch.empty(N, dtype=torch.float32, device=d)
            self.s_x = torch.empty(4, dtype=torch.float32, device=d)
            self.act_ws = torch.empty(B.sp24_act_scale_workspace_bytes(), dtype=torch.uint8,
                                      device=d)
            self.Xq = torch.empty((M, K), dtype=torch.int8, device=d)
        self.wanda = wl.mode == "wanda"

    # number of library kernel launches per step (see the calls below)
    def launches_per_step(self) -> int:
        if self.wl.int8:
            return 1 + 7 + 1 + 1             # weight conversion, act_scale, quantize, gemm
        if self.wanda:
            # the library forms the column norms inside the prune kernel when
            # row tiles x calibration rows is small, else launches colnorm first
            fused = ((self.N + 127) // 128) * self.wl.Xc.shape[0] <= 8192
            if self.wl.progressive:
                return (1 if fused else 2) + 1       # [colnorm +] progressive prune, gemm
            return (1 if fused else 2) + 1 + 1   # [colnorm +] prune, prune_compress, gemm
        return 1 + 1                         # prune_compress, gemm

    def step(self, ev=None):
        """Enqueues one step; `ev` = list of 4 events: start, after pruning,
        after compression, after the GEMM."""
        rec = (lambda i: ev[i].record()) if ev else (lambda i: None)
        wl = self.wl
        rec(0)
        if wl.int8:
            # weight side: 2:4 mask, per-channel scale and int8 compression in
            # one pass over W; activation side: per-tensor scale, quantisation
            B.sp24_prune_compress_int8(self.W, 0.9999, self.mask2, self.s_w, self.vals,
                                       self.meta)
            rec(1)
            B.sp24_act_scale(self.X, 0.9999, self.s_x, self.act_ws)
            B.sp24_quantize(self.X, self.s_x, self.Xq)
            rec(2)
            self.gemm_call()
        elif self.wanda and wl.progressive:
            # one pass: norms, the 3:4 mask, the 2:4 mask on the survivors and
            # the compressed operand
            rec(1)
            B.sp24_prune_progressive(self.W, self.Xc, B.SP24_WANDA, self.mask1, self.mask2,
                                     self.vals, self.meta, self.ws)
            rec(2)
            self.gemm_call()
        elif self.wanda:
            # prune also leaves the float64 column norms in its workspace
            n_keep = 2
            B.sp24_prune(self.W, self.Xc, B.SP24_WANDA, n_keep, None, self.mask1, self.ws)
            rec(1)
            B.sp24_prune_compress(self.W, B.SP24_WANDA, self.ws, None, None, B.SP24_BF16,
                                  None, self.vals, self.meta)
            rec(2)
            self.gemm_call()
        else:
            rec(1)
            B.sp24_prune_compress(self.W, B.SP24_MAGNITUDE, None, None, None, B.SP24_BF16, None,
                                  self.vals, self.meta)
            rec(2)
            self.gemm_call()
        rec(3)

    def prep_call(self):
        """The step's work before the GEMM (prune / compress, and for INT8 the
        weight conversion, activation scale and quantisation)."""
        wl = self.wl
        if wl.int8:
            B.sp24_prune_compress_int8(self.W, 0.9999, self.mask2, self.s_w, self.vals,
                                       self.meta)
            B.sp24_act_scale(self.X, 0.9999, self.s_x, self.act_ws)
            B.sp24_quantize(self.X, self.s_x, self.Xq)
        elif self.wanda and wl.progressive:
            B.sp24_prune_progressive(self.W, self.Xc, B.SP24_WANDA, self.mask1, self.mask2,
                                     self.vals, self.meta, self.ws)
        elif self.wanda:
            B.sp24_prune(self.W, self.Xc, B.SP24_WANDA, 2, None, self.mask1, self.ws)
            B.sp24_prune_compress(self.W, B.SP24_WANDA, self.ws, None, None, B.SP24_BF16,
                                  None, self.vals, self.meta)
        else:
            B.sp24_prune_compress(self.W, B.SP24_MAGNITUDE, None, None, None, B.SP24_BF16, None,
                                  self.vals, self.meta)

    def prep_bytes(self) -> float:
        """Algorithmic bytes of prep_call."""
        if self.wl.int8:
            return self.prune_bytes() + self.compress_bytes()
        return self.compress_bytes()

    def gemm_call(self):
        """The step's GEMM (its operands are the step's earlier outputs)."""
        if self.wl.int8:
            B.sp24_gemm(self.Xq, self.vals, self.meta, self.N, B.SP24_INT8, self.s_x, self.s_w,
                        B.SP24_OUT_BF16, None, self.Y)
        else:
            B.sp24_gemm(self.X, self.vals, self.meta, self.N, B.SP24_BF16, None, None,
                        B.SP24_OUT_BF16, None, self.Y)

    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K

    def gemm_bytes(self) -> float:
        return gemm_bytes(self.M, self.N, self.K, self.wl.int8)

    def compress_bytes(self) -> float:
        """Algorithmic bytes of the compression stage (fused prune+compress for
        bf16: read W, write values + metadata; INT8: the activation side)."""
        N, K, M = self.N, self.K, self.M
        if self.wl.int8:
            # activation scale (one pass over float32 X; the sample is
            # negligible) and quantisation (read X, write Xq)
            return 4 * M * K + 4 * M * K + M * K
        if self.wl.progressive:
            # one pass: read W (and Xc), write both masks, values and metadata
            mc = self.wl.Xc.shape[0] if self.wl.Xc is not None else 0
            return 2 * mc * K + 2 * N * K + 2 * N * K / 8 + N * K + N * K / 8
        return 2 * N * K + N * K + N * K / 8

    def prune_bytes(self) -> float:
        N, K = self.N, self.K
        if self.wl.int8:
            # one-pass weight conversion: read W, write mask, scales, int8
            # values and metadata
            return 2 * N * K + N * K / 8 + 4 * N + N * K / 2 + N * K / 8
        if self.wanda:
            mc = self.wl.Xc.shape[0]
            return 2 * mc * K + 8 * K + 2 * N * K + 8 * K + N * K / 8
        return 0.0

    def h2d_inputs(self):
        t = [self.wl.W, self.wl.X]
        if self.wl.Xc is not None:
            t.append(self.wl.Xc)
        return t


def gemm_bytes(m: int, n: int, k: int, int8: bool) -> float:
    """Algorithmic bytes of one sparse GEMM launch: X + values + metadata + Y
    (+ the per-channel scales for INT8)."""
    if int8:
        return m * k + n * k / 2 + n * k / 8 + 2 * m * n + 4 * n
    return 2 * m * k + n * k + n * k / 8 + 2 * m * n


def workload_config(wl: I.Workload, world: int) -> dict:
    """The `config` object of a JSON line (same for both arms)."""
    return {"workload": wl.name, "M": wl.M, "N": wl.N, "K": wl.K, "mode": wl.mode,
            "progressive": wl.progressive, "int8": wl.int8,
            "l2": ("flushed between steps (512 MB written then read back)"
                   + ("; W, X, Y also exceed L2" if wl.M * wl.K * 2 > (126 << 20) else "")),
            "parallelism": f"replicas{world}"}


COMMON_SOURCES = ["sp24_device.cuh", "sp24_host.h", "tma_host.h"]
FAMILY_SOURCES = {   # the files that define each GEMM kernel family and its launch
    "pair": ["gemm_pair.cuh", "gemm_epilogue.cuh"] + COMMON_SOURCES,
    "single": ["gemm_persistent.cuh", "gemm_epilogue.cuh"] + COMMON_SOURCES,
    "splitk": ["gemm_splitk.cuh"] + COMMON_SOURCES,
}


def family_of(plan_kernel: str) -> str:
    return "pair" if plan_kernel.startswith("pair") else plan_kernel


def gemm_src_hash(family: str) -> str:
    """Hash of the sources of one GEMM kernel family (the traffic table records
    the one each capture was made with)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "structured_sparse_gemm_sp24_b200", "csrc")
    for n in FAMILY_SOURCES[family]:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_rows(path: str = TRAFFIC_TABLE):
    if not os.path.exists(path):
        return []
    with open(path) as f:
        return json.load(f).get("rows", [])


def gemm_traffic(workload: str, plan_kernel: str, path: str = TRAFFIC_TABLE):
    """DRAM bytes (read + write) of one GEMM launch on this workload from the
    committed ncu traffic table, or None when there is no row for it, the plan
    now picks another kernel, or that kernel's sources changed since."""
    if family_of(plan_kernel) not in FAMILY_SOURCES:
        return None
    cur = gemm_src_hash(family_of(plan_kernel))
    for r in traffic_rows(path):
        if r["workload"] == workload and r["plan"] == plan_kernel and r["family_src_hash"] == cur:
            return int(r["traffic_bytes"])
    return None


def time_steps(runner, steps, flush, use_graph=True, stage_steps=None):
    """Step and stage times (ms), L2 flushed before every step (outside the
    events).
    1. Step time: the step captured once in a CUDA graph and replayed `steps`
       times, CUDA events around each replay.
    2. Stage times: `stage_steps` steps, each captured in its own graph with
       events between its stages (external event-record nodes), replayed
       once.  A record node costs the device about 2 us, so these intervals
       are slightly long; that is why they are not taken in pass 1.
    With use_graph=False both passes are plain launches."""
    stage_steps = steps if stage_steps is None else min(stage_steps, steps)
    tot = []
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            runner.step()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            flush_l2(flush)
            ev[i][0].record()
            graph.replay()
            ev[i][1].record()
        torch.cuda.synchronize()
        tot = [a.elapsed_time(b) for a, b in ev]
        del graph
    inner = [[torch.cuda.Event(enable_timing=True, external=use_graph) for _ in range(4)]
             for _ in range(stage_steps)]
    graphs = []
    if use_graph:
        for i in range(stage_steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                runner.step(inner[i])
            graphs.append(g)
        torch.cuda.synchronize()
    for i in range(stage_steps):
        flush_l2(flush)
        if use_graph:
            graphs[i].replay()
        else:
            runner.step(inner[i])
    torch.cuda.synchronize()
    if not use_graph:
        tot = [e[0].elapsed_time(e[3]) for e in inner]
    prune = [e[0].elapsed_time(e[1]) for e in inner]
    comp = [e[1].elapsed_time(e[2]) for e in inner]
    gemm = [e[2].elapsed_time(e[3]) for e in inner]
    del graphs
    return tot, prune, comp, gemm


def count_step_kernels(runner):
    """Kernels in one step, counted as the kernel nodes of a CUDA graph captured
    from it (every kernel in the step is a library kernel); None if the graph
    cannot be inspected."""
    try:
        from cuda.bindings import runtime as cudart
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            runner.step()
        raw = g.raw_cuda_graph()
        h = raw if isinstance(raw, cudart.cudaGraph_t) else cudart.cudaGraph_t(init_value=int(raw))
        err, _, n = cudart.cudaGraphGetNodes(h, 0)
        if err != cudart.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = cudart.cudaGraphGetNodes(h, n)
        if err != cudart.cudaError_t.cudaSuccess:
            return None
        kern = cudart.cudaGraphNodeType.cudaGraphNodeTypeKernel
        count = 0
        for nd in nodes[:n]:
            e2, t = cudart.cudaGraphNodeGetType(nd)
            if e2 == cudart.cudaError_t.cudaSuccess and t == kern:
                count += 1
        g.reset()
        return count
    except Exception as exc:   # no cuda-python or no raw graph access
        print(f"bench: could not count graph kernel nodes ({exc})", file=sys.stderr)
        return None


class nvtx_range:
    """An NVTX range around a phase of the bench (timeline tools show the
    phases; nothing is recorded without one attached)."""

    def __init__(self, name: str):
        self.name = name

    def __enter__(self):
        torch.cuda.nvtx.range_push(self.name)
        return self

    def __exit__(self, *exc):
        torch.cuda.nvtx.range_pop()
        return False


def max_over_ranks(value: float, device) -> float:
    """The maximum of a per-rank time over all ranks (every rank calls it at the
    same point; all_reduce MAX), or the value itself in a single process."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, steps: int, flops_per_step: float, total_ms: float) -> float:
    """Whole-job throughput under weak scaling: every rank runs `steps` steps of
    its own replica; the job takes the slowest rank's time."""
    return world * steps * flops_per_step / (total_ms * 1e-3) / 1e12


def time_e2e(runner, steps):
    """Same step through host buffers: pinned H2D copies of the step's inputs and
    a D2H copy of Y inside the timed region, one after the other on one stream.
    Returns (ms per step, H2D bytes, D2H bytes)."""
    host_in = [t.pin_memory() for t in runner.h2d_inputs()]
    dev_in = [runner.W, runner.X] + ([runner.Xc] if runner.Xc is not None else [])
    host_y = torch.empty(runner.Y.shape, dtype=runner.Y.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_y.numel() * host_y.element_size()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        for hd, dd in zip(host_in, dev_in):
            dd.copy_(hd, non_blocking=True)
        runner.step()
        host_y.copy_(runner.Y, non_blocking=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(steps):
        for hd, dd in zip(host_in, dev_in):
            dd.copy_(hd, non_blocking=True)
        runner.step()
        host_y.copy_(runner.Y, non_blocking=True)
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps, h2d, d2h


def time_e2e_pipelined(runner, steps):
    """The same steps through host buffers, pipelined as a serving loop runs
    them: step i's inputs go up (pinned host -> device) on one copy stream
    while step i-1 computes, and step i's Y comes down on another while step
    i+1 computes (two device copies of the inputs and of Y, two host copies of
    Y).  Every step's copies are inside the timed region; only their overlap
    with each other and with the compute differs from time_e2e.  Returns ms
    per step."""
    host_in = [t.pin_memory() for t in runner.h2d_inputs()]
    names = ["W", "X"] + (["Xc"] if runner.Xc is not None else [])
    sets = [[getattr(runner, nm) for nm in names]]
    sets.append([torch.empty_like(t) for t in sets[0]])
    ys = [runner.Y, torch.empty_like(runner.Y)]
    host_y = [torch.empty(runner.Y.shape, dtype=runner.Y.dtype).pin_memory() for _ in range(2)]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of set j landed
    ev_done = [torch.cuda.Event() for _ in range(2)]   # the step on set j finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # Y of set j is on the host

    def run(i):
        j = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev_done[j])      # the step two back is done with set j
            for hd, dd in zip(host_in, sets[j]):
                dd.copy_(hd, non_blocking=True)
            ev_in[j].record(up)
        comp.wait_event(ev_in[j])
        if i >= 2:
            comp.wait_event(ev_out[j])         # Y of set j has gone down
        for nm, t in zip(names, sets[j]):
            setattr(runner, nm, t)
        runner.Y = ys[j]
        runner.step()
        ev_done[j].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[j])
            host_y[j].copy_(ys[j], non_blocking=True)
            ev_out[j].record(down)

    try:
        for i in range(2):
            run(i)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(comp)
        for i in range(2, 2 + steps):
            run(i)
        comp.wait_stream(up)
        comp.wait_stream(down)
        e.record(comp)
        torch.cuda.synchronize()
        return s.elapsed_time(e) / steps
    finally:
        for nm, t in zip(names, sets[0]):
            setattr(runner, nm, t)
        runner.Y = ys[0]


# ------------------------------------------------------------ per-config block
def roofline_entry(runner, gemm_ms, peaks, sustained):
    """GEMM roofline figures for one workload: bound, achieved, peak, frac."""
    int8 = runner.wl.int8
    peak = sparse_peak(peaks, int8, sustained)
    tflops = runner.flops() / (gemm_ms * 1e-3) / 1e12
    gbs = runner.gemm_bytes() / (gemm_ms * 1e-3) / 1e9
    t_tensor = runner.flops() / (peak * 1e12)
    t_hbm = runner.gemm_bytes() / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        return {"bound": "tensor", "achieved": tflops, "peak": peak,
                "unit": "TOPS" if int8 else "TFLOP/s", "frac": tflops / peak}
    return {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"]}


def measure_config(name, device, flush, peaks, steps):
    """Step, GEMM and prune/compress figures of one configured workload (rank 0,
    after the headline run; short runs, so the burst peaks apply)."""
    wl = I.by_name(name)
    runner = Runner(wl, device)
    for _ in range(3):
        flush_l2(flush)
        runner.step()
    torch.cuda.synchronize()
    tot, prune, comp, gemm = time_steps(runner, steps, flush)
    # the GEMM again, five launches back to back in one graph (per launch):
    # how it runs between other kernels of a model, without the event nodes
    # of the stage timing
    b2b_ms = time_graph(lambda: [runner.gemm_call() for _ in range(5)], flush) / 5
    prep_b2b_ms = time_graph(lambda: [runner.prep_call() for _ in range(5)], flush) / 5
    if B.sp24_device_status() != B.SP24_OK:
        raise SystemExit(f"device status not OK after config {name}")
    gemm_ms, comp_ms = statistics.median(gemm), statistics.median(comp)
    plan = B.sp24_gemm_plan(wl.M, wl.N, wl.K, B.SP24_INT8 if wl.int8 else B.SP24_BF16)
    roof = roofline_entry(runner, gemm_ms, peaks, sustained=False)
    c_gbs = runner.compress_bytes() / (comp_ms * 1e-3) / 1e9
    out = {
        "workload": wl.name, "M": wl.M, "N": wl.N, "K": wl.K,
        "dtype": "int8" if wl.int8 else "bf16",
        "step_us": 1e3 * statistics.median(tot),
        "gemm": {"us": 1e3 * gemm_ms, "plan": plan["kernel"],
                 "tflops_dense_equiv": runner.flops() / (gemm_ms * 1e-3) / 1e12,
                 "gbs": runner.gemm_bytes() / (gemm_ms * 1e-3) / 1e9,
                 "bound": roof["bound"], "frac": roof["frac"],
                 "frac_of": ("sparse tensor peak" if roof["bound"] == "tensor" else "HBM") +
                            " (measured burst)",
                 "traffic": gemm_traffic(wl.name, plan["kernel"]),
                 "back_to_back_us": 1e3 * b2b_ms,
                 "frac_back_to_back": roofline_entry(runner, b2b_ms, peaks,
                                                     sustained=False)["frac"]},
        "prune_compress": {"us": 1e3 * comp_ms, "gbs": c_gbs,
                           "frac_hbm": c_gbs / peaks["hbm_gbs"],
                           "prune_us": 1e3 * statistics.median(prune)},
    }
    prep_gbs = runner.prep_bytes() / (prep_b2b_ms * 1e-3) / 1e9
    out["prune_compress"]["back_to_back_us"] = 1e3 * prep_b2b_ms
    out["prune_compress"]["back_to_back_gbs"] = prep_gbs
    out["prune_compress"]["frac_hbm_back_to_back"] = prep_gbs / peaks["hbm_gbs"]
    if wl.int8:
        # INT8: the first stage is the one-pass weight conversion, the second
        # the activation side (scale and quantisation)
        prune_ms = statistics.median(prune)
        p_gbs = runner.prune_bytes() / (prune_ms * 1e-3) / 1e9
        out["prune_compress"]["stages"] = ("prune_us: weight conversion (mask, scales, int8 "
                                           "compression); us: activation scale + quantisation")
        out["prune_compress"]["prune_gbs"] = p_gbs
        out["prune_compress"]["prune_frac_hbm"] = p_gbs / peaks["hbm_gbs"]
        out["prune_compress"]["prep_us"] = 1e3 * (prune_ms + comp_ms)
    del runner
    torch.cuda.empty_cache()
    return out


def time_graph(fn, flush, reps=10):
    """Median CUDA-event time (ms) of one replay of a graph of `fn`, L2
    flushed before each replay."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    ts = []
    for _ in range(reps):
        flush_l2(flush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    del g
    return statistics.median(ts)


def measure_extras(device, flush, peaks):
    """The rows after the path proper: the 3x3 convolution as an implicit GEMM
    against the explicit gather + GEMM (ResNet stage-2 shape, batch 32), and
    the Sparse-QAT forward fake-quantisation of the INT8 workload's weight."""
    from structured_sparse_gemm_sp24_b200 import pipeline as P
    out = {}
    b, h, w, c, cout = 32, 28, 28, 128, 128
    w4 = I.normal_bf16((cout, 3, 3, c), 0.05, 51).to(device)
    x = I.normal_bf16((b, h, w, c), 1.0, 52).to(device)
    vals, meta = P.prune_compress(w4.view(cout, 9 * c), B.SP24_MAGNITUDE)
    a = torch.empty((b * h * w, 9 * c), dtype=torch.bfloat16, device=device)
    y = torch.empty((b * h * w, cout), dtype=torch.bfloat16, device=device)
    yi = torch.empty((b, h, w, cout), dtype=torch.bfloat16, device=device)
    t_imp = time_graph(lambda: B.sp24_conv3x3(x, vals, meta, cout, B.SP24_BF16, None, None,
                                              B.SP24_OUT_BF16, None, yi), flush)
    t_exp = time_graph(lambda: (B.sp24_im2col3x3(x, a),
                                B.sp24_gemm(a, vals, meta, cout, B.SP24_BF16, None, None,
                                            B.SP24_OUT_BF16, None, y)), flush)
    m, k = b * h * w, 9 * c
    flops = 2.0 * m * cout * k
    out["conv3x3"] = {"shape": f"NHWC {b}x{h}x{w}x{c} -> {cout}, 3x3, stride 1, pad 1",
                      "implicit_us": 1e3 * t_imp, "explicit_gather_gemm_us": 1e3 * t_exp,
                      "implicit_tflops_dense_equiv": flops / (t_imp * 1e-3) / 1e12,
                      "speedup_vs_explicit": t_exp / t_imp}
    wl = I.int8_long_tail()
    W = wl.W.to(device)
    mask = P.prune(W, B.SP24_MAGNITUDE, 2)
    s_w = P.wscale(W, mask)
    wfq = torch.empty_like(W)
    t_fq = time_graph(lambda: B.sp24_fake_quant(W, mask, s_w, wfq), flush)
    n, kk = W.shape
    fq_bytes = 2 * n * kk + n * kk / 8 + 4 * n + 2 * n * kk
    out["fake_quant"] = {"shape": f"W {n}x{kk}", "us": 1e3 * t_fq,
                         "gbs": fq_bytes / (t_fq * 1e-3) / 1e9,
                         "frac_hbm": fq_bytes / (t_fq * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    if B.sp24_device_status() != B.SP24_OK:
        raise SystemExit("device status not OK after the extra rows")
    return out


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(wl: I.Workload, budget_s: float):
    """Times the CPU oracle (as it stands) on a bounded sample of the workload
    and extrapolates to one full step.

    Prune + compress run on slices of W rows (64, 128, 256, ... rows, while
    the time stays within 40 % of the budget; pruning is row-independent), the
    GEMM on slices of X rows against the largest pruned W slice (8, 16, 32,
    ... rows, within the rest of the budget).  The full step time is taken as
    t_prune/row * N + t_gemm/(row pair) * M * N.  Returns (dense-equivalent
    flops of one step, extrapolated seconds of one step, description, threads)."""
    from oracle import sp24_oracle as O
    import threadpoolctl

    n, k, m = wl.N, wl.K, wl.M
    xc = wl.Xc.to(torch.float64).numpy() if wl.Xc is not None else None
    mode = O.WANDA if wl.mode == "wanda" else O.MAGNITUDE
    done_w, t_prune, last = 0, 0.0, 0   # rows pruned in all slices, time, largest slice
    vals = meta = s_w = None
    t_last = 0.0
    # the next slice (twice the rows) takes about twice as long: start it only
    # if it still fits 40 % of the budget
    while last < n and (last == 0 or t_prune + 2.0 * t_last < 0.4 * budget_s):
        r = min(2 * last if last else 64, n)
        w = wl.W[:r].to(torch.float64).numpy()
        t0 = time.perf_counter()
        if wl.int8:
            keep = O.prune(w, O.MAGNITUDE, 2)
            s_w = O.channel_scales(w, keep)
            vals, meta = O.compress(O.quantize(w, s_w[:, None]), keep)
        else:
            keep = O.progressive(w, mode, xc)[1] if wl.progressive else O.prune(w, mode, 2, xc=xc)
            vals, meta = O.compress(w, keep)
        t_last = time.perf_counter() - t0
        t_prune += t_last
        done_w += r
        last = r
    def gemm_rows(r):
        if wl.int8:
            x = wl.X[:r].numpy()
            s_x = O.tensor_scale(x)   # per-sample scale: same arithmetic, bounded cost
            acc = O.gemm_int8_acc(O.quantize(x, s_x), vals, meta, k)
            O.dequant_bf16(acc, s_x, s_w)
        else:
            O.gemm(wl.X[:r].to(torch.float64).numpy(), vals, meta, k)

    # a probe of 16 rows sizes one call that fills the rest of the budget (the
    # oracle rebuilds the dense weight on every call, so one large call is
    # timed rather than many small ones)
    r = min(16, m)
    t1 = time.perf_counter()
    gemm_rows(r)
    t_probe = time.perf_counter() - t1
    x_rows, t_gemm = r, t_probe
    left = budget_s - t_prune - t_probe
    if x_rows < m and left > 0:
        r = int(min(m, max(16, left / max(t_probe, 1e-9) * 16)))
        t1 = time.perf_counter()
        gemm_rows(r)
        x_rows, t_gemm = r, time.perf_counter() - t1
    step_s = t_prune / done_w * n + t_gemm / (x_rows * last) * m * n
    cores = None
    for info in threadpoolctl.threadpool_info():
        cores = max(cores or 0, int(info.get("num_threads", 0)))
    full = x_rows >= m and last >= n
    sample = (f"prune+compress of W row slices up to {last} of {n} rows ({done_w} rows, "
              f"{t_prune:.2f}s) + GEMM of {x_rows} of {m} X rows x {last} W rows "
              f"({t_gemm:.2f}s); "
              + ("the whole step, time per row" if full else "step time extrapolated by rows"))
    return 2.0 * m * n * k, step_s, sample, cores or os.cpu_count()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = I.by_name(args.workload)
    per_step = []
    sample = ""
    cores = os.cpu_count()
    budget = max(0.3, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        flops, secs, sample, cores = oracle_sample(wl, budget)
        if i >= args.warmup:
            per_step.append((flops, secs))
    flops = sum(f for f, _ in per_step)
    secs = sum(s for _, s in per_step)
    value = flops / secs / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / max(1, len(per_step)), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, args.gpus),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------- main
def run_permute_search(args):
    """Times the channel permutation search on the workload's weight shape
    (channel-scaled synthetic weights, magnitude scores, keep 2 of 4): CUDA
    events on the stream around the whole blocking call, set-up included.
    Prints one JSON line."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    B.lib()
    from structured_sparse_gemm_sp24_b200 import pipeline as P
    wl = I.by_name(args.workload)
    n, k = wl.W.shape
    w = I.channel_scaled_bf16((n, k), 0.02, 5).to(device)
    limit = args.permute_max_swaps if args.permute_max_swaps is not None else 64 * k
    for _ in range(args.warmup):
        perm, res = P.permute_search(w, 2, None, limit)
    times = []
    for _ in range(args.steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        perm, res = P.permute_search(w, 2, None, limit)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    if B.sp24_device_status() != B.SP24_OK:
        raise SystemExit("device status not OK after the permutation search")
    ms = statistics.median(times)
    swaps = int(res["swaps"])
    line = {
        "metric": "channel permutation search time", "value": round(ms, 3), "unit": "ms",
        "higher_is_better": False, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "dtype": "int32/int64", "data": "synthetic",
        "config": {"workload": f"{args.workload}_weight_permute", "N": n, "K": k, "n_keep": 2,
                   "max_swaps": limit, "weights": "channel_scaled_bf16 sigma 0.02 seed 5"},
        "swaps": swaps, "us_per_swap": round(1e3 * ms / max(swaps, 1), 2),
        "kept_gain_pct": round(100.0 * (res["kept_after"] / max(res["kept_before"], 1) - 1), 4),
        "converged": swaps < limit,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sp24", choices=["sp24", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration block after the headline")
    ap.add_argument("--config-steps", type=int, default=20,
                    help="timed steps per configuration in the `configs` block")
    ap.add_argument("--no-graph", action="store_true",
                    help="time plain launches instead of a CUDA-graph replay of the step")
    ap.add_argument("--permute-search", action="store_true",
                    help="time the channel permutation search on the workload's weight shape")
    ap.add_argument("--permute-max-swaps", type=int, default=None)
    args = ap.parse_args(argv)
    if args.permute_search:
        return run_permute_search(args)
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return run_reference(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    B.lib()

    wl = I.by_name(args.workload)
    runner = Runner(wl, device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    for _ in range(args.warmup):
        flush_l2(flush)
        runner.step()
    torch.cuda.synchronize()
    if B.sp24_device_status() != B.SP24_OK:
        raise SystemExit("device status not OK after warm-up")

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    counted = count_step_kernels(runner)
    step_kernels = counted if counted is not None else runner.launches_per_step()
    if counted is not None and counted != runner.launches_per_step():
        print(f"bench: step graph holds {counted} kernels, expected "
              f"{runner.launches_per_step()}", file=sys.stderr)
    barrier()
    with ClockSampler(local) as clk, nvtx_range(f"sp24 timed steps: {wl.name}"):
        tot, prune, comp, gemm = time_steps(runner, args.steps, flush,
                                            use_graph=not args.no_graph, stage_steps=50)
    barrier()
    total_ms = max_over_ranks(sum(tot), device)
    ms_per_step = total_ms / args.steps
    value = job_tflops(world, args.steps, runner.flops(), total_ms)

    e2e_steps = max(3, min(args.steps, 50 if wl.N * wl.K < (1 << 26) else 10))
    with nvtx_range("sp24 end to end (serial, then pipelined)"):
        serial_ms, h2d, d2h = time_e2e(runner, e2e_steps)
        e2e_ms = time_e2e_pipelined(runner, e2e_steps)
    serial_ms = max_over_ranks(serial_ms, device)
    e2e_ms = max_over_ranks(e2e_ms, device)
    e2e_value = job_tflops(world, 1, runner.flops(), e2e_ms)
    e2e_serial_value = job_tflops(world, 1, runner.flops(), serial_ms)
    if B.sp24_device_status() != B.SP24_OK:
        raise SystemExit("device status not OK after timing")

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    peaks = load_peaks()
    gemm_ms = statistics.mean(gemm)
    comp_ms = statistics.mean(comp)
    prune_ms = statistics.mean(prune)
    # the step runs back to back for about a second or more: the GEMM is a
    # kernel timed inside a long step, so its primary denominator is the
    # sustained (power-capped) peak; the burst fraction is reported beside it
    roof = roofline_entry(runner, gemm_ms, peaks, sustained=True)
    burst = roofline_entry(runner, gemm_ms, peaks, sustained=False)
    roof["frac_of_burst_peak"] = burst["frac"]
    roof["burst_peak"] = burst["peak"]
    roof["peak_source"] = (f"{peaks['source']}: {'4' if wl.int8 else '2'}x dense bf16 "
                           "sustained (burst beside it)")
    plan = B.sp24_gemm_plan(wl.M, wl.N, wl.K, B.SP24_INT8 if wl.int8 else B.SP24_BF16)
    roof["traffic"] = gemm_traffic(wl.name, plan["kernel"])
    roof["algorithmic_bytes"] = runner.gemm_bytes()
    roof["kernel"] = "sp24 gemm " + plan["kernel"]
    roof["plan"] = plan
    c_gbs = runner.compress_bytes() / (comp_ms * 1e-3) / 1e9

    cfg = workload_config(wl, world)
    cfg["timing"] = ("plain launches" if args.no_graph else
                     "step: CUDA graph of one step; stages: 50 steps, event nodes between "
                     "stages (about 2 us each)")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8" if wl.int8 else "bf16", "data": "synthetic",
        "config": cfg,
        "gemm": {"ms": gemm_ms, "tflops_dense_equiv": runner.flops() / (gemm_ms * 1e-3) / 1e12,
                 "gbs": runner.gemm_bytes() / (gemm_ms * 1e-3) / 1e9,
                 "frac_sparse_peak_sustained": roof["frac"],
                 "frac_sparse_peak_burst": burst["frac"]},
        "prune_compress": {"ms": comp_ms, "gbs": c_gbs, "frac_hbm": c_gbs / peaks["hbm_gbs"],
                           "prune_ms": prune_ms},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "pipelined": "copies up and down on their own streams, overlapping the "
                             "neighbouring steps' compute",
                "serial_value": e2e_serial_value,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": step_kernels * args.steps,
        "clocks": clk.summary(),
    }
    del runner
    torch.cuda.empty_cache()
    if world == 1 and not args.no_configs:
        with nvtx_range("sp24 configured workloads"):
            line["configs"] = [measure_config(n, device, flush, peaks, args.config_steps)
                               for n in CONFIG_WORKLOADS if n != wl.name]
        with nvtx_range("sp24 extra rows"):
            line["extras"] = measure_extras(device, flush, peaks)
    if world == 1 and not args.no_cpu_baseline:
        flops, secs, sample, cores = oracle_sample(wl, args.cpu_budget)
        line["cpu_baseline"] = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle", "sample": sample}
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
