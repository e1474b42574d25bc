#!/usr/bin/env python
"""Benchmark of the virtual-rank all-reduce on one B200 (or N independent replicas).

One step = one all-reduce call (VRAR_ALGO_AUTO: the per-size selector plus the
kernel it picks) over one batch of synthetic input: P = 8 virtual ranks, a
prefill-shaped message of 16,384 tokens x hidden 7168 bf16 (224 MiB per rank,
1.88 GB of inputs over the 8 ranks), values N(0, 0.02), seed 0: the largest
workload that fits one GPU, a 16k-token prefill at 8-way tensor parallelism.

Timing: W warm-up steps, then EXACTLY K steps captured as one CUDA graph. The
graph is replayed R times; each replay is bracketed by a barrier and a device
synchronise and timed with CUDA events on the launching stream, and the
reported time per step is the median replay divided by K. Every step reads
1.88 GB of inputs and writes 1.88 GB of outputs, far more than the 126 MB L2,
so every step reads its inputs from HBM (smaller shapes rotate through buffer
sets whose total is more than 3x the L2 size). busbw = algbw * 2(P-1)/P with
algbw = n * bytes-per-element / t (the nccl-tests convention). The roofline
fraction uses the algorithm-independent minimum traffic B_min = 2 * P * n * s
(every input read once, every output written once) against the measured HBM
copy bandwidth.

Other keys: e2e (same metric with the inputs copied from pinned host memory
and the outputs copied back inside the timed region), cpu_baseline (the CPU
oracle on one pinned host core, on a contiguous slice of the workload),
per_algo (each algorithm on the step's workload) and sweep (the other
workload shapes and sizes: the decode message of 64 tokens x 8192 with its
warm-L2 and start/end-barrier rows, 128 KiB - 2 MiB per rank with recursive
doubling timed over graphs of 1000 calls, 2 ranks of small integers, 32 ranks
as 4 groups of 8, fp16 and fp32 partials on the wire).

--impl reference times the CPU oracle instead (the only reference that exists
for this method), on bounded slices of the same workload.

Multi-GPU: replicas only. Each rank runs the same single-GPU workload on its
own device; the time is the maximum over ranks and value sums all ranks' work.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "all-reduce busbw GB/s & % of HBM roofline vs size, P virtual ranks, 1 B200"
UNIT = "GB/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0

WORKLOAD = dict(name="prefill 16384x7168 bf16, P=8 virtual ranks (224 MiB per rank), N(0,0.02), seed 0",
                key="prefill_p8_224mib", P=8, n=16384 * 7168, dtype="bf16", dist="normal:0,0.02", seed=0)
DECODE = dict(name="decode 64x8192 bf16, P=8 virtual ranks (1 MiB per rank), N(0,1), seed 0",
              P=8, n=64 * 8192, dtype="bf16", dist="normal:0,1", seed=0)

HEADLINE_REPLAYS = 15   # replays of the K-step graph; the median is reported
SWEEP_REPLAYS = 5
RD_CALLS = 1000         # recursive doubling rows: graphs of 1000 back-to-back calls (flag reuse)
PER_ALGO_STEPS = 10     # graph length of the per-algorithm rows on the headline workload

SWEEP = (
    [dict(DECODE, algos=("oneshot", "twostage", "twostage_write", "rd", "auto"), collectives=("rs", "ag"),
          warm=("auto", "oneshot", "twostage", "twostage_write", "rd"),
          edge=("oneshot", "twostage_write"), fp8=("oneshot", "twostage", "twostage_write"))]
    + [dict(name=f"P=8 sweep {b >> 10} KiB per rank, N(0,1)", P=8, n=b // 2, dtype="bf16", dist="normal:0,1",
            algos=("oneshot", "twostage", "twostage_write", "rd", "auto"), collectives=("rs", "ag"),
            edge=("oneshot", "twostage_write") if b == 2 << 20 else (),
            fp8=("oneshot", "twostage_write") if b == 2 << 20 else ())
       for b in (128 << 10, 256 << 10, 512 << 10, 2 << 20)]
    + [dict(name="P=2 ints 128 KiB per rank", P=2, n=65536, dtype="bf16", dist="int8",
            algos=("oneshot", "rd", "auto"))]
    + [dict(name=f"P=32 hier 4x8 {b >> 10} KiB per rank, uniform(-1,1)", P=32, n=b // 2, dtype="bf16",
            dist="uniform:-1,1", L=8, algos=("hier", "oneshot", "twostage_write", "auto")) for b in
       (256 << 10, 2 << 20)]
    + [dict(name=f"P=8 fp16 {b >> 10} KiB per rank, N(0,1)", P=8, n=b // 2, dtype="fp16", dist="normal:0,1",
            algos=("oneshot", "twostage_write", "rd", "auto")) for b in (1 << 20, 2 << 20)]
    + [dict(name=f"P=8 bf16 {b >> 10} KiB per rank, N(0,1), RD with fp32 partials on the wire", P=8, n=b // 2,
            dtype="bf16", dist="normal:0,1", algos=("rd",), wire="fp32") for b in (128 << 10, 2 << 20)]
    + [dict(name="P=32 hier 4x8 2048 KiB per rank, uniform(-1,1), fp32 partials on the wire", P=32,
            n=(2 << 20) // 2, dtype="bf16", dist="uniform:-1,1", L=8, algos=("hier",), wire="fp32")]
)

# The oracle algorithm the reference arm times: the same summation the GPU
# path's choice for the workload computes (the three custom all-reduce variants
# share one order, so any of them gives the same bits).
REFERENCE_ALGO = "twostage_write"
REFERENCE_SAMPLE = 1 << 21  # elements per rank of each reference step (4 MiB of bf16)

TDT = {"bf16": torch.bfloat16, "fp32": torch.float32, "fp16": torch.float16}
ESZ = {"bf16": 2, "fp32": 4, "fp16": 2}


# ---- small helpers (host logic; tested on the CPU) ---------------------------------------------

def busbw_gbs(P: int, n: int, esz: int, seconds: float) -> float:
    """nccl-tests bus bandwidth of one all-reduce of n elements per rank."""
    if seconds <= 0:
        return float("nan")
    return n * esz / seconds * (2.0 * (P - 1) / P if P > 1 else 1.0) / 1e9


def b_min_bytes(P: int, n: int, esz: int) -> int:
    """Minimum HBM traffic of one all-reduce: every input read once, every output written once."""
    return 2 * P * n * esz


def b_alg_bytes(algo: str, P: int, n: int, esz: int, L: int = 8, fp32_wire: bool = False) -> int:
    """Bytes an algorithm's own loads and stores ask for (each input and output
    counted at every access; repeat reads may hit L2). One-shot: every rank
    reads all P inputs, (P^2 + P) n s. Two-stage pull: (3P - 1) n s. Write mode:
    2 P n s. Recursive doubling: inputs and outputs plus, per step, every rank's
    payload words written and read, 2 n s each way ({32 data bits | 32-bit
    sequence} per 8 bytes; fp32 partials of 16-bit data double that). HIER:
    2 P n s plus the same payload traffic on 1/L of the data over log2(P/L)
    steps."""
    wire = 2 if (fp32_wire and esz == 2) else 1
    if algo == "oneshot":
        return (P * P + P) * n * esz
    if algo == "twostage":
        return (3 * P - 1) * n * esz
    if algo == "twostage_write":
        return 2 * P * n * esz
    if algo == "rd":
        return P * n * esz * (2 + 4 * wire * int(math.log2(P)))
    if algo == "hier":
        return int((2 * P + 4 * wire * math.log2(P // L) * P / L) * n * esz)
    raise ValueError(algo)


def rotation_sets(set_bytes: int, l2_bytes: int = L2_BYTES, cap: int = 64) -> int:
    """Buffer sets to rotate through so that the total exceeds 3x the L2 size."""
    return max(1, min(cap, math.ceil(3 * l2_bytes / max(1, set_bytes))))


def load_peaks(path: str = os.path.join(ROOT, "MEASURED_PEAKS.json")):
    """The measured HBM copy bandwidth (GB/s): the first numeric "hbm_gbs" in
    the file, at the top level or nested; else the fallback."""
    def find(d):
        if isinstance(d, dict):
            v = d.get("hbm_gbs")
            if isinstance(v, (int, float)) and v > 0:
                return float(v)
            for x in d.values():
                r = find(x)
                if r:
                    return r
        elif isinstance(d, list):
            for x in d:
                r = find(x)
                if r:
                    return r
        return None
    try:
        with open(path) as f:
            v = find(json.load(f))
        if v:
            return v, "measured"
    except Exception:
        pass
    return FALLBACK_HBM_GBS, "fallback"


def parse_clocks_csv(text: str):
    """Median SM clock under load, the max clock and the throttle reasons seen."""
    rows = [r.strip() for r in text.splitlines() if r.strip() and not r.startswith("index")]
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        f = [c.strip() for c in r.split(",")]
        if len(f) < 9:
            continue
        try:
            cur = float(f[1].split()[0])
            mx = float(f[2].split()[0])
            pw = float(f[3].split()[0]) if f[3].split()[0] not in ("[N/A]", "N/A") else 0.0
        except ValueError:
            continue
        smax.append(mx)
        if pw > 150.0 or cur > 0.6 * mx:  # under load
            sm.append(cur)
        for name, val in zip(names, f[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons), "samples_under_load": len(sm), "samples": len(rows)}


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index  # nvidia-smi -i target: PCI bus id or index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}", "--format=csv,noheader",
                 "-lms", "50"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvidia-smi unavailable"}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        with open(self.file.name) as f:
            text = f.read()
        os.unlink(self.file.name)
        return parse_clocks_csv(text)


def gpu_bus_id(device, fallback):
    """PCI bus id of a torch device in nvidia-smi's form (CUDA ordinals and
    nvidia-smi indices need not agree)."""
    try:
        p = torch.cuda.get_device_properties(device)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return str(fallback)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank number over all ranks (a timing reduction, not data)."""
    if world <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index] if device is not None and device.type == "cuda" else None)


def source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "collective_all_reduce_virtual_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, or None when there is none or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None, None
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != source_hash():
        return None, None
    return e.get("dram_bytes_per_launch"), e.get("summary")


# ---- GPU timing -------------------------------------------------------------------------------

class Workload:
    """Rotating device buffer sets holding the same seeded inputs."""

    def __init__(self, spec, device, rotate=True):
        import collective_all_reduce_virtual_b200 as vrar
        self.vrar = vrar
        self.spec = spec
        self.P, self.n, self.dt = spec["P"], spec["n"], spec["dtype"]
        self.esz = ESZ[self.dt]
        dist = synth.parse_dist(spec["dist"])
        gen_dev = device if self.n * self.P >= (1 << 24) else "cpu"
        base = synth.make_inputs(self.P, self.n, TDT[self.dt], dist, seed=spec.get("seed", 0), device=gen_dev,
                                 block=1 << 25)
        self.base = [t.to(device) for t in base]
        set_bytes = b_min_bytes(self.P, self.n, self.esz)
        self.R = rotation_sets(set_bytes) if rotate else 1
        self.ins = [self.base] + [[t.clone() for t in self.base] for _ in range(self.R - 1)]
        self.outs = [[torch.empty_like(t) for t in self.base] for _ in range(self.R)]
        self.in_arr = [vrar.ptr_array([t.data_ptr() for t in s]) for s in self.ins]
        self.out_arr = [vrar.ptr_array([t.data_ptr() for t in s]) for s in self.outs]
        self.lib = vrar.lib()
        self.dtc = vrar.DTYPES[TDT[self.dt]]
        self.small = None

    def call(self, i: int, algo: str, stream_handle: int):
        r = i % self.R
        rc = self.lib.vrar_allreduce(self.in_arr[r], self.out_arr[r], self.P, self.n, self.dtc,
                                     self.vrar.ALGOS[algo], stream_handle)
        if rc != 0:
            raise self.vrar.VrarError(rc, f"vrar_allreduce({algo})")

    def graph(self, algo: str, count: int, offset: int = 0):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            h = torch.cuda.current_stream().cuda_stream
            for i in range(count):
                self.call(offset + i, algo, h)
        return g

    def collective_call(self, i: int, kind: str, stream_handle: int):
        """Standalone reduce-scatter ('rs': inputs -> n/P slices) or all-gather
        ('ag': n/P slices -> outputs) on this workload's buffer set i % R."""
        if self.small is None:
            m = self.n // self.P
            self.small = [[torch.empty(m, dtype=self.base[0].dtype, device=self.base[0].device)
                           for _ in range(self.P)] for _ in range(self.R)]
            self.small_arr = [self.vrar.ptr_array([t.data_ptr() for t in s]) for s in self.small]
        r = i % self.R
        if kind == "rs":
            rc = self.lib.vrar_reduce_scatter(self.in_arr[r], self.small_arr[r], self.P, self.n, self.dtc,
                                              stream_handle)
        else:
            rc = self.lib.vrar_all_gather(self.small_arr[r], self.out_arr[r], self.P, self.n, self.dtc,
                                          stream_handle)
        if rc != 0:
            raise self.vrar.VrarError(rc, kind)

    def free(self):
        self.ins = self.outs = self.base = self.small = None


def upload_graph(g) -> bool:
    """Move an instantiated graph to the device ahead of its first launch, so
    that the timed replay does not include the one-time upload."""
    try:
        from cuda.bindings import driver as cu
        (err,) = cu.cuGraphUpload(cu.CUgraphExec(g.raw_cuda_graph_exec()),
                                  cu.CUstream(torch.cuda.current_stream().cuda_stream))
        torch.cuda.synchronize()
        return int(err) == 0
    except Exception:
        return False


def time_graph(g, world=1, device=None, replays: int = 1) -> float:
    """Milliseconds of one replay of a captured graph: the median of `replays`
    replays, each bracketed by a barrier and a device synchronise and timed
    with CUDA events on the launching stream."""
    upload_graph(g)
    s = torch.cuda.current_stream()
    times = []
    for _ in range(max(1, replays)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world, device)
        torch.cuda.synchronize()
        e0.record(s)
        g.replay()
        e1.record(s)
        e1.synchronize()
        torch.cuda.synchronize()
        barrier(world, device)
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def measure_algo(wl: Workload, algo: str, steps: int, warmup: int, world=1, device=None, replays: int = 1):
    """Milliseconds per call: a graph of `warmup` calls replayed once, then a
    graph of `steps` calls timed over `replays` replays (median), max over ranks."""
    wl.call(0, algo, torch.cuda.current_stream().cuda_stream)  # sizes the workspace outside capture
    torch.cuda.synchronize()
    gw = wl.graph(algo, warmup)
    gt = wl.graph(algo, steps, offset=warmup)
    gw.replay()
    torch.cuda.synchronize()
    ms = max_over_ranks(time_graph(gt, world, device, replays), world, device)
    rc, info = wl.vrar.query_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} {info} after {algo}")
    del gw, gt
    return ms / steps


def measure_collective(wl: Workload, kind: str, steps: int, warmup: int, world=1, device=None, replays: int = 1):
    """Milliseconds per call of the standalone reduce-scatter ('rs') or
    all-gather ('ag') on the workload's shape (graph of `steps` calls)."""
    wl.collective_call(0, kind, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()

    def graph(count, offset):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            h = torch.cuda.current_stream().cuda_stream
            for i in range(count):
                wl.collective_call(offset + i, kind, h)
        return g

    gw, gt = graph(warmup, 0), graph(steps, warmup)
    gw.replay()
    torch.cuda.synchronize()
    ms = max_over_ranks(time_graph(gt, world, device, replays), world, device)
    del gw, gt
    return ms / steps


class nvtx:
    """An NVTX range around a phase of the benchmark (visible in profilers)."""

    def __init__(self, name: str):
        self.name = name

    def __enter__(self):
        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        torch.cuda.nvtx.range_pop()


def entry(wl: Workload, t_s: float, peak: float, algo: str):
    """One timing: busbw, and the fraction of the measured HBM bandwidth on
    B_min (algorithm-independent) and on B_alg (the algorithm's own traffic)."""
    bw = busbw_gbs(wl.P, wl.n, wl.esz, t_s)
    ach = b_min_bytes(wl.P, wl.n, wl.esz) / t_s / 1e9
    if algo == "auto":
        algo = wl.vrar.select_algo(wl.P, wl.n, TDT[wl.dt])
    b_alg = b_alg_bytes(algo, wl.P, wl.n, wl.esz, wl.spec.get("L", 8), wl.spec.get("wire") == "fp32")
    return {"us": round(t_s * 1e6, 3), "algbw_gbs": round(wl.n * wl.esz / t_s / 1e9, 1), "busbw_gbs": round(bw, 1),
            "hbm_gbs_bmin": round(ach, 1), "frac_bmin": round(ach / peak, 4),
            "frac_alg": round(b_alg / t_s / 1e9 / peak, 4)}


def measure_e2e(wl: Workload, algo: str, steps: int, warmup: int, world=1, device=None):
    """Every step copies its P inputs from pinned host memory to the device,
    runs the all-reduce through the public binding (the C ABI), and copies its
    P outputs back to pinned host memory. Steps are pipelined the way a user
    streaming batches would: copies in (one stream), the all-reduce (another)
    and copies out (a third) of consecutive steps overlap, on two device buffer
    sets; the host link carries both directions at once."""
    vrar = wl.vrar
    # The P rank buffers of a set are rows of one [P, n] block, so that a step
    # moves its inputs in one copy and its outputs out in one copy.
    dev = wl.base[0].device
    shape, dtype = (wl.P, wl.n), wl.base[0].dtype
    h_in = torch.empty(shape, dtype=dtype, pin_memory=True)
    for p, t in enumerate(wl.base):
        h_in[p].copy_(t)
    # One host output block: the copies out are ordered on their own stream,
    # and nothing reads the host copy inside the timed region.
    h_out = torch.empty(shape, dtype=dtype, pin_memory=True)
    sets = 2
    d_in_blk = [torch.empty(shape, dtype=dtype, device=dev) for _ in range(sets)]
    d_out_blk = [torch.empty(shape, dtype=dtype, device=dev) for _ in range(sets)]
    d_in = [list(blk.unbind(0)) for blk in d_in_blk]
    d_out = [list(blk.unbind(0)) for blk in d_out_blk]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    run_done = [ev(), ev()]
    out_done = [ev(), ev()]
    for e in run_done + out_done:
        e.record(torch.cuda.current_stream())

    def step(i):
        b = i % sets
        s_in.wait_event(run_done[b])          # the step two back has read these inputs
        with torch.cuda.stream(s_in):
            d_in_blk[b].copy_(h_in, non_blocking=True)
        in_done = ev()
        in_done.record(s_in)
        s_run.wait_event(in_done)
        s_run.wait_event(out_done[b])         # the step two back has copied these outputs out
        vrar.all_reduce(d_in[b], d_out[b], algo=algo, stream=s_run)
        run_done[b].record(s_run)
        s_out.wait_event(run_done[b])
        with torch.cuda.stream(s_out):
            h_out.copy_(d_out_blk[b], non_blocking=True)
        out_done[b].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    e1.record(s_out)
    e1.synchronize()
    torch.cuda.synchronize()
    barrier(world, device)
    ms = max_over_ranks(e0.elapsed_time(e1), world, device) / steps
    # The last step's outputs are on the host: check one rank against another.
    if not torch.equal(h_out[0].view(torch.int16), h_out[wl.P - 1].view(torch.int16)):
        raise RuntimeError("e2e: rank outputs differ after the copy back")
    bytes_in = h_in.numel() * h_in.element_size()
    bytes_out = h_out.numel() * h_out.element_size()
    del d_in_blk, d_out_blk, d_in, d_out, h_in, h_out
    return ms, bytes_in, bytes_out


# ---- CPU oracle timing ----------------------------------------------------------------------------

def host_description() -> dict:
    """Host facts reported beside the CPU oracle's time."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        allowed = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        allowed = None
    return {"nproc": os.cpu_count(), "cpus_allowed": allowed, "cpu_model": model}


class one_core:
    """Pin this process to one of its allowed cores for the duration (the
    oracle is single-threaded; pinning keeps it from migrating)."""

    def __enter__(self):
        self.old = None
        self.core = None
        try:
            self.old = os.sched_getaffinity(0)
            self.core = min(self.old)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            self.old = None
        return self

    def __exit__(self, *exc):
        if self.old is not None:
            os.sched_setaffinity(0, self.old)

    def describe(self) -> str:
        return f"os.sched_setaffinity to core {self.core}" if self.core is not None else "not pinned"


def oracle_inputs(spec, n_sample: int, device=None):
    """The first n_sample elements of every rank's input of the workload (the
    counter-based generator gives the same values as the full-size buffers),
    as numpy arrays for the oracle."""
    P, dt = spec["P"], spec["dtype"]
    m = min(spec["n"], n_sample)
    xs = synth.make_inputs(P, m, TDT[dt], synth.parse_dist(spec["dist"]), seed=spec.get("seed", 0),
                           device=device or "cpu", block=1 << 24)
    return [t.cpu().view(torch.int16).numpy().view(np.uint16) if dt != "fp32" else t.cpu().numpy() for t in xs], m


def oracle_samples(spec, algo: str, min_seconds: float, n_sample: int, device=None):
    """Time the CPU oracle, pinned to one core, on a contiguous slice of
    n_sample elements per rank of the workload; returns (seconds per full-size
    call scaled by n / n_sample, calls, sample text, host facts)."""
    import oracle
    P, n, dt = spec["P"], spec["n"], spec["dtype"]
    xs, m = oracle_inputs(spec, n_sample, device)
    L = spec.get("L", 8)
    oracle.allreduce(algo, xs, dt, L=L)  # builds/loads the library outside the timing
    with one_core() as pin:
        calls, t0 = 0, time.perf_counter()
        while True:
            oracle.allreduce(algo, xs, dt, L=L)
            calls += 1
            el = time.perf_counter() - t0
            if el >= min_seconds:
                break
    per_call = el / calls * (n / m)
    sample = f"{calls} oracle calls of '{algo}' on {P} x {m} {dt} elements" + \
             ("" if m == n else f" (the first {m} elements of every rank; time scaled by {n}/{m})")
    return per_call, calls, sample, dict(host_description(), affinity=pin.describe(), threads=1)


# ---- arms -------------------------------------------------------------------------------------------

def with_flags(algo: str):
    """'twostage_write+edge+fp8' -> ('twostage_write', edge=True, fp8=True): the
    algorithm with the start/end barriers and / or the fp8 payloads on."""
    parts = algo.split("+")
    return parts[0], "edge" in parts[1:], "fp8" in parts[1:]


class flags_set:
    """Turn the settings a row's suffixes name on for its capture (a graph keeps
    the settings its calls were queued with), and back off after."""

    def __init__(self, vrar, algo):
        self.vrar, (self.base, self.edge, self.fp8) = vrar, with_flags(algo)

    def __enter__(self):
        self.vrar.set_edge_sync(self.edge)
        self.vrar.set_fp8_quant(self.fp8)
        return self.base

    def __exit__(self, *exc):
        self.vrar.set_edge_sync(False)
        self.vrar.set_fp8_quant(False)


def measure_row(vrar, w: Workload, algo: str, steps: int, warmup: int, world, device, replays: int):
    with flags_set(vrar, algo) as base:
        return measure_algo(w, base, steps, warmup, world, device, replays)


def spin_row(vrar, w: Workload, algo: str, calls: int) -> dict:
    """Spin statistics of the waits of `calls` calls (a separate, instrumented
    graph: the counters cost a few atomics per warp and wait, so the timed rows
    run without them)."""
    with flags_set(vrar, algo) as base:
        vrar.set_spin_stats(True)
        try:
            w.call(0, base, torch.cuda.current_stream().cuda_stream)
            torch.cuda.synchronize()
            g = w.graph(base, calls)
            vrar.get_spin_stats(reset=True)
            g.replay()
            torch.cuda.synchronize()
        finally:
            vrar.set_spin_stats(False)
    st = vrar.get_spin_stats(reset=True)
    rc, _ = vrar.query_status()
    del g
    return {"calls": calls, "status": rc, **st}


def run_vrar(args):
    import collective_all_reduce_virtual_b200 as vrar

    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    peak, peak_src = load_peaks()

    clocks = ClockSampler(gpu_bus_id(device, local)).start()
    time.sleep(0.3)
    wl = Workload(WORKLOAD, device)
    algo_auto = vrar.select_algo(wl.P, wl.n, TDT[wl.dt])

    # The timed steps: exactly K AUTO calls per graph replay, median of R replays.
    with nvtx("timed steps"):
        t_step_ms = measure_algo(wl, "auto", args.steps, args.warmup, world, device, args.replays)
    t_s = t_step_ms / 1e3

    # e2e through the public call with host buffers.
    with nvtx("e2e"):
        e2e_ms, h2d, d2h = measure_e2e(wl, "auto", max(3, min(args.steps, 50)), args.warmup, world, device)

    per_algo = {}
    if not args.quick:
        for algo in ("oneshot", "twostage", "twostage_write", "rd", "twostage_write+fp8", "oneshot+fp8"):
            per_algo[algo] = entry(wl, measure_row(vrar, wl, algo, PER_ALGO_STEPS, 3, world, device, 3) / 1e3,
                                   peak, with_flags(algo)[0])
        for kind in ("rs", "ag"):
            t = measure_collective(wl, kind, PER_ALGO_STEPS, 3, world, device, 3) / 1e3
            ach = (wl.P + 1) * wl.n * wl.esz / t / 1e9  # (P + 1) n s either way
            per_algo["reduce_scatter" if kind == "rs" else "all_gather"] = {
                "us": round(t * 1e6, 3), "hbm_gbs": round(ach, 1), "frac": round(ach / peak, 4)}
    wl.free()
    del wl
    torch.cuda.empty_cache()

    sweep = []
    if not args.quick:
        for spec in SWEEP:
            if spec.get("L"):
                vrar.set_group_size(spec["L"])
            vrar.set_payload_wire(spec.get("wire", "element"))
            w = Workload(spec, device)
            row = {"workload": spec["name"], "P": w.P, "n": w.n, "rotating_sets": w.R,
                   "selected": vrar.select_algo(w.P, w.n, TDT[w.dt]),
                   "kernel": vrar.kernel_name(w.P, w.n, TDT[w.dt], "auto")}
            for algo in spec["algos"]:
                k = RD_CALLS if algo == "rd" else spec.get("steps", 200)
                row[algo] = entry(w, measure_algo(w, algo, k, 3, world, device, SWEEP_REPLAYS) / 1e3, peak, algo)
                if algo == "rd":
                    row[algo]["calls_per_graph"] = k
            for algo in spec.get("edge", ()):
                key = f"{algo}+edge"
                row[key] = entry(w, measure_row(vrar, w, key, 200, 3, world, device, SWEEP_REPLAYS) / 1e3, peak,
                                 algo)
                row[key]["spin"] = spin_row(vrar, w, key, 1000)
            for algo in spec.get("fp8", ()):
                key = f"{algo}+fp8"
                row[key] = entry(w, measure_row(vrar, w, key, 200, 3, world, device, SWEEP_REPLAYS) / 1e3, peak,
                                 algo)
            for kind in spec.get("collectives", ()):
                # RS moves P*n*s in and n*s out; AG n*s in and P*n*s out: (P+1)*n*s either way.
                t = measure_collective(w, kind, spec.get("steps", 200), 3, world, device, SWEEP_REPLAYS) / 1e3
                ach = (w.P + 1) * w.n * w.esz / t / 1e9
                row["reduce_scatter" if kind == "rs" else "all_gather"] = {
                    "us": round(t * 1e6, 3), "hbm_gbs": round(ach, 1), "frac": round(ach / peak, 4)}
            w.free()
            if spec.get("warm"):
                # The same buffers every call: the working set stays in L2. Beside the
                # cold numbers, never the headline.
                ww = Workload(spec, device, rotate=False)
                row["warm_l2"] = {a: entry(ww, measure_algo(ww, a, 200, 3, world, device, SWEEP_REPLAYS) / 1e3,
                                           peak, a) for a in spec["warm"]}
                ww.free()
            torch.cuda.empty_cache()
            vrar.set_group_size(8)
            vrar.set_payload_wire("element")
            if "wire" in spec:
                row["wire"] = spec["wire"]
            sweep.append(row)
    clk = clocks.stop()

    P, n, esz = WORKLOAD["P"], WORKLOAD["n"], ESZ[WORKLOAD["dtype"]]
    value = world * busbw_gbs(P, n, esz, t_s)
    achieved = b_min_bytes(P, n, esz) / t_s / 1e9
    kernel = vrar.kernel_name(P, n, TDT[WORKLOAD["dtype"]], "auto")
    traffic, traffic_src = profiled_traffic(kernel, WORKLOAD["key"])

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_step_ms, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD["name"], "P": P, "n": n, "algo": f"auto -> {algo_auto}",
                   "l2": f"inputs larger than L2: every step reads {P * n * esz / 1e9:.2f} GB of inputs and "
                         f"writes as much, against the 126 MB L2",
                   "timing": f"K = {args.steps} calls captured in one CUDA graph; the graph replayed "
                             f"R = {args.replays} times, each replay bracketed by a barrier and a device "
                             f"synchronise and timed with CUDA events on the launching stream; "
                             f"ms_per_step = median replay / K",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU, P virtual ranks"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6650 GB/s",
                     "bytes_per_launch": b_min_bytes(P, n, esz), "kernel": kernel,
                     "traffic_source": traffic_src},
        "e2e": {"value": round(world * busbw_gbs(P, n, esz, e2e_ms / 1e3), 3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": args.steps * args.replays,
        "gpu_launches_note": "one kernel per step: K steps in each of the R timed replays",
        "clocks": clk,
        "per_algo": per_algo,
        "sweep": sweep,
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per_call, calls, sample, host = oracle_samples(WORKLOAD, algo_auto, min_seconds=args.cpu_seconds,
                                                       n_sample=args.cpu_sample, device=device)
        line["cpu_baseline"] = {"value": round(busbw_gbs(P, n, esz, per_call), 4), "unit": UNIT, "cores": 1,
                                "kind": "oracle", "sample": sample, **host}
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return line if rank == 0 else None


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on one pinned host core.
    Each step is the oracle on a contiguous slice of the workload (the first
    REFERENCE_SAMPLE elements of every rank); busbw is scaled to the full size."""
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    P, n, esz = WORKLOAD["P"], WORKLOAD["n"], ESZ[WORKLOAD["dtype"]]
    algo = REFERENCE_ALGO
    xs, m = oracle_inputs(WORKLOAD, REFERENCE_SAMPLE)
    oracle.allreduce(algo, xs, "bf16")  # loads the library
    with one_core() as pin:
        for _ in range(args.warmup):
            oracle.allreduce(algo, xs, "bf16")
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle.allreduce(algo, xs, "bf16")
        el = time.perf_counter() - t0
    per_full = el / args.steps * (n / m)
    v = busbw_gbs(P, n, esz, per_full)
    sample = (f"each step: oracle '{algo}' on the first {m} elements of each of the {P} ranks of the workload; "
              f"time scaled by {n}/{m}")
    return {"metric": METRIC, "value": round(v, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD["name"], "P": P, "n": n, "algo": algo},
            "cpu_baseline": {"value": round(v, 4), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                             **host_description(), "affinity": pin.describe(), "threads": 1},
            "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# Bytes per rank (KiB) of the selector table's columns: 32 KiB to 8 MiB in
# powers of two, then 16 and 32 MiB, and 64 MiB for everything above.
SELECTOR_KIB = (32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768, 65536)


def run_selector_sweep(args):
    """Every algorithm at every (P, bytes per rank) of the selector table, as
    JSON lines (one per shape). The write-mode kernel is the one this process
    runs (VRAR_WRITE_KERNEL=plain|staged|async|batched forces one; with staged,
    async or batched only the write mode is timed). --sweep-kib limits the
    sizes; --fp8 turns the fp8 payloads on (one-shot, write mode and the pull
    2-stage; recursive doubling has no fp8 form)."""
    import collective_all_reduce_virtual_b200 as vrar
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    kernel = os.environ.get("VRAR_WRITE_KERNEL", "auto")
    sizes = [int(k) for k in args.sweep_kib.split(",")] if args.sweep_kib else SELECTOR_KIB
    vrar.set_fp8_quant(bool(args.fp8))
    for P in (2, 4, 8, 16, 32):
        for kib in sizes:
            spec = dict(DECODE, P=P, n=kib * 512, name=f"P={P} {kib} KiB per rank")
            wl = Workload(spec, device)
            row = {"P": P, "kib": kib, "write_kernel": kernel, "fp8": bool(args.fp8),
                   "selected": vrar.select_algo(P, wl.n, TDT[wl.dt]),
                   "kernel": vrar.kernel_name(P, wl.n, TDT[wl.dt], "auto")}
            steps = 200 if kib <= 4096 else 50 if kib <= 16384 else 10
            algos = ("oneshot", "twostage_write", "twostage", "rd") \
                if kernel not in ("staged", "async", "batched") else ("twostage_write",)
            for algo in algos:
                if algo == "rd" and (P & (P - 1) or args.fp8):
                    continue
                row[algo] = round(min(measure_algo(wl, algo, steps, 3) for _ in range(3)) * 1e3, 3)
            wl.free()
            torch.cuda.empty_cache()
            print(json.dumps(row), flush=True)


def run_case(spec_text: str):
    """A few back-to-back calls of one algorithm on one shape (for profilers):
    'algo,P,KiB[,calls]', algo an all-reduce algorithm (with '+edge' and / or
    '+fp8' for the start/end barriers and the fp8 payloads) or 'rs' / 'ag' (the
    standalone reduce-scatter / all-gather; KiB is the full per-rank vector).
    Exits non-zero if the device status is not clean."""
    import collective_all_reduce_virtual_b200 as vrar
    parts = spec_text.split(",")
    algo, P, kib = parts[0], int(parts[1]), int(parts[2])
    calls = int(parts[3]) if len(parts) > 3 else 6
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wl = Workload(dict(DECODE, P=P, n=kib * 512, name=spec_text), device)
    h = torch.cuda.current_stream().cuda_stream
    with flags_set(vrar, algo) as base:
        for i in range(calls):
            if base in ("rs", "ag"):
                wl.collective_call(i, base, h)
            else:
                wl.call(i, base, h)
        torch.cuda.synchronize()
    rc, info = vrar.query_status()
    print(json.dumps({"case": spec_text, "status": rc, "info": info}))
    return rc


def run_spin_stats(args):
    """Spin statistics of the cross-rank waits over many calls (JSON lines):
    for each algorithm with waits, `--spin-stats N` calls on the decode
    workload (8 ranks x 1 MiB), as graphs of 1000 calls."""
    import collective_all_reduce_virtual_b200 as vrar
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wl = Workload(DECODE, device)
    per = 1000
    for algo, edge in (("twostage", False), ("twostage_write", True), ("rd", False)):
        vrar.set_edge_sync(edge)
        vrar.set_spin_stats(True)  # before capture: a graph keeps the arguments of its calls
        wl.call(0, algo, torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        g = wl.graph(algo, per)
        vrar.get_spin_stats(reset=True)
        t0 = time.perf_counter()
        reps = max(1, args.spin_stats // per)
        for _ in range(reps):
            g.replay()
        torch.cuda.synchronize()
        el = time.perf_counter() - t0
        vrar.set_spin_stats(False)
        st = vrar.get_spin_stats(reset=True)
        rc, info = vrar.query_status()
        print(json.dumps({"algo": algo, "edge_sync": edge, "calls": reps * per, "seconds": round(el, 2),
                          "status": rc, **st}), flush=True)
        del g
    vrar.set_edge_sync(False)


def run_floor(args):
    """Where the time of a small call goes (JSON lines). For P = 2 and 8 ranks:
    the per-call cost of a call on one 16-byte item per rank (launch, one
    DRAM round trip, the tail), and calls from 8 KiB to 8 MiB per rank, cold
    (inputs rotated through more than 3x L2) and warm (one buffer set, so the
    working set stays in L2), each the median of graph replays of 1000 (small)
    or 200 back-to-back calls. The write-mode kernel is whichever this process
    runs (VRAR_WRITE_KERNEL forces one). A straight-line fit of the cold times
    from 512 KiB per rank up, t = t0 + B_min / BW, splits each call into a
    fixed part t0 and a streaming part."""
    import collective_all_reduce_virtual_b200 as vrar
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    kernel = os.environ.get("VRAR_WRITE_KERNEL", "auto")
    for P in (2, 8):
        tiny = Workload(dict(DECODE, P=P, n=8, name="one item"), device)
        row = {"P": P, "write_kernel": kernel, "one_item_us": {}}
        for algo in ("oneshot", "twostage_write", "twostage", "rd"):
            row["one_item_us"][algo] = round(measure_algo(tiny, algo, 1000, 3, replays=5) * 1e3, 3)
        tiny.free()
        pts = []
        for kib in (8, 32, 128, 512, 1024, 2048, 4096, 8192):
            n = kib * 512
            spec = dict(DECODE, P=P, n=n, name=f"P={P} {kib} KiB")
            steps = 1000 if kib <= 512 else 200
            cold, warm = Workload(spec, device), Workload(spec, device, rotate=False)
            e = {"kib": kib, "bmin_bytes": b_min_bytes(P, n, 2),
                 "kernel": vrar.kernel_name(P, n, TDT["bf16"], "auto")}
            for algo in ("oneshot", "twostage_write"):
                e[algo] = {"cold_us": round(measure_algo(cold, algo, steps, 3, replays=5) * 1e3, 3),
                           "warm_us": round(measure_algo(warm, algo, steps, 3, replays=5) * 1e3, 3)}
            cold.free()
            warm.free()
            torch.cuda.empty_cache()
            pts.append(e)
        row["sizes"] = pts
        for algo in ("oneshot", "twostage_write"):
            xs = [p["bmin_bytes"] for p in pts if p["kib"] >= 512]
            ys = [p[algo]["cold_us"] * 1e-6 for p in pts if p["kib"] >= 512]
            mx, my = sum(xs) / len(xs), sum(ys) / len(ys)
            slope = sum((x - mx) * (y - my) for x, y in zip(xs, ys)) / sum((x - mx) ** 2 for x in xs)
            row[f"fit_{algo}"] = {"t0_us": round((my - slope * mx) * 1e6, 3),
                                  "stream_gbs": round(1 / slope / 1e9, 1) if slope > 0 else None}
        print(json.dumps(row), flush=True)


class TboPrefill:
    """Two micro-batches of a 16k-token prefill through L row-parallel linear
    layers with P virtual ranks. In each layer rank p multiplies its K/P slice
    of the micro-batch's activations with its K/P rows of the layer's weight (a
    plain cuBLAS GEMM through torch: the compute the all-reduce overlaps with),
    and the P partial outputs are all-reduced; the next layer of that
    micro-batch reads its slice of the all-reduced output. Random weights; no
    model is needed."""

    def __init__(self, device, P=8, tokens=8192, hidden=7168, layers=4, seed=0):
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        self.P, self.T, self.K, self.H, self.L = P, tokens, hidden, hidden, layers
        kp = hidden // P
        self.kp = kp
        self.x = [torch.randn(tokens, hidden, device=device, dtype=torch.bfloat16, generator=g) for _ in range(2)]
        self.w = [torch.randn(hidden, hidden, device=device, dtype=torch.bfloat16, generator=g) * 0.02
                  for _ in range(layers)]
        self.part = [[torch.empty(tokens, hidden, device=device, dtype=torch.bfloat16) for _ in range(P)]
                     for _ in range(2)]
        self.out = [[torch.empty(tokens, hidden, device=device, dtype=torch.bfloat16) for _ in range(P)]
                    for _ in range(2)]

    def gemm(self, u, layer):
        kp = self.kp
        for p in range(self.P):
            src = self.x[u] if layer == 0 else self.out[u][p]
            torch.matmul(src[:, p * kp:(p + 1) * kp], self.w[layer][p * kp:(p + 1) * kp, :], out=self.part[u][p])

    def allreduce(self, u, stream=None):
        import collective_all_reduce_virtual_b200 as vrar
        vrar.all_reduce(self.part[u], self.out[u], algo="auto", stream=stream)

    def step_sequential(self):
        for layer in range(self.L):
            for u in (0, 1):
                self.gemm(u, layer)
                self.allreduce(u)

    def step_overlapped(self, comm):
        """Each all-reduce runs on the comm stream while the other micro-batch
        computes; a micro-batch's next layer waits for its own all-reduce."""
        main = torch.cuda.current_stream()
        done = [None, None]
        for layer in range(self.L):
            for u in (0, 1):
                if done[u] is not None:
                    main.wait_event(done[u])
                self.gemm(u, layer)
                ready = torch.cuda.Event()
                ready.record(main)
                comm.wait_event(ready)
                with torch.cuda.stream(comm):
                    self.allreduce(u, comm)
                done[u] = torch.cuda.Event()
                done[u].record(comm)
        main.wait_stream(comm)


def run_overlap(args):
    """NEXT-1 shape: sequential vs overlapped 2-micro-batch prefill step."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    m = TboPrefill(device)
    comm = torch.cuda.Stream()

    def timed(fn, iters):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / iters

    import collective_all_reduce_virtual_b200 as vrar
    it = max(3, args.steps // 20)
    gemm_flop = m.L * 2 * 2 * m.T * m.K * m.H
    ar_bytes = m.L * 2 * 2 * m.P * m.T * m.H * 2
    base = {"workload": f"2 micro-batches x {m.T} tokens, {m.L} layers, hidden {m.H}, row-parallel linear over "
                        f"P={m.P} virtual ranks (K/P = {m.K // m.P}), bf16, each followed by the all-reduce of "
                        f"the P partials"}
    base["gemm_ms"] = timed(lambda: [m.gemm(u, l) for l in range(m.L) for u in (0, 1)], it)
    base["gemm_tflops"] = gemm_flop / (base["gemm_ms"] * 1e-3) / 1e12
    base["sequential_ms"] = timed(m.step_sequential, it)
    rows = []
    for cap in (0, 148, 96, 64, 48, 32, 24, 16):  # CTA budget of each all-reduce (0 = whole GPU)
        vrar.set_max_ctas(cap)
        r = {"max_ctas": cap, "allreduce_ms": timed(lambda: [m.allreduce(u) for _ in range(m.L) for u in (0, 1)], it),
             "overlapped_ms": timed(lambda: m.step_overlapped(comm), it)}
        r["allreduce_hbm_gbs"] = ar_bytes / (r["allreduce_ms"] * 1e-3) / 1e9
        r["speedup_vs_sequential"] = base["sequential_ms"] / r["overlapped_ms"]
        rows.append({k: (round(v, 4) if isinstance(v, float) else v) for k, v in r.items()})
    vrar.set_max_ctas(0)
    rc, info = vrar.query_status()
    base["status"] = rc
    base["budgets"] = rows
    best = min(rows, key=lambda r: r["overlapped_ms"])
    base["best_overlapped_ms"], base["best_max_ctas"] = best["overlapped_ms"], best["max_ctas"]
    base["saved_ms"] = base["sequential_ms"] - best["overlapped_ms"]
    print(json.dumps({k: (round(v, 4) if isinstance(v, float) else v) for k, v in base.items()}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("vrar", "reference"), default="vrar")
    ap.add_argument("--quick", action="store_true", help="skip the per-algorithm table and the sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--replays", type=int, default=HEADLINE_REPLAYS,
                    help="timed replays of the K-step graph (the median is reported)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-sample", type=int, default=1 << 23,
                    help="elements per rank of the slice the CPU oracle baseline runs on")
    ap.add_argument("--case", metavar="ALGO,P,KIB[,CALLS]",
                    help="run a few calls of one algorithm on one shape and exit (for profilers)")
    ap.add_argument("--spin-stats", type=int, metavar="CALLS", default=0,
                    help="spin statistics of the waits over CALLS calls per algorithm (JSON lines) and exit")
    ap.add_argument("--overlap", action="store_true",
                    help="sequential vs overlapped two-micro-batch prefill step (JSON line) and exit")
    ap.add_argument("--floor", action="store_true",
                    help="per-call fixed cost and size ladder at 2 and 8 ranks (JSON lines) and exit")
    ap.add_argument("--selector-sweep", action="store_true",
                    help="print per-shape timings of every algorithm (JSON lines) and exit")
    ap.add_argument("--sweep-kib", metavar="KIB,...", help="bytes per rank (KiB) the selector sweep covers")
    ap.add_argument("--fp8", action="store_true", help="selector sweep with fp8 payloads on")
    args = ap.parse_args(argv)
    if args.selector_sweep:
        run_selector_sweep(args)
        return
    if args.floor:
        run_floor(args)
        return
    if args.case:
        sys.exit(1 if run_case(args.case) else 0)
    if args.spin_stats:
        run_spin_stats(args)
        return
    if args.overlap:
        run_overlap(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    line = run_reference(args) if args.impl == "reference" else run_vrar(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
