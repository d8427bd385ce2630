"""Benchmark of the retention hot path on B200: prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload layer200m|layer3b|long7b|decode7b] [--chunk C]
                    [--form chunkwise|parallel] [--backward] [--seqlen n]
                    [--batch B] [--tokens T] [--no-overlap]

One step = one pass of the whole hot path over one batch of the workload:
rotation prologue, chunkwise prefill with the state carried out, the
GroupNorm + swish gate epilogue (when the workload has a gate), then one
recurrent decode step for every sequence from that state.  `value` counts
the tokens of the step (batch * seqlen prefill tokens + batch decode
tokens) per second of device time, max over ranks; inputs are resident in
HBM.  Three input sets rotate so that every step reads inputs that are not
in L2 (each set is larger than a third of the 126 MB L2 and three together
are well beyond it).

The default workload is the largest single-GPU prefill, the 7B-like long
prefill (B=1, H=16, n=8192, d=256, bf16, chunk 512, final state out).  The
default line adds two measurements of their own (skip with --no-legs):
"decode_legs", the decode configuration (H=16, d=256, states seeded by an
8192-token prefill) at batch 32 and 128, where the state (269 MB, 1.08 GB)
is beyond L2, each with its HBM roofline; and "secondary", the 200M-layer
step (B=8, H=4, n=2048, gate) at chunk 512 and at chunk 64, measured the
same way as the main workload.

The K timed steps are captured once as a CUDA graph and replayed (after one
warm-up replay), so the GPU runs them back to back without host launch
gaps; that replay holds no timer events.  The dominant kernel's time comes
from a second capture of the same steps in which the library's kernel timer
brackets that kernel with event-record nodes, and the roofline uses it.
The same K steps launched one by one from Python are reported under
"eager".

Other modes print their own line with their own metric:
  --form parallel    the parallel form instead of the chunkwise prefill
                     (prefill only, no state, no decode step);
  --backward         the backward pass of the prefill (dq, dk, dv);
  --layer            the multi-scale retention layer: Q/K/V/G projection
                     GEMM, gated prefill, output projection GEMM (random
                     weights; hidden = the workload's gate width, or H d);
  --workload decode7b [--batch B] [--tokens T]
                     decode steps (T = 1) or T-token recurrent calls from
                     states seeded by an 8192-token prefill;
  --seqlen n         the workload's shape at another sequence length.

Under torchrun each rank runs its own replica on its own sequences (no
data-path collective; weak scaling).  `--impl reference` times the CPU
oracle (float64 numpy) on rank 0 on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "retention prefill tokens/s and decode steps/s on 1 B200; % of roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload_config(w: wl.Workload, chunk: int, form: str = "chunkwise") -> dict:
    if form == "parallel":
        what = "parallel form over the whole sequence" + \
            (" + GroupNorm/swish gate" if w.hidden else "") + " (prefill only, no state)"
    else:
        what = f"chunk {chunk}" + (" + GroupNorm/swish gate" if w.hidden else "") + \
            " + 1 decode step"
    cfg = {
        "workload": f"{w.name}: B={w.batch} H={w.heads} n={w.seqlen} d={w.d} {w.dtype} " + what,
        "batch": w.batch, "heads": w.heads, "seqlen": w.seqlen, "dk": w.d, "dv": w.d,
        "chunk": chunk if form == "chunkwise" else None, "form": form, "gate": bool(w.hidden),
        "l2": "3 rotating input sets, each beyond 1/3 of the 126 MB L2",
    }
    if form == "chunkwise" and chunk < 128 and w.dtype == "bf16" and w.d == 256:
        cfg["computed_as"] = ("128-token chunks on the tensor cores: the chunkwise form's "
                              "outputs do not depend on the chunk length, so only the "
                              "rounding order differs from chunk " + str(chunk))
    return cfg


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a
# kernel on a workload, from one ncu capture.  Each figure is kept with the
# SHA-256 of the kernel's source at capture time: its section of the .cu file
# (from its banner line to the next) and the device headers it includes.
# The figure is reported only while that source is unchanged.
NCU_TRAFFIC = {
    ("tc_output", "long7b"): {
        "source": "chunkwise_tc.cu", "section": "output pass",
        "headers": ["sm100.cuh", "common.cuh"],
        "sha256": "2135b4b483203581f984438dece09b44b415da3e3335562b3b0a0389e1c1b9af",
        "bytes": 277.97e6,
    },
}
SECTION_BANNER = "// " + "-" * 66 + " "


def kernel_source_sha(source: str, section: str, headers) -> str | None:
    """SHA-256 over one banner-delimited section of a .cu file and the headers."""
    import hashlib
    csrc = os.path.join(ROOT, "linear_recurrent_sequence_02_b200", "csrc")
    try:
        with open(os.path.join(csrc, source), encoding="utf-8") as f:
            lines = f.read().split("\n")
        start = lines.index(SECTION_BANNER + section)
        end = next((i for i in range(start + 1, len(lines))
                    if lines[i].startswith(SECTION_BANNER)), len(lines))
        h = hashlib.sha256("\n".join(lines[start:end]).encode())
        for name in headers:
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
    except (OSError, ValueError):
        return None
    return h.hexdigest()


def measured_traffic(kernel: str, workload: str):
    rec = NCU_TRAFFIC.get((kernel, workload))
    if not rec or not rec["sha256"] or rec["bytes"] is None:
        return None
    sha = kernel_source_sha(rec["source"], rec["section"], rec["headers"])
    return rec["bytes"] if sha == rec["sha256"] else None


def output_kernel_bytes(batch: int, heads: int, n: int, d: int, chunk: int, gate: bool) -> int:
    """Algorithmic HBM bytes of one output-pass launch: Qt, Kt, V read and O
    written once (bf16), G read once when gated, and S_prev (bf16 d x d) read
    once for every chunk after the first."""
    th = batch * heads * n
    nchunks = (n + chunk - 1) // chunk
    return th * 2 * d * (3 + (2 if gate else 1)) + batch * heads * (nchunks - 1) * d * d * 2


def algorithmic_flops_per_token_head(d: int, chunk: int) -> int:
    # causal Q K^T and P V inside a chunk, plus the state update and the
    # cross-chunk product: (dk + dv)(C + 1) + 4 dk dv
    return 2 * d * (chunk + 1) + 4 * d * d


def output_kernel_flops_per_token_head(d: int, chunk: int) -> int:
    return 2 * d * (chunk + 1) + 2 * d * d


def state_kernel_flops_per_token_head(d: int) -> int:
    return 2 * d * d


def prep_kernel_bytes_per_token_head(d: int) -> int:
    # the rotation and decay fold: q and k read, Qt and Kt written, bf16
    return 4 * d * 2


def parallel_flops_per_token_head(d: int, n: int) -> int:
    # causal Q K^T and P V over the whole sequence: 2 d (n + 1) on average
    return 2 * d * (n + 1)


def executed_flops_per_token_head(d: int, chunk: int, n: int, parallel: bool = False) -> float:
    """Flops the tensor-core prefill executes per token-head (the tensor
    path, n a multiple of the chunk): 128-key tiles up to the diagonal,
    the diagonal tile whole, upper tiles skipped.  A row block r of a chunk
    runs r + 1 tiles of Q K^T and P V, 4 * 128 * d flops per row each, so a
    chunk of R = C / 128 row blocks averages 256 d (R + 1) per token; the
    chunkwise form adds Qt S_prev (2 d^2) for every chunk after the first
    and the state pass's Kt^T V (2 d^2).  Chunks below 128 are computed as
    128; the parallel form is one chunk of ceil(n / 128) row blocks."""
    if parallel:
        return 256.0 * d * ((n + 127) // 128 + 1)
    c = max(chunk, 128)
    nchunks = (n + c - 1) // c
    return 256.0 * d * (c // 128 + 1) + 2.0 * d * d * (nchunks - 1) / nchunks + 2.0 * d * d


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML on a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((mhz, int(reasons)))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(self.period)

    def start(self):
        if self.nv is None:
            return
        self._sample()
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def stop(self) -> dict:
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        if self._thread:
            self._thread.join()
        self._sample()
        mhz = [s[0] for s in self.samples]
        active = set()
        for _, r in self.samples:
            for name, bit in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    active.add(name)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(active), "samples": len(mhz)}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ------------------------------------------------------------------ oracle arm
def oracle_step(inputs, gam, chunk, b):
    """The hot path on the CPU oracle for sequence b: prefill + 1 decode step."""
    import oracle
    q, k, v, g, qd, kd, vd = inputs
    sl = slice(b, b + 1)
    y, s = oracle.retention_prefill(q[sl], k[sl], v[sl], gam, chunk,
                                    gate=None if g is None else g[sl])
    n = q.shape[1]
    o, _ = oracle.retention_step(oracle.xpos_rotate(qd[sl][:, None], n)[:, 0],
                                 oracle.xpos_rotate(kd[sl][:, None], n)[:, 0], vd[sl], gam, s)
    return y, o


# ------------------------------------------------------------- ranks (N > 1)
# Every rank runs its own replica of the workload on its own sequences (no
# data-path collective); the job's time is the slowest rank's, and the
# job's throughput counts the units of all ranks.
def rank_env():
    """(rank, world size, local rank) from torchrun's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_seed(seed: int, rank: int) -> int:
    """Seed of a rank's replica: rank 0 keeps the workload's own seed."""
    return seed + 7919 * rank


def max_over_ranks(x: float, dist, device) -> float:
    """The largest value over the ranks (the job's time is the slowest rank's)."""
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_step: int, steps: int, ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the time."""
    return world * units_per_step * steps / (ms / 1e3)


def host_inputs(w: wl.Workload, rank: int = 0):
    seed = shard_seed(w.seed, rank)
    q, k, v, g = wl.make_prefill_inputs(w.batch, w.heads, w.seqlen, w.d, w.dtype, w.scale,
                                        seed, hidden=w.hidden)
    qd, kd, vd = (x[0] for x in wl.make_decode_inputs(w.batch, w.heads, 1, w.d, w.dtype,
                                                      w.scale, seed + 100))
    return q, k, v, g, qd, kd, vd


def cpu_baseline(w, chunk, min_seconds=10.0):
    inputs = host_inputs(w)
    gam = np.float32([1 - 2.0 ** (-5 - h) for h in range(w.heads)])
    t0 = time.perf_counter()
    seqs = 0
    while True:
        oracle_step(inputs, gam, chunk, seqs % w.batch)
        seqs += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or seqs >= 4 * w.batch:
            break
    tokens = seqs * (w.seqlen + 1)
    return {"value": tokens / el, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{seqs} sequence(s) of {w.seqlen} prefill tokens + 1 decode step each, "
                      f"all {w.heads} heads, float64 numpy, {el:.1f} s"}


def run_reference(args, w, chunk):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inputs = host_inputs(w)
    gam = np.float32([1 - 2.0 ** (-5 - h) for h in range(w.heads)])
    for i in range(args.warmup):
        oracle_step(inputs, gam, chunk, i % w.batch)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_step(inputs, gam, chunk, i % w.batch)
    el = time.perf_counter() - t0
    value = args.steps * (w.seqlen + 1) / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, chunk),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"each step: 1 of {w.batch} sequences ({w.seqlen} prefill "
                                   f"tokens + 1 decode step), all heads, float64 numpy"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
def run_ours(args, w, chunk):
    import torch
    import torch.distributed as dist

    import linear_recurrent_sequence_02_b200 as rn

    rank, world, local = rank_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    from linear_recurrent_sequence_02_b200.build import build
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    rn.load_library()
    rn.retnet_set_launch_overlap(not args.no_overlap)
    if args.pairs is not None:
        rn.retnet_set_output_pairing(args.pairs)

    line = measure_prefill(args, w, chunk, rank, world, dev, full=True)
    line["output_pairs"] = args.pairs
    if args.form == "chunkwise" and not args.no_legs:
        # the decode configuration at the batches whose state is beyond L2,
        # and the 200M-layer step as a second prefill shape
        dw = wl.WORKLOADS["decode7b"]
        line["decode_legs"] = {f"batch{b}": measure_decode(args, dw, b, 1, dev, world)
                               for b in (32, 128)}
        if w.name != "layer200m":
            # the 200M-layer step at its chunk 512 and at its second chunk
            # length, 64 (computed as 128-token chunks on the tensor cores)
            sw = wl.WORKLOADS["layer200m"]
            line["secondary"] = {
                "layer200m": measure_prefill(args, sw, sw.chunk, rank, world, dev, full=False),
                "layer200m_chunk64": measure_prefill(args, sw, 64, rank, world, dev, full=False),
            }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_prefill(args, w, chunk, rank, world, dev, full=True):
    """Times K steps of the workload (prefill + one decode step per sequence)
    as one CUDA graph replay; returns the bench line's fields.  `full` adds
    the eager timing, the end-to-end leg and the CPU baseline."""
    import torch
    import torch.distributed as dist

    import linear_recurrent_sequence_02_b200 as rn

    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q, k, v, g, qd, kd, vd = host_inputs(w, rank)

    def pinned(x):
        return torch.from_numpy(x).to(tdt).pin_memory()

    host = [pinned(x) if x is not None else None for x in (q, k, v, g, qd, kd, vd)]
    nsets = 3
    sets = []
    for _ in range(nsets):
        sets.append([None if x is None else x.to(dev, non_blocking=True) for x in host])
    B, n, H, d = w.batch, w.seqlen, w.heads, w.d
    gam = rn.retnet_default_gammas(H)
    y = torch.empty(B, n, H, d, dtype=tdt, device=dev)
    o = torch.empty(B, H, d, dtype=tdt, device=dev)
    state = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    par = args.form == "parallel"
    wsb = rn.retnet_parallel_workspace_size(B, H, n, d, d, tdt) if par else \
        rn.retnet_chunkwise_workspace_size(B, H, n, d, d, tdt, chunk, args.algo)

    def prefill(qq, kk, vv, gg, st, out, wsp):
        if par:
            rn.retnet_retention_parallel(qq, kk, vv, gam, gate=gg, out=out, workspace=wsp)
        else:
            rn.retnet_retention_chunkwise(qq, kk, vv, gam, chunk, state_out=st, gate=gg, out=out,
                                          workspace=wsp, algo=args.algo)

    ws = rn.retnet_workspace(wsb, dev)

    def step(s):
        qq, kk, vv, gg, q1, k1, v1 = s
        prefill(qq, kk, vv, gg, state, y, ws)
        if not par:     # the parallel form leaves no state to decode from
            rn.retnet_retention_step(q1, k1, v1, gam, state, n, out=o)

    torch.cuda.synchronize()
    for i in range(args.warmup):
        step(sets[i % nsets])
    torch.cuda.synchronize()
    # Three more steps with every kernel timed: the per-kernel breakdown
    # ("kernels") and the choice of the dominant kernel come from these.
    rn.retnet_profiler_select(None)
    rn.retnet_profiler_reset()
    rn.retnet_profiler_enable(True)
    for i in range(3):
        step(sets[i % nsets])
    torch.cuda.synchronize()
    rn.retnet_profiler_enable(False)
    kern_warm = rn.retnet_profiler_read()
    rn.retnet_check_device_errors(dev)
    dom = max(kern_warm.items(), key=lambda kv: kv[1][0])[0] if kern_warm else None

    stream = torch.cuda.current_stream(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)

    # ---- the same steps launched one by one from Python (reported as "eager")
    eager_ms = None
    if full:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for i in range(args.steps):
            step(sets[i % nsets])
        ev1.record(stream)
        torch.cuda.synchronize()
        eager_ms = ev0.elapsed_time(ev1)
        if world > 1:
            eager_ms = max_over_ranks(eager_ms, dist, dev)

    # ---- device-timed region: the K steps captured once as a CUDA graph
    # (inputs of each step baked into its nodes), replayed once to warm up and
    # once timed.  No timer events inside it, so consecutive kernels keep
    # their launch overlap.
    launches0 = rn.retnet_kernel_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.steps):
            step(sets[i % nsets])
    launches = rn.retnet_kernel_launch_count() - launches0
    graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    ev0.record(stream)
    graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    del graph

    # ---- the dominant kernel's own time: the same K steps captured again
    # with the kernel timer bracketing that kernel alone (event-record nodes)
    rn.retnet_profiler_reset()
    rn.retnet_profiler_select(dom)
    rn.retnet_profiler_enable(True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.steps):
            step(sets[i % nsets])
    rn.retnet_profiler_enable(False)
    rn.retnet_profiler_select(None)
    graph.replay()
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    # the captured events hold the times of the latest (second) replay
    kern = rn.retnet_profiler_read()
    del graph
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)
    rn.retnet_check_device_errors(dev)

    tokens_per_step = B * n + (0 if par else B)
    value = job_rate(world, tokens_per_step, args.steps, ms)

    # ---- end to end through the public API with host buffers
    # Every step copies its inputs from pinned host memory, runs the hot path
    # and copies y and the decode output back.  Copies run on their own
    # streams, double-buffered, so step i's upload overlaps step i-1's
    # compute and download (PCIe is full duplex).
    e2e = None
    if full:
        h2d = sum(x.numel() * x.element_size() for x in host[:4 if par else 7] if x is not None)
        d2h = y.numel() * y.element_size() + (0 if par else o.numel() * o.element_size())
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        dsets = [[None if x is None else torch.empty_like(x, device=dev) for x in host]
                 for _ in range(2)]
        ys = [torch.empty_like(y) for _ in range(2)]
        os_ = [torch.empty_like(o) for _ in range(2)]
        yh = [torch.empty_like(y, device="cpu").pin_memory() for _ in range(2)]
        oh = [torch.empty_like(o, device="cpu").pin_memory() for _ in range(2)]
        st2 = [torch.empty_like(state) for _ in range(2)]
        ws2 = [rn.retnet_workspace(wsb, dev) for _ in range(2)]
        nin = 4 if par else 7                 # the parallel form uploads no decode inputs

        def run_e2e(nsteps):
            in_ready = [torch.cuda.Event() for _ in range(nsteps)]
            done = [torch.cuda.Event() for _ in range(nsteps)]
            out_done = [torch.cuda.Event() for _ in range(nsteps)]
            for i in range(nsteps):
                j = i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(done[i - 2])
                    for dst, src in zip(dsets[j][:nin], host[:nin]):
                        if src is not None:
                            dst.copy_(src, non_blocking=True)
                    in_ready[i].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(in_ready[i])
                    if i >= 2:
                        s_cmp.wait_event(out_done[i - 2])
                    qq, kk, vv, gg, q1, k1, v1 = dsets[j]
                    prefill(qq, kk, vv, gg, st2[j], ys[j], ws2[j])
                    if not par:
                        rn.retnet_retention_step(q1, k1, v1, gam, st2[j], n, out=os_[j])
                    done[i].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done[i])
                    yh[j].copy_(ys[j], non_blocking=True)
                    if not par:
                        oh[j].copy_(os_[j], non_blocking=True)
                    out_done[i].record(s_out)
            return out_done[-1]

        run_e2e(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_cmp.wait_stream(s_in)
        s_out.wait_stream(s_in)
        last = run_e2e(e2e_steps)
        s_in.wait_event(last)
        s_in.wait_stream(s_cmp)
        e1.record(s_in)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        if world > 1:
            e2e_ms = max_over_ranks(e2e_ms, dist, dev)
        e2e = {"value": job_rate(world, tokens_per_step, e2e_steps, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}
        del dsets, ys, os_, yh, oh, st2, ws2

    # ---- roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    roof = None
    kernels_json = {}                      # every kernel, from the warm-up steps
    for name, (tot, cnt) in kern_warm.items():
        kernels_json[name] = {"avg_us": 1e3 * tot / cnt, "launches": cnt,
                              "share": tot / max(sum(v[0] for v in kern_warm.values()), 1e-12)}
    if dom is not None and dom in kern:
        tot, cnt = kern[dom]
        avg_s = tot / cnt / 1e3
        th = B * n * H
        if dom in ("tc_output", "simt_output"):
            # the tensor-core kernels compute chunks below 128 as 128-token
            # chunks: the work they do is that chunk length's
            kc = max(chunk, 128) if dom.startswith("tc") else chunk
            flops = (parallel_flops_per_token_head(d, n) if par else
                     output_kernel_flops_per_token_head(d, kc)) * th
            achieved = flops / avg_s / 1e12
            if dom.startswith("tc"):
                # the binding roof of min(tensor peak, HBM bandwidth x intensity):
                # the larger of the two floors, flops / peak and bytes / bandwidth
                nbytes = None if par else output_kernel_bytes(B, H, n, d, kc, bool(w.hidden))
                tensor = {"achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": achieved / peaks["bf16_tflops"], "work_per_launch": flops}
                hbm = None
                if nbytes:
                    gbs = nbytes / avg_s / 1e9
                    hbm = {"achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": gbs / peaks["hbm_gbs"], "work_per_launch": nbytes}
                binding = hbm if hbm and hbm["frac"] > tensor["frac"] else tensor
                roof = {"kernel": dom, "bound": "hbm" if binding is hbm else "tensor",
                        "achieved": binding["achieved"], "peak": binding["peak"],
                        "unit": binding["unit"], "frac": binding["frac"],
                        "traffic": None if par else measured_traffic(dom, w.name),
                        "peak_source": peak_src, "work_per_launch": binding["work_per_launch"],
                        "avg_us": avg_s * 1e6, "tensor": tensor, "hbm": hbm,
                        "intensity_flop_per_byte": flops / nbytes if nbytes else None,
                        "chunk_computed": None if par else kc}
            else:   # float32 FFMA: 148 SMs x 128 lanes x 2 flop x max SM clock
                peak = 148 * 128 * 2 * (peaks.get("sm_max_mhz", 1965.0) * 1e6) / 1e12
                roof = {"kernel": dom, "bound": "alu", "achieved": achieved, "peak": peak,
                        "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                        "peak_source": peak_src, "work_per_launch": flops,
                        "avg_us": avg_s * 1e6}
        elif dom in ("tc_state", "simt_state"):
            flops = state_kernel_flops_per_token_head(d) * th
            achieved = flops / avg_s / 1e12
            bound = "tensor" if dom.startswith("tc") else "alu"
            peak = peaks["bf16_tflops"] if bound == "tensor" else \
                148 * 128 * 2 * (peaks.get("sm_max_mhz", 1965.0) * 1e6) / 1e12
            roof = {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak,
                    "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                    "peak_source": peak_src, "work_per_launch": flops, "avg_us": avg_s * 1e6}
        elif dom == "tc_prep":
            # q and k read, Qt and Kt written once (bf16)
            nbytes = prep_kernel_bytes_per_token_head(d) * th
            gbs = nbytes / avg_s / 1e9
            roof = {"kernel": dom, "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                    "peak_source": peak_src, "work_per_launch": nbytes, "avg_us": avg_s * 1e6}
        else:
            roof = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": None, "traffic": None, "peak_source": peak_src}

    # whole prefill against the tensor peak (algorithmic flops at this chunk):
    # the timed step time less the decode kernel's warm-up average
    dec_ms = (kern_warm["retention_step"][0] / kern_warm["retention_step"][1]
              if "retention_step" in kern_warm else 0.0)
    pre_ms = ms / max(args.steps, 1) - dec_ms
    prefill_info = None
    if pre_ms > 0:
        alg = (parallel_flops_per_token_head(d, n) if par else
               algorithmic_flops_per_token_head(d, chunk)) * B * n * H
        prefill_info = {"tokens_per_s": B * n / (pre_ms / 1e3), "ms": pre_ms,
                        "tflops_algorithmic": alg / (pre_ms / 1e3) / 1e12,
                        "frac_of_bf16_peak": alg / (pre_ms / 1e3) / 1e12 / peaks["bf16_tflops"]}
        if d == 256 and w.dtype == "bf16" and args.algo != "simt":   # the tensor-core path
            exe = executed_flops_per_token_head(d, chunk, n, par) * B * n * H
            prefill_info["flop_executed_per_token_head"] = exe / (B * n * H)
            prefill_info["tflops_executed"] = exe / (pre_ms / 1e3) / 1e12
    step_decode = None
    if "retention_step" in kern_warm:
        tot, cnt = kern_warm["retention_step"]
        avg_s = tot / cnt / 1e3
        step_decode = {"batch": B, "us_per_step": avg_s * 1e6,
                       "note": f"the step's own decode of {B} sequence(s), state just written "
                               "by the prefill and L2-resident; the HBM-bound decode "
                               "measurement is decode_legs"}

    cpu = None
    if full and rank == 0 and world == 1 and not args.no_cpu_baseline and not par:
        cpu = cpu_baseline(w, chunk)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic", "config": workload_config(w, chunk, args.form),
        "algo": "tensor" if par else args.algo, "roofline": roof, "prefill": prefill_info,
        "step_decode": step_decode, "kernels": kernels_json, "gpu_launches": launches,
        "clocks": clock_info,
        "timing": "one replay of a CUDA graph holding the K timed steps; the roofline "
                  "kernel is timed in a second replay of the same steps captured with "
                  "event-record nodes around it; 'kernels' are 3 steps after the warm-up "
                  "with every kernel bracketed by events",
        "launch_overlap": not args.no_overlap,
    }
    if full:
        line["cpu_baseline"] = cpu
        line["e2e"] = e2e
        line["eager"] = {"value": job_rate(world, tokens_per_step, args.steps, eager_ms),
                         "ms_per_step": eager_ms / args.steps}
    del sets, ws, y, o, state
    torch.cuda.empty_cache()
    return line


def run_backward(args, w, chunk):
    """Backward pass (retnet_retention_backward) of the prefill without
    epilogue: one timed step = dq, dk, dv for the whole batch, given dO."""
    import torch

    import linear_recurrent_sequence_02_b200 as rn
    from linear_recurrent_sequence_02_b200.build import build

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    build()
    rn.load_library()
    rn.retnet_set_launch_overlap(not args.no_overlap)
    if args.pairs is not None:
        rn.retnet_set_output_pairing(args.pairs)
    B, n, H, d = w.batch, w.seqlen, w.heads, w.d
    gam = rn.retnet_default_gammas(H)
    sets = []
    for i in range(3):                                  # rotating inputs, each beyond L2/3
        q, k, v = wl.make_prefill_inputs_device(B, H, n, d, w.scale, w.seed + 31 * i, dev)
        gen = torch.Generator(device=dev)
        gen.manual_seed(w.seed + 31 * i + 5)
        do = torch.randn(B, n, H, d, generator=gen, device=dev).to(torch.bfloat16)
        sets.append((q, k, v, do))
    dq, dk, dv = (torch.empty(B, n, H, d, dtype=torch.bfloat16, device=dev) for _ in range(3))
    ws = rn.retnet_workspace(rn.retnet_backward_workspace_size(B, H, n, d, d, torch.bfloat16,
                                                               chunk, args.algo), dev)

    def step(i):
        q, k, v, do = sets[i % 3]
        rn.retnet_retention_backward(q, k, v, do, gam, chunk, algo=args.algo, dq=dq, dk=dk,
                                     dv=dv, workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    rn.retnet_profiler_reset()
    rn.retnet_profiler_select(None)
    rn.retnet_profiler_enable(True)
    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    rn.retnet_profiler_enable(False)
    kern = rn.retnet_profiler_read()
    rn.retnet_check_device_errors(dev)
    launches0 = rn.retnet_kernel_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.steps):
            step(i)
    launches = rn.retnet_kernel_launch_count() - launches0
    graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    ev0.record(stream)
    graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    del graph
    rn.retnet_check_device_errors(dev)
    peaks, src = load_peaks()
    # three forward retentions: 3 x the forward's algorithmic flops at this chunk
    alg = 3 * algorithmic_flops_per_token_head(d, chunk) * B * n * H
    step_s = ms / args.steps / 1e3
    total = sum(v[0] for v in kern.values())
    line = {
        "metric": "retention backward tokens/s (dq, dk, dv of the prefill)",
        "value": B * n / step_s, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": f"{w.name} backward: B={B} H={H} n={n} d={d} bf16 chunk {chunk}, "
                               "no epilogue, zero initial state",
                   "batch": B, "heads": H, "seqlen": n, "chunk": chunk,
                   "l2": "3 rotating input sets"},
        "tflops_algorithmic": alg / step_s / 1e12,
        "frac_of_bf16_peak": alg / step_s / 1e12 / peaks["bf16_tflops"],
        "kernels": {k: {"avg_us": 1e3 * v[0] / v[1], "launches_per_step": v[1] / 3,
                        "share": v[0] / max(total, 1e-12)} for k, v in kern.items()},
        "gpu_launches": launches, "clocks": clock_info, "peak_source": src,
        "timing": "one replay of a CUDA graph holding the K timed steps; 'kernels' are 3 "
                  "steps with every kernel bracketed by events",
    }
    print(json.dumps(line), flush=True)


def measure_decode(args, w, B, T, dev, world=1):
    """Decode at batch B from states seeded by an 8192-token GPU prefill:
    K steps (T = 1) or T-token recurrent calls, captured as one CUDA graph
    and replayed; returns the measurement's fields (max over ranks)."""
    import torch

    import linear_recurrent_sequence_02_b200 as rn

    H, d, n = w.heads, w.d, w.seqlen
    gam = rn.retnet_default_gammas(H)
    state = torch.empty(B, H, d, d, device=dev)
    for b0 in range(0, B, 16):                       # seed the state slice by slice
        b1 = min(B, b0 + 16)
        q, k, v = wl.make_prefill_inputs_device(b1 - b0, H, n, d, w.scale, w.seed + b0, dev)
        rn.retnet_retention_chunkwise(q, k, v, gam, w.chunk, state_out=state[b0:b1])
        del q, k, v
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 7)
    steps = max(args.steps, 20)
    if T == 1:
        pool = w.decode_steps
        qd, kd, vd = ((torch.randn(pool, B, H, d, generator=gen, device=dev) * w.scale)
                      .to(torch.bfloat16) for _ in range(3))
        o = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)

        def step(i):
            rn.retnet_retention_step(qd[i % pool], kd[i % pool], vd[i % pool], gam, state,
                                     n + i, out=o)
    else:
        # T tokens per call (multi-token decode) through the recurrent form;
        # a pool of four input sets, each call at its own positions
        pool = 4
        qd, kd, vd = ((torch.randn(pool, B, T, H, d, generator=gen, device=dev) * w.scale)
                      .to(torch.bfloat16) for _ in range(3))
        o = torch.empty(B, T, H, d, dtype=torch.bfloat16, device=dev)

        def step(i):
            rn.retnet_retention_recurrent(qd[i % pool], kd[i % pool], vd[i % pool], gam,
                                          state, n + i * T, out=o)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index or 0)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream(dev)
    rn.retnet_profiler_reset()
    rn.retnet_profiler_enable(True)
    launches0 = rn.retnet_kernel_launch_count()
    clocks.start()
    ev0.record(stream)
    for i in range(steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    rn.retnet_profiler_enable(False)
    kern = rn.retnet_profiler_read()
    eager_ms = ev0.elapsed_time(ev1)
    launches_eager = rn.retnet_kernel_launch_count() - launches0

    # The same number of steps captured once as a CUDA graph (each node keeps
    # its own inputs and position) and replayed: no host work per step.
    graph = torch.cuda.CUDAGraph()
    launches1 = rn.retnet_kernel_launch_count()
    with torch.cuda.graph(graph):
        for i in range(steps):
            step(steps + i)
    graph_launches = rn.retnet_kernel_launch_count() - launches1
    graph.replay()                                    # warm-up replay
    torch.cuda.synchronize()
    clocks2 = ClockSampler(dev.index or 0)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks2.start()
    ev0.record(stream)
    graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    clock_info2 = clocks2.stop()
    ms = ev0.elapsed_time(ev1)
    if world > 1:
        import torch.distributed as dist
        ms = max_over_ranks(ms, dist, dev)
    del graph
    rn.retnet_check_device_errors(dev)
    peaks, src = load_peaks()
    tot, cnt = kern["retention_step"]
    eager_avg_s = tot / cnt / 1e3          # includes launch latency when the host lags
    avg_s = ms / steps / 1e3               # graph replay: kernel time plus node gaps
    bytes_step = B * H * (8 * d * d + T * 2 * 4 * d)
    res = {
        "batch": B, "tokens_per_call": T, "steps": steps,
        "steps_per_s": world * steps / (ms / 1e3) if T == 1 else None,
        "calls_per_s": world * steps / (ms / 1e3) if T > 1 else None,
        "tokens_per_s": world * B * T * steps / (ms / 1e3),
        "us_per_step": avg_s * 1e6,
        "l2": "state larger than L2" if bytes_step > 126e6 else "state fits in L2 (L2-resident)",
        "roofline": {"kernel": "retention_step", "bound": "hbm",
                     "state_l2_resident": bytes_step <= 126e6,
                     "achieved": bytes_step / avg_s / 1e9,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": bytes_step / avg_s / 1e9 / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": src, "work_per_launch": bytes_step},
        "gpu_launches": graph_launches, "clocks": clock_info2,
        "eager": {"ms_per_step": eager_ms / steps, "kernel_event_us": eager_avg_s * 1e6,
                  "clocks": clock_info, "gpu_launches": launches_eager},
        "timing": "one replay of a CUDA graph holding all timed steps (one kernel per step); "
                  "the roofline divides the algorithmic bytes by the replay's time per step",
    }
    if T > 1:
        # the state update and the output cost 4 dk dv flops per head-token
        # (float32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 flop x clock)
        flops = B * H * T * 4 * d * d
        alu_peak = 148 * 128 * 2 * (peaks.get("sm_max_mhz", 1965.0) * 1e6) / 1e12
        res["roofline_alu"] = {"bound": "alu", "achieved": flops / avg_s / 1e12,
                               "peak": alu_peak, "unit": "TFLOP/s",
                               "frac": flops / avg_s / 1e12 / alu_peak, "work_per_launch": flops}
    del state, qd, kd, vd, o
    torch.cuda.empty_cache()
    return res


def run_decode(args, w):
    """Decode-only line: one timed step = one recurrent step for every
    sequence of the batch (state seeded by an 8192-token GPU prefill)."""
    import torch

    import linear_recurrent_sequence_02_b200 as rn
    from linear_recurrent_sequence_02_b200.build import build

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    build()
    rn.load_library()
    rn.retnet_set_launch_overlap(not args.no_overlap)
    B, T = args.batch, args.tokens
    r = measure_decode(args, w, B, T, dev)
    H, d, n = w.heads, w.d, w.seqlen
    line = {
        "metric": "decode steps/s (all sequences advance one token)" if T == 1 else
                  f"multi-token decode calls/s (all sequences advance {T} tokens per call)",
        "value": r["steps_per_s"] if T == 1 else r["calls_per_s"],
        "unit": "steps/s" if T == 1 else "calls/s", "tokens_per_call": T,
        "n_gpus": 1, "steps": r["steps"], "warmup": args.warmup,
        "ms_per_step": r["us_per_step"] / 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 state, bf16 q/k/v", "data": "synthetic",
        "config": {"workload": f"decode7b: H={H} d={d} batch {B}, state from an {n}-token prefill"
                               + ("" if T == 1 else f", {T} tokens per call"),
                   "batch": B, "tokens_per_call": T, "l2": r["l2"]},
        "timing": r["timing"], "eager": r["eager"], "tokens_per_s": r["tokens_per_s"],
        "roofline": r["roofline"], "kernel_avg_us": r["us_per_step"],
        "gpu_launches": r["gpu_launches"], "clocks": r["clocks"],
        "launch_overlap": not args.no_overlap,
    }
    if "roofline_alu" in r:
        line["roofline_alu"] = r["roofline_alu"]
    print(json.dumps(line), flush=True)


def run_layer(args, w, chunk):
    """The multi-scale retention layer (retnet_msr_layer): Q/K/V/G projection
    GEMM, the gated chunkwise prefill, and the output projection GEMM.  One
    timed step = one layer pass over the workload's batch."""
    import torch

    import linear_recurrent_sequence_02_b200 as rn
    from linear_recurrent_sequence_02_b200.build import build

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    build()
    rn.load_library()
    rn.retnet_set_launch_overlap(not args.no_overlap)
    if args.pairs is not None:
        rn.retnet_set_output_pairing(args.pairs)
    B, n, H, d = w.batch, w.seqlen, w.heads, w.d
    hidden = w.hidden or H * d
    gam = rn.retnet_default_gammas(H)
    sets = []
    for i in range(3):                                # rotating inputs
        x, wqkvg, wo = wl.make_msr_inputs(B, n, hidden, H, d, w.seed + 17 * i)
        sets.append(tuple(torch.from_numpy(a).to(torch.bfloat16).to(dev)
                          for a in (x, wqkvg, wo)))
    y = torch.empty(B, n, hidden, dtype=torch.bfloat16, device=dev)
    st = torch.empty(B, H, d, d, device=dev)
    ws = rn.retnet_workspace(rn.retnet_msr_workspace_size(B, H, n, d, hidden, chunk), dev)

    def step(i):
        x, wqkvg, wo = sets[i % 3]
        rn.retnet_msr_layer(x, wqkvg, wo, gam, chunk, state_out=st, out=y, workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    rn.retnet_profiler_reset()
    rn.retnet_profiler_select(None)
    rn.retnet_profiler_enable(True)
    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    rn.retnet_profiler_enable(False)
    kern = rn.retnet_profiler_read()
    rn.retnet_check_device_errors(dev)
    launches0 = rn.retnet_kernel_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.steps):
            step(i)
    launches = rn.retnet_kernel_launch_count() - launches0
    graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    ev0.record(stream)
    graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    del graph
    rn.retnet_check_device_errors(dev)
    peaks, src = load_peaks()
    rows = B * n
    gemm_flops = {"gemm_qkvg": 2 * rows * 4 * H * d * hidden,
                  "gemm_out": 2 * rows * hidden * H * d}
    gemms = {}
    for name, fl in gemm_flops.items():
        if name in kern:
            tot, cnt = kern[name]
            avg_s = tot / cnt / 1e3
            gemms[name] = {"avg_us": avg_s * 1e6, "achieved": fl / avg_s / 1e12,
                           "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                           "frac": fl / avg_s / 1e12 / peaks["bf16_tflops"],
                           "work_per_launch": fl}
    step_s = ms / args.steps / 1e3
    total_kern = sum(v[0] for v in kern.values())
    alg = sum(gemm_flops.values()) + algorithmic_flops_per_token_head(d, chunk) * rows * H
    line = {
        "metric": "MSR layer tokens/s (Q/K/V/G projection, gated chunkwise retention, "
                  "output projection)",
        "value": rows / step_s, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name} MSR layer: B={B} n={n} hidden={hidden} H={H} d={d} "
                               f"chunk {chunk}, random weights",
                   "batch": B, "seqlen": n, "hidden": hidden, "heads": H, "d": d,
                   "chunk": chunk,
                   "l2": "3 rotating input sets; the five [B n, H d] intermediates of a step "
                         "exceed L2"},
        "roofline": dict(gemms.get("gemm_qkvg", {}), kernel="gemm_qkvg", bound="tensor",
                         peak_source=src, traffic=None),
        "gemms": gemms,
        "tflops_algorithmic": alg / step_s / 1e12,
        "frac_of_bf16_peak": alg / step_s / 1e12 / peaks["bf16_tflops"],
        "kernels": {k: {"avg_us": 1e3 * v[0] / v[1], "launches_per_step": v[1] / 3,
                        "share": v[0] / max(total_kern, 1e-12)} for k, v in kern.items()},
        "gpu_launches": launches, "clocks": clock_info, "peak_source": src,
        "timing": "one replay of a CUDA graph holding the K timed steps; 'kernels' are 3 "
                  "steps with every kernel bracketed by events",
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["layer200m", "layer3b", "long7b", "decode7b"],
                    default="long7b")
    ap.add_argument("--batch", type=int, default=128, help="decode7b batch")
    ap.add_argument("--tokens", type=int, default=1,
                    help="decode7b: tokens per call (above 1: the recurrent form)")
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's sequence length (length sweeps)")
    ap.add_argument("--algo", choices=["auto", "simt", "tensor"], default="auto")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the decode legs (batch 32, 128) and the secondary prefill shape")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass of the prefill (no epilogue) instead")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch kernels without programmatic launch overlap")
    ap.add_argument("--pairs", type=int, choices=[0, 1, 2], default=None,
                    help="output pass: 1 CTA pairs folding q, 2 CTA pairs with q folded by the "
                         "prep pass, 0 single CTAs (default: the library's own default)")
    ap.add_argument("--layer", action="store_true",
                    help="time the whole multi-scale retention layer (projections included)")
    ap.add_argument("--form", choices=["chunkwise", "parallel"], default="chunkwise",
                    help="prefill form; 'parallel' times the parallel form alone (no decode)")
    args = ap.parse_args()
    w = wl.WORKLOADS[args.workload]
    if args.seqlen:
        # same shape with another sequence length (a length sweep, not a
        # configuration of its own); the workload name records it
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}@n{args.seqlen}", seqlen=args.seqlen)
    chunk = args.chunk or w.chunk
    if args.impl == "reference":
        run_reference(args, w, chunk)
    elif args.workload == "decode7b":
        run_decode(args, w)
    elif args.backward:
        run_backward(args, w, chunk)
    elif args.layer:
        run_layer(args, w, chunk)
    else:
        run_ours(args, w, chunk)


if __name__ == "__main__":
    main()
