"""Benchmark of the online 2:4 prune + compress + quantize + error-energy path.

Workload (one step): a batch of B = 8 linear-layer inputs X, each bf16
4096 x 4096, Student-t (nu = 4, unit variance) with 8 outlier channels x50.
A step runs every row of the hot path once over the batch, pass by pass; each
pass is one batched call over all 8 operands (one kernel launch), so each
pass reads its operands from HBM (the batch is 256 MiB, twice the L2):
  1. per-tensor FP8 scale and per-row amax of each X       ss24_amax_rows
  2. fused 2:4 magnitude prune + compress + FP8 E4M3 of the
     kept values + energies (E_total, E_prune, E_q)        ss24_prune24_quant_fused
  3. dense FP8 E4M3 partner (same scale) + energy          ss24_quantize_fp8
  4. dense INT8, one scale per row (from the row amax),
     partner + energy                                      ss24_quantize_int_rows
  5. predicted R against both partners (one launch each)   ss24_predicted_ratio
The whole step is one CUDA graph, the passes chained by programmatic dependent
launch. Every 8th step of the timed region instead replays a copy of that graph
with an event-record node at every pass boundary, the nodes pointed at that
step's own events: the per-kernel durations are CUDA events on the launching
stream inside the timed region (an event node ends the overlap of the launches
it separates, so those steps are a little slower, and are counted).

Prints ONE JSON line (rank 0). ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fused 2:4 prune+compress+quant HBM GB/s and % of peak/memcpy; Gelem/s"
WORKLOAD = ("linear-input X bf16 4096x4096 (Student-t nu=4 /sqrt2, 8 outlier channels x50), batch of 8 per step: "
            "FP8 tensor scale, fused 2:4 magnitude prune+compress+FP8 E4M3 kept values, dense FP8 and dense INT8 "
            "per-row partners, energies, predicted R")
M = K = 4096
BATCH = 8
EVENT_EVERY = 8   # steps per evented step in the timed region


def algorithmic_bytes(m=M, k=K):
    """Bytes each pass must move per operand (bf16 in; see the DESIGN notes)."""
    n = m * k
    return {
        "tensor_scale": 2 * n + 4 * m,                 # read X; write the row amax
        "fused_24_fp8": 2 * n + n // 2 + n // 8,       # read X; write FP8 codes (k/2) + metadata (k/8)
        "dense_fp8": 2 * n + n,                        # read X; write FP8 codes
        "dense_int8_row": 2 * n + 4 * m + n + 4 * m,   # read X and the row amax; write INT8 codes + row scales
        "ratio": 0,
    }


# The sources the step's kernels are built from: the stream kernel (its
# template, helpers, dispatch and bf16 instantiations), the ratio kernel and the
# launch code. The ncu traffic figures are valid while these hash the same.
STEP_KERNEL_SOURCES = ("device.cuh", "internal.cuh", "pass_impl.cuh", "pass_dispatch.cuh", "pass_bf16.cu",
                       "misc.cu", "abi.cu")


def kernel_source_sha():
    """Hash of the step kernels' CUDA sources (the ncu traffic figures are valid for one)."""
    import hashlib
    h = hashlib.sha256()
    src = os.path.join(ROOT, "semi_structured_sparsity_online_b200", "csrc")
    for name in STEP_KERNEL_SOURCES:
        with open(os.path.join(src, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(pass_name):
    """DRAM bytes per launch of a pass from the committed ncu capture, or None
    when the kernels changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("source_sha") != kernel_source_sha():
        return None
    return t.get(pass_name)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read-only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x2: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x4: "applications_clocks_setting", 0x10: "sync_boost", 0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def make_batch(seed0=1):
    from semi_structured_sparsity_online_b200 import synth
    xs = []
    for b in range(BATCH):
        x, _ = synth.linear_input(M, K, seed=seed0 + b)
        xs.append(x)
    return xs


class Cudart:
    """The few runtime calls torch does not expose: event-record nodes in a
    captured graph, repointed to fresh events before every replay."""
    EVENT_RECORD_EXTERNAL = 0x1
    NODE_TYPE_EVENT_RECORD = 7

    def __init__(self):
        import ctypes
        self.c = ctypes
        self.rt = ctypes.CDLL("libcudart.so.12")

    def check(self, err, what):
        if err != 0:
            raise RuntimeError(f"{what} failed with CUDA error {err}")

    def event_create(self):
        ev = self.c.c_void_p()
        self.check(self.rt.cudaEventCreate(self.c.byref(ev)), "cudaEventCreate")
        return ev

    def record_external(self, ev, stream):
        self.check(self.rt.cudaEventRecordWithFlags(ev, self.c.c_void_p(stream), self.EVENT_RECORD_EXTERNAL),
                   "cudaEventRecordWithFlags")

    def elapsed_ms(self, a, b):
        ms = self.c.c_float()
        self.check(self.rt.cudaEventElapsedTime(self.c.byref(ms), a, b), "cudaEventElapsedTime")
        return ms.value

    def event_nodes(self, graph):
        """{event handle value: node} for the event-record nodes of a graph."""
        c = self.c
        n = c.c_size_t(0)
        g = c.c_void_p(graph)
        self.check(self.rt.cudaGraphGetNodes(g, None, c.byref(n)), "cudaGraphGetNodes")
        nodes = (c.c_void_p * n.value)()
        self.check(self.rt.cudaGraphGetNodes(g, nodes, c.byref(n)), "cudaGraphGetNodes")
        out = {}
        for i in range(n.value):
            t = c.c_int()
            self.check(self.rt.cudaGraphNodeGetType(c.c_void_p(nodes[i]), c.byref(t)), "cudaGraphNodeGetType")
            if t.value == self.NODE_TYPE_EVENT_RECORD:
                ev = c.c_void_p()
                self.check(self.rt.cudaGraphEventRecordNodeGetEvent(c.c_void_p(nodes[i]), c.byref(ev)),
                           "cudaGraphEventRecordNodeGetEvent")
                out[ev.value] = c.c_void_p(nodes[i])
        return out

    def set_node_event(self, graph_exec, node, ev):
        self.check(self.rt.cudaGraphExecEventRecordNodeSetEvent(self.c.c_void_p(graph_exec), node, ev),
                   "cudaGraphExecEventRecordNodeSetEvent")


class Step:
    """Device buffers and per-pass CUDA graphs for one step over the batch.
    Each pass is one batched call (one kernel launch over all 8 operands)."""

    def __init__(self, ss, x_dev, stream):
        import torch
        self.ss, self.torch, self.stream = ss, torch, stream
        self.x = x_dev                                                # [BATCH, M, K]
        dev = x_dev.device
        self.ws = ss.Workspace(dev, stream)
        self.scale = torch.empty(BATCH, dtype=torch.float32, device=dev)
        self.row_amax = torch.empty((BATCH, M), dtype=torch.float32, device=dev)
        self.sp = ss._alloc_outputs(M, K, ss.SPARSE_24, ss.make_format("fp8"), torch.bfloat16, dev, BATCH)
        self.d8 = ss._alloc_outputs(M, K, ss.DENSE, ss.make_format("fp8"), torch.bfloat16, dev, BATCH)
        self.di = ss._alloc_outputs(M, K, ss.DENSE, ss.make_format("int", 8, 0), torch.bfloat16, dev, BATCH)
        self.e = torch.zeros((3, BATCH, 4), dtype=torch.float64, device=dev)   # sparse, dense fp8, dense int8
        self.r = torch.zeros((2, BATCH, 4), dtype=torch.float64, device=dev)   # R vs fp8, R vs int8
        self.passes = ["tensor_scale", "fused_24_fp8", "dense_fp8", "dense_int8_row", "ratio"]
        self.launches_per_step = 4 + 2

    def run_pass(self, name):
        ss, s, x = self.ss, self.stream, self.x
        if name == "tensor_scale":
            # the FP8 tensor scale and the per-row amax of the INT8 partner in
            # one read (magnitude score: the kept amax equals the amax of all)
            ss.amax_rows(x, pattern=ss.DENSE, scale_fmt="fp8", ws=self.ws, stream=s, out=self.row_amax,
                         scale_out=self.scale)
        elif name == "fused_24_fp8":
            ss.run(x, pattern=ss.SPARSE_24, fmt="fp8", tensor_scale=self.scale, energy=self.e[0], ws=self.ws,
                   stream=s, out=self.sp)
        elif name == "dense_fp8":
            # for the magnitude score the kept amax equals the amax of all values,
            # so the 2:4 scales are the dense FP8 scales too
            ss.run(x, pattern=ss.DENSE, fmt="fp8", tensor_scale=self.scale, energy=self.e[1], ws=self.ws,
                   stream=s, out=self.d8)
        elif name == "dense_int8_row":
            ss.run_int_rows(x, self.row_amax, pattern=ss.DENSE, bits=8, energy=self.e[2], ws=self.ws, stream=s,
                            out=self.di)
        elif name == "ratio":
            ss.predicted_ratio(self.e[0], self.e[1], out=self.r[0], stream=s)
            ss.predicted_ratio(self.e[0], self.e[2], out=self.r[1], stream=s)

    def run_eager(self):
        for p in self.passes:
            self.run_pass(p)

    def capture(self, rt):
        """The whole step as one CUDA graph (the passes chained by
        programmatic dependent launch), with an event-record node before each
        pass and after the last one. Before each replay the nodes are pointed
        at that step's own events, so every step's pass boundaries are timed
        with CUDA events on the launching stream."""
        torch = self.torch
        self.rt = rt
        marks = [rt.event_create() for _ in range(len(self.passes) + 1)]
        self.graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(self.graph, stream=self.stream):
            for i, p in enumerate(self.passes):
                rt.record_external(marks[i], self.stream.cuda_stream)
                self.run_pass(p)
            rt.record_external(marks[-1], self.stream.cuda_stream)
        nodes = rt.event_nodes(self.graph.raw_cuda_graph())
        self.nodes = [nodes[m.value] for m in marks]
        self.graph.instantiate()
        self.exec = self.graph.raw_cuda_graph_exec()
        # the same step without event nodes: every pass boundary stays a
        # programmatic (overlapping) launch
        self.plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.plain, stream=self.stream):
            self.run_eager()

    def replay(self, events=None):
        """One step. With events (len(passes) + 1 fresh events) the evented
        graph runs and records the pass boundaries; else the plain graph."""
        if events is None:
            self.plain.replay()
            return
        for node, ev in zip(self.nodes, events):
            self.rt.set_node_event(self.exec, node, ev)
        self.graph.replay()


def memcpy_gbps(torch, dev, nbytes=1 << 30, iters=10):
    a = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=dev)
    b = torch.empty_like(a)
    b.copy_(a)
    torch.cuda.synchronize()
    best = None
    for _ in range(iters):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        b.copy_(a)
        e.record()
        e.synchronize()
        t = s.elapsed_time(e) / 1e3
        best = t if best is None else min(best, t)
    del a, b
    return 2 * nbytes / best / 1e9


def cpu_baseline_sample(xs_host, rows=96):
    """The oracle, as it stands, on a bounded sample: the first `rows` rows of
    every operand of the batch through the same passes (each sample treated as
    its own operand). Returns (GB/s of algorithmic bytes, seconds, cores)."""
    import oracle
    t0 = time.perf_counter()
    for x in xs_host:
        xs = np.ascontiguousarray(x[:rows])
        ts = oracle.tensor_scale(xs, "fp8")
        sp = oracle.run(xs, pattern=oracle.SPARSE_24, fmt="fp8", tensor_scale=ts)["energy"]
        d8 = oracle.run(xs, pattern=oracle.DENSE, fmt="fp8", tensor_scale=ts)["energy"]
        di = oracle.run(xs, pattern=oracle.DENSE, fmt="int", bits=8, group=0)["energy"]
        oracle.ratio(sp, d8)
        oracle.ratio(sp, di)
    dt = time.perf_counter() - t0
    nbytes = sum(algorithmic_bytes(rows, K).values()) * len(xs_host)
    return nbytes / dt / 1e9, dt, 1


def run_cuda(args):
    import torch
    import torch.distributed as dist

    from semi_structured_sparsity_online_b200 import ss24 as ss

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    ss.lib()
    stream = torch.cuda.Stream(device=dev)

    # each rank draws its own batch (independent problems: weak scaling)
    xs_host = make_batch(seed0=1 + 100 * rank)
    x_pinned = torch.from_numpy(np.stack(xs_host).view(np.int16)).view(torch.bfloat16).pin_memory()
    x_dev = torch.empty((BATCH, M, K), dtype=torch.bfloat16, device=dev)
    with torch.cuda.stream(stream):
        x_dev.copy_(x_pinned, non_blocking=True)
    stream.synchronize()

    step = Step(ss, x_dev, stream)
    with torch.cuda.stream(stream):
        step.run_eager()          # first launches: kernel attributes, tensor-map entry point
    stream.synchronize()
    rt = Cudart()
    step.capture(rt)
    with torch.cuda.stream(stream):       # graph replays launch on the current stream
        for _ in range(args.warmup):
            step.replay()
        step.replay([rt.event_create() for _ in range(len(step.passes) + 1)])   # the evented graph too
    stream.synchronize()
    if step.ws.error(stream) != 0:
        raise RuntimeError("a kernel wait timed out during warm-up")

    # ---- timed region: K steps; every EVENT_EVERY-th step runs the evented
    # graph (its pass boundaries timed by CUDA events), the others the plain one ----
    n_ev = len(step.passes) + 1
    timed = [i for i in range(args.steps) if i % EVENT_EVERY == 0]
    evs = {i: [rt.event_create() for _ in range(n_ev)] for i in timed}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with clocks, torch.cuda.stream(stream):
        start.record(stream)
        for i in range(args.steps):
            step.replay(evs.get(i))
        end.record(stream)
        end.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_s = start.elapsed_time(end) / 1e3
    per_pass = {p: 0.0 for p in step.passes}
    for i in timed:
        for j, p in enumerate(step.passes):
            per_pass[p] += rt.elapsed_ms(evs[i][j], evs[i][j + 1]) / 1e3
    if world > 1:
        t = torch.tensor([elapsed_s], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_s = t.item()
    err = step.ws.error(stream)
    if err != 0:
        raise RuntimeError(f"a kernel wait timed out (code {err})")

    ab = algorithmic_bytes()
    step_bytes = BATCH * sum(ab.values())
    ms_per_step = elapsed_s / args.steps * 1e3
    value = world * step_bytes * args.steps / elapsed_s / 1e9
    elems = world * BATCH * M * K * args.steps / elapsed_s / 1e9

    # ---- end to end through the public API with host buffers ----
    e2e_steps = max(3, min(20, args.steps // 10))
    r_host = torch.empty((2, BATCH, 4), dtype=torch.float64).pin_memory()
    h2d = BATCH * M * K * 2
    d2h = r_host.numel() * 8
    with torch.cuda.stream(stream):
        x_dev.copy_(x_pinned, non_blocking=True)     # warm-up of the copy path
        step.replay()
        r_host.copy_(step.r, non_blocking=True)
    stream.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            x_dev.copy_(x_pinned, non_blocking=True)
            step.replay()
            r_host.copy_(step.r, non_blocking=True)
        e1.record(stream)
    e1.synchronize()
    e2e_s = e0.elapsed_time(e1) / 1e3
    if world > 1:
        t = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_s = t.item()
    e2e_value = world * step_bytes * e2e_steps / e2e_s / 1e9

    peak, peak_kind = load_peaks()
    mc = memcpy_gbps(torch, dev)

    # dominant kernel: the pass with the largest device time
    dom = max((p for p in step.passes if ab[p] > 0), key=lambda p: per_pass[p])
    # one launch per pass covers the whole batch (the ratio pass is two tiny launches)
    dom_us = per_pass[dom] / len(timed) * 1e6
    achieved = BATCH * ab[dom] / (dom_us * 1e-6) / 1e9
    passes = {}
    for p in step.passes:
        us = per_pass[p] / len(timed) * 1e6
        passes[p] = {"us_per_step": round(us, 3),
                     "gbps": round(BATCH * ab[p] / (us * 1e-6) / 1e9, 1) if ab[p] else None,
                     "bytes_per_launch": BATCH * ab[p]}
    traffic = measured_traffic(dom)

    r = step.r.cpu().numpy()
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "operands_per_step": BATCH, "m": M, "k": K, "input_dtype": "bf16",
                   "l2": "inputs larger than L2: 8 x 32 MiB per step; each pass is one launch over all 8 "
                         "operands before the next pass", "parallelism": f"dp{world} (independent batches)"},
        "gelem_per_s": round(elems, 2),
        "frac_of_peak": round(value / world / peak, 4),
        "memcpy_gbps": round(mc, 1),
        "frac_of_memcpy": round(value / world / mc, 4),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "algorithmic_bytes_per_launch": BATCH * ab[dom]},
        "passes": passes,
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": clocks.summary(),
        "predicted_r": {"vs_dense_fp8": round(float(r[0, 0, 3]), 4), "vs_dense_int8_row": round(float(r[1, 0, 3]), 4),
                        "energy_loss_24": round(float(r[0, 0, 0]), 5)},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbps, dt, cores = cpu_baseline_sample(xs_host, rows=args.cpu_rows)
        result["cpu_baseline"] = {"value": round(gbps, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                                  "sample": f"first {args.cpu_rows} rows of each of the 8 operands, all passes "
                                            f"({dt:.1f} s of CPU work)"}
    if world > 1:
        del step
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def run_reference(args):
    """The oracle on the host cores, per step a bounded sample of the workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    xs_host = make_batch()
    rows = args.ref_rows
    for _ in range(args.warmup):
        cpu_baseline_sample(xs_host[:1], rows=rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cpu_baseline_sample(xs_host[:1], rows=rows)
    dt = time.perf_counter() - t0
    nbytes = sum(algorithmic_bytes(rows, K).values()) * args.steps
    value = nbytes / dt / 1e9
    sample = f"per step: first {rows} rows of one 4096x4096 operand through all passes"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ss24", "reference"], default="ss24")
    ap.add_argument("--cpu-rows", type=int, default=4096)
    ap.add_argument("--ref-rows", type=int, default=8, help="rows of one operand per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
