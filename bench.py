"""Benchmark of the differentiable sparse SPD solve on B200.

One step = the whole hot path on the 2-D 5-point Poisson system on a 1024x1024
grid (n = 1,048,576, nnz = 5,238,784): a fixed 1000-iteration Jacobi-PCG
forward solve, the 1000-iteration adjoint solve A^T lambda = x - x*, and the
sparse value gradient -lambda_i x_j (torch-sla summary page, "Experimental
results": 10^6 DOF, 1000 CG iterations; "Methodology" 2 for the adjoint).

value      = CG iterations per second over all ranks (2000 per step per rank),
             inputs resident in HBM, L2 flushed between steps, CUDA events.
e2e        = the same metric through the public autograd API (CSR.solve +
             backward) with the step's inputs copied from pinned host memory
             and the loss read back every step.
roofline   = the persistent CG kernel: algorithmic bytes per launch (1000
             iterations x the per-iteration traffic of a two-pass fused PCG:
             one sweep of A plus 11 vector passes) / its CUDA-event duration.
cpu_baseline = the CPU oracle (single thread) on a bounded sample of the step.

Multi-GPU (torchrun): every rank solves its own independent system (replicas;
the single system is not partitioned), time = max over ranks.
`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CG iter/s & fwd+adjoint solve ms; SpMV/CG HBM GB/s vs B200 peak (1 GPU)"
UNIT = "CG iterations/s"
N_GRID, ITERS = 1024, 1000
FALLBACK_HBM_GBS = 6650.0


def per_iteration_bytes(n: int, nnz: int, vbytes: int) -> int:
    """Two-pass fused PCG: A once ((vbytes + 4) nnz + 4 (n + 1)) + 11 vector passes."""
    return (vbytes + 4) * nnz + 4 * (n + 1) + 11 * vbytes * n


def grad_bytes(n: int, nnz: int, vbytes: int) -> int:
    """Value gradient: colind + gradient per entry, lambda, x and rowptr per row."""
    return (4 + vbytes) * nnz + (2 * vbytes + 4) * n


def edge_metrics(n: int, nnz: int, E: int, B: int, vbytes: int, asm_ms: float, grad_ms: float):
    """Algorithmic bytes of the edge kernels: assembly reads the shared pattern
    (row pointers, columns, entry-to-edge map) once and per system the weights,
    writing the values; the fused gradient reads the edge list once and per
    system lambda and x, writing dL/dw (the shift gradient's sum is included)."""
    asm_bytes = 4 * (n + 1) + 8 * nnz + B * vbytes * (E + nnz + 1)
    grad_bytes_ = 8 * E + B * vbytes * (2 * n + E + 1)
    return {"assemble_ms": asm_ms, "assemble_gbs": asm_bytes / (asm_ms / 1000.0) / 1e9,
            "assemble_bytes": asm_bytes, "edge_grad_bytes": grad_bytes_,
            "edge_grad_gbs": grad_bytes_ / (grad_ms / 1000.0) / 1e9}


def source_digest(files=None) -> str:
    """sha256 (16 hex digits) of the library source: every file of csrc/, or
    only `files` (names in csrc/), those a profiled kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "differentiable_sparse_linear_csr_b200", "csrc")
    for f in sorted(files if files else os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def profile_digest_matches(text: str) -> bool:
    """A summary's `source_digest` against the current source: over the files
    its `source_files` line names when it has one (the profiled kernel's own
    sources), else over all of csrc/."""
    d = re.search(r"source_digest:\s*([0-9a-f]+)", text)
    if not d:
        return False
    f = re.search(r"^source_files:\s*(.+)$", text, re.M)
    try:
        return d.group(1) == source_digest(f.group(1).split() if f else None)
    except OSError:
        return False


def profile_traffic(kernel_key: str, iters_per_launch: float):
    """DRAM bytes per launch from a committed ncu summary whose source digest
    matches the library source: either a per-launch figure, or a per-iteration
    figure (for kernels whose traffic grows with the iteration count) scaled to
    this launch's iterations."""
    path = os.path.join(ROOT, "profiles", f"{kernel_key}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    if not profile_digest_matches(text):
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if m:
        return float(m.group(1))
    m = re.search(r"traffic_bytes_per_iteration:\s*([0-9.eE+]+)", text)
    if m:
        return float(m.group(1)) * iters_per_launch
    return None


def profile_metric(kernel_key: str, name: str):
    """A named figure (`name: value`) from a committed ncu summary, or None."""
    path = os.path.join(ROOT, "profiles", f"{kernel_key}.md")
    if not os.path.exists(path):
        return None
    m = re.search(rf"^{re.escape(name)}:\s*([0-9.eE+-]+)", open(path).read(), re.M)
    return float(m.group(1)) if m else None


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region.

    NVML (read-only queries) from a thread every 5 ms, so that timed regions of
    a few tens of milliseconds still get samples; nvidia-smi at 200 ms when
    NVML cannot be used."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index: int):
        import threading
        self.proc = None
        self.samples = []
        self.stop_evt = threading.Event()
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)

            def run():
                while not self.stop_evt.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx,
                                             int(reasons_fn(h))))
                    except Exception:
                        pass
                    self.stop_evt.wait(0.005)
            self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx, int(reasons_fn(h))))
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            sm = [float(a) for a, _, _ in self.samples]
            mx = [float(b) for _, b, _ in self.samples]
            reasons = {name for _, _, r in self.samples for name, bit in self.BITS.items() if r & bit}
            if not sm:
                return None
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                    "reasons": sorted(reasons), "source": "nvml"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons), "source": "nvidia-smi"}


_WORKLOAD = {}

WORKLOADS = ("c2", "c1", "c3", "c4", "c5", "c5rcm", "c4list", "c3b4")
CPU_ITERS = {"c1": 1000, "c2": 300, "c3": 100, "c4": 2000, "c5": 12, "c5rcm": 12, "c4list": 60,
             "c3b4": 100}


def split_workload(w, world: int, rank: int):
    """Rank `rank`'s contiguous shard of the batch of `w` (the same batch on
    every rank; see sharding.shard_range)."""
    import dataclasses
    from differentiable_sparse_linear_csr_b200.sharding import shard_range
    lo, hi = shard_range(w.batch, world, rank)
    return dataclasses.replace(
        w, values=w.values[lo:hi], b=w.b[lo:hi], xstar=w.xstar[lo:hi],
        weights=None if w.weights is None else w.weights[lo:hi])


def load_workload(name: str, rank: int = 0):
    """The synthetic workload `name`; every rank gets its own seed (replicas)."""
    from differentiable_sparse_linear_csr_b200 import workloads as W
    key = (name, rank)
    if key not in _WORKLOAD:
        if name == "c1":
            w = W.c1_poisson64(seed=1 + 10 * rank)
        elif name == "c2":
            w = W.c2_poisson1024(seed=2 + 10 * rank, N=N_GRID, iters=ITERS)
        elif name == "c3":
            w = W.c3_diffusion3d(seed=3 + 10 * rank)
        elif name == "c4":
            w = W.c4_batched(seed=4 + 10 * rank)
        elif name == "c5":
            w = W.c5_knn(seed=5 + 10 * rank)
        elif name == "c5rcm":
            w = W.c5_knn(seed=5 + 10 * rank, order="rcm")
        elif name == "c4list":
            w = W.list_of_grids(seed=6 + 10 * rank)
        elif name == "c3b4":
            w = W.c3_batched(seed=3 + 10 * rank, B=4)
        else:
            raise ValueError(name)
        _WORKLOAD[key] = w
    return _WORKLOAD[key]


def oracle_sample(dtype_name: str, k_iters: int, name: str = "c2", edges: bool = False):
    """Oracle on a bounded sample of the step: k forward + k adjoint iterations +
    gradient, on system 0 of the workload (with edges: assembly from the edge
    weights first and the chain rule to them last)."""
    import numpy as np
    from oracle import oracle as O
    w = load_workload(name)
    npdt = np.float64 if dtype_name == "f64" else np.float32
    v, b, xs = w.values[0].astype(npdt), w.b[0].astype(npdt), w.xstar[0].astype(npdt)
    O.build()
    if w.item_rows is not None:
        # a list: its first 32 items, each k forward + k adjoint iterations
        ir = w.item_rows[:33]
        e = int(w.rowptr[ir[-1]])
        rp, ci = w.rowptr[:ir[-1] + 1], w.colind[:e]
        t0 = time.perf_counter()
        x, _ = O.pcg_list(ir, rp, ci, v[:e], b[:ir[-1]], fixed_iters=k_iters)
        lam, _ = O.pcg_list(ir, rp, ci, v[:e], (x - xs[:ir[-1]]).astype(npdt), adjoint=True,
                            fixed_iters=k_iters)
        O.grad_values(rp, ci, lam, x)
        dt = time.perf_counter() - t0
        return 2 * 32 * k_iters / dt, dt, x
    t0 = time.perf_counter()
    if edges:
        v = O.laplacian_assemble(w.rowptr, w.colind, w.edges[0], w.edges[1],
                                 w.weights[0].astype(npdt), w.shift)
    x, _ = O.pcg(w.rowptr, w.colind, v, b, fixed_iters=k_iters)
    lam, _ = O.cg_adjoint(w.rowptr, w.colind, v, (x - xs).astype(npdt), fixed_iters=k_iters)
    G = O.grad_values(w.rowptr, w.colind, lam, x)
    if edges:
        O.laplacian_grad_values(w.rowptr, w.colind, w.edges[0], w.edges[1], G)
    dt = time.perf_counter() - t0
    return 2 * k_iters / dt, dt, x


def host_cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_all_cores(args, k: int, x_single):
    """The same oracle sample with the oracle's source built with OpenMP, on
    every core this process may use, in a child process; its forward solution
    is checked against the single-threaded one to the parity tolerance (only
    the order of the dot products' additions differs)."""
    import tempfile
    import numpy as np
    cores = len(os.sched_getaffinity(0))
    with tempfile.TemporaryDirectory() as tmp:
        out = os.path.join(tmp, "x.npy")
        code = (f"import sys, json, numpy as np; sys.path.insert(0, {ROOT!r}); import bench; "
                f"r, t, x = bench.oracle_sample({args.dtype!r}, {k}, {args.workload!r}, {bool(args.edges)}); "
                f"np.save({out!r}, x); print(json.dumps([r, t]))")
        env = dict(os.environ, SLA_ORACLE_OPENMP="1", OMP_NUM_THREADS=str(cores), OMP_PROC_BIND="close")
        res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                             timeout=900)
        if res.returncode != 0:
            return {"error": res.stderr.strip().splitlines()[-1:] or ["failed"]}
        rate, secs = json.loads(res.stdout.strip().splitlines()[-1])
        x_omp = np.load(out)
    xs = np.asarray(x_single, np.float64)
    err = float(np.linalg.norm(np.asarray(x_omp, np.float64) - xs) / max(np.linalg.norm(xs), 1e-300))
    tol = 1e-8 if args.dtype == "f64" else 1e-4
    return {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle, OpenMP build of the same source",
            "cpu_model": host_cpu_model(), "seconds": secs,
            "x_rel_diff_vs_single_thread": err, "within_parity_tolerance": err <= tol}


def reduce_over_ranks(total_ms: float, iters_per_step: float, device):
    """Across ranks: the slowest rank's time (max) and every rank's work (sum).

    Replicas solve independent systems, so the job's throughput is all ranks'
    iterations over the slowest rank's time.  Single-rank runs pass through.
    """
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    w = torch.tensor([float(iters_per_step)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t.item()), float(w.item())


def spmv_bytes(n: int, nnz: int, vbytes: int) -> int:
    """One y = A x: the matrix once ((vbytes + 4) nnz + 4 (n + 1)), x once (ideal
    gather) and y written once."""
    return (vbytes + 4) * nnz + 4 * (n + 1) + 2 * vbytes * n


def time_kernel_ms(fn, flush, reps: int = 20, warmup: int = 3) -> float:
    """Mean CUDA-event time of fn() on the current stream, L2 flushed (outside
    the events) before every launch."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush.zero_()
        fn()
    total = 0.0
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        e1.synchronize()
        total += e0.elapsed_time(e1)
    return total / reps


def spmv_block(A, vals, n: int, nnz: int, B: int, vbytes: int, dt, dev, flush, peak: float) -> dict:
    """The standalone `.matvec` (sla_spmv, y = A x) on the workload's matrix."""
    import torch
    from differentiable_sparse_linear_csr_b200 import _lib as L
    x = torch.linspace(-1.0, 1.0, B * n, dtype=dt, device=dev).reshape(B, n)
    y = torch.empty(B, n, dtype=dt, device=dev)
    ms = time_kernel_ms(lambda: L.sla_spmv(A.handle, vals, x, y, 0, 1.0, 0.0), flush)
    by = spmv_bytes(n, nnz, vbytes) * B
    gbs = by / (ms / 1000.0) / 1e9
    # context for a launch this short: torch's own reduction reading the same
    # number of bytes, timed the same way (the same L2 flush before each)
    buf = torch.empty(by // 8, dtype=torch.float64, device=dev).uniform_()
    ms_read = time_kernel_ms(lambda: torch.sum(buf), flush)
    read_gbs = by / (ms_read / 1000.0) / 1e9
    del buf
    kernel = ("sla_spmv, pipelined one-thread rows: 256-row chunks copied to shared memory one chunk "
              "ahead (cp.async)" if A.props.lanes == 1 else "sla_spmv, sub-warp rows")
    return {"ms": ms, "algorithmic_bytes": by, "gbs": gbs, "frac_of_hbm_peak": gbs / peak,
            "same_bytes_read_gbs": read_gbs, "frac_of_same_bytes_read": gbs / read_gbs,
            "same_bytes_read": "torch.sum over a buffer of the same bytes, same flush before each",
            "kernel": kernel}


def l2_stream_peak_gbs(dev) -> float:
    """Bandwidth of an L2-resident copy: torch's vectorised copy of one 24 MB
    buffer into another (both stay in the 126 MB L2), 100 copies back to back
    in one CUDA graph, less the same graph of 4 KB copies (the per-launch cost),
    counting bytes read plus written.  The denominator of kernels whose working
    set stays in L2."""
    import torch

    def graph_ms(numel: int) -> float:
        src = torch.ones(numel, dtype=torch.float64, device=dev)
        dst = torch.empty_like(src)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            for _ in range(3):
                dst.copy_(src)
        torch.cuda.current_stream(dev).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(100):
                dst.copy_(src)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        best = float("inf")
        for _ in range(5):
            e0.record()
            g.replay()
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del g
        return best

    big = 3 << 20                                   # 3 Mi doubles = 24 MB
    t = graph_ms(big) - graph_ms(512)
    return 2 * big * 8 * 100 / (t / 1000.0) / 1e9


def secondary_workload(args, name: str, dev, flush, peak: float, peak_kind: str) -> dict:
    """The HBM-streaming 3-D diffusion workload measured beside the headline:
    the same step (forward PCG, g = x - x*, adjoint, value gradient), timed the
    same way, with its solve kernel's roofline and its standalone SpMV."""
    import torch
    import differentiable_sparse_linear_csr_b200 as sla
    from differentiable_sparse_linear_csr_b200 import _lib as L
    w = load_workload(name)
    dt = torch.float64 if args.dtype == "f64" else torch.float32
    vbytes = 8 if args.dtype == "f64" else 4
    n, nnz, B = w.n, w.nnz, w.batch
    A = sla.CSR(torch.from_numpy(w.rowptr).to(dev), torch.from_numpy(w.colind).to(dev),
                batch=B, dtype=dt, symmetric=True)
    vals = torch.from_numpy(w.values).to(dev, dt).contiguous()
    b = torch.from_numpy(w.b).to(dev, dt).contiguous()
    xs = torch.from_numpy(w.xstar).to(dev, dt).contiguous()
    x, g, lam = (torch.empty(B, n, dtype=dt, device=dev) for _ in range(3))
    G = torch.empty(B, nnz, dtype=dt, device=dev)
    fi = [torch.empty(B, dtype=t, device=dev) for t in (torch.int32, torch.float64, torch.int32)]
    ai = [torch.empty(B, dtype=t, device=dev) for t in (torch.int32, torch.float64, torch.int32)]
    ws = torch.empty(L.sla_workspace_bytes(A.handle, L.SLA_OP_ADJOINT), dtype=torch.uint8, device=dev)
    opts = L.make_opts(rtol=w.rtol, fixed_iters=w.fixed_iters)
    stream = torch.cuda.current_stream()
    evs = []
    for k in range(args.warmup + args.steps):
        flush.zero_()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        e[0].record(stream)
        L.sla_cg_solve(A.handle, vals, b, x, opts, L.make_info(*fi), ws)
        e[1].record(stream)
        torch.sub(x, xs, out=g)
        e[2].record(stream)
        L.sla_cg_adjoint(A.handle, vals, g, lam, opts, L.make_info(*ai), ws)
        e[3].record(stream)
        L.sla_grad_values(A.handle, lam, x, G, 0)
        e[4].record(stream)
        if k >= args.warmup:
            evs.append(e)
    torch.cuda.synchronize()
    step_ms = statistics.mean(e[0].elapsed_time(e[4]) for e in evs)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    solve_ms = fwd_ms + statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    grad_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in evs)
    fwd_it, adj_it = int(fi[0].sum().item()), int(ai[0].sum().item())
    it_bytes = per_iteration_bytes(n, nnz, vbytes)
    achieved = (fwd_it + adj_it) * it_bytes / (solve_ms / 1000.0) / 1e9
    traffic = profile_traffic(f"cg_kernel_{name}_{args.dtype}", (fwd_it + adj_it) / 2)
    launch_ms = solve_ms / 2
    out = {"workload": f"{w.description}: forward and adjoint to relative residual {w.rtol:g} "
                       f"Jacobi-PCG iterations + sparse value gradient",
           "name": name, "n": n, "nnz": nnz, "value_dtype": args.dtype,
           "value": (fwd_it + adj_it) / (step_ms / 1000.0), "unit": UNIT,
           "fwd_adj_grad_ms": step_ms, "forward_ms": fwd_ms, "grad_ms": grad_ms,
           "forward_iters": fwd_it, "adjoint_iters": adj_it,
           "statuses": sorted(set(fi[2].tolist()) | set(ai[2].tolist())),
           "grad_gbs": grad_bytes(n, nnz, vbytes) * B / (grad_ms / 1000.0) / 1e9,
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "peak_source": peak_kind,
                        "traffic": traffic,
                        "traffic_gbs": None if traffic is None else traffic / (launch_ms / 1000.0) / 1e9,
                        "traffic_frac": None if traffic is None else
                        traffic / (launch_ms / 1000.0) / 1e9 / peak,
                        "kernel": f"PCG solve kernel (grid_onchip={A.props.grid_onchip}, "
                                  f"sliced={A.props.sliced}), one launch per solve",
                        "bytes_per_iteration": it_bytes, "launch_ms": launch_ms},
           "spmv": spmv_block(A, vals, n, nnz, B, vbytes, dt, dev, flush, peak)}
    del A
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    k = args.ref_iters
    for _ in range(args.warmup):
        oracle_sample(args.dtype, k, args.workload, args.edges)
    total_it, total_t = 0, 0.0
    for _ in range(args.steps):
        rate, dt, _ = oracle_sample(args.dtype, k, args.workload, args.edges)
        total_it += rate * dt                     # iterations of the sample (items x 2k for a list)
        total_t += dt
    v = total_it / total_t
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * total_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
            "config": workload_config(args),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"each step: {k} forward + {k} adjoint PCG iterations "
                                       f"{'of each of the first 32 items ' if args.workload == 'c4list' else ''}+ "
                                       f"{'edge-weight' if args.edges else 'value'} gradient of "
                                       f"system 0 of workload {args.workload}"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(args, w=None):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if w is None:
        w = load_workload(args.workload)
    mode = (f"fixed {w.fixed_iters} forward + {w.fixed_iters} adjoint" if w.fixed_iters
            else f"forward and adjoint to relative residual {w.rtol:g}")
    if args.edges:
        what = (f"{w.description}: assembly from the {len(w.edges[0])} edge weights, {mode} "
                f"Jacobi-PCG iterations, gradient to the edge weights and the shift")
    else:
        what = f"{w.description}: {mode} Jacobi-PCG iterations + sparse value gradient"
    return {"workload": what, "edges": bool(args.edges),
            "name": args.workload, "n": int(w.n), "nnz": int(w.nnz), "batch": int(w.batch),
            **({"items": int(len(w.item_rows) - 1)} if w.item_rows is not None else {}),
            "value_dtype": args.dtype, "l2": "flushed between steps (write of a 256 MiB buffer)",
            "parallelism": (f"one batch split along its systems x{world}" if getattr(args, "split_batch", False)
                            else f"replicas x{world}")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="sla", choices=["sla", "reference"])
    ap.add_argument("--dtype", default="f64", choices=["f64", "f32"])
    ap.add_argument("--ref-iters", type=int, default=40)
    ap.add_argument("--cpu-iters", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cpu-all-cores", action="store_true",
                    help="skip the OpenMP build of the oracle on all host cores")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the standalone SpMV and, on the default workload, the 3-D diffusion "
                         "block measured beside it")
    ap.add_argument("--strategy", type=int, default=0)
    ap.add_argument("--iters", type=int, default=0,
                    help="override the fixed iteration count (short profiler captures)")
    ap.add_argument("--workload", default="c2", choices=WORKLOADS)
    ap.add_argument("--split-batch", action="store_true",
                    help="shared-pattern batches (c4, c3b4): the ranks split one batch along the "
                         "systems instead of each solving its own replica (strong scaling)")
    ap.add_argument("--edges", action="store_true",
                    help="edge-weighted workloads (c3, c4, c5, c5rcm): assemble the values from "
                         "the edge weights and take the gradient back to them")
    args = ap.parse_args()
    if args.edges and args.workload not in ("c3", "c4", "c5", "c5rcm", "c3b4"):
        ap.error("--edges needs an edge-weighted workload (c3, c4, c5, c5rcm, c3b4)")
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch
    import torch.distributed as dist

    import differentiable_sparse_linear_csr_b200 as sla
    from differentiable_sparse_linear_csr_b200 import _lib as L
    from differentiable_sparse_linear_csr_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))

    dt = torch.float64 if args.dtype == "f64" else torch.float32
    vbytes = 8 if args.dtype == "f64" else 4
    if args.split_batch:
        w_all = load_workload(args.workload, 0)
        if w_all.item_rows is not None or w_all.batch < world:
            ap.error(f"--split-batch needs a shared-pattern batch of at least {world} systems")
        w = split_workload(w_all, world, rank)
    else:
        w = load_workload(args.workload, rank)
    n, nnz, B = w.n, w.nnz, w.batch
    fixed = args.iters if args.iters > 0 else w.fixed_iters
    if w.item_rows is not None:
        A = sla.CSRList(torch.from_numpy(w.item_rows).to(dev), torch.from_numpy(w.rowptr).to(dev),
                        torch.from_numpy(w.colind).to(dev), dtype=dt, symmetric=True)
    else:
        A = sla.CSR(torch.from_numpy(w.rowptr).to(dev), torch.from_numpy(w.colind).to(dev),
                    batch=B, dtype=dt, symmetric=True)
    vals = torch.from_numpy(w.values).to(dev, dt).contiguous()
    b = torch.from_numpy(w.b).to(dev, dt).contiguous()
    xs = torch.from_numpy(w.xstar).to(dev, dt).contiguous()
    x = torch.empty(B, n, dtype=dt, device=dev)
    g = torch.empty(B, n, dtype=dt, device=dev)
    lam = torch.empty(B, n, dtype=dt, device=dev)
    G = torch.empty(B, nnz, dtype=dt, device=dev)
    finfo = [torch.empty(A.n_info, dtype=t, device=dev) for t in (torch.int32, torch.float64, torch.int32)]
    ainfo = [torch.empty(A.n_info, dtype=t, device=dev) for t in (torch.int32, torch.float64, torch.int32)]
    ws = torch.empty(L.sla_workspace_bytes(A.handle, L.SLA_OP_ADJOINT), dtype=torch.uint8, device=dev)
    opts = L.make_opts(rtol=w.rtol, fixed_iters=fixed, strategy=args.strategy)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    if args.edges:
        E = len(w.edges[0])
        Ed = sla.EdgeLaplacian(A, torch.from_numpy(w.edges[0].astype(np.int32)).to(dev),
                               torch.from_numpy(w.edges[1].astype(np.int32)).to(dev))
        wts = torch.from_numpy(w.weights).to(dev, dt).contiguous()
        shift_t = torch.full((B,), w.shift, dtype=dt, device=dev)
        dwt = torch.empty(B, E, dtype=dt, device=dev)
        dst = torch.empty(B, dtype=dt, device=dev)
        ews = torch.empty(max(L.sla_edges_workspace_bytes(Ed.plan), 1), dtype=torch.uint8, device=dev)

    def step(e=None):
        if e: e[0].record(stream)
        if args.edges:
            L.sla_laplacian_assemble(Ed.plan, wts, shift_t, vals)
        if e: e[1].record(stream)
        L.sla_cg_solve(A.handle, vals, b, x, opts, L.make_info(*finfo), ws)
        if e: e[2].record(stream)
        torch.sub(x, xs, out=g)                       # dL/dx of L = 0.5 ||x - x*||^2
        if e: e[3].record(stream)
        L.sla_cg_adjoint(A.handle, vals, g, lam, opts, L.make_info(*ainfo), ws)
        if e: e[4].record(stream)
        if args.edges:
            L.sla_laplacian_grad(Ed.plan, lam, x, dwt, dst, 0, ews)
        else:
            L.sla_grad_values(A.handle, lam, x, G, 0)
        if e: e[5].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local) if rank == 0 else None
    events = [[ev() for _ in range(6)] for _ in range(args.steps)]
    for k in range(args.steps):
        flush.zero_()                                  # L2 flush, outside the step's events
        step(events[k])
    torch.cuda.synchronize()
    clock_info = clocks.stop() if clocks else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = [e[0].elapsed_time(e[5]) for e in events]
    asm_ms = [e[0].elapsed_time(e[1]) for e in events]
    fwd_ms = [e[1].elapsed_time(e[2]) for e in events]
    adj_ms = [e[3].elapsed_time(e[4]) for e in events]
    grad_ms = [e[4].elapsed_time(e[5]) for e in events]
    # every step does the same work (deterministic solver): iterations of the last one
    fwd_it = int(finfo[0].sum().item())
    adj_it = int(ainfo[0].sum().item())
    statuses = sorted(set(finfo[2].tolist()) | set(ainfo[2].tolist()))
    total_ms, per_step = reduce_over_ranks(sum(step_ms), fwd_it + adj_it, dev)
    iters_done = per_step * args.steps
    value = iters_done / (total_ms / 1000.0)

    # ---- end to end through the public API, host buffers, loss read back
    e2e = None
    if not args.no_e2e:
        # the step's inputs: the values (or the edge weights), b and x*
        vh = torch.from_numpy(w.weights if args.edges else w.values).to(dt).pin_memory()
        bh = torch.from_numpy(w.b).to(dt).pin_memory()
        xh = torch.from_numpy(w.xstar).to(dt).pin_memory()
        vd = torch.empty(vh.shape, dtype=dt, device=dev)
        bd = torch.empty_like(b)
        xd = torch.empty_like(xs)

        def e2e_step():
            vd.copy_(vh, non_blocking=True)
            bd.copy_(bh, non_blocking=True)
            xd.copy_(xh, non_blocking=True)
            vv = vd.requires_grad_(True)
            if args.edges:
                xx = Ed.solve(vv, bd, w.shift, rtol=w.rtol, fixed_iters=fixed, strategy=args.strategy)
            else:
                xx = A.solve(vv, bd, rtol=w.rtol, fixed_iters=fixed, strategy=args.strategy)
            loss = 0.5 * ((xx - xd) ** 2).sum()
            loss.backward()
            vv.grad = None
            vd.requires_grad_(False)
            return loss.item()

        for _ in range(args.warmup):
            flush.zero_()
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e2e_ms = 0.0
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = ev(), ev()
            e0.record(stream)
            e2e_step()
            e1.record(stream)
            torch.cuda.synchronize()
            e2e_ms += e0.elapsed_time(e1)
        e2e_total, _ = reduce_over_ranks(e2e_ms, 0.0, dev)
        e2e = {"value": iters_done / (e2e_total / 1000.0), "unit": UNIT,
               "h2d_bytes_per_step": int(vh.numel() * vh.element_size() + bh.numel() * bh.element_size()
                                         + xh.numel() * xh.element_size()),
               "d2h_bytes_per_step": 8}

    if rank == 0:
        peak, peak_kind = measured_hbm_peak()
        # per system-iteration (a list: the mean item's bytes per item-iteration)
        if w.item_rows is not None:
            it_bytes = per_iteration_bytes(n // A.n_info, nnz // A.n_info, vbytes)
        else:
            it_bytes = per_iteration_bytes(n, nnz, vbytes)
        cg_ms = statistics.mean(fwd_ms) + statistics.mean(adj_ms)
        achieved = (fwd_it + adj_it) * it_bytes / (cg_ms / 1000.0) / 1e9
        props = A.props
        uses_cluster = args.strategy == 3 or (args.strategy == 0 and props.cluster_fits
                                              and w.batch * 8 <= 148)
        uses_grid = not uses_cluster and not (args.strategy == 2 or
                                              (args.strategy == 0 and props.block_fits))
        # per solve: the solver kernel (+ the sliced-value gather); then the gradient
        launches_per_step = 2 * (1 + (1 if (uses_grid and props.sliced) else 0)) + 1
        if args.edges:
            # assembly; the edge gradient (per edge) and the shift gradient (tile sums, finish)
            launches_per_step += 1 + 2
        if w.item_rows is not None:
            uses_cluster = uses_grid = False
            launches_per_step = 3
            variant = "one block per item, largest items first"
        elif uses_cluster:
            variant = "thread-block cluster per system, DSMEM"
        elif not uses_grid:
            variant = ("block-per-system, whole system in shared memory" if props.block_resident
                       else "block-per-system, vectors in shared memory")
        elif props.interleaved:
            variant = "persistent grid, batch interleaved [entry][system], vectors in HBM"
            launches_per_step = 2 * 4 + 1          # layouts in and out, values, solver
        elif props.grid_onchip == 2:
            variant = "persistent grid, x, r, M^-1 on chip, two barriers an iteration"
        elif props.grid_onchip:
            variant = "persistent grid, x, r, M^-1 on chip"
        else:
            variant = "persistent grid, vectors in HBM"
        traffic = profile_traffic(f"cg_kernel_{args.workload}_{args.dtype}", (fwd_it + adj_it) / 2)
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                # DRAM bytes of the profile at this launch's time: how busy DRAM is
                "traffic_gbs": None if traffic is None else traffic / (cg_ms / 2 / 1000.0) / 1e9,
                "traffic_frac": None if traffic is None else traffic / (cg_ms / 2 / 1000.0) / 1e9 / peak,
                "kernel": f"PCG solve kernel ({variant}), one launch per solve",
                "algorithmic_bytes_per_launch": (fwd_it + adj_it) * it_bytes / 2,
                "bytes_per_iteration": it_bytes,
                "launch_ms": cg_ms / 2}
        if uses_grid and props.grid_onchip and not props.interleaved:
            # The on-chip solver keeps x, r, M^-1 in shared memory; the matrix and p
            # it sweeps every iteration stay in L2 after the first pass, so its
            # bandwidth roof is L2's, measured here.
            l2 = l2_stream_peak_gbs(dev)
            roof.update({"bound": "l2", "peak": l2, "frac": achieved / l2,
                         "peak_source": "measured in this run: L2-resident 24 MB copies (torch) in a "
                                        "CUDA graph, less the per-launch cost, bytes read plus written",
                         "hbm_peak": peak, "hbm_peak_source": peak_kind, "frac_of_hbm_peak": achieved / peak,
                         "ncu_lts_throughput_frac": profile_metric(
                             f"cg_kernel_{args.workload}_{args.dtype}", "lts_throughput_frac")})
        spmv = None
        if w.item_rows is None and not args.no_secondary:
            spmv = spmv_block(A, vals, n, nnz, B, vbytes, dt, dev, flush, peak)
        secondary = None
        if world == 1 and not args.no_secondary and args.workload == "c2" and not args.edges:
            secondary = secondary_workload(args, "c3", dev, flush, peak, peak_kind)
        gb = grad_bytes(n, nnz, vbytes) * B
        cpu = cpu_all = None
        if not args.no_cpu_baseline and world == 1:
            k = args.cpu_iters if args.cpu_iters > 0 else CPU_ITERS[args.workload]
            v_cpu, t_cpu, x_cpu = oracle_sample(args.dtype, k, args.workload, args.edges)
            sample = (f"{k} forward + {k} adjoint PCG iterations + "
                      f"{'assembly and edge-weight' if args.edges else 'value'} gradient of "
                      f"{'the first 32 items' if w.item_rows is not None else 'system 0'}")
            cpu = {"value": v_cpu, "unit": UNIT, "cores": 1, "kind": "oracle",
                   "cpu_model": host_cpu_model(),
                   "sample": f"{sample}, single-threaded C ({t_cpu:.1f} s)"}
            if not args.no_cpu_all_cores:
                cpu_all = cpu_all_cores(args, k, x_cpu)
                cpu_all["sample"] = sample
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "strong" if args.split_batch else "weak",
                "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
                "config": workload_config(args, w_all if args.split_batch else w),
                "fwd_adj_grad_ms": statistics.mean(step_ms),
                "forward_ms": statistics.mean(fwd_ms), "adjoint_ms": statistics.mean(adj_ms),
                "grad_ms": statistics.mean(grad_ms),
                "forward_iters": fwd_it, "adjoint_iters": adj_it, "statuses": statuses,
                "grad_gbs": None if args.edges else gb / (statistics.mean(grad_ms) / 1000.0) / 1e9,
                **(edge_metrics(n, nnz, len(w.edges[0]), B, vbytes, statistics.mean(asm_ms),
                                statistics.mean(grad_ms)) if args.edges else {}),
                "roofline": roof, "spmv": spmv, "hbm_workload": secondary,
                "cpu_baseline": cpu, "cpu_baseline_all_cores": cpu_all, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps,
                "clocks": clock_info}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
