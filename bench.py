"""Benchmark: PCG iterations/s of the differentiable sparse SPD solve on B200.

One step = the whole hot path on one batch of synthetic input: the forward PCG solve
x = A^-1 b, the adjoint solve A lambda = w (w = dL/dx for L = w.x) and the pattern
gradient dL/dA_ij = -lambda_i x_j.  The default workload is the largest single-GPU one:
the SPAI-preconditioned power-law SPD system (n = 4,194,304, 212.7M stored entries, fp32
values and vectors, fp64 reductions, M^-1 = G G^T + 3e-3 I, tolerance 1e-6).  value = PCG
iterations (forward + adjoint) per second over all ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 1..6]

Multi-GPU (torchrun): every rank solves its own replica (the single-system solve does not
shard here), weak scaling; time is the max over ranks.  --impl reference times the fp64
CPU oracle on the host cores (bounded sample per step).
"""
from __future__ import annotations

import argparse
import gc
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import sla_workloads as W  # noqa: E402  (seeded inputs; no method arithmetic)

METRIC = "PCG iterations/sec and SpMV HBM GB/s (fraction of ~8 TB/s) at 1 B200"
UNIT = "iterations/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=5)
    ap.add_argument("--size", default="full", choices=["full", "small", "tiny"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-reps", type=int, default=20)
    ap.add_argument("--engine", default="auto", choices=["auto", "graph", "persistent"])
    return ap.parse_args()


# ------------------------------------------------------------------------- byte model
def nrhs_of(w) -> int:
    return 1 if w.B.ndim == 1 else int(w.B.shape[1])


def vbytes(dtype) -> int:
    return np.dtype(dtype).itemsize


def matrix_bytes(n, nnz, sv) -> int:
    """Algorithmic bytes to stream one CSR matrix: values + column indices + row_ptr."""
    return nnz * (sv + 4) + (n + 1) * 4


def stream_bytes(A, sv) -> int:
    """Algorithmic bytes to stream matrix A: CSR as above; BSR one column index and b*b
    values per block plus the block row pointers."""
    if isinstance(A, W.BSR):
        return A.nnzb * (A.b * A.b * sv + 4) + (A.n_brows + 1) * 4
    return matrix_bytes(A.n_rows, A.nnz, sv)


def oracle_matrix(ora, A):
    """The matrix as the oracle takes it: a BSR matrix as its scalar CSR expansion."""
    return ora.bsr_to_csr(A)[0] if isinstance(A, W.BSR) else A


def kernel_bytes(w) -> dict:
    """Algorithmic bytes per launch of each kernel of one PCG iteration (K right-hand sides)."""
    A = w.A
    n, nnz, sv = A.n_rows, A.nnz, vbytes(w.dtype)
    K = w.nrhs
    out = {"q_spmv": stream_bytes(A, sv) + 4 * n * K * sv}   # read z, p_old; write p_new, q
    if w.precond == "spai":
        ng = w.G.nnz
        out["update_gt_spmv"] = matrix_bytes(n, ng, sv) + 7 * n * K * sv   # r,q gathered; p,x; write r,x,y
        out["z_g_spmv"] = matrix_bytes(n, ng, sv) + 3 * n * K * sv         # y gathered, r; write z
    else:
        out["update_jacobi"] = 8 * n * K * sv + n * sv                     # x,p,r,q,(D^-1); write x,r,z
    return out


# ------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[str] = []
        self.t = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        """Host time of a point in the run (samples are kept from the window between two marks)."""
        return time.time()

    def wait_first_sample(self, limit_s: float = 10.0):
        """nvidia-smi's start-up takes driver locks; begin timing only once it samples."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < limit_s:
            time.sleep(0.05)
        time.sleep(0.25)

    def stop(self, window: tuple[float, float] | None = None) -> dict:
        """Stop sampling; summarise the samples taken inside `window` (host times), or all."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = [ln for ts, ln in self.lines if window is None or window[0] <= ts <= window[1] + 0.25]
        if not lines and self.lines:              # a timed region shorter than the sampling period
            lines = [self.lines[-1][1]]
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(max(smax)) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_bus_id(dev: int) -> str | None:
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


# ------------------------------------------------------------------------- helpers
def measured_peaks() -> tuple[float, str]:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# The files that define each profiled kernel's code: its ncu traffic stays valid while they
# are unchanged (other kernels' sources do not move it).
KERNEL_SOURCES = {
    "k_pcg_persistent": ("persist.cuh", "sell.cuh", "pcg_ops.cuh"),
    # the long-row single-RHS product (column-sorted segments) of the graph engine
    "q_spmv": ("csb.cuh", "pcg_ops.cuh", "tile_engine.cuh"),
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the code that defines a kernel (its ncu traffic is tied to it): the listed
    sources with their // comments and blank lines left out, so an edit of a comment does
    not detach a capture from the code it measured."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "differentiable_sparse_linear_b200", "csrc")
    for fn in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, units: float = 1.0) -> int | None:
    """DRAM bytes (read + write) of one launch, from the committed ncu summary if it was
    taken on the current kernel sources: the summary holds bytes per unit (per launch, or per
    PCG iteration for the persistent solver), scaled here by the launch's units."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    if kernel not in KERNEL_SOURCES:
        return None
    src = kernel_source_hash(kernel)
    for ln in open(path):
        parts = ln.split()
        if len(parts) >= 4 and not ln.startswith("#") and parts[0] == kernel and parts[1] == workload:
            if parts[3] == src:
                return int(float(parts[2]) * units)
    return None


def _oracle_problem(ora, w):
    """(A, b, preconditioner) of the workload as the oracle takes them: system 0 of a list,
    a BSR matrix as its scalar CSR; the preconditioner (and G^T) is built once, outside any
    timed region."""
    B = w.B if w.B.ndim == 1 else w.B[:, 0]
    A = oracle_matrix(ora, w.A)
    if A.sys_row_off is not None:
        A = ora.system(A, 0)
        B = B[: A.n_rows]
    P = ora._precond(A, w.precond, w.G, w.eps)
    return A, B, P


def _time_oracle(ora, A, B, P, budget_s: float) -> tuple[int, float]:
    """Fixed PCG iterations of the forward solve for about budget_s seconds: (iters, s)."""
    t0 = time.perf_counter()
    ora.pcg(A, B, fixed_iters=2, _P=P)
    per = (time.perf_counter() - t0) / 2
    iters = int(max(2, min(5000, budget_s / max(per, 1e-9))))
    t0 = time.perf_counter()
    r = ora.pcg(A, B, fixed_iters=iters, _P=P)
    return r.iters, time.perf_counter() - t0


def cpu_baseline(w, budget_s: float = 10.0) -> dict:
    """The fp64 oracle on a bounded sample (fixed PCG iterations of the forward solve), once
    on one host thread and once in its OpenMP build on every host core (same source, same
    bits; row-parallel products and vector updates, sequential dot products)."""
    import oracle
    seq, par = oracle.get(), oracle.get_omp()
    A, B, P = _oracle_problem(seq, w)
    it1, dt1 = _time_oracle(seq, A, B, P, budget_s)
    itn, dtn = _time_oracle(par, A, B, P, budget_s)
    cores = os.cpu_count() or 1
    part = "system 0 of the " if w.A.sys_row_off is not None else ""
    return {"value": itn / dtn, "unit": UNIT, "cores": cores, "kind": "oracle",
            "value_1_thread": it1 / dt1,
            "sample": f"fixed PCG iterations of the forward solve on {part}the same workload: "
                      f"{itn} on all {cores} host cores (OpenMP build, {dtn:.1f} s) and {it1} on one "
                      f"thread ({dt1:.1f} s); preconditioner set-up outside the timed sample"}


# ------------------------------------------------------------------------- ranks
def reduce_over_ranks(ms: float, iters: float, world: int, device) -> tuple[float, float]:
    """Whole-job numbers of a replicated run: the slowest rank's time and the iterations of
    all ranks (each rank solves its own replica).  One rank: the inputs unchanged."""
    if world <= 1:
        return float(ms), float(iters)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms), float(iters)], dtype=torch.float64, device=device)
    tm = t.clone()
    dist.all_reduce(tm, op=dist.ReduceOp.MAX)
    ti = t.clone()
    dist.all_reduce(ti, op=dist.ReduceOp.SUM)
    return float(tm[0]), float(ti[1])


# ------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import sla_workloads as W
    w = W.workload(args.config, args.size)
    import oracle
    ora = oracle.get_omp()
    A, B, P = _oracle_problem(ora, w)
    t0 = time.perf_counter()
    ora.pcg(A, B, fixed_iters=2, _P=P)
    per = (time.perf_counter() - t0) / 2
    per_step = int(max(2, min(2000, 2.0 / max(per, 1e-9))))     # about 2 s of CPU per step
    for _ in range(args.warmup):
        ora.pcg(A, B, fixed_iters=per_step, _P=P)
    t0 = time.perf_counter()
    total = 0
    for _ in range(args.steps):
        total += ora.pcg(A, B, fixed_iters=per_step, _P=P).iters
    dt = time.perf_counter() - t0
    value = total / dt
    cores = os.cpu_count() or 1
    sample = (f"{per_step} fixed forward PCG iterations per step of the fp64 oracle (OpenMP build, "
              f"all {cores} host cores) on {w.name}; preconditioner set-up outside the timed steps")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "n": int(A.n_rows), "nnz": int(A.nnz)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    import differentiable_sparse_linear_b200 as sla
    import sla_workloads as W

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = W.workload(args.config, args.size)
    A = w.A
    t_setup = time.perf_counter()
    rp = torch.from_numpy(A.row_ptr).to(dev)
    ci = torch.from_numpy(A.col).to(dev)
    va = torch.from_numpy(A.val).to(dev)
    is_list = A.sys_row_off is not None
    if is_list:
        Ad = sla.sla_csr_create_list(list(A.sys_row_off), rp, ci, va)
    elif isinstance(A, W.BSR):
        Ad = sla.sla_bsr_create(rp, ci, va)
    else:
        Ad = sla.sla_csr_create(rp, ci, va)
    Gd = None
    if w.precond == "spai":
        Gd = sla.sla_csr_create(torch.from_numpy(w.G.row_ptr).to(dev), torch.from_numpy(w.G.col).to(dev),
                                torch.from_numpy(w.G.val).to(dev))
        M = sla.sla_precond_spai(Ad, Gd, w.eps)
    else:
        M = sla.sla_precond_jacobi(Ad)
    b = torch.from_numpy(np.ascontiguousarray(w.B)).to(dev)
    wl = torch.from_numpy(np.ascontiguousarray(w.W)).to(dev)
    X = torch.empty_like(b)
    torch.cuda.synchronize()
    setup_s = time.perf_counter() - t_setup
    nrhs = w.nrhs
    multi = is_list or nrhs > 1
    # graph engine: matrices with rows of more than 16 entries (and BSR matrices) get their
    # operand vectors formed by an elementwise kernel first (Q: k_ep + SpMV; U_S: k_er + SpMV)
    spai = w.precond == "spai"
    form_a = isinstance(A, W.BSR) or (not is_list and int(np.diff(A.row_ptr).max(initial=0)) > 16)
    form_gt = spai and int(np.bincount(w.G.col, minlength=A.n_rows).max(initial=0)) > 16
    # single-RHS long-row matrices run on column-sorted copies whose values (and per-segment
    # row bounds) are gathered from the CSR values before every graph-engine solve: two
    # kernels per such matrix; with fp32 values and vectors each of their products is
    # preceded by the max |v| kernel of its fixed-point row sums
    one_col = nrhs_of(w) == 1 and not is_list and not isinstance(A, W.BSR)
    form_g = spai and int(np.diff(w.G.row_ptr).max(initial=0)) > 16
    fx = int(one_col and vbytes(w.dtype) == 4)
    q_k = (2 + fx) if form_a else 1
    us_k = (2 + fx) if form_gt else 1
    z_k = 1 + fx * int(form_g)
    csb_gathers = 2 * (int(form_a) + int(form_g) + int(form_gt)) if one_col else 0
    body_kernels = 2 * (q_k + us_k + z_k) if spai else 2 * (q_k + 1)   # two iterations per loop body
    prologue = us_k + z_k if spai else 1
    engines_seen = set()

    def launches(iters: int, engine: str) -> int:
        """Kernels one solve launches: init, the solve (persistent: the sliced values of each
        matrix gathered from CSR -- A, and G and G^T with SPAI -- then one kernel; graph:
        the column-sorted copies' value gathers, prologue and loop bodies of two iterations
        each), copy-out."""
        if engine == "persistent":
            return 3 + (3 if spai else 1)
        return 2 + csb_gathers + prologue + body_kernels * ((iters + 1) // 2)

    # outputs allocated once, so a step allocates nothing
    lam_buf = torch.empty_like(b)
    g_buf = torch.empty(A.nnz, dtype=va.dtype, device=dev)

    fwd_events = []                 # (start, end) CUDA events around each forward solve
    fwd_iters = []                  # its iterations (single systems)

    def step(bv, wv, x_out, record=False):
        if record:
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            fwd_events.append((f0, f1))
            f0.record()
        if multi:
            x, inf = sla.sla_pcg_solve_batched(Ad, M, bv, x_out, rtol=w.tol, engine=args.engine)
            if record:
                fwd_events[-1][1].record()
                if not is_list:     # one iteration advances every right-hand side
                    fwd_iters.append(int(inf.iters.max()))
            lam, g, ainf = sla.sla_pcg_adjoint_batched(Ad, M, x, wv, rtol=w.tol, engine=args.engine,
                                                       dLdB=lam_buf, dLdA=g_buf)
            # the per-system results are read as arrays (PcgInfoList), not system by system
            engines_seen.update(inf.engines | ainf.engines)
            if is_list:
                return int(inf.iters.sum()) + int(ainf.iters.sum()), 2, x, lam
            it = int(inf.iters.max()), int(ainf.iters.max())
            return (int(inf.iters.sum()) + int(ainf.iters.sum()),
                    launches(it[0], inf[0].engine) + launches(it[1], ainf[0].engine) + 1, x, lam)
        x, inf = sla.sla_pcg_solve(Ad, M, bv, x_out, rtol=w.tol, engine=args.engine)
        if record:
            fwd_events[-1][1].record()
            fwd_iters.append(inf.iters)
        lam, g, ainf = sla.sla_pcg_adjoint(Ad, M, x, wv, rtol=w.tol, engine=args.engine, dLdb=lam_buf, dLdA=g_buf)
        engines_seen.update((inf.engine, ainf.engine))
        if inf.status != 0 or ainf.status != 0:
            raise RuntimeError(f"solve did not converge: {inf} {ainf}")
        return (inf.iters + ainf.iters, launches(inf.iters, inf.engine) + launches(ainf.iters, ainf.engine) + 1,
                x, lam)

    # Between timed steps the L2 (126 MB) must not hold this step's inputs.  Workloads whose
    # matrices stream well over the L2's size per product evict it themselves; the others
    # are flushed: write 512 MiB (evicts every line of ours), then read 256 MiB so the lines
    # the write dirtied are back in HBM before the next timed launch (otherwise that launch
    # would pay their write-back).  The flush runs inside the timed step; its two kernels
    # are torch's, not counted in gpu_launches.
    L2_BYTES = 126 << 20
    big = stream_bytes(A, vbytes(w.dtype)) > 4 * L2_BYTES
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    drain = torch.zeros(64 << 20, dtype=torch.float32, device=dev)
    l2_note = (f"no flush: inputs larger than L2 (the matrix streams "
               f"{stream_bytes(A, vbytes(w.dtype)) / 1e9:.2f} GB per product, L2 is 126 MB)" if big else
               "flushed between steps inside the timed step (512 MiB write, then a 256 MiB read that "
               "writes the dirtied lines back; 2 torch kernels per step, not in gpu_launches)")

    def flush_l2(force=False):
        if big and not force:
            return
        flush.zero_()
        drain.sum()

    flush_l2()

    def barrier():
        if world > 1:
            dist.barrier()

    # the clock sampler starts before the warm-up, so its start-up stays out of the timed
    # region; only the samples taken inside the timed region are summarised
    clocks = ClockSampler(gpu_bus_id(local) if rank == 0 else None)
    if rank == 0:
        clocks.start()
        clocks.wait_first_sample()
    # the first step also builds the matrices' solver layouts (once per pattern): timed apart
    t_first = time.perf_counter()
    step(b, wl, X)
    torch.cuda.synchronize()
    first_step_s = time.perf_counter() - t_first
    for _ in range(args.warmup):
        flush_l2()
        step(b, wl, X)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    total_iters = 0
    total_launch = 0
    gc.collect()
    gc.disable()            # no collector pause inside the timed region
    t_begin = clocks.mark()
    ev0.record()
    fwd_iters.clear()
    for k in range(args.steps):
        flush_l2()
        it, nl, _, _ = step(b, wl, X, record=True)
        evs[k].record()
        total_iters += it
        total_launch += nl
    ev1.record()
    torch.cuda.synchronize()
    gc.enable()
    t_end = clocks.mark()
    barrier()
    clk = clocks.stop((t_begin, t_end)) if rank == 0 else {}
    ms = ev0.elapsed_time(ev1)
    step_ms = [ev0.elapsed_time(evs[0])] + [evs[k - 1].elapsed_time(evs[k]) for k in range(1, args.steps)]
    ms_max, iters_all = reduce_over_ranks(ms, total_iters, world, dev)
    value = iters_all / (ms_max / 1e3)

    # end to end: host inputs in pinned memory, result read back every step
    hb = torch.from_numpy(np.ascontiguousarray(w.B)).pin_memory()
    hw = torch.from_numpy(np.ascontiguousarray(w.W)).pin_memory()
    hx = torch.empty(hb.shape, dtype=hb.dtype).pin_memory()
    hl = torch.empty(hb.shape, dtype=hb.dtype).pin_memory()
    bd = torch.empty_like(b)
    wd = torch.empty_like(wl)
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e_iters = 0
    gc.collect()
    gc.disable()
    e0.record()
    for _ in range(args.steps):
        flush_l2()
        bd.copy_(hb, non_blocking=True)
        wd.copy_(hw, non_blocking=True)
        it, _, x, lam = step(bd, wd, X)
        hx.copy_(x, non_blocking=True)
        hl.copy_(lam, non_blocking=True)
        e_iters += it
    e1.record()
    torch.cuda.synchronize()
    gc.enable()
    barrier()
    ems = e0.elapsed_time(e1)
    ems, e_iters = reduce_over_ranks(ems, e_iters, world, dev)
    e2e = {"value": e_iters / (ems / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": int(hb.numel() * hb.element_size() + hw.numel() * hw.element_size()),
           "d2h_bytes_per_step": int(hx.numel() * hx.element_size() + hl.numel() * hl.element_size())}

    # dominant kernel: per-launch device time inside the iteration sequence
    peak, peak_kind = measured_peaks()
    roofline = None
    kernels = {}
    spmv = None
    if not is_list and engines_seen == {"persistent"}:
        # the whole solve is one launch of the persistent kernel: time forward solves alone
        # (L2 flushed before each; the launch brackets also hold the two small set-up and
        # copy-out kernels) and take the algorithmic bytes of every phase the launch ran
        kb = kernel_bytes(w)
        names = list(kb)
        reps = 3
        tot = 0.0
        for r in range(reps + 1):
            flush_l2()
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record()
            if multi:
                sla.sla_pcg_solve_batched(Ad, M, b, X, rtol=w.tol, engine=args.engine)
            else:
                sla.sla_pcg_solve(Ad, M, b, X, rtol=w.tol, engine=args.engine)
            s1.record()
            torch.cuda.synchronize()
            if r >= 1:
                tot += s0.elapsed_time(s1)
        launch_ms = tot / reps
        pms, pcnt = sla.sla_pcg_phase_times(Ad, M, nrhs)
        slot = {"q_spmv": 0, "update_gt_spmv": 1, "z_g_spmv": 2, "update_jacobi": 3}
        launch_bytes = 0
        for nm in names:
            i = slot[nm]
            launch_bytes += kb[nm] * pcnt[i]
            kernels[nm] = {"ms": pms[i], "phases": pcnt[i], "bytes": kb[nm],
                           "gbs": kb[nm] / (pms[i] * 1e6) if pms[i] > 0 else None,
                           "timing": "in-kernel, grid barrier to grid barrier (block 0)"}
        ach = launch_bytes / (launch_ms * 1e6)
        roofline = {"bound": "hbm", "kernel": "k_pcg_persistent", "achieved": ach, "peak": peak, "unit": "GB/s",
                    "frac": ach / peak,
                    "traffic": profiled_traffic("k_pcg_persistent", w.name, units=pcnt[0]),
                    "peak_source": peak_kind, "algorithmic_bytes": launch_bytes, "ms_per_launch": launch_ms,
                    "units_per_launch": {nm: pcnt[slot[nm]] for nm in names},
                    "note": "one launch = one forward solve; bytes = per-phase algorithmic bytes x phases run"}
    elif is_list:
        # one launch of the list kernel = one batched solve (a block per system); bytes per
        # system iteration in the streaming form: the system's matrix + 13 vector passes
        sys_off = np.asarray(A.sys_row_off, dtype=np.int64)
        sys_n = np.diff(sys_off)
        sys_nnz = A.row_ptr[sys_off[1:]].astype(np.int64) - A.row_ptr[sys_off[:-1]].astype(np.int64)
        sv = vbytes(w.dtype)
        per_iter = sys_nnz * (sv + 4) + (sys_n + 1) * 4 + 13 * sys_n * sv
        reps = 3
        tot = 0.0
        infos = None
        # the list kernel alone: the library records CUDA events on the solve stream right
        # around its launch (the call's result copy and host work stay outside)
        for r in range(reps + 1):
            flush_l2()
            _, infos = sla.sla_pcg_solve_batched(Ad, M, b, X, rtol=w.tol)
            if r >= 1:
                tot += sla.sla_list_kernel_ms(Ad)
        launch_ms = tot / reps
        its = np.asarray(infos.iters, dtype=np.int64)
        launch_bytes = int((per_iter * its).sum())
        ach = launch_bytes / (launch_ms * 1e6)
        roofline = {"bound": "hbm", "kernel": "k_list_pcg", "achieved": ach, "peak": peak, "unit": "GB/s",
                    "frac": ach / peak, "traffic": None, "peak_source": peak_kind,
                    "algorithmic_bytes": launch_bytes, "ms_per_launch": launch_ms,
                    "units_per_launch": {"system_iterations": int(its.sum())},
                    "note": "one launch = one batched forward solve; bytes per system iteration = "
                            "nnz_s*(s_v+4) + (n_s+1)*4 + 13*n_s*s_v (streaming form; the kernel keeps "
                            "each system's vectors in shared memory)"}
    elif not is_list:
        # graph engine: every kernel of one iteration launched alone in loop order, each
        # bracketed by CUDA events on the launching stream (the loop itself runs inside a
        # graph, where events cannot bracket single kernels)
        kt = sla.sla_pcg_kernel_times(Ad, M, nrhs, reps=args.kernel_reps)
        names = list(kernel_bytes(w))
        kb = kernel_bytes(w)
        for i, nm in enumerate(names):
            kernels[nm] = {"ms": kt[i], "bytes": kb[nm], "gbs": kb[nm] / (kt[i] * 1e6) if kt[i] > 0 else None}
        dom = max(names, key=lambda k: kernels[k]["ms"])
        ach = kernels[dom]["gbs"]
        tr = profiled_traffic(dom, w.name)
        roofline = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": peak, "unit": "GB/s",
                    "frac": ach / peak, "traffic": tr, "peak_source": peak_kind,
                    "algorithmic_bytes": kb[dom], "ms_per_launch": kernels[dom]["ms"]}
    iteration = None
    if not is_list and fwd_events:
        # the full PCG iteration, measured live: the forward solves of the timed steps (CUDA
        # events on the solve stream around each solve call, which also holds the solve's
        # small set-up and copy-out kernels) against the algorithmic bytes of the iterations
        # they ran -- one product with A, and with SPAI one with G^T and one with G, plus 16
        # vector passes (SPAI) or 13 (Jacobi) of n x nrhs elements
        fwd_ms = sum(a.elapsed_time(b_) for a, b_ in fwd_events)
        sv = vbytes(w.dtype)
        per_iter = stream_bytes(A, sv) + (16 if spai else 13) * A.n_rows * nrhs * sv
        if spai:
            per_iter += 2 * matrix_bytes(A.n_rows, w.G.nnz, sv)
        its = sum(fwd_iters)
        ach_i = per_iter * its / (fwd_ms * 1e6)
        iteration = {"bound": "hbm", "achieved": ach_i, "peak": peak, "unit": "GB/s", "frac": ach_i / peak,
                     "bytes_per_iteration": per_iter, "iterations": its, "ms": fwd_ms,
                     "ms_per_iteration": fwd_ms / max(its, 1), "peak_source": peak_kind,
                     "timing": "forward solves inside the timed steps, CUDA events on the solve stream"}
    if not is_list:
        # standalone SpMV y = A x, L2 flushed before each launch: on a handle whose values are
        # declared static (SLA_STATIC_VALUES, the matrix of this benchmark never changes) and
        # on the handle above, which reads the CSR values at every call
        xs = torch.randn(A.n_rows * nrhs, dtype=va.dtype, device=dev).reshape(b.shape)
        ys = torch.empty_like(xs)
        As = None
        if not isinstance(A, W.BSR):
            As = sla.sla_csr_create(rp, ci, va, static_values=True)
        sb = stream_bytes(A, vbytes(w.dtype)) + 2 * A.n_rows * nrhs * vbytes(w.dtype)

        def time_spmv(H, reps=20):
            tot = 0.0
            for r in range(reps + 2):
                flush_l2(force=True)
                s0 = torch.cuda.Event(enable_timing=True)
                s1 = torch.cuda.Event(enable_timing=True)
                s0.record()
                if nrhs > 1:
                    sla.sla_spmv_multi(H, xs, ys)
                else:
                    sla.sla_spmv(H, xs, ys)
                s1.record()
                torch.cuda.synchronize()
                if r >= 2:
                    tot += s0.elapsed_time(s1)
            return tot / reps

        sp_ms = time_spmv(As if As is not None else Ad)
        spmv = {"gbs": sb / (sp_ms * 1e6), "frac": sb / (sp_ms * 1e6) / peak, "ms": sp_ms, "bytes": sb,
                "values": "static (SLA_STATIC_VALUES)" if As is not None else "read from CSR each call",
                "l2": "flushed before each launch (512 MiB write + 256 MiB read)"}
        if As is not None:
            dyn_ms = time_spmv(Ad)
            spmv["csr_values_each_call"] = {"gbs": sb / (dyn_ms * 1e6), "frac": sb / (dyn_ms * 1e6) / peak,
                                            "ms": dyn_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        iters_per_step = total_iters / args.steps
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32" if w.dtype == np.float32 else "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "n": int(A.n_rows), "nnz": int(A.nnz),
                       "nnz_G": int(w.G.nnz) if w.G is not None else 0, "nrhs": nrhs,
                       "batch": int(A.batch), "precond": w.precond, "tol": w.tol,
                       "iters_per_step": iters_per_step,
                       "step": "forward PCG solve + adjoint PCG solve + pattern gradient",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": l2_note, "setup_s": setup_s, "first_step_s": first_step_s,
                       "engine": "+".join(sorted(engines_seen))},
            "step_ms": {"min": min(step_ms), "median": float(np.median(step_ms)), "max": max(step_ms),
                        "argmax": int(np.argmax(step_ms))},
            "roofline": roofline, "iteration_roofline": iteration, "spmv": spmv, "kernels": kernels,
            "gpu_launches": total_launch, "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
