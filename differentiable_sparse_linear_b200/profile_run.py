"""One solve of a seeded workload, for profiler captures (ncu) of the solver kernels.

    python -m differentiable_sparse_linear_b200.profile_run --config 2 [--size full]
        [--engine auto|graph|persistent] [--maxit N] [--solves S] [--kernel-times R]

Builds the workload's matrices and preconditioner on cuda:0, runs S forward solves (the
first one also sets the solver up) with an optional iteration cap, so a capture of the
solve kernel stays short, and prints the iteration counts and the engine that ran.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import differentiable_sparse_linear_b200 as sla  # noqa: E402
import sla_workloads as W  # noqa: E402


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--size", default="full", choices=["full", "medium", "small", "tiny"])
    ap.add_argument("--engine", default="auto", choices=["auto", "graph", "persistent"])
    ap.add_argument("--maxit", type=int, default=0)
    ap.add_argument("--solves", type=int, default=1)
    ap.add_argument("--kernel-times", type=int, default=0,
                    help="then launch one iteration's kernels alone this many times (graph engine: "
                         "profilers do not see the kernels of a graph with a conditional node)")
    a = ap.parse_args(argv)
    w = W.workload(a.config, a.size)
    d = torch.device("cuda", 0)

    def dev(arr):
        return torch.from_numpy(np.ascontiguousarray(arr)).to(d)

    if w.A.sys_row_off is not None:
        Ad = sla.sla_csr_create_list(list(w.A.sys_row_off), dev(w.A.row_ptr), dev(w.A.col), dev(w.A.val))
    elif isinstance(w.A, W.BSR):
        Ad = sla.sla_bsr_create(dev(w.A.row_ptr), dev(w.A.col), dev(w.A.val))
    else:
        Ad = sla.sla_csr_create(dev(w.A.row_ptr), dev(w.A.col), dev(w.A.val))
    if w.precond == "spai":
        Gd = sla.sla_csr_create(dev(w.G.row_ptr), dev(w.G.col), dev(w.G.val))
        M = sla.sla_precond_spai(Ad, Gd, w.eps)
    else:
        M = sla.sla_precond_jacobi(Ad)
    b = dev(w.B)
    for s in range(a.solves):
        if w.nrhs > 1 or w.A.sys_row_off is not None:
            _, infos = sla.sla_pcg_solve_batched(Ad, M, b, rtol=w.tol, maxit=a.maxit, engine=a.engine)
        else:
            _, info = sla.sla_pcg_solve(Ad, M, b, rtol=w.tol, maxit=a.maxit, engine=a.engine)
            infos = [info]
        torch.cuda.synchronize()
        print(f"solve {s}: {w.name} iters {[i.iters for i in infos][:8]} status "
              f"{sorted(set(i.status for i in infos))} engine {infos[0].engine}", flush=True)
    if a.kernel_times > 0 and w.A.sys_row_off is None:
        ms = sla.sla_pcg_kernel_times(Ad, M, w.nrhs, reps=a.kernel_times)
        torch.cuda.synchronize()
        print(f"kernel times (ms): {[round(t, 4) for t in ms]}", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
