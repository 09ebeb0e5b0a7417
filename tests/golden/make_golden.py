"""Write the oracle's results for the full-size workloads to tests/golden/full_<cfg>.json.

Calls only the fp64 CPU oracle (oracle/) on the seeded inputs (sla_workloads/).  The GPU
parity tests at full size compare iteration counts with these and the solution, adjoint
and gradient at sampled indices (the oracle cannot run inside a test at these sizes).

    python tests/golden/make_golden.py [cfg ...]        (default: 1 2 3 4 5)
"""
from __future__ import annotations

import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import sla_workloads as W  # noqa: E402

N_SAMPLE = 96


def sample_idx(n: int, seed: int) -> list[int]:
    rng = np.random.default_rng(seed)
    idx = set(np.linspace(0, n - 1, N_SAMPLE // 2).astype(np.int64).tolist())
    idx |= set(rng.integers(0, n, size=N_SAMPLE // 2).tolist())
    return sorted(int(i) for i in idx)


def run(cfg: int) -> dict:
    ora = oracle.get()
    t0 = time.time()
    w = W.workload(cfg, "full")
    A = w.A
    kw = dict(precond=w.precond, G=w.G, eps=w.eps, tol=w.tol)
    out = {"workload": w.name, "n": int(A.n_rows), "nnz": int(A.nnz), "tol": w.tol,
           "precond": w.precond, "generated_by": "tests/golden/make_golden.py (oracle/ only)"}
    rows = sample_idx(A.n_rows, 77 + cfg)
    ents = sample_idx(A.nnz, 99 + cfg)
    out["rows"] = rows
    out["entries"] = ents
    if A.sys_row_off is not None:                       # list of systems
        x, fw = ora.pcg_list(A, w.B, precond=w.precond, tol=w.tol)
        lam, g, ad = ora.adjoint_list(A, x, w.W, precond=w.precond, tol=w.tol)
        out["fwd_iters"] = [r.iters for r in fw]
        out["adj_iters"] = [r.iters for r in ad]
        out["status"] = max(max(r.status for r in fw), max(r.status for r in ad))
    elif w.nrhs > 1:                                     # shared pattern, several RHS
        x, fw = ora.pcg_multi(A, w.B, **kw)
        lam, g, ad = ora.adjoint_multi(A, x, w.W, **kw)
        out["fwd_iters"] = [r.iters for r in fw]
        out["adj_iters"] = [r.iters for r in ad]
        out["status"] = max(max(r.status for r in fw), max(r.status for r in ad))
    else:
        fw = ora.pcg(A, w.B, **kw)
        ad = ora.adjoint(A, fw.x, w.W, **kw)
        x, lam, g = fw.x, ad.lam, ad.grad
        out["fwd_iters"] = [fw.iters]
        out["adj_iters"] = [ad.iters]
        out["fwd_relres"] = fw.relres
        out["adj_relres"] = ad.relres
        out["status"] = max(fw.status, ad.status)
    x2 = x.reshape(A.n_rows, -1)
    l2 = lam.reshape(A.n_rows, -1)
    out["x"] = x2[rows].tolist()
    out["lam"] = l2[rows].tolist()
    out["grad"] = np.asarray(g)[ents].tolist()
    out["x_norm"] = float(np.linalg.norm(x))
    out["lam_norm"] = float(np.linalg.norm(lam))
    out["grad_norm"] = float(np.linalg.norm(g))
    out["seconds"] = time.time() - t0
    return out


def main(cfgs):
    for cfg in cfgs:
        res = run(cfg)
        path = os.path.join(HERE, f"full_{cfg}.json")
        with open(path, "w") as f:
            json.dump(res, f)
        print(f"config {cfg}: fwd {res['fwd_iters'][:8]} adj {res['adj_iters'][:8]} "
              f"({res['seconds']:.0f} s) -> {path}", flush=True)


if __name__ == "__main__":
    main([int(a) for a in sys.argv[1:]] or [1, 2, 3, 4, 5])
