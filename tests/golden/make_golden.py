"""Write the oracle's results for the full-size workloads to tests/golden/full_<cfg>.{json,npz}.

Calls only the fp64 CPU oracle (oracle/) on the seeded inputs (sla_workloads/).  The GPU
parity tests at full size compare iteration counts with these and the solution, adjoint
and gradient at sampled indices (the oracle cannot run inside a test at these sizes).
It runs the oracle's OpenMP build (the same oracle.c with its independent row and element
loops on every core, whose results are bit-identical to the one-thread build).

full_<cfg>.json holds the scalars: iteration counts of the fp64 oracle and, for workloads
whose vectors are fp32, of its fp32-storage mode (the precision in which an fp32-vector
solver takes its stopping decision), residuals, norms.  full_<cfg>.npz holds the sampled
values: x and lambda at N_ROWS sampled rows (all right-hand sides) and the gradient at
N_ENTRIES sampled stored entries, in fp64.  The sample positions are not stored: they are
sample_idx(n, seed) of this file, recomputed by the tests.

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

N_VALUES = 131072          # sampled values per stored vector (rows x right-hand sides)
N_ENTRIES = 131072         # sampled gradient entries


def sample_idx(n: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct indices in [0, n): all of them when n <= count, else half evenly
    spaced (first and last included) and half uniform random from `seed`."""
    if n <= count:
        return np.arange(n, dtype=np.int64)
    rng = np.random.default_rng(seed)
    idx = set(np.linspace(0, n - 1, count // 2).astype(np.int64).tolist())
    while len(idx) < count:
        idx |= set(rng.integers(0, n, size=count - len(idx)).tolist())
    return np.array(sorted(idx), dtype=np.int64)


def row_sample(w, cfg: int) -> np.ndarray:
    return sample_idx(w.A.n_rows, max(1, N_VALUES // w.nrhs), 77 + cfg)


def entry_sample(w, cfg: int) -> np.ndarray:
    return sample_idx(w.A.nnz, N_ENTRIES, 99 + cfg)


def _solve(ora, w, store_f32: bool):
    A = w.A
    kw = dict(precond=w.precond, G=w.G, eps=w.eps, tol=w.tol)
    if A.sys_row_off is not None:                       # list of systems
        x, fw = ora.pcg_list(A, w.B, precond=w.precond, tol=w.tol, store_f32=store_f32)
        lam, g, ad = ora.adjoint_list(A, x, w.W, precond=w.precond, tol=w.tol, store_f32=store_f32)
    elif w.nrhs > 1:                                     # shared pattern, several RHS
        x, fw = ora.pcg_multi(A, w.B, store_f32=store_f32, **kw)
        lam, g, ad = ora.adjoint_multi(A, x, w.W, store_f32=store_f32, **kw)
    else:
        f = ora.pcg(A, w.B, store_f32=store_f32, **kw)
        a = ora.adjoint(A, f.x, w.W, store_f32=store_f32, **kw)
        x, lam, g, fw, ad = f.x, a.lam, a.grad, [f], [a]
    return x, lam, g, fw, ad


def run(cfg: int) -> tuple[dict, dict]:
    ora = oracle.get_omp()       # the same source on every host core; bit-identical results
    t0 = time.time()
    w = W.workload(cfg, "full")
    A = w.A
    out = {"workload": w.name, "n": int(A.n_rows), "nnz": int(A.nnz), "tol": w.tol,
           "precond": w.precond, "nrhs": int(w.nrhs),
           "generated_by": "tests/golden/make_golden.py (oracle/ only)",
           "n_rows_sampled": 0, "n_entries_sampled": 0}
    x, lam, g, fw, ad = _solve(ora, w, False)
    out["fwd_iters"] = [r.iters for r in fw]
    out["adj_iters"] = [r.iters for r in ad]
    out["fwd_relres"] = [r.relres for r in fw][:16]
    out["adj_relres"] = [r.relres for r in ad][:16]
    out["status"] = max(max(r.status for r in fw), max(r.status for r in ad))
    if w.dtype == np.float32:
        _, _, _, fw32, ad32 = _solve(ora, w, True)
        out["fwd_iters_f32"] = [r.iters for r in fw32]
        out["adj_iters_f32"] = [r.iters for r in ad32]
    rows = row_sample(w, cfg)
    ents = entry_sample(w, cfg)
    out["n_rows_sampled"] = int(rows.size)
    out["n_entries_sampled"] = int(ents.size)
    x2 = np.asarray(x).reshape(A.n_rows, -1)
    l2 = np.asarray(lam).reshape(A.n_rows, -1)
    arrays = {"x": x2[rows], "lam": l2[rows], "grad": np.asarray(g)[ents]}
    out["x_norm"] = float(np.linalg.norm(x))
    out["lam_norm"] = float(np.linalg.norm(lam))
    out["grad_norm"] = float(np.linalg.norm(g))
    out["seconds"] = time.time() - t0
    return out, arrays


def main(cfgs):
    for cfg in cfgs:
        res, arrays = run(cfg)
        with open(os.path.join(HERE, f"full_{cfg}.json"), "w") as f:
            json.dump(res, f, indent=0)
        np.savez_compressed(os.path.join(HERE, f"full_{cfg}.npz"), **arrays)
        print(f"config {cfg}: fwd {res['fwd_iters'][:8]} adj {res['adj_iters'][:8]} "
              f"f32 {res.get('fwd_iters_f32', [])[:8]} {res.get('adj_iters_f32', [])[:8]} "
              f"({res['seconds']:.0f} s)", flush=True)


if __name__ == "__main__":
    main([int(a) for a in sys.argv[1:]] or [1, 2, 3, 4, 5])
