"""The iteration-step calls (sla_vec_dot, sla_pcg_update, sla_pcg_direction, sla_vec_gather,
sla_vec_scatter_add) against numpy, and the row-block distributed PCG over libsla's kernels
with its ranks as threads of one process on one GPU (ThreadComm: every wait is a host-side
rendezvous; no kernel waits for another), compared with the oracle on the whole system."""
import threading

import numpy as np
import pytest
import torch

import sla_workloads as W
from differentiable_sparse_linear_b200 import distributed as D
from gpu_helpers import SOL_TOL, dev, host, iters_close, rel, relmax

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ora():
    import oracle
    return oracle.get()


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [0, 1, 1000, 300001])
def test_step_calls(dtype, n):
    import differentiable_sparse_linear_b200 as sla
    rng = np.random.default_rng(n)
    p, q, x, r, d = (rng.uniform(-1, 1, n).astype(dtype) for _ in range(5))
    P, Q, X, R, Dv = (dev(a) for a in (p, q, x, r, d))
    Z = torch.empty_like(R)
    got = host(sla.sla_vec_dot(P, Q))
    assert abs(got[0] - float(np.dot(p.astype(np.float64), q.astype(np.float64)))) <= 1e-12 * max(1.0, n)
    alpha = 0.37
    out = host(sla.sla_pcg_update(alpha, P, Q, X, R, Dv, Z))
    if dtype == np.float32:
        a32 = np.float32(alpha)
        xr = (x.astype(np.float64) + np.float64(a32) * p).astype(np.float32)   # one fused multiply-add
        rr = (r.astype(np.float64) - np.float64(a32) * q).astype(np.float32)
    else:
        xr, rr = x + alpha * p, r - alpha * q
    zr = (rr.astype(np.float64) * d.astype(np.float64)).astype(dtype)
    tol = 1e-15 if dtype == np.float64 else 1e-7
    assert relmax(host(X), xr) <= tol and relmax(host(R), rr) <= tol and relmax(host(Z), zr) <= tol
    assert abs(out[0] - float(rr.astype(np.float64) @ rr)) <= 1e-12 * max(1.0, n)
    assert abs(out[1] - float(rr.astype(np.float64) @ zr)) <= 1e-12 * max(1.0, n)
    sla.sla_pcg_direction(0.5, Z, P)
    pr = (zr.astype(np.float64) + np.float64(np.asarray(0.5, dtype)) * p).astype(dtype)
    assert relmax(host(P), pr) <= tol
    if n:
        idx = rng.permutation(n)[: max(1, n // 3)].astype(np.int32)
        dst = torch.empty(idx.size, dtype=P.dtype, device="cuda")
        sla.sla_vec_gather(dev(idx), Q, dst)
        assert np.array_equal(host(dst), q[idx].astype(np.float64))
        acc = Q.clone()
        sla.sla_vec_scatter_add(dev(idx), dst, acc)
        ref = q.copy()
        ref[idx] = (q[idx].astype(np.float64) + q[idx].astype(np.float64)).astype(dtype)
        assert np.array_equal(host(acc), ref.astype(np.float64))


def _run_ranks(world, A, b, w, tol, dtype, nonsym=None):
    hub = D.ThreadHub(world)
    off = D.partition_rows(A.row_ptr, world)
    res, errs = {}, []

    def body(rank):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                comm = D.ThreadComm(hub, rank, stream=s)
                ops = D.CudaOps()
                blk = D.build_local(A.row_ptr, A.col, A.val, off, rank, comm)
                r0, r1 = int(off[rank]), int(off[rank + 1])
                solver = D.DistributedPCG(blk, ops, comm, dtype, precond="jacobi")
                x, info = solver.solve(ops.tensor(b[r0:r1]), tol)
                lam, g, ainfo = solver.adjoint(x, ops.tensor(w[r0:r1]), tol)
                out = dict(x=host(x), lam=host(lam), g=host(g), it=info.iters, st=info.status,
                           ait=ainfo.iters, ast=ainfo.status, halo=blk.n_halo)
                if nonsym is not None:
                    offn = D.partition_rows(nonsym.row_ptr, world)
                    bn = D.build_local(nonsym.row_ptr, nonsym.col, nonsym.val, offn, rank, comm)
                    sn = D.DistributedPCG(bn, ops, comm, dtype, precond="none")
                    v = np.random.default_rng(44).uniform(-1, 1, nonsym.n_rows).astype(nonsym.val.dtype)
                    out["ATv"] = host(sn.rmatvec(ops.tensor(v[int(offn[rank]):int(offn[rank + 1])])))
                s.synchronize()
                res[rank] = out
        except Exception as e:          # reported by the test thread
            errs.append(e)
            hub.barrier.abort()

    ts = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(timeout=600)
    if errs:
        raise errs[0]
    return res


def _nonsym(dtype):
    rng = np.random.default_rng(43)
    n = 2000
    m = 20000
    i = rng.integers(0, n, m)
    j = rng.integers(0, n, m)
    key = np.unique(i * n + j)
    i, j = key // n, key % n
    rp = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(np.bincount(i, minlength=n), out=rp[1:])
    return W.CSR(n, n, rp.astype(np.int32), j.astype(np.int32), rng.uniform(-1, 1, key.size).astype(dtype))


@pytest.mark.parametrize("world,cfg,size", [(2, 1, "full"), (3, 1, "full"), (2, 2, "small"), (4, 5, "small")])
def test_distributed_threads(ora, world, cfg, size):
    w = W.workload(cfg, size)
    A = w.A
    dt = torch.float64 if w.dtype == np.float64 else torch.float32
    N = _nonsym(w.dtype)
    got = _run_ranks(world, A, w.B, w.W, w.tol, dt, nonsym=N)
    # Jacobi throughout (the distributed solver's preconditioner)
    f32 = w.dtype == np.float32
    ref = ora.pcg(A, w.B, precond="jacobi", tol=w.tol)
    adj = ora.adjoint(A, ref.x, w.W, precond="jacobi", tol=w.tol)
    cnt = ora.pcg(A, w.B, precond="jacobi", tol=w.tol, store_f32=True) if f32 else ref
    acnt = ora.adjoint(A, cnt.x, w.W, precond="jacobi", tol=w.tol, store_f32=True) if f32 else adj
    for r in range(world):
        assert got[r]["st"] == 0 and got[r]["ast"] == 0 and got[r]["halo"] > 0
        assert iters_close(got[r]["it"], cnt.iters), (got[r]["it"], cnt.iters, ref.iters)
        assert iters_close(got[r]["ait"], acnt.iters), (got[r]["ait"], acnt.iters, adj.iters)
    x = np.concatenate([got[r]["x"] for r in range(world)])
    lam = np.concatenate([got[r]["lam"] for r in range(world)])
    g = np.concatenate([got[r]["g"] for r in range(world)])
    t = SOL_TOL[np.float32 if f32 else np.float64]
    assert rel(x, ref.x) <= t and rel(lam, adj.lam) <= t and rel(g, adj.grad) <= t
    assert relmax(g, adj.grad) <= 10 * t
    v = np.random.default_rng(44).uniform(-1, 1, N.n_rows).astype(N.val.dtype)
    ATv = np.concatenate([got[r]["ATv"] for r in range(world)])
    assert rel(ATv, ora.spmv(ora.transpose(N), v)) <= (1e-14 if not f32 else 1e-6)
