"""The row-block distributed PCG on two and three gloo ranks on CPU: partition and halo
lists, the forward halo exchange, the reverse (sum-into-owner) exchange of a transposed
product, the distributed solve, adjoint and gradient -- each compared with the oracle on
the whole system.  The ranks' numeric steps are the oracle-backed CPU stand-in
(tests/dist_ops_cpu.py); the GPU path runs the same host logic over libsla's kernels
(tests/test_gpu_distributed.py)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import sla_workloads as W
from differentiable_sparse_linear_b200 import distributed as D

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _system(kind):
    if kind == "poisson":
        w = W.workload(1, "tiny")
        return w.A, w.B, w.W, w.tol
    if kind == "poisson64":
        w = W.workload(1, "full")
        return w.A, w.B, w.W, w.tol
    A = W.random_spd_list(1, 300, seed=41, dtype=np.float64)
    A.sys_row_off = None
    rng = np.random.default_rng(42)
    return A, rng.uniform(-1, 1, A.n_rows), rng.uniform(-1, 1, A.n_rows), 1e-10


def _nonsym():
    rng = np.random.default_rng(43)
    n = 120
    D_ = np.zeros((n, n))
    D_[rng.uniform(size=(n, n)) < 0.05] = 1.0
    D_ *= rng.uniform(-1, 1, size=(n, n))
    rp = [0]
    ci, v = [], []
    for i in range(n):
        nz = np.nonzero(D_[i])[0]
        ci += nz.tolist()
        v += D_[i, nz].tolist()
        rp.append(len(ci))
    return W.CSR(n, n, np.array(rp, np.int32), np.array(ci, np.int32), np.array(v))


def _rank_main(rank, world, port, kind, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    from dist_ops_cpu import OracleOps
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        comm = D.TorchComm()
        ops = OracleOps()
        A, b, w, tol = _system(kind)
        off = D.partition_rows(A.row_ptr, world)
        blk = D.build_local(A.row_ptr, A.col, A.val, off, rank, comm)
        r0, r1 = int(off[rank]), int(off[rank + 1])
        solver = D.DistributedPCG(blk, ops, comm, torch.float64, precond="jacobi")
        x, info = solver.solve(torch.from_numpy(b[r0:r1].copy()), tol)
        lam, g, ainfo = solver.adjoint(x, torch.from_numpy(w[r0:r1].copy()), tol)
        Ax = solver.matvec(x)
        N = _nonsym()
        offn = D.partition_rows(N.row_ptr, world)
        blkn = D.build_local(N.row_ptr, N.col, N.val, offn, rank, comm)
        sn = D.DistributedPCG(blkn, ops, comm, torch.float64, precond="none")
        v = np.random.default_rng(44).uniform(-1, 1, N.n_rows)
        a0, a1 = int(offn[rank]), int(offn[rank + 1])
        ATv = sn.rmatvec(torch.from_numpy(v[a0:a1].copy()))
        out.put((rank, dict(x=x.numpy(), lam=lam.numpy(), g=g.numpy(), it=info.iters, st=info.status,
                            ait=ainfo.iters, ast=ainfo.status, Ax=Ax.numpy(), ATv=ATv.numpy(),
                            halo=blk.n_halo)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,kind", [(2, "poisson"), (2, "random"), (3, "random"), (2, "poisson64")])
def test_distributed_pcg_gloo(world, kind):
    import oracle
    ora = oracle.get()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, kind, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    A, b, w, tol = _system(kind)
    ref = ora.pcg(A, b, precond="jacobi", tol=tol)
    adj = ora.adjoint(A, ref.x, w, precond="jacobi", tol=tol)
    x = np.concatenate([got[r]["x"] for r in range(world)])
    lam = np.concatenate([got[r]["lam"] for r in range(world)])
    g = np.concatenate([got[r]["g"] for r in range(world)])
    assert all(got[r]["st"] == 0 and got[r]["ast"] == 0 for r in range(world))
    assert all(got[r]["halo"] > 0 for r in range(world))
    for r in range(world):
        assert abs(got[r]["it"] - ref.iters) <= 0.02 * ref.iters, (got[r]["it"], ref.iters)
        assert abs(got[r]["ait"] - adj.iters) <= 0.02 * adj.iters
    rel = lambda a, b_: np.linalg.norm(a - b_) / np.linalg.norm(b_)
    assert rel(x, ref.x) <= 1e-8
    assert rel(lam, adj.lam) <= 1e-8
    assert rel(g, adj.grad) <= 1e-8
    assert np.max(np.abs(g - adj.grad)) <= 1e-7 * np.max(np.abs(adj.grad))
    Ax = np.concatenate([got[r]["Ax"] for r in range(world)])
    assert rel(Ax, ora.spmv(A, x)) <= 1e-14
    N = _nonsym()
    v = np.random.default_rng(44).uniform(-1, 1, N.n_rows)
    ATv = np.concatenate([got[r]["ATv"] for r in range(world)])
    assert rel(ATv, ora.spmv(ora.transpose(N), v)) <= 1e-14


def test_partition_rows_balanced():
    A = W.workload(5, "tiny").A
    for world in (1, 2, 3, 8):
        off = D.partition_rows(A.row_ptr, world)
        assert off[0] == 0 and off[-1] == A.n_rows and np.all(np.diff(off) >= 0)
        cost = np.array([A.row_ptr[off[r + 1]] - A.row_ptr[off[r]] + off[r + 1] - off[r] for r in range(world)])
        total = A.nnz + A.n_rows
        assert cost.max() <= total / world + np.diff(A.row_ptr).max() + 1


class _LoneComm:
    def all_gather_object(self, obj):
        return [obj]


def test_local_block_single_rank_is_the_matrix():
    A = W.workload(1, "tiny").A
    blk = D.build_local(A.row_ptr, A.col, A.val, np.array([0, A.n_rows]), 0, _LoneComm())
    assert blk.n_halo == 0 and not blk.send_to and not blk.recv_from
    assert np.array_equal(blk.row_ptr, A.row_ptr) and np.array_equal(blk.col, A.col)
    assert np.array_equal(blk.perm, np.arange(A.nnz))
