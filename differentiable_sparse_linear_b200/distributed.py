"""Row-block distributed PCG with halo exchange, and its adjoint.

"torch-sla: Differentiable Sparse Linear Algebra with Adjoint Solvers and Sparse Tensor
Parallelism for PyTorch", Methodology §3 (distributed layer): the matrix is split into
contiguous blocks of rows, one per rank; before each product a rank receives the values of
the columns its rows touch but other ranks own (its halo); the scalars of the recurrence are
all-reduced; the backward pass of an operator applied transposed sends the contributions a
rank computed for other ranks' entries back to their owners, which sum them
(sum-into-owner).  For an SPD matrix the adjoint solve applies A itself, so it uses the
forward exchange; the gradient dL/dA_ij = -lambda_i x_j needs x at the halo columns, which
one more forward exchange of x supplies.

Layout on a rank that owns global rows [row0, row1) (n_own rows):
  * its rows as a square CSR of n_own + n_halo rows: owned columns are renumbered 0..n_own-1,
    halo columns n_own..n_own+n_halo-1 (grouped by owning rank, ascending global index), the
    halo rows are empty; entries are re-sorted by local column inside each row (`perm` maps a
    local entry to its position among the owned rows' entries of the global CSR);
  * every vector is local: n_own owned values followed by the n_halo halo slots.
The exchange receives straight into the halo slots of the receiver's own vector (NCCL or
gloo point-to-point), one contiguous slice per neighbour; senders pack what a neighbour
needs with a gather kernel.

Everything numeric runs in libsla's kernels through an `ops` object (CudaOps below); the
communication goes through a `comm` object: TorchComm (torch.distributed -- NCCL on GPUs,
gloo on CPUs) or ThreadComm (ranks as threads of one process, each on its own CUDA stream;
a test transport for one GPU, where the ranks' kernels never wait on one another -- all
waiting happens on the host).  Set-up (partition, halo lists, local CSR) is host numpy.
"""
from __future__ import annotations

import math
import threading
from dataclasses import dataclass, field
from typing import Optional

import numpy as np


# ----------------------------------------------------------------------------- partition
def partition_rows(row_ptr: np.ndarray, world: int) -> np.ndarray:
    """world+1 row offsets: contiguous blocks with about equal (stored entries + rows)."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    n = row_ptr.size - 1
    cost = np.cumsum(np.diff(row_ptr) + 1)
    total = int(cost[-1]) if n > 0 else 0
    off = np.zeros(world + 1, dtype=np.int64)
    for r in range(1, world):
        off[r] = int(np.searchsorted(cost, r * total / world, side="left")) + 1 if n > 0 else 0
    off[world] = n
    return np.maximum.accumulate(np.minimum(off, n))


@dataclass
class LocalBlock:
    """The part of a row-partitioned matrix one rank holds (host arrays)."""
    rank: int
    world: int
    offsets: np.ndarray            # world+1 global row offsets
    n_own: int
    n_halo: int
    row_ptr: np.ndarray            # int32, n_own + n_halo + 1 (halo rows empty)
    col: np.ndarray                # int32 local columns, ascending in each row
    val: np.ndarray                # values in local entry order
    perm: np.ndarray               # int32: local entry -> position among the owned rows' global entries
    halo_global: np.ndarray        # int64 global index of each halo slot
    recv_from: list = field(default_factory=list)    # [(rank q, first halo slot, count)]
    send_to: list = field(default_factory=list)      # [(rank q, int32 owned local indices, in q's order)]

    @property
    def n_loc(self) -> int:
        return self.n_own + self.n_halo

    @property
    def row0(self) -> int:
        return int(self.offsets[self.rank])


def _owner(offsets: np.ndarray, g: np.ndarray) -> np.ndarray:
    return np.searchsorted(offsets, g, side="right") - 1


def build_local(row_ptr: np.ndarray, col: np.ndarray, val: np.ndarray, offsets: np.ndarray, rank: int,
                comm) -> LocalBlock:
    """This rank's block of a global CSR (host arrays; only rows [row0, row1) are read) and
    its halo lists.  The send lists come from one all-gather of every rank's requests."""
    world = offsets.size - 1
    r0, r1 = int(offsets[rank]), int(offsets[rank + 1])
    k0, k1 = int(row_ptr[r0]), int(row_ptr[r1])
    rp = np.asarray(row_ptr[r0:r1 + 1], dtype=np.int64) - k0
    gcol = np.asarray(col[k0:k1], dtype=np.int64)
    n_own = r1 - r0
    own = (gcol >= r0) & (gcol < r1)
    halo_g = np.unique(gcol[~own])                           # ascending global = grouped by owner
    hown = _owner(offsets, halo_g)
    lcol = np.empty(gcol.size, dtype=np.int64)
    lcol[own] = gcol[own] - r0
    lcol[~own] = n_own + np.searchsorted(halo_g, gcol[~own])
    # re-sort each row's entries by local column
    rows = np.repeat(np.arange(n_own, dtype=np.int64), np.diff(rp))
    order = np.lexsort((lcol, rows))
    n_halo = int(halo_g.size)
    rp_loc = np.concatenate([rp, np.full(n_halo, rp[-1], dtype=np.int64)])
    recv_from = []
    requests = []
    for q in range(world):
        sel = np.nonzero(hown == q)[0]
        if sel.size:
            recv_from.append((q, int(sel[0]), int(sel.size)))
        requests.append(halo_g[sel].astype(np.int64))
    # every rank's requests, so each rank learns what its neighbours need from it
    all_req = comm.all_gather_object(requests)
    send_to = []
    for q in range(world):
        if q == rank:
            continue
        need = np.asarray(all_req[q][rank], dtype=np.int64)
        if need.size:
            send_to.append((q, (need - r0).astype(np.int32)))
    return LocalBlock(rank, world, np.asarray(offsets, dtype=np.int64), n_own, n_halo,
                      rp_loc.astype(np.int32), lcol[order].astype(np.int32),
                      np.asarray(val[k0:k1])[order], order.astype(np.int32), halo_g,
                      recv_from, send_to)


def transpose_local(blk: LocalBlock) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Square CSR (n_loc rows) of the transpose of the rank's rows: row j lists the owned
    rows i that store column j.  Used for products with A^T (then summed into owners)."""
    n = blk.n_loc
    rows = np.repeat(np.arange(blk.n_own, dtype=np.int64), np.diff(blk.row_ptr[:blk.n_own + 1]))
    c = blk.col.astype(np.int64)
    order = np.lexsort((rows, c))
    counts = np.bincount(c, minlength=n)
    rp = np.zeros(n + 1, dtype=np.int64)
    np.cumsum(counts, out=rp[1:])
    return rp.astype(np.int32), rows[order].astype(np.int32), blk.val[order]


# ----------------------------------------------------------------------------- transports
class TorchComm:
    """torch.distributed point-to-point and all-reduce (NCCL on GPUs, gloo on CPUs)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather_object(self, obj):
        out = [None] * self.world
        self.dist.all_gather_object(out, obj, group=self.group)
        return out

    def exchange(self, sends, recvs):
        """sends / recvs: lists of (peer, tensor); all posted at once, then waited on."""
        ops = [self.dist.P2POp(self.dist.isend, t, p, group=self.group) for p, t in sends]
        ops += [self.dist.P2POp(self.dist.irecv, t, p, group=self.group) for p, t in recvs]
        if ops:
            for w in self.dist.batch_isend_irecv(ops):
                w.wait()

    def all_reduce_sum(self, t):
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
        return t


class ThreadHub:
    """Shared state of ThreadComm ranks (one per thread of one process)."""

    def __init__(self, world: int):
        self.world = world
        self.barrier = threading.Barrier(world)
        self.slots = {}
        self.lock = threading.Lock()
        self.gather = [None] * world


class ThreadComm:
    """Ranks as threads of one process (each with its own CUDA stream): a transport for
    testing the multi-rank path on one GPU.  Every collective is a host-side rendezvous;
    no kernel ever waits for another rank's kernel.  Reductions sum the ranks' values in rank
    order on the host (fp64), so they are deterministic."""

    def __init__(self, hub: ThreadHub, rank: int, stream=None):
        self.hub, self.rank, self.world = hub, rank, hub.world
        self.stream = stream

    def _sync(self):
        if self.stream is not None:
            self.stream.synchronize()

    def all_gather_object(self, obj):
        self.hub.gather[self.rank] = obj
        self.hub.barrier.wait()
        out = list(self.hub.gather)
        self.hub.barrier.wait()
        return out

    def exchange(self, sends, recvs):
        self._sync()
        with self.hub.lock:
            for p, t in sends:
                self.hub.slots[(self.rank, p)] = t
        self.hub.barrier.wait()
        for p, t in recvs:
            t.copy_(self.hub.slots[(p, self.rank)])
        self._sync()
        self.hub.barrier.wait()
        with self.hub.lock:
            for p, _ in sends:
                self.hub.slots.pop((self.rank, p), None)

    def all_reduce_sum(self, t):
        self._sync()
        vals = self.all_gather_object(t.detach().to("cpu", copy=True).double().numpy())
        tot = np.zeros_like(vals[0])
        for v in vals:
            tot = tot + v
        import torch
        t.copy_(torch.from_numpy(tot).to(t.dtype))
        return t


# ----------------------------------------------------------------------------- kernels
class CudaOps:
    """The numeric steps on the GPU, all in libsla's kernels."""

    def __init__(self, device=None, stream=None):
        import torch
        self.torch = torch
        self.device = torch.device("cuda") if device is None else torch.device(device)
        self.stream = stream

    def tensor(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a)).to(self.device)

    def zeros(self, n, dtype):
        return self.torch.zeros(n, dtype=dtype, device=self.device)

    def matrix(self, rp, ci, val):
        import differentiable_sparse_linear_b200 as sla
        return sla.sla_csr_create(self.tensor(rp), self.tensor(ci), self.tensor(val), stream=self.stream)

    def spmv(self, A, x, y):
        import differentiable_sparse_linear_b200 as sla
        sla.sla_spmv(A, x, y, stream=self.stream)

    def dot(self, x, y, n):
        import differentiable_sparse_linear_b200 as sla
        return sla.sla_vec_dot(x[:n], y[:n], stream=self.stream)

    def update(self, alpha, p, q, x, r, dinv, z, n):
        import differentiable_sparse_linear_b200 as sla
        return sla.sla_pcg_update(alpha, p, q, x, r, dinv, z, n=n, stream=self.stream)

    def direction(self, beta, z, p, n):
        import differentiable_sparse_linear_b200 as sla
        sla.sla_pcg_direction(beta, z, p, n=n, stream=self.stream)

    def gather(self, idx, src, dst):
        import differentiable_sparse_linear_b200 as sla
        sla.sla_vec_gather(idx, src, dst, stream=self.stream)

    def scatter_add(self, idx, src, dst):
        import differentiable_sparse_linear_b200 as sla
        sla.sla_vec_scatter_add(idx, src, dst, stream=self.stream)

    def pattern_grad(self, A, lam, x):
        import differentiable_sparse_linear_b200 as sla
        return sla.sla_pattern_grad(A, lam, x, stream=self.stream)

    def jacobi(self, blk: LocalBlock, dtype):
        """1 / A_ii of the owned rows (from the local values; set-up on the host)."""
        rows = np.repeat(np.arange(blk.n_own), np.diff(blk.row_ptr[:blk.n_own + 1]))
        d = np.zeros(blk.n_loc, dtype=np.float64)
        diag = blk.col.astype(np.int64) == rows
        d[rows[diag]] = np.asarray(blk.val, dtype=np.float64)[diag]
        if np.any(d[:blk.n_own] <= 0):
            raise ValueError("every owned row needs a positive diagonal entry")
        inv = np.zeros(blk.n_loc, dtype=np.float64)
        inv[:blk.n_own] = 1.0 / d[:blk.n_own]
        return self.tensor(inv.astype(np.dtype(str(dtype).replace("torch.", ""))))

    def host(self, t):
        return t.detach().to("cpu").numpy()


# ----------------------------------------------------------------------------- exchange
class HaloExchange:
    """Forward (owner -> halo copies) and reverse (halo contributions summed into owners)."""

    def __init__(self, blk: LocalBlock, ops, comm, dtype):
        self.blk, self.ops, self.comm = blk, ops, comm
        self.send_idx = [(q, ops.tensor(idx)) for q, idx in blk.send_to]
        self.send_buf = [(q, ops.zeros(int(idx.size), dtype)) for q, idx in blk.send_to]

    def forward(self, v):
        """Fill v's halo slots with the owners' values."""
        for (q, idx), (_, buf) in zip(self.send_idx, self.send_buf):
            self.ops.gather(idx, v, buf)
        n = self.blk.n_own
        recvs = [(q, v[n + a:n + a + c]) for q, a, c in self.blk.recv_from]
        self.comm.exchange(list(self.send_buf), recvs)

    def reverse_add(self, v):
        """Send v's halo slots to their owners, which add them to the owned entries (in rank
        order, so the sums are deterministic); the halo slots are zeroed."""
        n = self.blk.n_own
        sends = [(q, v[n + a:n + a + c]) for q, a, c in self.blk.recv_from]
        recvs = list(self.send_buf)
        self.comm.exchange(sends, recvs)
        for (q, idx), (_, buf) in zip(self.send_idx, self.send_buf):
            self.ops.scatter_add(idx, buf, v)
        if self.blk.n_halo:
            v[n:].zero_()


# ----------------------------------------------------------------------------- solver
@dataclass
class DistInfo:
    iters: int
    relres: float
    status: int            # 0 converged, 1 maxit, 2 breakdown


class DistributedPCG:
    """Jacobi-preconditioned (or plain) CG on a row-partitioned SPD matrix; one rank's side.

    Every rank calls the same methods in the same order (SPMD).  Per iteration: one halo
    exchange of p, the local product, one all-reduce of p.q, the fused update with the
    all-reduce of (r.r, r.z), and the direction update -- the recurrence of the single-GPU
    solver, with the stopping test on the recursive residual."""

    def __init__(self, blk: LocalBlock, ops, comm, dtype, precond: str = "jacobi"):
        self.blk, self.ops, self.comm, self.dtype = blk, ops, comm, dtype
        self.A = ops.matrix(blk.row_ptr, blk.col, blk.val)
        self.halo = HaloExchange(blk, ops, comm, dtype)
        self.dinv = ops.jacobi(blk, dtype) if precond == "jacobi" else None
        self._AT = None
        n = blk.n_loc
        self.p, self.q, self.r, self.z, self.x = (ops.zeros(n, dtype) for _ in range(5))

    def _allreduce(self, t):
        return self.ops.host(self.comm.all_reduce_sum(t))

    def solve(self, b_own, tol: float, maxit: Optional[int] = None) -> tuple:
        """x_own with A x = b (global system); b_own: this rank's n_own values (device)."""
        blk, ops = self.blk, self.ops
        n = blk.n_own
        nglob = int(blk.offsets[-1])
        maxit = 10 * max(nglob, 1) if maxit is None else int(maxit)
        for t in (self.p, self.q, self.x, self.z, self.r):
            t.zero_()
        self.r[:n].copy_(b_own)
        bn = math.sqrt(float(self._allreduce(ops.dot(self.r, self.r, n))[0]))
        if bn == 0.0:
            return self.x[:n].clone(), DistInfo(0, 0.0, 0)
        s = self._allreduce(ops.update(0.0, self.p, self.q, self.x, self.r, self.dinv, self.z, n))
        rho = float(s[1])
        if not (rho > 0.0) or not math.isfinite(rho):
            return self.x[:n].clone(), DistInfo(0, 1.0, 2)
        ops.direction(0.0, self.z, self.p, n)
        k, relres, status = 0, 1.0, 1
        while k < maxit:
            k += 1
            self.halo.forward(self.p)
            ops.spmv(self.A, self.p, self.q)
            pq = float(self._allreduce(ops.dot(self.p, self.q, n))[0])
            if not (pq > 0.0) or not math.isfinite(pq):
                status = 2
                break
            alpha = rho / pq
            s = self._allreduce(ops.update(alpha, self.p, self.q, self.x, self.r, self.dinv, self.z, n))
            relres = math.sqrt(float(s[0])) / bn
            if not math.isfinite(relres):
                status = 2
                break
            if relres <= tol:
                status = 0
                break
            rz = float(s[1])
            if not (rz > 0.0):
                status = 2
                break
            ops.direction(rz / rho, self.z, self.p, n)
            rho = rz
        return self.x[:n].clone(), DistInfo(k, relres, status)

    def adjoint(self, x_own, w_own, tol: float, maxit: Optional[int] = None) -> tuple:
        """lambda_own (A^T lambda = w with A^T = A) and dL/dA_ij = -lambda_i x_j for this
        rank's stored entries, in the global CSR order of its rows."""
        blk, ops = self.blk, self.ops
        n = blk.n_own
        lam_own, info = self.solve(w_own, tol, maxit)
        xl = ops.zeros(blk.n_loc, self.dtype)
        xl[:n].copy_(x_own)
        self.halo.forward(xl)                      # x at the halo columns
        lam = ops.zeros(blk.n_loc, self.dtype)
        lam[:n].copy_(lam_own)
        g_loc = ops.pattern_grad(self.A, lam, xl)
        g = ops.zeros(int(blk.col.size), self.dtype)
        ops.scatter_add(ops.tensor(blk.perm), g_loc, g)      # back to the global entry order
        return lam_own, g, info

    def rmatvec(self, v_own):
        """A^T v for a (possibly non-symmetric) row-partitioned A: the local transposed
        product gives contributions to owned and halo columns; the halo ones are summed into
        their owners (sum-into-owner)."""
        blk, ops = self.blk, self.ops
        if self._AT is None:
            self._AT = ops.matrix(*transpose_local(blk))
        v = ops.zeros(blk.n_loc, self.dtype)
        v[:blk.n_own].copy_(v_own)
        y = ops.zeros(blk.n_loc, self.dtype)
        ops.spmv(self._AT, v, y)
        self.halo.reverse_add(y)
        return y[:blk.n_own].clone()

    def matvec(self, v_own):
        """A v (forward exchange, then the local product)."""
        blk, ops = self.blk, self.ops
        v = ops.zeros(blk.n_loc, self.dtype)
        v[:blk.n_own].copy_(v_own)
        self.halo.forward(v)
        y = ops.zeros(blk.n_loc, self.dtype)
        ops.spmv(self.A, v, y)
        return y[:blk.n_own].clone()
