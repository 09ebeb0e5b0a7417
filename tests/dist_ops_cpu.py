"""CPU stand-in for the distributed solver's numeric steps, for testing the multi-rank host
logic (partition, halo lists, exchanges, the SPMD recurrence) with gloo ranks on CPU.

Test infrastructure: the local product is the oracle's SpMV; the vector steps are numpy
fp64 restatements of what libsla's iteration-step calls do.  The product path (CudaOps in
differentiable_sparse_linear_b200.distributed) never uses this."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sla_workloads import CSR


class OracleOps:
    def __init__(self):
        self.ora = oracle.get()

    def tensor(self, a):
        return torch.from_numpy(np.ascontiguousarray(a).copy())

    def zeros(self, n, dtype):
        return torch.zeros(n, dtype=dtype)

    def matrix(self, rp, ci, val):
        n = len(rp) - 1
        return CSR(n, n, np.asarray(rp, np.int32), np.asarray(ci, np.int32), np.asarray(val))

    def spmv(self, A, x, y):
        y.copy_(torch.from_numpy(self.ora.spmv(A, x.numpy())).to(y.dtype))

    def dot(self, x, y, n):
        return torch.tensor([float(np.dot(x[:n].double().numpy(), y[:n].double().numpy()))], dtype=torch.float64)

    def update(self, alpha, p, q, x, r, dinv, z, n):
        x[:n] += alpha * p[:n]
        r[:n] -= alpha * q[:n]
        z[:n] = r[:n] * dinv[:n] if dinv is not None else r[:n]
        rr = float(np.dot(r[:n].double().numpy(), r[:n].double().numpy()))
        rz = float(np.dot(r[:n].double().numpy(), z[:n].double().numpy()))
        return torch.tensor([rr, rz], dtype=torch.float64)

    def direction(self, beta, z, p, n):
        p[:n] = z[:n] + beta * p[:n]

    def gather(self, idx, src, dst):
        dst.copy_(src[idx.long()])

    def scatter_add(self, idx, src, dst):
        il = idx.long()
        dst[il] = dst[il] + src

    def pattern_grad(self, A, lam, x):
        return torch.from_numpy(self.ora.grad(A, lam.double().numpy(), x.double().numpy())).to(lam.dtype)

    def jacobi(self, blk, dtype):
        rows = np.repeat(np.arange(blk.n_own), np.diff(blk.row_ptr[:blk.n_own + 1]))
        inv = np.zeros(blk.n_loc, dtype=np.float64)
        diag = blk.col.astype(np.int64) == rows
        inv[rows[diag]] = 1.0 / np.asarray(blk.val, dtype=np.float64)[diag]
        return torch.from_numpy(inv).to(dtype)

    def host(self, t):
        return t.detach().numpy()
