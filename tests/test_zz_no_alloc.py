"""The list solve entry point that allocates nothing, checked against the regular one.

Callers under a device-memory budget or pool, or that may not allocate after start-up, use
sla_pcg_solve_batched_noalloc: its per-system results go through a fixed array inside the
library instead of a per-call allocation.  This file is collected last so that, if it fails,
a run that stops at the first failure has already run every other test; it also passes on
its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import sla_workloads as W

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _rel(a, b):
    a = a.detach().cpu().numpy().astype(np.float64)
    b = b.detach().cpu().numpy().astype(np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("size", ["tiny", "small"])
def test_noalloc_matches_regular_list_solve(size):
    import differentiable_sparse_linear_b200 as sla
    w = W.workload(4, size)
    A = w.A
    Ad = sla.sla_csr_create_list(list(A.sys_row_off), _dev(A.row_ptr), _dev(A.col), _dev(A.val))
    M = sla.sla_precond_jacobi(Ad)
    b = _dev(w.B)
    x_ref, info_ref = sla.sla_pcg_solve_batched(Ad, M, b, rtol=w.tol)
    for call in range(2):                      # two calls in a row share the fixed array
        b2 = _dev(w.B) * (1.0 + call)          # the second call solves a scaled right-hand side
        x, info = sla.sla_pcg_solve_batched_noalloc(Ad, M, b2, rtol=w.tol)
        torch.cuda.synchronize()
        assert len(info) == A.batch
        assert _rel(x, x_ref * (1.0 + call)) <= 1e-8
        for a, r in zip(info, info_ref):
            assert a.status == r.status == 0
            assert a.iters == r.iters


def test_noalloc_rejects_too_many_systems():
    import differentiable_sparse_linear_b200 as sla
    nsys = 65537                               # one more than the fixed array holds
    rp = torch.arange(nsys + 1, dtype=torch.int32, device="cuda")
    ci = torch.arange(nsys, dtype=torch.int32, device="cuda")
    v = torch.ones(nsys, dtype=torch.float64, device="cuda")
    Ad = sla.sla_csr_create_list(list(range(nsys + 1)), rp, ci, v)
    with pytest.raises(sla.SlaError) as e:
        sla.sla_pcg_solve_batched_noalloc(Ad, None, torch.ones(nsys, dtype=torch.float64, device="cuda"))
    assert e.value.status == sla.SLA_ERR_INVALID_ARG
    assert "65536" in str(e.value)
