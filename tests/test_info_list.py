"""PcgInfoList (host only): the per-system results of a batched solve read in bulk from the
library's result structs behave as a sequence of PcgInfo."""
import differentiable_sparse_linear_b200 as sla
from differentiable_sparse_linear_b200 import _lib


def _arr(n):
    a = (_lib.sla_pcg_info * n)()
    for i in range(n):
        a[i].iters = 3 * i
        a[i].relres = 0.5 ** i
        a[i].status = i % 2
        a[i].engine = 3 if i % 3 else 1
    return a


def test_sequence_reads_every_field():
    infos = sla._infos(_arr(5))
    assert len(infos) == 5
    assert [i.iters for i in infos] == [0, 3, 6, 9, 12]
    assert infos[2] == sla.PcgInfo(6, 0.25, 0, "list")
    assert infos[-1].iters == 12 and infos[3].engine == "graph" and not infos[1].converged
    assert [i.iters for i in infos[1:3]] == [3, 6]
    assert int(infos.iters.sum()) == 30 and infos.engines == {"list", "graph"}


def test_concatenation_and_empty():
    a, b = sla._infos(_arr(2)), sla._infos(_arr(3))
    both = a + b
    assert isinstance(both, list) and [i.iters for i in both] == [0, 3, 0, 3, 6]
    assert [i.iters for i in [sla.PcgInfo(1, 0.0, 0)] + a] == [1, 0, 3]
    empty = sla._infos(_arr(0))
    assert len(empty) == 0 and list(empty) == [] and empty.engines == set()
