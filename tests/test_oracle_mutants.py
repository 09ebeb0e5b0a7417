"""Planted mistakes: each case copies oracle.c, plants one plausible mistake, builds the copy
on the CPU and requires that at least one oracle pin fails on it.  This shows the pins
would catch a dropped term, a wrong sign or index, or a transposed operand."""
import os
import shutil
import tempfile

import pytest

import oracle
import oracle_checks as OC
from oracle import build as obuild

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

MUTANTS = {
    "spmv_wrong_index": ("s += val[k] * x[col[k]];", "s += val[k] * x[i];"),
    "spmv_drops_last_entry": ("for (int64_t k = row_ptr[i]; k < row_ptr[i + 1]; ++k)\n            s +=",
                              "for (int64_t k = row_ptr[i]; k < row_ptr[i + 1] - 1; ++k)\n            s +="),
    "transpose_keeps_column": ("ciT[dst] = (int32_t)i;", "ciT[dst] = (int32_t)ci[k];"),
    "jacobi_multiplies": ("z[i] = r[i] / M->diag[i];", "z[i] = r[i] * M->diag[i];"),
    "spai_drops_eps": ("z[i] = z[i] + M->eps * r[i];", "z[i] = z[i];"),
    "spai_transposed_order": (
        "ora_spmv(n, M->gt_rp, M->gt_ci, M->gt_v, r, work);   /* y = G^T r */\n"
        "        if (store_f32)\n"
        "            ora_round_f32(n, work);\n"
        "        ora_spmv(n, M->g_rp, M->g_ci, M->g_v, work, z);      /* z = G y   */",
        "ora_spmv(n, M->g_rp, M->g_ci, M->g_v, r, work);\n"
        "        ora_spmv(n, M->gt_rp, M->gt_ci, M->gt_v, work, z);"),
    "first_direction_unpreconditioned": ("p[i] = z[i];\n    rho =", "p[i] = r[i];\n    rho ="),
    "rho_uses_r_dot_r": ("rho_new = ora_dot(n, r, z);", "rho_new = ora_dot(n, r, r);"),
    "beta_dropped": ("p[i] = z[i] + beta * p[i];", "p[i] = z[i];"),
    "x_update_uses_q": ("x[i] = x[i] + alpha * p[i];", "x[i] = x[i] + alpha * q[i];"),
    "residual_sign": ("r[i] = r[i] - alpha * q[i];", "r[i] = r[i] + alpha * q[i];"),
    "absolute_stop_test": ("*relres = rnorm / bnorm;", "*relres = rnorm;"),
    "grad_sign": ("g[k] = -lam[i] * x[ci[k]];", "g[k] = lam[i] * x[ci[k]];"),
    "grad_transposed": ("g[k] = -lam[i] * x[ci[k]];", "g[k] = -lam[ci[k]] * x[i];"),
    "bsr_block_transposed": ("s += val[k * b * b + (int64_t)r * b + c] * x[(int64_t)ci[k] * b + c];",
                             "s += val[k * b * b + (int64_t)c * b + r] * x[(int64_t)ci[k] * b + c];"),
    "bsr_operand_row": ("s += val[k * b * b + (int64_t)r * b + c] * x[(int64_t)ci[k] * b + c];",
                        "s += val[k * b * b + (int64_t)r * b + c] * x[(int64_t)ci[k] * b + r];"),
    "bsr_expansion_position": ("const int64_t p = k * b * b + (int64_t)r * b + c;",
                               "const int64_t p = k * b * b + (int64_t)c * b + r;"),
    "store_f32_keeps_q": ("        if (store_f32)\n            ora_round_f32(n, q);\n", ""),
    "store_f32_keeps_x": ("            ora_round_f32(n, x);\n", ""),
    "eigen_grad_sign": ("g[k] = v[i] * v[ci[k]];", "g[k] = -v[i] * v[ci[k]];"),
    "eigen_grad_row_only": ("g[k] = v[i] * v[ci[k]];", "g[k] = v[i] * v[i];"),
    "add_diagonal_first_entry": ("            if (ci[k] == i) {\n                out[k] = v[k] + c[i];",
                                 "            if (k == rp[i]) {\n                out[k] = v[k] + c[i];"),
    "bsr_expansion_column": ("out_ci[e] = (int32_t)((int64_t)ci[k] * b + c);",
                             "out_ci[e] = (int32_t)((int64_t)ci[k] + c);"),
}


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(workdir, name):
    old, new = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique or missing"
    path = os.path.join(workdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = obuild.build(src=path, out=os.path.join(workdir, f"lib{name}.so"), force=True)
    mut = oracle.Oracle(lib)
    failed = []
    for check in OC.ALL_CHECKS:
        try:
            check(mut)
        except AssertionError:
            failed.append(check.__name__)
        except Exception as e:                  # a crash-free numerical failure is also a catch
            failed.append(f"{check.__name__}:{type(e).__name__}")
    assert failed, f"no pin catches the planted mistake {name}"
