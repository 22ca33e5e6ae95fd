"""Planted mistakes in the oracle: each edit below makes one plausible error
in oracle/eaga_oracle.c (a dropped term, a wrong sign, index, column or
operand), and the oracle's pins (test_oracle_pins.py) must catch every one.

Each mutant is compiled from a copy of the oracle in a temporary directory,
and the pin suite runs against that copy in a subprocess.  The unmodified
copy must pass.  Nothing here touches the repository's own oracle build.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# name: (text in eaga_oracle.c, replacement).  Only edits that change some
# output belong here: leaving dO of a masked row unzeroed, for instance, does
# not (its row has a = 0, so that dO reaches nothing), and no pin could catch it.
MUTANTS = {
    # forward
    "drop_beta": ("sp[j] = s * (1.0 + gam) + bet;", "sp[j] = s * (1.0 + gam);"),
    "gamma_without_one": ("sp[j] = s * (1.0 + gam) + bet;", "sp[j] = s * gam + bet;"),
    "no_score_scale": ("return acc / sqrt((double)d->dh);", "return acc;"),
    "film_wrong_column": ("acc += e[c] * Wfe[(long)c * 2 * d->H + k];",
                          "acc += e[c] * Wfe[(long)c * 2 * d->H + (k + 1) % (2 * d->H)];"),
    "edge_update_shifted_index": ("double coef = arow[(long)h * n + j];\n                    if (variant == ORC_UNNORMALISED) {\n                        const double sp = srow[(long)h * n + j] * (1.0 + frow[(long)j * 2 * H + h]) +",
                                  "double coef = arow[(long)h * n + (j + 1) % n];\n                    if (variant == ORC_UNNORMALISED) {\n                        const double sp = srow[(long)h * n + j] * (1.0 + frow[(long)j * 2 * H + h]) +"),
    "mask_rows_only": ("if (mb[j] && sp[j] > m) m = sp[j];", "if (sp[j] > m) m = sp[j];"),
    # backward
    "dS_sign": ("const double dsp = a * (dA[(long)h * n + j] - D)",
                "const double dsp = a * (dA[(long)h * n + j] + D)"),
    "dE_missing_film_term": ("acc += df[(long)j * F + k] * Wfe[(long)c * F + k];",
                             "acc += 0 * df[(long)j * F + k];"),
    "dq_without_film_factor": ("const double ds = dsp * (1.0 + gam);", "const double ds = dsp;"),
    "dk_without_film_factor": ("const double ds = dsp * (1.0 + f[h]);", "const double ds = dsp;"),
    "dv_transposed": ("dV[r * hd + h * dh + t] += a * dO[ri * hd + h * dh + t];",
                      "dV[r * hd + h * dh + t] += a * dO[r * hd + h * dh + t];"),
    "dWe_wrong_operand": ("pWe[(long)h * de + c] += coef * dEout[e0 + c];",
                          "pWe[(long)h * de + c] += coef * E[e0 + c];"),
    "lse_without_log": ("lse[h] = valid ? m + log(l) : -INFINITY;", "lse[h] = valid ? m + l : -INFINITY;"),
    # node residual and output projection
    "out_proj_not_masked": ("Xout[r * dx + o] = X[r * dx + o] + (mi != 0.0 ? acc : 0.0);",
                            "Xout[r * dx + o] = X[r * dx + o] + acc;"),
    "out_proj_no_residual": ("Xout[r * dx + o] = X[r * dx + o] + (mi != 0.0 ? acc : 0.0);",
                             "Xout[r * dx + o] = (mi != 0.0 ? acc : 0.0);"),
    "dWo_dbo_not_masked": ("if (!M[r]) continue;", "if (0) continue;"),
    "dWo_wrong_operand": ("gr->Wo[(long)k * dx + o] += O[r * hd + k] * dXout[r * dx + o];",
                          "gr->Wo[(long)k * dx + o] += V[r * hd + k] * dXout[r * dx + o];"),
    # gradients of the FiLM maps and of y
    "dWfe_wrong_operand": ("pWfe[(long)c * F + k] += E[e0 + c] * df[(long)j * F + k];",
                           "pWfe[(long)c * F + k] += dEout[e0 + c] * df[(long)j * F + k];"),
    "dWfy_shifted_column": ("gr->Wfy[(long)c * F + k] += y[(long)b * dyd + c] * dg[(long)b * F + k];",
                            "gr->Wfy[(long)c * F + k] += y[(long)b * dyd + c] * dg[(long)b * F + (k + 1) % F];"),
    "dbf_missing": ("gr->bf[k] += dg[(long)b * F + k];", "gr->bf[k] += 0.0 * dg[(long)b * F + k];"),
    "dy_shifted_column": ("acc += dg[(long)b * F + k] * w->Wfy[(long)c * F + k];",
                          "acc += dg[(long)b * F + k] * w->Wfy[(long)c * F + (k + 1) % F];"),
    # ablation variants (unnormalised edge update, Light Edge)
    "unnormalised_update_uses_a": ("coef = valid ? sp : 0.0;\n                    }\n                    acc += coef",
                                   "coef = arow[(long)h * n + j];\n                    }\n                    acc += coef"),
    "unnormalised_update_unmasked": ("coef = valid ? sp : 0.0;\n                    }\n                    acc += coef",
                                     "coef = sp;\n                    }\n                    acc += coef"),
    "unnormalised_D_keeps_edge_term": ("dA[(long)h * n + j] = unnorm ? dov : dov + u;",
                                       "dA[(long)h * n + j] = dov + u;"),
    "unnormalised_row_dS_without_u": ("+ (unnorm ? urow[j] : 0.0);", "+ 0.0;"),
    "unnormalised_column_dS_without_u": ("a * (dov - Dst[ri * H + h]) + u :", "a * (dov - Dst[ri * H + h]) :"),
    "unnormalised_dWe_uses_a": ("coef = valid ? sp : 0.0;\n                    }\n                    pWe",
                                "coef = arow[(long)h * n + j];\n                    }\n                    pWe"),
    "light_edge_keeps_Wfe": ("const double *Wfe = variant == ORC_LIGHT_EDGE ? Wfe0 : w->Wfe;\n    double *Q",
                             "const double *Wfe = w->Wfe;\n    double *Q"),
    "light_edge_dWfe_not_zeroed": ("if (variant == ORC_LIGHT_EDGE) memset(gr->Wfe", "if (0) memset(gr->Wfe"),
    "dX_without_dK_term": ("for (int p = 0; p < 3; ++p)\n                for (int k = 0; k < hd; ++k) acc += dN[p]",
                           "for (int p = 0; p < 3; p += 2)\n                for (int k = 0; k < hd; ++k) acc += dN[p]"),
}


def _copy_tree(dst, oracle_src):
    os.makedirs(os.path.join(dst, "oracle"))
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), os.path.join(dst, "oracle"))
    with open(os.path.join(dst, "oracle", "eaga_oracle.c"), "w") as f:
        f.write(oracle_src)
    os.makedirs(os.path.join(dst, "tests"))
    for name in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(dst, "tests"))
    os.makedirs(os.path.join(dst, "edge_aware_graph_b200"))
    for name in ("__init__.py", "inputs.py"):
        shutil.copy(os.path.join(ROOT, "edge_aware_graph_b200", name), os.path.join(dst, "edge_aware_graph_b200"))


def _run_pins(dst):
    env = dict(os.environ, PYTHONPATH=dst, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "tests/test_oracle_pins.py"],
                       cwd=dst, env=env, capture_output=True, text=True, timeout=900)
    lines = r.stdout.strip().splitlines()
    return r.returncode, (lines[-1] if lines else r.stderr[-500:])


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    src = open(os.path.join(ROOT, "oracle", "eaga_oracle.c")).read()
    jobs = {"unmodified": src}
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, f"{name}: the text to mutate is not in the oracle exactly once"
        jobs[name] = src.replace(old, new)
    base = tmp_path_factory.mktemp("oracle_mutants")
    dirs = {}
    for name, text in jobs.items():
        dirs[name] = str(base / name)
        _copy_tree(dirs[name], text)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
        futs = {name: ex.submit(_run_pins, d) for name, d in dirs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_unmodified_copy_passes_the_pins(results):
    rc, summary = results["unmodified"]
    assert rc == 0, summary


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(results, name):
    rc, summary = results[name]
    # exit code 1: the suite ran and at least one pin failed (not a build or
    # collection error, which would be 2 or more)
    assert rc == 1 and "failed" in summary, summary
