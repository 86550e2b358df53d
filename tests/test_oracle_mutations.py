"""Planted mistakes in the oracle must fail its pins.

Each case copies the oracle and its pin tests to a scratch directory, plants
one plausible mistake in its C source or its Python composition of the
steps, and runs the pins (tests/test_oracle_pins.py
and the worked examples of tests/golden/) against it.  The run must fail: the
pins are meant to catch a dropped term, a wrong tie rule, a wrong index or
threshold, a missing normalisation or scale anywhere in the oracle."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
# scratch runs in parallel, each oracle with a share of the cores
WORKERS = max(1, min(8, (os.cpu_count() or 2) // 2))
THREADS = max(1, (os.cpu_count() or 2) // WORKERS)

MUTATIONS = [
    ("assign ties to the highest id",
     "if (mode == ORC_EUCLID ? (s < bs) : (s > bs))", "if (mode == ORC_EUCLID ? (s <= bs) : (s >= bs))"),
    ("no query normalisation",
     "xs[i * d + t] = (nr > 0.0) ? (double)xi[t] / nr : 0.0;", "xs[i * d + t] = (double)xi[t];"),
    ("mean divides by count + 1",
     "(float)(s[t] / (double)cnt[j])", "(float)(s[t] / (double)(cnt[j] + 1))"),
    ("spherical update not normalised",
     "cent[(int64_t)j * d + t] = (float)(s[t] / nr2);", "cent[(int64_t)j * d + t] = (float)(s[t]);"),
    ("empty cluster zeroed",
     "if (cnt[j] == 0) continue;",
     "if (cnt[j] == 0) { for (int t = 0; t < d; t++) cent[(int64_t)j * d + t] = 0.0f; continue; }"),
    ("initial centroid row shifted by one",
     "int64_t r = ((int64_t)j * nr) / k;", "int64_t r = (((int64_t)j * nr) / k + 1) % nr;"),
    ("threshold test not strict",
     "if (!(dl[r] < tau)) U[keep++] = U[r];", "if (!(dl[r] <= tau)) U[keep++] = U[r];"),
    ("MEAN_X rule uses the sum", "tau = tau_value * (s / (double)nu);", "tau = tau_value * s;"),
    ("upper median radius", "tau = tau_value * rs[(m - 1) / 2];", "tau = tau_value * rs[m / 2];"),
    ("squared distance", "        acc = acc + df * df;\n    }\n    return sqrt(acc);",
     "        acc = acc + df * df;\n    }\n    return acc;"),
    ("stage size m0 at every stage", "        if (t == 0) mt = m0;\n        else {", "        if (1) mt = m0;\n        else {"),
    ("no N_max test", "        if (nc >= nmax) { F = 1; break; }\n", ""),
    ("no final reassignment",
     "        orc_assign(mode, n, NULL, d, xs, nc, cent, 0, assign, dist);\n        for (int j = 0; j < nc; j++) count[j] = 0;",
     "        for (int64_t i = 0; i < n; i++) assign[i] = 0;\n        for (int j = 0; j < nc; j++) count[j] = 0;"),
    ("selection score without the mean query norm", "return (rbar * dot) * scale;", "return dot * scale;"),
    ("selection weights without the cluster sizes",
     "double w = (double)k_count[b] * exp(s[b] - m);", "double w = exp(s[b] - m);"),
    ("top-p cut strict", "if (top_p < 1.0 && cum >= top_p) break;", "if (top_p < 1.0 && cum > top_p) break;"),
    ("attention scale 1/d", "        double *o = out + r * d;", "        double *o = out + r * d; scale = 1.0 / (double)d;"),
    ("Quest score keeps only the max-bound term", "acc = acc + (hi > lo ? hi : lo);", "acc = acc + hi;"),
    ("key lower bound takes the max", "if (x[t] < m[t]) m[t] = x[t];", "if (x[t] > m[t]) m[t] = x[t];"),
    ("cluster sort not stable", "for (int64_t i = 0; i < n; i++) perm[pos[assign[i]]++] = (int32_t)i;",
     "for (int64_t i = n - 1; i >= 0; i--) perm[pos[assign[i]]++] = (int32_t)i;"),
    ("selection ties to the higher id", "return (a->b > b->b) - (a->b < b->b);", "return (a->b < b->b) - (a->b > b->b);"),
    ("argtopk keeps one too many", "for (int r = 0; r < np && r < top_k; r++) keep[pb[r].b] = 1;",
     "for (int r = 0; r < np && r <= top_k; r++) keep[pb[r].b] = 1;"),
    ("later steps not warm-started", "rq = kmeans(xq, nq, spec.iters, SPHERE, init=prev.q.cent[:nq])",
     "rq = kmeans(xq, nq, spec.iters, SPHERE, init=None)", "__init__.py"),
    ("text keys clustered", "    if spec.text_keys:\n        k = k[:k.shape[0] - spec.text_keys]\n", "", "__init__.py"),
    ("mean query norm is the sum", "mean_norm[j] = c[j] ? (float)(s[j] / (double)c[j]) : 0.0f;",
     "mean_norm[j] = c[j] ? (float)(s[j]) : 0.0f;"),
    ("sparse attention over every key",
     "for (int c = 0; c < sel_cnt[a]; c++) allow[sel_idx[(int64_t)a * kk_stride + c]] = 1;",
     "for (int c = 0; c < kk; c++) allow[c] = 1;"),
    ("no final k-means assignment",
     "    double o = orc_assign(mode, nr, rows, d, xs, k, cent, 0, assign, dist);\n    if (obj_trace) obj_trace[2 * iters] = o;",
     "    double o = 0.0;\n    if (obj_trace) obj_trace[2 * iters] = o;"),
    ("pair count with query and key sizes swapped",
     "keys += k_count[sel_idx[(int64_t)a * kk_stride + c]];", "keys += q_count[sel_idx[(int64_t)a * kk_stride + c] % kq];"),
    ("pair count of the last query cluster dropped", "for (int a = 0; a < kq; a++) {\n        int64_t keys = 0;",
     "for (int a = 0; a < kq - 1; a++) {\n        int64_t keys = 0;"),
    ("per-query score of the normalised query", "    q_rows = _f32(q_rows)\n    n = q_rows.shape[0]",
     "    q_rows = _f32(q_rows / np.linalg.norm(q_rows, axis=1, keepdims=True))\n    n = q_rows.shape[0]",
     "__init__.py"),
    ("per-query rows attend with their cluster's selection",
     "out = attend_per_query(q, k, v, k_assign, nv + (1 if spec.text_keys else 0), sq, cq, rows)",
     "out = attention_rows(q, k, v, rq.assign, k_assign, nv + (1 if spec.text_keys else 0), sel, cnt, dense, rows)",
     "__init__.py"),
    ("text group also for empty query clusters",
     "live = np.nonzero(np.asarray(rq.count)[:sel.shape[0]] > 0)[0]", "live = np.arange(sel.shape[0])",
     "__init__.py"),
]


def _copy(dst):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "clustered_sparse_attention_head_b200"),
                    os.path.join(dst, "clustered_sparse_attention_head_b200"),
                    ignore=shutil.ignore_patterns("*.so", "_build", "csrc", "__pycache__"))
    os.makedirs(os.path.join(dst, "tests"))
    for f in ("conftest.py", "test_oracle_pins.py", "test_golden.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))


def _run(base, i, mut):
    name, old, new = mut[:3]
    fname = mut[3] if len(mut) > 3 else "adacluster_oracle.c"
    dst = os.path.join(base, f"m{i}")
    _copy(dst)
    src = os.path.join(dst, "oracle", fname)
    s = open(src).read()
    if s.count(old) != 1:
        return None
    open(src, "w").write(s.replace(old, new))
    env = dict(os.environ, OMP_NUM_THREADS=str(THREADS))
    return subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                           "tests/test_oracle_pins.py", "tests/test_golden.py"],
                          cwd=dst, capture_output=True, text=True, timeout=600, env=env)


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Every planted mistake, run in parallel (one scratch copy each)."""
    from concurrent.futures import ThreadPoolExecutor
    base = str(tmp_path_factory.mktemp("mutations"))
    with ThreadPoolExecutor(WORKERS) as ex:
        futs = [ex.submit(_run, base, i, m) for i, m in enumerate(MUTATIONS)]
        return [f.result() for f in futs]


@pytest.mark.parametrize("i", range(len(MUTATIONS)), ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(outcomes, i):
    name = MUTATIONS[i][0]
    r = outcomes[i]
    assert r is not None, f"the mistake's site is no longer unique: {name}"
    assert r.returncode not in (0, 5), f"no pin failed with '{name}' planted"
    assert "FAILED" in r.stdout, f"'{name}': the pins did not fail cleanly:\n{r.stdout[-1500:]}\n{r.stderr[-800:]}"
