"""The oracle against the hand-derived worked examples in ``tests/golden/``.

The pages print no numeric worked example of the method, so each fixture is a
small case whose result follows by hand from the passage it cites (the
derivation is stored beside the numbers).  These pin the oracle to values that
do not come from the oracle itself."""
import glob
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        g = json.load(f)
    assert g["cite"].startswith("AdaCluster: Adaptive Query-Key Clustering")
    assert g["derivation"]
    return g


def test_every_fixture_is_used():
    names = sorted(os.path.basename(p) for p in glob.glob(os.path.join(GOLDEN, "*.json")))
    assert names == sorted(["attention_two_keys.json", "kmeans_euclid_1d.json", "kmeans_sphere_2d.json",
                            "multistage_four_groups.json", "multistage_strict_tau.json",
                            "select_size_and_score.json"])


@pytest.mark.parametrize("name", ["kmeans_euclid_1d.json", "kmeans_sphere_2d.json"])
def test_kmeans_worked_example(orc, name):
    g = _load(name)
    mode = orc.EUCLID if g["mode"] == "euclid" else orc.SPHERE
    x = np.array(g["x"], np.float32)
    xs, nrm = orc.prepare(x, mode)
    r = orc.kmeans(xs, g["k"], g["iters"], mode, trace=True)
    e, tol = g["expected"], g["tolerance"]
    np.testing.assert_array_equal(r.assign, e["assign"])
    np.testing.assert_array_equal(r.count, e["count"])
    if "rel_cent" in tol:
        np.testing.assert_allclose(r.cent, e["cent"], rtol=tol["rel_cent"], atol=tol["abs"])
    else:
        np.testing.assert_allclose(r.cent, e["cent"], atol=tol["abs"])
    if "dist" in e:
        np.testing.assert_allclose(r.dist, e["dist"], atol=tol["abs"])
    if "objective" in e:
        assert abs(r.trace[-1] - e["objective"]) <= tol["abs"]
    if "mean_norm" in e:
        np.testing.assert_allclose(orc.cluster_mean_norm(nrm, r.assign, g["k"]), e["mean_norm"], atol=tol["abs"])
    if "expected_iters0" in g:
        r0 = orc.kmeans(xs, g["k"], 0, mode)
        e0 = g["expected_iters0"]
        np.testing.assert_array_equal(r0.assign, e0["assign"])
        np.testing.assert_array_equal(r0.count, e0["count"])
        np.testing.assert_allclose(r0.cent, e0["cent"], atol=tol["abs"])


def test_attention_worked_example(orc):
    g = _load("attention_two_keys.json")
    q, k, v = (np.array(g[n], np.float32) for n in "qkv")
    out = orc.attention_rows(q, k, v, None, None, None, None, None, None, np.arange(len(q)))
    np.testing.assert_allclose(out, g["expected"]["out"], atol=g["tolerance"]["abs"])


def test_select_worked_example(orc):
    g = _load("select_size_and_score.json")
    d = g["d"]
    for c in g["cases"]:
        t = np.array(c["t"], np.float64)
        if "p" in c:
            s = c["rbar"] * t / math.sqrt(d)
            w = np.exp(s - s.max())
            np.testing.assert_allclose(w / w.sum(), c["p"], rtol=1e-12)
        qc = np.zeros((1, d), np.float32)
        qc[0, 0] = 1
        kc = np.zeros((len(t), d), np.float32)
        kc[:, 0] = t
        for top_p, kept in c["kept"].items():
            sel, cnt = orc.select(qc, np.array([c["rbar"]], np.float32), np.array([1], np.int32), kc,
                                  np.array(c["counts"], np.int32), float(top_p))
            assert sorted(sel[0, :cnt[0]].tolist()) == kept, (c["name"], top_p)


def test_multistage_worked_example(orc):
    g = _load("multistage_four_groups.json")
    inp = g["input"]
    rng = np.random.default_rng(inp["seed"])
    pts = [np.array(c) + rng.uniform(-inp["jitter"], inp["jitter"], (inp["per_group"], 2)) for c in inp["centres"]]
    pts.append(np.array(inp["pair"]))
    x = np.concatenate(pts).astype(np.float32)
    r = orc.multistage(x.astype(np.float64), g["m0"], g["iters"], orc.TAU_ABS, g["tau_abs"], g["nmax"], orc.EUCLID)
    e = g["expected"]
    assert (r.nclusters, r.dense, r.nstages) == (e["nclusters"], e["dense"], e["nstages"])
    np.testing.assert_array_equal(np.sort(r.count[:r.nclusters]), e["sorted_count"])
    n = len(x)
    assert r.assign[n - 2] == r.assign[n - 1] == e["pair_cluster"]
    np.testing.assert_allclose(r.cent[e["pair_cluster"]], e["pair_centre"], atol=g["tolerance"]["abs"])


def test_multistage_strict_threshold(orc):
    g = _load("multistage_strict_tau.json")
    x = np.array(g["x"], np.float64)
    r = orc.multistage(x, g["m0"], g["iters"], orc.TAU_ABS, g["tau_abs"], g["nmax"], orc.EUCLID)
    e = g["expected"]
    assert (r.nclusters, r.dense, r.nstages) == (e["nclusters"], e["dense"], e["nstages"])
    np.testing.assert_array_equal(r.cent[:r.nclusters], e["cent"])
