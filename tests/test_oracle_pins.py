"""Pins for the CPU oracle: each test checks it against something other than
itself (brute force, closed forms, invariants, textbook routines, hand-derived
examples).  Rules cited from "AdaCluster: Adaptive Query-Key Clustering for
Sparse Attention in Video Generation" (Tan et al.)."""
import itertools
import math

import numpy as np
import pytest

from clustered_sparse_attention_head_b200 import workloads as W


def _gmm(n, d, comps, seed, sigma=0.3):
    rng = np.random.default_rng(seed)
    mu = rng.standard_normal((comps, d)).astype(np.float32)
    lab = rng.integers(0, comps, n)
    return (mu[lab] + sigma * rng.standard_normal((n, d))).astype(np.float32)


# ---------------------------------------------------------------- assignment
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_assign_euclid_bruteforce_with_ties(orc, seed):
    """§3.2.1: keys go to the Euclidean-closest centre.  Small integers make
    every distance exact, duplicated centroids force exact ties -> lowest id."""
    rng = np.random.default_rng(seed)
    n, k, d = 40, 7, 3
    x = rng.integers(-3, 4, (n, d)).astype(np.float32)
    c = rng.integers(-3, 4, (k, d)).astype(np.float32)
    c[5] = c[2]
    ids, dist, obj = orc.assign(x.astype(np.float64), c, orc.EUCLID)
    for i in range(n):
        d2 = [sum((float(x[i, t]) - float(c[j, t])) ** 2 for t in range(d)) for j in range(k)]
        best = min(range(k), key=lambda j: (d2[j], j))
        assert ids[i] == best
        assert dist[i] == math.sqrt(d2[best])
    assert 5 not in ids.tolist()


@pytest.mark.parametrize("seed", [0, 1])
def test_assign_sphere_bruteforce(orc, seed):
    """§3.1: normalised queries go to the centre of largest cosine; for unit
    centroids that is also the Euclidean-closest centre on the sphere."""
    rng = np.random.default_rng(seed)
    n, k, d = 50, 6, 4
    x = rng.standard_normal((n, d)).astype(np.float32)
    c = rng.standard_normal((k, d))
    c = (c / np.linalg.norm(c, axis=1, keepdims=True)).astype(np.float32)
    c[4] = c[1]
    xs, nrm = orc.prepare(x, orc.SPHERE)
    ids, dist, _ = orc.assign(xs, c, orc.SPHERE)
    for i in range(n):
        xi = [float(v) for v in x[i]]
        r = math.sqrt(sum(v * v for v in xi))
        cos = [sum(xi[t] / r * float(c[j, t]) for t in range(d)) for j in range(k)]
        eu = [sum((xi[t] / r - float(c[j, t])) ** 2 for t in range(d)) for j in range(k)]
        best = max(range(k), key=lambda j: (cos[j], -j))
        assert ids[i] == best
        assert min(range(k), key=lambda j: (eu[j], j)) == best or abs(eu[best] - min(eu)) < 1e-12
        assert abs(dist[i] - math.sqrt(eu[best])) < 1e-12
    assert 4 not in ids.tolist()


def test_normalise_unit_and_zero(orc):
    """§3.1 normalisation: unit length, a zero query stays zero (and ties every
    centroid, so it lands in cluster 0)."""
    x = _gmm(30, 8, 3, 5)
    x[7] = 0
    xs, nrm = orc.prepare(x, orc.SPHERE)
    np.testing.assert_allclose(np.linalg.norm(xs, axis=1)[np.arange(30) != 7], 1.0, atol=1e-15)
    assert np.all(xs[7] == 0) and nrm[7] == 0
    c = xs[[0, 10, 20]].astype(np.float32)
    ids, _, _ = orc.assign(xs, c, orc.SPHERE)
    assert ids[7] == 0


def test_sphere_scale_invariance(orc):
    """§3.1: the ranking of q.k over keys does not depend on ||q||, so query
    clusters must not either.  Power-of-two scalings keep q/||q|| bit-identical."""
    x = _gmm(400, 16, 6, 11)
    s = (2.0 ** np.random.default_rng(3).integers(-6, 7, 400)).astype(np.float32)
    a = orc.kmeans(orc.prepare(x, orc.SPHERE)[0], 6, 8, orc.SPHERE)
    b = orc.kmeans(orc.prepare(x * s[:, None], orc.SPHERE)[0], 6, 8, orc.SPHERE)
    assert np.array_equal(a.assign, b.assign)
    assert np.array_equal(a.cent, b.cent)


# ------------------------------------------------------------------- k-means
@pytest.mark.parametrize("mode", [0, 1])
def test_kmeans_objective_monotone(orc, mode):
    """Lloyd's algorithm never increases its objective (assign and update both
    minimise it); fp32 storage of centroids allows a relative 1e-6 slack."""
    x = _gmm(3000, 32, 12, 21, sigma=0.8)
    xs, _ = orc.prepare(x, mode)
    r = orc.kmeans(xs, 20, 10, mode, trace=True)
    tr = r.trace
    assert np.all(np.diff(tr) <= 1e-6 * np.abs(tr[:-1]) + 1e-9), tr


def test_kmeans_k1_closed_form(orc):
    """k = 1: the Euclidean centre is the mean; the spherical centre is the
    normalised sum of the unit vectors (textbook closed forms)."""
    x = _gmm(500, 12, 3, 8)
    r = orc.kmeans(x.astype(np.float64), 1, 3, orc.EUCLID)
    np.testing.assert_array_equal(r.cent[0], x.astype(np.float64).mean(0).astype(np.float32))
    xs, _ = orc.prepare(x, orc.SPHERE)
    r2 = orc.kmeans(xs, 1, 3, orc.SPHERE)
    u = x / np.linalg.norm(x.astype(np.float64), axis=1, keepdims=True)
    s = u.sum(0)
    np.testing.assert_allclose(r2.cent[0], (s / np.linalg.norm(s)).astype(np.float32), rtol=0, atol=1e-7)
    assert np.all(r.assign == 0) and r.count[0] == 500


def test_kmeans_separated_recovers_components(orc):
    """Well-separated components with one seed per component: k-means returns the
    component means (each centre = its component's sample mean)."""
    rng = np.random.default_rng(4)
    d, comps, per = 8, 5, 60
    mu = 20.0 * rng.standard_normal((comps, d))
    x = np.concatenate([mu[c] + 0.1 * rng.standard_normal((per, d)) for c in range(comps)]).astype(np.float32)
    r = orc.kmeans(x.astype(np.float64), comps, 5, orc.EUCLID)
    for c in range(comps):
        np.testing.assert_array_equal(r.assign[c * per:(c + 1) * per], c)
        np.testing.assert_allclose(r.cent[c], x[c * per:(c + 1) * per].astype(np.float64).mean(0), rtol=1e-6)


def test_update_empty_cluster_keeps_centroid(orc):
    x = _gmm(200, 4, 2, 9)
    c = np.array([x[0], x[100], [1e4, 1e4, 1e4, 1e4]], np.float32)
    ids, _, _ = orc.assign(x.astype(np.float64), c, orc.EUCLID)
    c2, cnt = orc.update(x.astype(np.float64), ids, c, orc.EUCLID)
    assert cnt[2] == 0 and np.array_equal(c2[2], c[2])


def test_cauchy_schwarz_bound(orc):
    """§3.2.1: |q.c(k) - q.k| <= ||q|| ||k - c(k)|| for every key and query."""
    k = _gmm(800, 16, 8, 2)
    q = _gmm(50, 16, 8, 3)
    r = orc.kmeans(k.astype(np.float64), 8, 6, orc.EUCLID)
    c = r.cent[r.assign].astype(np.float64)
    lhs = np.abs(q.astype(np.float64) @ (c - k).T)
    rhs = np.linalg.norm(q, axis=1)[:, None] * r.dist[None, :]
    assert np.all(lhs <= rhs * (1 + 1e-12) + 1e-12)
    np.testing.assert_allclose(r.dist, np.linalg.norm(k - c, axis=1), rtol=1e-12)


# -------------------------------------------------------------- Algorithm 1
def _four_groups():
    """Three tight groups of 100 (spread 0.5) and a far pair, in 2-D."""
    rng = np.random.default_rng(7)
    cen = [(0.0, 0.0), (10.0, 0.0), (0.0, 10.0)]
    pts = [np.array(c) + rng.uniform(-0.25, 0.25, (100, 2)) for c in cen]
    pts.append(np.array([[30.0, 25.0], [31.0, 25.0]]))
    return np.concatenate(pts).astype(np.float32)


def test_multistage_hand_trace(orc):
    """Algorithm 1 on a hand-built case (the Figure 5 idea): stage 0 (m0 = 3)
    finds the three groups (the far pair joins the group at (10,0), whose centre
    moves by < 0.6, so every group point stays within tau = 3); only the far pair
    is left in U; stage 1 uses m_1 = ceil(3*2/302) = 1 cluster, whose centre is
    the pair's midpoint (distance 0.5 < tau), so U empties: |C| = 4, F = False,
    two stages; the final reassignment gives counts 100/100/100/2."""
    x = _four_groups()
    r = orc.multistage(x.astype(np.float64), 3, 10, orc.TAU_ABS, 3.0, 50, orc.EUCLID)
    assert (r.nclusters, r.dense, r.nstages) == (4, 0, 2)
    np.testing.assert_array_equal(np.sort(r.count), [2, 100, 100, 100])
    for g in range(3):
        assert len(set(r.assign[100 * g:100 * (g + 1)].tolist())) == 1
    assert r.assign[300] == r.assign[301] == 3
    np.testing.assert_allclose(r.cent[3], [30.5, 25.0], atol=1e-6)


def test_multistage_nmax_sets_flag(orc):
    """Algorithm 1's N_max test: U is non-empty after stage 0 and |C| = 3 >= N_max = 3,
    so F is set and no further stage runs."""
    x = _four_groups()
    r = orc.multistage(x.astype(np.float64), 3, 10, orc.TAU_ABS, 3.0, 3, orc.EUCLID)
    assert (r.nclusters, r.dense, r.nstages) == (3, 1, 1)


def test_multistage_tau_zero_closed_form(orc):
    """tau = 0 removes nothing (d_i < 0 never holds), so each stage adds m0
    clusters until |C| >= N_max: ceil(N_max / m0) stages, F = True."""
    x = _gmm(500, 6, 5, 1)
    for m0, nmax in [(4, 10), (5, 5), (7, 30)]:
        r = orc.multistage(x.astype(np.float64), m0, 3, orc.TAU_ABS, 0.0, nmax, orc.EUCLID)
        st = -(-nmax // m0)
        assert (r.nstages, r.nclusters, r.dense) == (st, st * m0, 1)


def test_multistage_tau_inf_is_plain_kmeans(orc):
    """tau = +inf empties U after stage 0: one stage of k-means with m0 centres,
    F = False, and the final reassignment equals k-means' own final assignment."""
    x = _gmm(600, 8, 6, 2)
    for mode in (0, 1):
        xs, _ = orc.prepare(x, mode)
        r = orc.multistage(xs, 6, 5, orc.TAU_ABS, np.inf, 100, mode)
        k = orc.kmeans(xs, 6, 5, mode)
        assert (r.nclusters, r.dense, r.nstages) == (6, 0, 1)
        assert np.array_equal(r.assign, k.assign) and np.array_equal(r.cent, k.cent)


def test_multistage_terminates_and_partitions(orc):
    """Every stage adds >= 1 centre, so the loop ends; the final assignment
    covers every token and ids are < |C|; the capacity bound N_max + m0 holds."""
    x = _gmm(2000, 16, 30, 6, sigma=1.0)
    for rule, val in [(orc.TAU_MEAN_X, 1.0), (orc.TAU_MEDIAN_RADIUS_X, 0.5), (orc.TAU_ABS, 2.0)]:
        r = orc.multistage(x.astype(np.float64), 16, 4, rule, val, 120, orc.EUCLID)
        assert r.nclusters <= 120 + 16 and r.count.sum() == 2000
        assert r.assign.min() >= 0 and r.assign.max() < r.nclusters
        assert r.dense == (1 if r.nclusters >= 120 else 0) or r.dense == 0


def test_tau_mean_rule_matches_stage0(orc):
    """§4.1: tau = 1.5 x the mean token-to-centre distance of the first stage.
    Stage 0 is plain k-means with m0 centres, so tau must equal 1.5 x the mean
    of that run's distances, and rerunning with that tau as an absolute value
    must reproduce the result."""
    x = _gmm(1500, 16, 20, 8, sigma=0.7)
    xs = x.astype(np.float64)
    r = orc.multistage(xs, 10, 5, orc.TAU_MEAN_X, 1.5, 200, orc.EUCLID)
    k0 = orc.kmeans(xs, 10, 5, orc.EUCLID)
    assert r.tau == pytest.approx(1.5 * k0.dist.mean(), rel=1e-12)
    r2 = orc.multistage(xs, 10, 5, orc.TAU_ABS, r.tau, 200, orc.EUCLID)
    assert np.array_equal(r.assign, r2.assign) and r.nclusters == r2.nclusters


def test_tau_median_radius_rule(orc):
    x = _gmm(1500, 16, 20, 8, sigma=0.7)
    xs = x.astype(np.float64)
    r = orc.multistage(xs, 10, 5, orc.TAU_MEDIAN_RADIUS_X, 0.5, 200, orc.EUCLID)
    k0 = orc.kmeans(xs, 10, 5, orc.EUCLID)
    radii = sorted(k0.dist[k0.assign == j].mean() for j in range(10) if np.any(k0.assign == j))
    assert r.tau == pytest.approx(0.5 * radii[(len(radii) - 1) // 2], rel=1e-12)


# ---------------------------------------------------------------- selection
def _sel(orc, t, counts, top_p, rbar=2.0, qcount=1):
    """One query cluster with centroid e_0, mean norm rbar, d = 4 (so
    s_b = rbar * t_b / 2), key centroids t_b * e_0."""
    d = 4
    qc = np.zeros((1, d), np.float32)
    qc[0, 0] = 1
    kc = np.zeros((len(t), d), np.float32)
    kc[:, 0] = t
    s, c = orc.select(qc, np.array([rbar], np.float32), np.array([qcount], np.int32), kc,
                      np.array(counts, np.int32), top_p)
    return sorted(s[0, :c[0]].tolist())


def test_select_hand_example_sizes(orc):
    """Equal scores: p_b is the size share n_b / sum n = [.1,.2,.3,.4]."""
    assert _sel(orc, [0, 0, 0, 0], [1, 2, 3, 4], 0.5) == [2, 3]
    assert _sel(orc, [0, 0, 0, 0], [1, 2, 3, 4], 0.4) == [3]
    assert _sel(orc, [0, 0, 0, 0], [1, 2, 3, 4], 0.71) == [1, 2, 3]
    assert _sel(orc, [0, 0, 0, 0], [1, 2, 3, 4], 1.0) == [0, 1, 2, 3]


def test_select_hand_example_scores(orc):
    """Scores s_b = t_b (rbar = 2, sqrt(d) = 2), unit sizes:
    p = e^{t-2} / sum = [0.0900, 0.2447, 0.6652]."""
    e = [math.exp(t - 2) for t in (0, 1, 2)]
    p = [v / sum(e) for v in e]
    assert abs(p[2] - 0.6652) < 1e-4
    assert _sel(orc, [0, 1, 2], [1, 1, 1], 0.6) == [2]
    assert _sel(orc, [0, 1, 2], [1, 1, 1], 0.7) == [1, 2]
    assert _sel(orc, [0, 1, 2], [1, 1, 1], 0.9) == [1, 2]
    assert _sel(orc, [0, 1, 2], [1, 1, 1], 0.95) == [0, 1, 2]
    # doubling rbar doubles the temperature-free scores: p = e^{2t-4}/sum
    assert _sel(orc, [0, 1, 2], [1, 1, 1], 0.85, rbar=4.0) == [2]


def test_select_ties_lower_index_first(orc):
    """Equal p: the lower cluster id is visited first."""
    assert _sel(orc, [0, 0, 0], [2, 2, 1], 0.3) == [0]
    assert _sel(orc, [0, 0, 0], [1, 2, 2], 0.3) == [1]


def test_select_empty_clusters(orc):
    assert _sel(orc, [5, 0, 0], [0, 1, 1], 1.0) == [1, 2]
    assert _sel(orc, [0, 0], [1, 1], 1.0, qcount=0) == []


def test_select_invariants(orc):
    """top_p = 1 keeps every non-empty key cluster; the kept set grows with
    top_p; one key cluster is always kept."""
    rng = np.random.default_rng(0)
    kq, kk, d = 20, 60, 16
    qc = rng.standard_normal((kq, d)).astype(np.float32)
    qc /= np.linalg.norm(qc, axis=1, keepdims=True)
    kc = rng.standard_normal((kk, d)).astype(np.float32)
    qn = rng.uniform(1, 8, kq).astype(np.float32)
    qcnt = rng.integers(0, 30, kq).astype(np.int32)
    kcnt = rng.integers(0, 30, kk).astype(np.int32)
    prev = None
    for p in [0.1, 0.5, 0.8, 0.9, 0.99, 1.0]:
        s, c = orc.select(qc, qn, qcnt, kc, kcnt, p)
        sets = [set(s[a, :c[a]].tolist()) for a in range(kq)]
        for a in range(kq):
            assert all(kcnt[b] > 0 for b in sets[a])
            assert (len(sets[a]) == 0) == (qcnt[a] == 0)
            if prev is not None:
                assert prev[a] <= sets[a]
        prev = sets
    for a in range(kq):
        if qcnt[a]:
            assert prev[a] == {b for b in range(kk) if kcnt[b] > 0}
    s, c = orc.select(qc, qn, qcnt, kc[:1], np.array([5], np.int32), 0.5)
    assert all(c[a] == (1 if qcnt[a] else 0) for a in range(kq))


# ---------------------------------------------------------------- attention
def _np_attention(q, k, v):
    s = (q.astype(np.float64) @ k.astype(np.float64).T) / math.sqrt(q.shape[1])
    s -= s.max(1, keepdims=True)
    e = np.exp(s)
    return (e @ v.astype(np.float64)) / e.sum(1, keepdims=True)


def test_attention_select_all_is_dense(orc):
    """Algorithm 3: with every key cluster selected (or F set) the sparse
    attention equals dense softmax attention (textbook definition in numpy)."""
    rng = np.random.default_rng(1)
    n, d = 300, 32
    q, k, v = (rng.standard_normal((n, d)).astype(np.float32) for _ in range(3))
    ref = _np_attention(q, k, v)
    rows = np.arange(n)
    out = orc.attention_rows(q, k, v, None, None, 0, None, None, 1, rows)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    qa = rng.integers(0, 5, n)
    ka = rng.integers(0, 7, n)
    sel = np.tile(np.arange(7, dtype=np.int32), (5, 1))
    out2 = orc.attention_rows(q, k, v, qa, ka, 7, sel, np.full(5, 7, np.int32), 0, rows)
    np.testing.assert_allclose(out2, ref, rtol=1e-12, atol=1e-12)


def test_attention_subset_is_attention_over_subset(orc):
    """Algorithm 3's gather and attention: attention over K* = K[Index], V* = V[Index]."""
    rng = np.random.default_rng(2)
    n, d, kq, kk = 400, 16, 6, 9
    q, k, v = (rng.standard_normal((n, d)).astype(np.float32) for _ in range(3))
    qa = rng.integers(0, kq, n).astype(np.int32)
    ka = rng.integers(0, kk, n).astype(np.int32)
    sel = np.full((kq, kk), -1, np.int32)
    cnt = np.zeros(kq, np.int32)
    for a in range(kq):
        s = np.sort(rng.choice(kk, rng.integers(1, kk + 1), replace=False))
        sel[a, :len(s)] = s
        cnt[a] = len(s)
    rows = np.arange(0, n, 7)
    out = orc.attention_rows(q, k, v, qa, ka, kk, sel, cnt, 0, rows)
    for r, i in enumerate(rows):
        keys = np.isin(ka, sel[qa[i], :cnt[qa[i]]])
        np.testing.assert_allclose(out[r], _np_attention(q[i:i + 1], k[keys], v[keys])[0], rtol=1e-12,
                                   atol=1e-12)


def test_attention_single_key(orc):
    rng = np.random.default_rng(3)
    n, d = 50, 8
    q, k, v = (rng.standard_normal((n, d)).astype(np.float32) for _ in range(3))
    ka = np.arange(n, dtype=np.int32)
    qa = np.zeros(n, np.int32)
    sel = np.array([[17]], np.int32)
    out = orc.attention_rows(q, k, v, qa, ka, n, sel, np.array([1], np.int32), 0, np.arange(n))
    np.testing.assert_array_equal(out, np.tile(v[17].astype(np.float64), (n, 1)))


# --------------------------------------------------------------------- sort
def test_cluster_sort_is_stable_argsort(orc):
    rng = np.random.default_rng(5)
    ids = rng.integers(0, 37, 5000).astype(np.int32)
    ids[ids == 11] = 12  # an empty cluster
    perm, off = orc.cluster_sort(ids, 37)
    np.testing.assert_array_equal(perm, np.argsort(ids, kind="stable"))
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(ids, minlength=37))]))


# --------------------------------------------------------- composed forward
def test_forward_head_top_p_one_is_dense(orc):
    """Algorithm 3 end to end: top_p = 1 selects every non-empty key cluster,
    so each row's output is dense attention."""
    w = W.small(W.WORKLOADS["gmm16-n2048-d64-f32"], 512)
    h = W.head_inputs(w, 0)
    spec = orc.HeadSpec(kq=8, kk=16, iters=4, top_p=1.0)
    r = orc.forward_head(h.q, h.k, h.v, spec, rows=np.arange(0, 512, 5))
    np.testing.assert_allclose(r.out_rows, _np_attention(h.q[::5], h.k, h.v), rtol=1e-10, atol=1e-12)
    assert r.dense == 0


def test_forward_head_dense_flag(orc):
    """Algorithm 3's dense branch: F set (N_max reached) -> full attention."""
    w = W.small(W.WORKLOADS["gmm16-n2048-d64-f32"], 400)
    h = W.head_inputs(w, 0)
    spec = orc.HeadSpec(kq=8, kk=16, iters=3, top_p=0.5, adaptive_k=True, tau_rule=orc.TAU_ABS,
                        tau_value=0.0, nmax_k=16)
    r = orc.forward_head(h.q, h.k, h.v, spec, rows=np.arange(0, 400, 9))
    assert r.dense == 1
    np.testing.assert_allclose(r.out_rows, _np_attention(h.q[::9], h.k, h.v), rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------
# Quest bounds (§3.2.3 eq. (1)) and the argtopk cut (Algorithm 3)
# --------------------------------------------------------------------------
def test_key_bounds_are_member_extremes(orc):
    """Per cluster and dimension: the largest / smallest member value (numpy's
    max/min over the members), zeros for an empty cluster."""
    rng = np.random.default_rng(21)
    n, d, kk = 300, 16, 9
    k = rng.standard_normal((n, d)).astype(np.float32)
    ids = rng.integers(0, kk - 1, size=n).astype(np.int32)  # cluster kk-1 stays empty
    kmax, kmin = orc.key_bounds(k, ids, kk)
    for b in range(kk):
        mem = k[ids == b]
        if len(mem):
            np.testing.assert_array_equal(kmax[b], mem.max(0))
            np.testing.assert_array_equal(kmin[b], mem.min(0))
        else:
            assert not kmax[b].any() and not kmin[b].any()


def test_quest_score_bounds_every_member_and_is_tight(orc):
    """Eq. (1) is an upper bound of qbar.k over the keys k of a page, attained
    when a page holds one key (or when every key sits at the page's corner)."""
    rng = np.random.default_rng(22)
    d, kq, kk = 32, 5, 7
    q_cent = rng.standard_normal((kq, d)).astype(np.float32)
    rbar = rng.uniform(0.5, 2.0, kq).astype(np.float32)
    pages = [rng.standard_normal((int(rng.integers(1, 9)), d)).astype(np.float32) for _ in range(kk)]
    pages[0] = pages[0][:1]  # a one-key page
    kmax = np.stack([p.max(0) for p in pages])
    kmin = np.stack([p.min(0) for p in pages])
    s = orc.scores(q_cent, rbar, score_mode=orc.SCORE_QUEST, k_max=kmax, k_min=kmin) * np.sqrt(d)
    for a in range(kq):
        qbar = rbar[a].astype(np.float64) * q_cent[a].astype(np.float64)
        for b in range(kk):
            dots = pages[b].astype(np.float64) @ qbar
            assert s[a, b] >= dots.max() - 1e-9 * (1 + abs(dots.max()))
        one = pages[0][0].astype(np.float64) @ qbar
        assert s[a, 0] == pytest.approx(one, rel=1e-12, abs=1e-12)
    # the corner key (per-dimension choice of max or min by the sign of qbar)
    # attains the bound exactly
    qbar = rbar[0].astype(np.float64) * q_cent[0].astype(np.float64)
    corner = np.where(qbar >= 0, kmax[3], kmin[3]).astype(np.float64)
    assert s[0, 3] == pytest.approx(corner @ qbar, rel=1e-12)


def test_quest_score_of_single_key_pages_is_the_centroid_score(orc):
    """With one key per page (max = min = the key = its centroid) the Quest
    bound is the centroid dot product, so both scores pick the same top-k."""
    rng = np.random.default_rng(23)
    d, kq, kk = 24, 6, 40
    q_cent = rng.standard_normal((kq, d)).astype(np.float32)
    rbar = rng.uniform(0.5, 2.0, kq).astype(np.float32)
    c = rng.standard_normal((kk, d)).astype(np.float32)
    s0 = orc.scores(q_cent, rbar, k_cent=c)
    s1 = orc.scores(q_cent, rbar, k_cent=c, score_mode=orc.SCORE_QUEST, k_max=c, k_min=c)
    np.testing.assert_allclose(s1, s0, rtol=1e-12, atol=1e-12)
    qc, kc = np.ones(kq, np.int32), np.ones(kk, np.int32)
    a0, n0 = orc.select2(q_cent, rbar, qc, c, kc, top_k=7)
    a1, n1 = orc.select2(q_cent, rbar, qc, c, kc, top_k=7, score_mode=orc.SCORE_QUEST, k_max=c, k_min=c)
    np.testing.assert_array_equal(n0, 7)
    np.testing.assert_array_equal(a0[:, :7], a1[:, :7])


def test_topk_hand_example(orc):
    """argtopk by score, ties to the lower cluster id, empty clusters never
    kept, k larger than the non-empty count keeps them all; the size weights
    of the top-p rule play no part."""
    mu = np.array([[1.0, 0.0]], np.float32)
    rbar = np.array([np.sqrt(2.0)], np.float32)  # s_b = c_b[0] exactly
    c = np.array([[3, 0], [1, 0], [2, 0], [2, 0], [9, 0]], np.float32)
    kc = np.array([1, 100, 5, 5, 0], np.int32)   # cluster 4 (best score) is empty
    qc = np.array([3], np.int32)
    s = orc.scores(mu, rbar, k_cent=c)
    np.testing.assert_allclose(s[0], [3, 1, 2, 2, 9], rtol=1e-6)
    sel, cnt = orc.select2(mu, rbar, qc, c, kc, top_k=2)
    assert cnt[0] == 2 and list(sel[0, :2]) == [0, 2]
    sel, cnt = orc.select2(mu, rbar, qc, c, kc, top_k=3)
    assert cnt[0] == 3 and list(sel[0, :3]) == [0, 2, 3]
    sel, cnt = orc.select2(mu, rbar, qc, c, kc, top_k=50)
    assert cnt[0] == 4 and list(sel[0, :4]) == [0, 1, 2, 3]


def test_quest_selects_a_page_with_an_aligned_outlier(orc):
    """A page whose centroid points away from the query but holds one key
    aligned with it: the centroid score ranks it last, the Quest bound first."""
    d = 4
    mu = np.array([[1.0, 0.0, 0.0, 0.0]], np.float32)
    rbar = np.array([1.0], np.float32)
    far = np.array([[-1, 0, 0, 0], [-1, 0, 0, 0], [-1, 0, 0, 0], [5, 0, 0, 0]], np.float32)  # mean (0.5, 0, 0, 0)
    near = np.array([[1, 0, 0, 0], [1, 0, 0, 0]], np.float32)
    pages = [far, near]
    c = np.stack([p.mean(0) for p in pages]).astype(np.float32)
    kmax = np.stack([p.max(0) for p in pages])
    kmin = np.stack([p.min(0) for p in pages])
    kc = np.array([4, 2], np.int32)
    qc = np.array([1], np.int32)
    sel0, _ = orc.select2(mu, rbar, qc, c, kc, top_k=1)
    sel1, _ = orc.select2(mu, rbar, qc, c, kc, top_k=1, score_mode=orc.SCORE_QUEST, k_max=kmax, k_min=kmin)
    assert sel0[0, 0] == 1 and sel1[0, 0] == 0


# --------------------------------------------------------------------------
# Multi-step driver (§3.2.2 "Efficient initialization", §4.1): counts and F of
# step 0 kept, k-means seeded with the previous step's centres
# --------------------------------------------------------------------------
def _drifting_gmm(steps, comps=6, per=40, d=16, drift=0.05, sep=12.0, seed=11):
    """Per step (q, k, v) of `comps` well-separated components (q and k share
    the component of a token); every step moves every point by drift * N(0, I).
    Returns the steps and the true component of each token."""
    rng = np.random.default_rng(seed)
    lab = np.repeat(np.arange(comps), per)
    mq = sep * rng.standard_normal((comps, d))
    mk = sep * rng.standard_normal((comps, d))
    q = mq[lab] + 0.2 * rng.standard_normal((len(lab), d))
    k = mk[lab] + 0.2 * rng.standard_normal((len(lab), d))
    v = rng.standard_normal((len(lab), d))
    out = []
    for _ in range(steps):
        out.append((q.astype(np.float32), k.astype(np.float32), v.astype(np.float32)))
        q = q + drift * rng.standard_normal(q.shape)
        k = k + drift * rng.standard_normal(k.shape)
        v = v + drift * rng.standard_normal(v.shape)
    return out, lab


def _same_partition(a, b):
    """a and b split the tokens into the same groups (labels may differ)."""
    pairs = set(zip(a.tolist(), b.tolist()))
    return len(pairs) == len(set(a.tolist())) == len(set(b.tolist()))


def test_steps_track_drifting_components(orc):
    """Every step re-clusters its own inputs: the assignments stay the true
    components while the points drift, and each key centre is the sample mean
    of its component at that step (closed form), not step 0's centre."""
    steps, lab = _drifting_gmm(4, drift=0.3)
    spec = orc.HeadSpec(kq=6, kk=6, iters=5, top_p=0.9)
    res = orc.forward_steps(steps, spec, rows=np.arange(0, len(lab), 7))
    for s, r in enumerate(res):
        assert _same_partition(r.q.assign, lab) and _same_partition(r.k.assign, lab), f"step {s}"
        k = steps[s][1].astype(np.float64)
        for c in range(6):
            m = r.k.assign == c
            np.testing.assert_allclose(r.k.cent[c], k[m].mean(0), rtol=1e-6, atol=1e-6)
    assert not np.array_equal(res[0].k.cent, res[3].k.cent)


def test_steps_fixed_point_without_drift(orc):
    """No drift and converged centres: every later step reproduces step 0
    exactly (assignments, centres, selection, output rows)."""
    steps, lab = _drifting_gmm(1)
    steps = steps * 3
    spec = orc.HeadSpec(kq=6, kk=6, iters=6, top_p=0.8)
    res = orc.forward_steps(steps, spec, rows=np.arange(0, len(lab), 5))
    for r in res[1:]:
        np.testing.assert_array_equal(r.q.assign, res[0].q.assign)
        np.testing.assert_array_equal(r.k.assign, res[0].k.assign)
        np.testing.assert_array_equal(r.q.cent, res[0].q.cent)
        np.testing.assert_array_equal(r.k.cent, res[0].k.cent)
        np.testing.assert_array_equal(r.sel_cnt, res[0].sel_cnt)
        np.testing.assert_array_equal(r.out_rows, res[0].out_rows)


def test_steps_keep_step0_counts(orc):
    """Later steps keep the counts Algorithm 1 chose at step 0, even where
    Algorithm 1 on that step's inputs would choose another count."""
    steps, lab = _drifting_gmm(3, comps=4, per=50, drift=0.0)
    # step 2: a fifth, far-away group appears among the tokens
    q2, k2, v2 = (a.copy() for a in steps[2])
    far = np.arange(0, len(lab), 4)
    k2[far] += 60.0
    q2[far] = -q2[far]
    steps[2] = (q2, k2, v2)
    spec = orc.HeadSpec(kq=4, kk=4, iters=4, top_p=0.9, adaptive_k=True, tau_rule=orc.TAU_ABS, tau_value=8.0,
                        nmax_k=64)
    res = orc.forward_steps(steps, spec, rows=np.arange(0, len(lab), 9))
    xs2, _ = orc.prepare(k2, orc.EUCLID)
    alone = orc.multistage(xs2, spec.kk, spec.iters, spec.tau_rule, spec.tau_value, spec.nmax_k, orc.EUCLID)
    assert alone.nclusters != res[0].k.nclusters
    assert [r.k.nclusters for r in res] == [res[0].k.nclusters] * 3
    assert all(r.dense == res[0].dense for r in res)


def test_steps_keep_dense_flag(orc):
    """F set at step 0 (N_max reached) keeps every later step dense: the rows
    are exact attention over all keys."""
    w = W.small(W.WORKLOADS["gmm16-n2048-d64-f32"], 300)
    steps = [(W.step_inputs(w, 0, s, drift=0.05).q, W.step_inputs(w, 0, s, drift=0.05).k,
              W.step_inputs(w, 0, s, drift=0.05).v) for s in range(3)]
    spec = orc.HeadSpec(kq=8, kk=16, iters=3, top_p=0.5, adaptive_k=True, tau_rule=orc.TAU_ABS,
                        tau_value=0.0, nmax_k=16)
    rows = np.arange(0, 300, 7)
    res = orc.forward_steps(steps, spec, rows=rows)
    for (q, k, v), r in zip(steps, res):
        assert r.dense == 1
        np.testing.assert_allclose(r.out_rows, _np_attention(q[rows], k, v), rtol=1e-10, atol=1e-12)


def test_step_inputs_drift(orc):
    """step_inputs: step 0 is head_inputs; step s differs from step s - 1 by
    about drift * N(0, 1) per element (before bf16 rounding)."""
    w = W.small(W.WORKLOADS["gmm16-n2048-d64-f32"], 256)
    h0 = W.head_inputs(w, 0)
    s0, s1, s2 = (W.step_inputs(w, 0, s, drift=0.1) for s in range(3))
    np.testing.assert_array_equal(s0.q, h0.q)
    d1, d2 = (s1.k - s0.k), (s2.k - s1.k)
    assert abs(d1.std() - 0.1) < 0.01 and abs(d2.std() - 0.1) < 0.01
    assert abs(np.corrcoef(d1.ravel(), d2.ravel())[0, 1]) < 0.05


# --------------------------------------------------------------------------
# Text keys always attended (a dense strip; a variant, not in the pages)
# --------------------------------------------------------------------------
def _with_text(n_video=360, n_text=24, d=16, seed=21):
    rng = np.random.default_rng(seed)
    steps, lab = _drifting_gmm(1, comps=6, per=n_video // 6, d=d, seed=seed)
    q, k, v = steps[0]
    tq, tk, tv = (rng.standard_normal((n_text, d)).astype(np.float32) for _ in range(3))
    return np.concatenate([q, tq]), np.concatenate([k, tk]), np.concatenate([v, tv]), n_text


def test_text_keys_in_every_key_set(orc):
    """Every query attends to the text keys plus the members of its cluster's
    selected video key clusters: the rows equal exact attention over that set."""
    q, k, v, T = _with_text()
    n = q.shape[0]
    spec = orc.HeadSpec(kq=6, kk=6, iters=5, top_p=0.3, text_keys=T)
    rows = np.arange(0, n, 7).astype(np.int32)
    r = orc.forward_head(q, k, v, spec, rows=rows)
    assert r.dense == 0
    nv = r.k.nclusters
    for i, row in enumerate(rows):
        a = r.q.assign[row]
        chosen = set(r.sel_idx[a, :r.sel_cnt[a]].tolist())
        assert nv in chosen, "the text group is always selected"
        keys = np.concatenate([np.nonzero(np.isin(r.k.assign, sorted(chosen - {nv})))[0], np.arange(n - T, n)])
        np.testing.assert_allclose(r.out_rows[i], _np_attention(q[row:row + 1], k[keys], v[keys])[0],
                                   rtol=1e-10, atol=1e-12)


def test_text_keys_not_clustered(orc):
    """The video keys are clustered exactly as on their own; the text keys get
    the extra group id."""
    q, k, v, T = _with_text()
    spec = orc.HeadSpec(kq=6, kk=6, iters=5, top_p=0.9, text_keys=T)
    r = orc.forward_head(q, k, v, spec, rows=np.arange(0, 10, dtype=np.int32))
    xs, _ = orc.prepare(k[:-T], orc.EUCLID)
    alone = orc.kmeans(xs, 6, 5, orc.EUCLID)
    np.testing.assert_array_equal(r.k.assign, alone.assign)
    np.testing.assert_array_equal(r.extra["k_assign"][-T:], 6)


def test_text_keys_zero_is_unchanged(orc):
    """text_keys = 0 gives exactly Algorithm 3 without the strip."""
    q, k, v, T = _with_text()
    rows = np.arange(0, q.shape[0], 11).astype(np.int32)
    a = orc.forward_head(q, k, v, orc.HeadSpec(kq=6, kk=6, iters=5, top_p=0.5), rows=rows)
    b = orc.forward_head(q, k, v, orc.HeadSpec(kq=6, kk=6, iters=5, top_p=0.5, text_keys=0), rows=rows)
    np.testing.assert_array_equal(a.out_rows, b.out_rows)
    np.testing.assert_array_equal(a.sel_cnt, b.sel_cnt)


def test_steps_zero_rounds_keep_the_previous_centres(orc):
    """With zero k-means rounds a later step's centres are exactly its seeds,
    the previous step's centres (§3.2.2 "Efficient initialization"), not rows
    of its own inputs."""
    steps, lab = _drifting_gmm(3, drift=0.3)
    spec = orc.HeadSpec(kq=6, kk=6, iters=0, top_p=0.9)
    res = orc.forward_steps(steps, spec, rows=np.arange(0, len(lab), 9))
    for r in res[1:]:
        np.testing.assert_array_equal(r.q.cent, res[0].q.cent)
        np.testing.assert_array_equal(r.k.cent, res[0].k.cent)
    # step 0's own seeds are rows of step 0 (strided), which the drift moves
    xq, _ = orc.prepare(steps[1][0], orc.SPHERE)
    assert not np.array_equal(res[1].q.cent, orc.init_centroids(xq, 6))


def test_text_group_skips_empty_query_clusters(orc):
    """An empty query cluster selects nothing, not even the text group: with
    four copies each of two query vectors and kq = 4, the strided seeds are
    a, a, b, b, every row goes to the lowest tied id, and clusters 1 and 3
    stay empty."""
    rng = np.random.default_rng(5)
    d, T = 8, 3
    a, b = rng.standard_normal((2, d)).astype(np.float32)
    q = np.stack([a] * 4 + [b] * 4 + [rng.standard_normal(d).astype(np.float32) for _ in range(T)])
    q[8:] = np.stack([a] * T)   # text-position queries also copy a
    k = rng.standard_normal((8 + T, d)).astype(np.float32)
    v = rng.standard_normal((8 + T, d)).astype(np.float32)
    spec = orc.HeadSpec(kq=4, kk=2, iters=3, top_p=0.5, text_keys=T)
    r = orc.forward_head(q, k, v, spec)
    assert list(r.q.count) == [7, 0, 4, 0]
    nv = r.k.nclusters
    assert r.sel_cnt[1] == 0 and r.sel_cnt[3] == 0
    for c in (0, 2):
        assert nv in r.sel_idx[c, :r.sel_cnt[c]].tolist()


@pytest.mark.parametrize("mode", ["euclid", "sphere"])
@pytest.mark.parametrize("rule, val", [("abs", 0.9), ("mean", 0.8), ("median", 0.8)])
def test_single_cluster_stages_are_complete_after_one_round(orc, mode, rule, val):
    """With m0 = 1 every stage of Algorithm 1 has one cluster.  Such a stage's
    k-means puts every row in cluster 0, so its first update gives the centre
    that every later round repeats: one round and ten give identical results
    (the fact the GPU path uses to run such stages for one round)."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((300, 3)) * np.array([1.0, 0.5, 0.25])).astype(np.float32)
    m = orc.EUCLID if mode == "euclid" else orc.SPHERE
    xs, _ = orc.prepare(x, m)
    r = {"abs": orc.TAU_ABS, "mean": orc.TAU_MEAN_X, "median": orc.TAU_MEDIAN_RADIUS_X}[rule]
    a = orc.multistage(xs, 1, 1, r, val, 60, m)
    b = orc.multistage(xs, 1, 10, r, val, 60, m)
    assert a.nstages > 5, "the case should run many stages"
    assert (a.nclusters, a.dense, a.nstages, a.tau) == (b.nclusters, b.dense, b.nstages, b.tau)
    np.testing.assert_array_equal(a.assign, b.assign)
    np.testing.assert_array_equal(a.count[:a.nclusters], b.count[:b.nclusters])
    np.testing.assert_array_equal(a.cent[:a.nclusters], b.cent[:b.nclusters])


# ------------------------------------------------------------ pair count
def test_pairs_hand_count(orc):
    """The pair count of §3.3 (each query of cluster a meets every key of each
    selected cluster b), counted by hand on an asymmetric case: 3 query clusters
    of 5, 0 and 2 queries, 4 key clusters of 3, 7, 0 and 11 keys; cluster 0
    selects {1, 3} (18 keys), the empty cluster 1 nothing, cluster 2 {0, 2}
    (3 keys).  5 * 18 + 0 + 2 * 3 = 96.  The sizes are unequal on the two
    sides, so a count that read one side's sizes for the other would differ."""
    q_count = np.array([5, 0, 2], np.int32)
    k_count = np.array([3, 7, 0, 11], np.int32)
    sel = np.full((3, 4), -1, np.int32)
    sel[0, :2] = [1, 3]
    sel[2, :2] = [0, 2]
    sel_cnt = np.array([2, 0, 2], np.int32)
    assert orc.pairs(q_count, k_count, sel, sel_cnt) == 96
    # a partial selection of a single cluster: 2 queries x 7 keys
    sel2 = np.full((3, 4), -1, np.int32)
    sel2[2, 0] = 1
    assert orc.pairs(q_count, k_count, sel2, np.array([0, 0, 1], np.int32)) == 14


def test_pairs_brute_force_over_tokens(orc):
    """Brute force over token pairs: count (i, j) with the key's cluster in the
    query's selected set, from random assignments with empty clusters and
    unequal query and key counts."""
    rng = np.random.default_rng(5)
    nq_tok, nk_tok, kq, kk = 57, 131, 6, 9
    qa = rng.integers(0, kq - 1, nq_tok)  # cluster kq-1 stays empty
    ka = rng.integers(1, kk, nk_tok)      # cluster 0 stays empty
    sel = np.full((kq, kk), -1, np.int32)
    sel_cnt = np.zeros(kq, np.int32)
    sets = []
    for a in range(kq):
        s = np.sort(rng.choice(kk, rng.integers(0, kk + 1), replace=False)).astype(np.int32)
        sel[a, :len(s)] = s
        sel_cnt[a] = len(s)
        sets.append(set(s.tolist()))
    brute = sum(1 for i in range(nq_tok) for j in range(nk_tok) if int(ka[j]) in sets[int(qa[i])])
    q_count = np.bincount(qa, minlength=kq).astype(np.int32)
    k_count = np.bincount(ka, minlength=kk).astype(np.int32)
    assert orc.pairs(q_count, k_count, sel, sel_cnt) == brute


# ------------------------------------------------- per-query selection (f2)
def _np_attention_row(q, k, v, allowed):
    s = (k[allowed].astype(np.float64) @ q.astype(np.float64)) / math.sqrt(q.shape[0])
    w = np.exp(s - s.max())
    return (w[:, None] * v[allowed].astype(np.float64)).sum(0) / w.sum()


def test_per_query_hand_example(orc):
    """Algorithm 3 selects along each row of S (one row per query): two queries
    of one query cluster that point at different key clusters each keep their
    own best cluster under argtopk with top_k = 1, and attend to its keys only;
    the per-cluster selection would give both the same cluster."""
    k = np.array([[3, 0], [2.5, 0.5], [0, 3], [0.5, 2.5]], np.float32)
    v = np.array([[1, 0], [2, 0], [0, 1], [0, 2]], np.float32)
    ka = np.array([0, 0, 1, 1], np.int32)
    cent = np.array([[2.75, 0.25], [0.25, 2.75]], np.float32)
    # one token count for queries and keys (rows 2 and 3 are not evaluated)
    q = np.array([[4, 0.1], [0.1, 4], [1, 1], [1, -1]], np.float32)
    sel, cnt = orc.select_per_query(q[:2], cent, np.array([2, 2], np.int32), top_k=1)
    assert cnt.tolist() == [1, 1] and sel[0, 0] == 0 and sel[1, 0] == 1
    out = orc.attend_per_query(q, k, v, ka, 2, sel, cnt, np.array([0, 1], np.int32))
    np.testing.assert_allclose(out[0], _np_attention_row(q[0], k, v, ka == 0), rtol=1e-12)
    np.testing.assert_allclose(out[1], _np_attention_row(q[1], k, v, ka == 1), rtol=1e-12)
    # as one cluster (representative = the mean of the two queries) both rows share one set
    qc = q[:2].mean(0, keepdims=True) / np.linalg.norm(q[:2].mean(0))
    sel_c, cnt_c = orc.select2(qc.astype(np.float32), np.array([np.linalg.norm(q[:2], axis=1).mean()], np.float32),
                               np.array([2], np.int32), cent, np.array([2, 2], np.int32), top_k=1)
    assert cnt_c.tolist() == [1]


def test_per_query_argtopk_matches_numpy_ranking(orc):
    """argtopk per row equals numpy's ranking of q . c_b (separated random data,
    no near-ties), empty clusters never kept; QUEST scores the Quest bound of
    the query itself."""
    rng = np.random.default_rng(12)
    d, kk, n = 16, 23, 40
    cent = rng.standard_normal((kk, d)).astype(np.float32)
    cnt = rng.integers(1, 9, kk).astype(np.int32)
    cnt[[4, 17]] = 0
    q = rng.standard_normal((n, d)).astype(np.float32)
    sel, c = orc.select_per_query(q, cent, cnt, top_k=5)
    s = q.astype(np.float64) @ cent.astype(np.float64).T
    s[:, cnt == 0] = -np.inf
    for i in range(n):
        want = np.sort(np.argsort(-s[i], kind="stable")[:5])
        assert c[i] == 5 and sel[i, :5].tolist() == want.tolist()
    kmax = cent + np.abs(rng.standard_normal((kk, d))).astype(np.float32)
    kmin = cent - np.abs(rng.standard_normal((kk, d))).astype(np.float32)
    sel, c = orc.select_per_query(q, cent, cnt, score_mode=orc.SCORE_QUEST, top_k=3, k_max=kmax, k_min=kmin)
    qd = q.astype(np.float64)[:, None, :]
    sq = np.maximum(qd * kmax[None].astype(np.float64), qd * kmin[None].astype(np.float64)).sum(2)
    sq[:, cnt == 0] = -np.inf
    for i in range(n):
        assert sel[i, :3].tolist() == np.sort(np.argsort(-sq[i], kind="stable")[:3]).tolist()


def test_per_query_top_p_matches_numpy_cut(orc):
    """The top-p cut per query row: weights n_b exp(q . c_b / sqrt(d)), shares
    in decreasing order (ties to the lower b), shortest prefix reaching top_p;
    the query is not normalised (its scale sets the softmax temperature)."""
    rng = np.random.default_rng(3)
    d, kk, n = 8, 12, 30
    cent = rng.standard_normal((kk, d)).astype(np.float32)
    cnt = rng.integers(1, 20, kk).astype(np.int32)
    q = (3.0 * rng.standard_normal((n, d))).astype(np.float32)
    for tp in (0.5, 0.9):
        sel, c = orc.select_per_query(q, cent, cnt, top_p=tp)
        s = (q.astype(np.float64) @ cent.astype(np.float64).T) / math.sqrt(d)
        for i in range(n):
            w = cnt * np.exp(s[i] - s[i].max())
            pr = w / w.sum()
            order = np.argsort(-pr, kind="stable")
            k = int(np.searchsorted(np.cumsum(pr[order]), tp) + 1)
            assert sel[i, :c[i]].tolist() == np.sort(order[:k]).tolist(), (tp, i)


def test_per_query_select_all_is_dense(orc):
    """top_k at least the number of key clusters: every row attends to every key."""
    rng = np.random.default_rng(8)
    n, d = 60, 8
    q, k, v = (rng.standard_normal((n, d)).astype(np.float32) for _ in range(3))
    spec = orc.HeadSpec(kq=4, kk=5, iters=3, top_k=5, per_query=True)
    r = orc.forward_head(q, k, v, spec, rows=np.arange(0, n, 7, dtype=np.int32))
    for i, row in enumerate(r.rows):
        np.testing.assert_allclose(r.out_rows[i], _np_attention_row(q[row], k, v, np.ones(n, bool)), rtol=1e-10)


def test_per_query_forward_rows_use_their_own_sets(orc):
    """forward_head with per-query argtopk (top_k = 2): each evaluated row
    attends exactly to the keys of the two key clusters whose centroids score
    highest against the row itself (numpy ranking of q . c over the oracle's
    key clustering), which differs from its query cluster's set on some rows."""
    w = W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 600, heads=1, seed=4, kq=3, kk=9, outlier_frac=0.0)
    x = W.head_inputs(w, 0)
    spec = orc.HeadSpec(kq=3, kk=9, iters=4, top_k=2, per_query=True)
    rows = np.arange(0, 600, 11, dtype=np.int32)
    r = orc.forward_head(x.q, x.k, x.v, spec, rows=rows)
    s = x.q[rows].astype(np.float64) @ r.k.cent.astype(np.float64).T
    s[:, np.asarray(r.k.count) == 0] = -np.inf
    differs = 0
    for i, row in enumerate(rows):
        top = np.argsort(-s[i], kind="stable")[:2]
        allowed = np.isin(r.extra["k_assign"], top)
        np.testing.assert_allclose(r.out_rows[i], _np_attention_row(x.q[row], x.k, x.v, allowed), rtol=1e-9, atol=1e-12)
        a = int(r.q.assign[row])
        differs += set(top.tolist()) != set(r.sel_idx[a, :r.sel_cnt[a]].tolist())
    assert differs > 0, "the per-query sets should differ from the per-cluster ones somewhere"
