"""CPU oracle for AdaCluster clustered sparse attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
library never calls it, and it shares no code with the CUDA path.

It wraps ``adacluster_oracle.c`` (plain C, fp64 arithmetic) through ctypes and
composes Algorithm 3 of "AdaCluster: Adaptive Query-Key Clustering for Sparse
Attention in Video Generation" (§3.3) from its steps:

  1. A_q, C_q <- KMeans(Normalize(Q))              (§3.1; or Algorithm 1 on Q)
  2. A_k, C_k, F <- MultiStageClustering(K, tau, N_max)  (§3.2.2, Algorithm 1;
     or plain Euclidean k-means with a fixed count, §3.2.1)
  3. F set -> dense attention; else select critical key clusters per query
     cluster and attend over their keys only (Algorithm 3, after the clustering).

Parity unpinned: the selection's score/weight reading (centroid-centroid score
scaled by the cluster's mean query norm, weighted by key-cluster size, top-p
cut) is not fixed by the paper; it is pinned only by invariants and a
hand-derived example.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "adacluster_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

EUCLID, SPHERE = 0, 1
TAU_ABS, TAU_MEAN_X, TAU_MEDIAN_RADIUS_X = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None
_P = ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.orc_prepare.argtypes = [i32, i64, i32, _P, _P, _P]
        lib.orc_assign.argtypes = [i32, i64, _P, i32, _P, i32, _P, ctypes.c_int32, _P, _P]
        lib.orc_assign.restype = dbl
        lib.orc_update.argtypes = [i32, i64, _P, i32, _P, _P, i32, _P, _P]
        lib.orc_init.argtypes = [i64, _P, i32, _P, i32, _P]
        lib.orc_kmeans.argtypes = [i32, i64, _P, i32, _P, i32, i32, _P, _P, _P, _P, _P]
        lib.orc_multistage.argtypes = [i32, i64, i32, _P, i32, i32, i32, dbl, i32, i32, _P, _P, _P,
                                       _P, _P, _P, _P, _P]
        lib.orc_multistage.restype = i32
        lib.orc_cluster_mean_norm.argtypes = [i64, _P, _P, i32, _P]
        lib.orc_select.argtypes = [i32, i32, _P, _P, _P, i32, _P, _P, dbl, i32, _P, _P]
        lib.orc_select2.argtypes = [i32, i32, _P, _P, _P, i32, _P, _P, _P, _P, i32, i32, dbl, i32, _P, _P]
        lib.orc_key_bounds.argtypes = [i64, i32, _P, _P, i32, _P, _P]
        lib.orc_scores.argtypes = [i32, i32, i32, _P, _P, i32, _P, _P, _P, _P]
        lib.orc_cluster_sort.argtypes = [i64, _P, i32, _P, _P]
        lib.orc_attention_rows.argtypes = [i64, i32, _P, _P, _P, _P, _P, i32, _P, _P, i32, i32, i64,
                                           _P, _P]
        lib.orc_pairs.argtypes = [i32, _P, _P, _P, _P, i32]
        lib.orc_pairs.restype = ctypes.c_int64
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def _i32(x):
    return np.ascontiguousarray(x, dtype=np.int32)


# --------------------------------------------------------------------------
# single steps
# --------------------------------------------------------------------------
def prepare(x, mode):
    """Working vectors in double (x itself, or x/||x|| for SPHERE) and ||x||."""
    x = _f32(x)
    n, d = x.shape
    xs = np.empty((n, d), np.float64)
    nrm = np.empty(n, np.float64)
    _load().orc_prepare(mode, n, d, _p(x), _p(xs), _p(nrm))
    return xs, nrm


def assign(xs, cent, mode, rows=None, id_base=0):
    """Closest centroid per row (ties -> lowest id); returns (ids, dist, objective)."""
    xs = np.ascontiguousarray(xs, np.float64)
    cent = _f32(cent)
    n, d = xs.shape
    rows_a = None if rows is None else _i32(rows)
    nr = n if rows is None else len(rows_a)
    ids = np.empty(nr, np.int32)
    dist = np.empty(nr, np.float64)
    obj = _load().orc_assign(mode, nr, _p(rows_a), d, _p(xs), cent.shape[0], _p(cent), id_base,
                             _p(ids), _p(dist))
    return ids, dist, obj


def update(xs, ids, cent, mode, rows=None):
    """One centroid update from local ids; returns (new centroids fp32, counts)."""
    xs = np.ascontiguousarray(xs, np.float64)
    c = _f32(cent).copy()
    ids = _i32(ids)
    rows_a = None if rows is None else _i32(rows)
    nr = len(ids)
    k, d = c.shape
    cnt = np.empty(k, np.int32)
    _load().orc_update(mode, nr, _p(rows_a), d, _p(xs), _p(ids), k, _p(c), _p(cnt))
    return c, cnt


def init_centroids(xs, k, rows=None):
    xs = np.ascontiguousarray(xs, np.float64)
    n, d = xs.shape
    rows_a = None if rows is None else _i32(rows)
    nr = n if rows is None else len(rows_a)
    c = np.empty((k, d), np.float32)
    _load().orc_init(nr, _p(rows_a), d, _p(xs), k, _p(c))
    return c


def kmeans(xs, k, iters, mode, init=None, trace=False):
    """Lloyd's k-means: iters x (assign, update) then a final assign."""
    xs = np.ascontiguousarray(xs, np.float64)
    n, d = xs.shape
    cent = init_centroids(xs, k) if init is None else _f32(init).copy()
    ids = np.empty(n, np.int32)
    cnt = np.empty(k, np.int32)
    dist = np.empty(n, np.float64)
    tr = np.empty(2 * iters + 1, np.float64) if trace else None
    _load().orc_kmeans(mode, n, None, d, _p(xs), k, iters, _p(cent), _p(ids), _p(cnt), _p(dist), _p(tr))
    return KMeansResult(cent, ids, cnt, dist, k, 0, 1, float("nan"), tr)


@dataclass
class KMeansResult:
    cent: np.ndarray
    assign: np.ndarray
    count: np.ndarray
    dist: np.ndarray
    nclusters: int
    dense: int
    nstages: int
    tau: float
    trace: np.ndarray | None = None


def multistage(xs, m0, iters, tau_rule, tau_value, nmax, mode):
    """Algorithm 1 (MultiStageClustering) on the working vectors xs."""
    xs = np.ascontiguousarray(xs, np.float64)
    n, d = xs.shape
    cap = nmax + m0
    cent = np.zeros((cap, d), np.float32)
    ids = np.empty(n, np.int32)
    cnt = np.zeros(cap, np.int32)
    dist = np.empty(n, np.float64)
    nc, fl, ns, tau = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_double()
    rc = _load().orc_multistage(mode, n, d, _p(xs), m0, iters, tau_rule, float(tau_value), nmax, cap,
                                _p(cent), _p(ids), _p(cnt), _p(dist), ctypes.byref(nc), ctypes.byref(fl),
                                ctypes.byref(ns), ctypes.byref(tau))
    if rc != 0:
        raise RuntimeError("multistage capacity overflow")
    k = nc.value
    return KMeansResult(cent[:k].copy(), ids, cnt[:k].copy(), dist, k, fl.value, ns.value, tau.value)


def cluster_mean_norm(norm, ids, k):
    out = np.empty(k, np.float32)
    _load().orc_cluster_mean_norm(len(ids), _p(np.ascontiguousarray(norm, np.float64)), _p(_i32(ids)), k,
                                  _p(out))
    return out


def select(q_cent, q_mean_norm, q_count, k_cent, k_count, top_p):
    """Per query cluster: selected key-cluster ids (ascending) as (sel_idx, sel_cnt)."""
    q_cent, k_cent = _f32(q_cent), _f32(k_cent)
    kq, d = q_cent.shape
    kk = k_cent.shape[0]
    sel = np.full((kq, max(kk, 1)), -1, np.int32)
    cnt = np.zeros(kq, np.int32)
    _load().orc_select(d, kq, _p(q_cent), _p(_f32(q_mean_norm)), _p(_i32(q_count)), kk, _p(k_cent),
                       _p(_i32(k_count)), float(top_p), sel.shape[1], _p(sel), _p(cnt))
    return sel, cnt


SCORE_CENTROID, SCORE_QUEST = 0, 1


def key_bounds(k, ids, kk):
    """Per key cluster and dimension: the largest and the smallest key value
    (Quest's page bounds, §3.2.3 eq. (1)); zeros for clusters without members."""
    k = _f32(k)
    n, d = k.shape
    kmax = np.empty((kk, d), np.float32)
    kmin = np.empty((kk, d), np.float32)
    _load().orc_key_bounds(n, d, _p(k), _p(_i32(ids)), kk, _p(kmax), _p(kmin))
    return kmax, kmin


def select2(q_cent, q_mean_norm, q_count, k_cent, k_count, top_p=0.9, score_mode=SCORE_CENTROID, top_k=0,
            k_max=None, k_min=None):
    """Selection with either score (centroid, or the Quest bound of eq. (1))
    and either cut (top-p, or Algorithm 3's argtopk when top_k > 0)."""
    q_cent, k_cent = _f32(q_cent), _f32(k_cent)
    kq, d = q_cent.shape
    kk = k_cent.shape[0]
    sel = np.full((kq, max(kk, 1)), -1, np.int32)
    cnt = np.zeros(kq, np.int32)
    km = _f32(k_max) if k_max is not None else None
    kn = _f32(k_min) if k_min is not None else None
    _load().orc_select2(d, kq, _p(q_cent), _p(_f32(q_mean_norm)), _p(_i32(q_count)), kk, _p(k_cent),
                        _p(_i32(k_count)), _p(km), _p(kn), int(score_mode), int(top_k), float(top_p), sel.shape[1],
                        _p(sel), _p(cnt))
    return sel, cnt


def select_per_query(q_rows, k_cent, k_count, top_p=0.9, score_mode=SCORE_CENTROID, top_k=0, k_max=None,
                     k_min=None):
    """Per-query selection (AdaCluster §3.3, Algorithm 3: the score matrix S has
    one row per query token and argtopk runs along each row).  Each query row is
    scored as its own one-member cluster: its representative is the query itself
    (centroid = q, mean norm 1), so s_ib = q_i . c_b / sqrt(d) (CENTROID) or the
    Quest bound of q_i against cluster b (QUEST), and the cut is select2's.
    Returns (sel_idx, sel_cnt) with one row per query row."""
    q_rows = _f32(q_rows)
    n = q_rows.shape[0]
    return select2(q_rows, np.ones(n, np.float32), np.ones(n, np.int32), k_cent, k_count, top_p, score_mode, top_k,
                   k_max, k_min)


def attend_per_query(q, k, v, k_assign, kk, sel_rows, cnt_rows, rows):
    """Attention of each listed query row over the keys of its own selected
    clusters (row i of sel_rows / cnt_rows belongs to rows[i])."""
    rows = _i32(rows)
    qa = np.zeros(q.shape[0], np.int32)
    qa[rows] = np.arange(len(rows), dtype=np.int32)
    return attention_rows(q, k, v, qa, k_assign, kk, sel_rows, cnt_rows, 0, rows)


def scores(q_cent, q_mean_norm, k_cent=None, score_mode=SCORE_CENTROID, k_max=None, k_min=None):
    """The selection score s_ab of every (query cluster, key cluster) pair."""
    q_cent = _f32(q_cent)
    kq, d = q_cent.shape
    kk = (k_cent if k_cent is not None else k_max).shape[0]
    out = np.empty((kq, kk), np.float64)
    _load().orc_scores(int(score_mode), d, kq, _p(q_cent), _p(_f32(q_mean_norm)), kk,
                       _p(_f32(k_cent)) if k_cent is not None else None,
                       _p(_f32(k_max)) if k_max is not None else None,
                       _p(_f32(k_min)) if k_min is not None else None, _p(out))
    return out


def cluster_sort(ids, k):
    ids = _i32(ids)
    perm = np.empty(len(ids), np.int32)
    off = np.empty(k + 1, np.int32)
    _load().orc_cluster_sort(len(ids), _p(ids), k, _p(perm), _p(off))
    return perm, off


def attention_rows(q, k, v, q_assign, k_assign, kk, sel_idx, sel_cnt, dense, rows):
    """Exact softmax attention (double) for the given query rows."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    n, d = q.shape
    rows = _i32(rows)
    out = np.empty((len(rows), d), np.float64)
    if sel_idx is None:
        sel_idx = np.zeros((1, 1), np.int32)
        sel_cnt = np.zeros(1, np.int32)
        q_assign = np.zeros(n, np.int32)
        k_assign = np.zeros(n, np.int32)
        kk = 1
        dense = 1
    sel_idx = _i32(sel_idx)
    _load().orc_attention_rows(n, d, _p(q), _p(k), _p(v), _p(_i32(q_assign)), _p(_i32(k_assign)), kk,
                               _p(sel_idx), _p(_i32(sel_cnt)), sel_idx.shape[1], int(dense), len(rows),
                               _p(rows), _p(out))
    return out


def pairs(q_count, k_count, sel_idx, sel_cnt):
    sel_idx = _i32(sel_idx)
    return int(_load().orc_pairs(len(q_count), _p(_i32(q_count)), _p(_i32(k_count)), _p(sel_idx),
                                 _p(_i32(sel_cnt)), sel_idx.shape[1]))


# --------------------------------------------------------------------------
# Algorithm 3, one head
# --------------------------------------------------------------------------
@dataclass
class HeadSpec:
    """Clustering parameters of one head (mirrors the library's ac_config)."""
    kq: int
    kk: int
    iters: int = 10
    top_p: float = 0.9
    adaptive_q: bool = False
    adaptive_k: bool = False
    tau_rule: int = TAU_ABS
    tau_value: float = 0.0
    nmax_q: int = 0
    nmax_k: int = 0
    score_mode: int = 0   # SCORE_CENTROID or SCORE_QUEST
    top_k: int = 0        # > 0: argtopk instead of top-p
    text_keys: int = 0    # > 0: the last text_keys keys are always attended, not clustered
    per_query: bool = False  # selection per query row (Algorithm 3's argtopk along S's rows)


@dataclass
class HeadResult:
    q: KMeansResult
    k: KMeansResult
    q_mean_norm: np.ndarray
    sel_idx: np.ndarray
    sel_cnt: np.ndarray
    dense: int
    out_rows: np.ndarray | None = None
    rows: np.ndarray | None = None
    extra: dict = field(default_factory=dict)


def cluster_q(q, spec: HeadSpec, init=None):
    xs, nrm = prepare(q, SPHERE)
    if spec.adaptive_q:
        r = multistage(xs, spec.kq, spec.iters, spec.tau_rule, spec.tau_value, spec.nmax_q, SPHERE)
    else:
        r = kmeans(xs, spec.kq, spec.iters, SPHERE, init=init)
    return r, cluster_mean_norm(nrm, r.assign, r.nclusters)


def cluster_k(k, spec: HeadSpec, init=None):
    """Key clustering; with spec.text_keys only the keys before the text strip."""
    if spec.text_keys:
        k = k[:k.shape[0] - spec.text_keys]
    xs, _ = prepare(k, EUCLID)
    if spec.adaptive_k:
        return multistage(xs, spec.kk, spec.iters, spec.tau_rule, spec.tau_value, spec.nmax_k, EUCLID)
    return kmeans(xs, spec.kk, spec.iters, EUCLID, init=init)


def forward_head(q, k, v, spec: HeadSpec, rows=None):
    """Algorithm 3 for one head; attention is evaluated for `rows` (all if None)."""
    rq, qmn = cluster_q(q, spec)
    rk = cluster_k(k, spec)
    return _select_attend(q, k, v, rq, rk, qmn, int(rq.dense or rk.dense), spec, rows)


def forward_steps(steps, spec: HeadSpec, rows=None):
    """One head over consecutive denoising steps (AdaCluster §3.2.2 "Efficient
    initialization", §4.1): step 0 is forward_head (Algorithm 1 counts when the
    spec is adaptive); every later step keeps step 0's cluster counts and dense
    flag F and runs fixed-count k-means (spec.iters rounds) seeded with the
    previous step's centres, then selection and attention as forward_head.
    `steps` is a list of (q, k, v); returns one HeadResult per step."""
    q0, k0, v0 = steps[0]
    res = [forward_head(q0, k0, v0, spec, rows)]
    nq, nk, dense = res[0].q.nclusters, res[0].k.nclusters, res[0].dense
    for q, k, v in steps[1:]:
        prev = res[-1]
        xq, nrm = prepare(q, SPHERE)
        rq = kmeans(xq, nq, spec.iters, SPHERE, init=prev.q.cent[:nq])
        qmn = cluster_mean_norm(nrm, rq.assign, rq.nclusters)
        xk, _ = prepare(k[:k.shape[0] - spec.text_keys], EUCLID)
        rk = kmeans(xk, nk, spec.iters, EUCLID, init=prev.k.cent[:nk])
        res.append(_select_attend(q, k, v, rq, rk, qmn, dense, spec, rows))
    return res


def _select_attend(q, k, v, rq, rk, qmn, dense, spec: HeadSpec, rows):
    """Algorithm 3's selection and attention for one head from its two clusterings.  With
    spec.text_keys the text keys form one more key group (id = the number of
    key clusters) that no score ranks and every query cluster selects."""
    nv = rk.nclusters
    kv = k[:k.shape[0] - spec.text_keys]
    k_assign = rk.assign
    if spec.text_keys:
        k_assign = np.concatenate([rk.assign, np.full(spec.text_keys, nv, np.int32)])
    if dense:
        sel = np.zeros((rq.nclusters, max(nv, 1)), np.int32)
        cnt = np.zeros(rq.nclusters, np.int32)
    else:
        kmax = kmin = None
        if spec.score_mode == SCORE_QUEST:
            kmax, kmin = key_bounds(kv, rk.assign, nv)
        sel, cnt = select2(rq.cent, qmn, rq.count, rk.cent[:nv], rk.count, spec.top_p, spec.score_mode,
                           spec.top_k, kmax, kmin)
        if spec.text_keys:
            # every non-empty query cluster (an empty one selects nothing)
            sel = np.concatenate([sel, np.full((sel.shape[0], 1), -1, np.int32)], axis=1)
            live = np.nonzero(np.asarray(rq.count)[:sel.shape[0]] > 0)[0]
            sel[live, cnt[live]] = nv
            cnt = cnt.copy()
            cnt[live] += 1
    if rows is None:
        rows = np.arange(q.shape[0], dtype=np.int32)
    if spec.per_query and not dense:
        # every evaluated row selects for itself; the per-cluster selection above
        # is kept in the result for reference
        kmax = kmin = None
        if spec.score_mode == SCORE_QUEST:
            kmax, kmin = key_bounds(kv, rk.assign, nv)
        rows = np.asarray(rows, np.int32)
        sq, cq = select_per_query(q[rows], rk.cent[:nv], rk.count, spec.top_p, spec.score_mode, spec.top_k, kmax,
                                  kmin)
        if spec.text_keys:
            sq = np.concatenate([sq, np.full((sq.shape[0], 1), -1, np.int32)], axis=1)
            sq[np.arange(len(rows)), cq] = nv
            cq = cq + 1
        out = attend_per_query(q, k, v, k_assign, nv + (1 if spec.text_keys else 0), sq, cq, rows)
        return HeadResult(rq, rk, qmn, sel, cnt, dense, out, rows,
                          extra={"k_assign": k_assign, "sel_rows": sq, "cnt_rows": cq})
    out = attention_rows(q, k, v, rq.assign, k_assign, nv + (1 if spec.text_keys else 0), sel, cnt, dense, rows)
    return HeadResult(rq, rk, qmn, sel, cnt, dense, out, np.asarray(rows, np.int32), extra={"k_assign": k_assign})
