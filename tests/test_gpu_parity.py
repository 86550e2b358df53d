"""GPU path vs the CPU oracle on identical seeded inputs, through the C ABI.

Stage-isolated: each GPU stage is fed the oracle's output of the previous
stage (one k-means assignment from the oracle's centroids, one iteration, the
selection from the oracle's clusters, the attention from the oracle's
clusters and selection).  End-to-end runs compare the whole chain.
Bit-exact: assignments, counts, permutations, selected sets.  Centroids:
1e-5 relative.  Attention: max-abs 2e-2, mean-abs 2e-3."""
import numpy as np
import pytest

from clustered_sparse_attention_head_b200 import workloads as W

from gpu_util import (ATT_MAX_ABS, CENT_RTOL, assert_assign_equal, attn_close, stack_heads, to_dev)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import build
    build()


def _ctx(w, **over):
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    cfg = Config.from_workload(w)
    for k, v in over.items():
        setattr(cfg, k, v)
    return AdaCluster(cfg)


CASES = {
    # name: (workload, n tokens, heads)
    "f32-d64": (W.WORKLOADS["gmm16-n2048-d64-f32"], 2048, 1),
    "bf16-d64-ragged": (W.small(W.WORKLOADS["cogvideox2b-n17776-h30-d64"], 3001, heads=2, seed=5, kq=20, kk=37), 0, 0),
    "bf16-d128-ragged": (W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 2777, heads=2, seed=6, kq=23, kk=41), 0, 0),
}


def _case(name):
    w, n, h = CASES[name]
    return w


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("mode", ["q", "k"])
def test_assign_from_oracle_centroids(orc, name, mode):
    """One assignment step from the oracle's (converged) centroids: bit-exact."""
    w = _case(name)
    q, k, v = stack_heads(w)
    x = q if mode == "q" else k
    om = orc.SPHERE if mode == "q" else orc.EUCLID
    kc = w.kq if mode == "q" else w.kk
    ctx = _ctx(w, iters=0)
    init = []
    ref = []
    for h in range(w.heads):
        xs, _ = orc.prepare(x[h], om)
        r = orc.kmeans(xs, kc, 3, om)
        init.append(r.cent)
        ids, _, _ = orc.assign(xs, r.cent, om)
        ref.append((xs, r.cent, ids))
    init_t = torch.from_numpy(np.stack(init)).cuda()
    fn = ctx.ac_cluster_q if mode == "q" else ctx.ac_cluster_k
    out = fn(to_dev(x, w.dtype), init_cent=init_t)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    got = out["assign"].cpu().numpy()
    cnt = out["count"].cpu().numpy()
    for h in range(w.heads):
        xs, cent, ids = ref[h]
        assert_assign_equal(orc, xs, cent, om, got[h], ids, f"{name}/{mode}/h{h}")
        np.testing.assert_array_equal(cnt[h, :kc], np.bincount(got[h], minlength=kc))


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("mode", ["q", "k"])
def test_kmeans_end_to_end(orc, name, mode):
    """Full k-means (strided init, 10 iterations): assignments and counts
    bit-exact, centroids within 1e-5 relative, query mean norms too."""
    w = _case(name)
    q, k, v = stack_heads(w)
    x = q if mode == "q" else k
    om = orc.SPHERE if mode == "q" else orc.EUCLID
    kc = w.kq if mode == "q" else w.kk
    ctx = _ctx(w)
    fn = ctx.ac_cluster_q if mode == "q" else ctx.ac_cluster_k
    out = fn(to_dev(x, w.dtype))
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    for h in range(w.heads):
        xs, nrm = orc.prepare(x[h], om)
        r = orc.kmeans(xs, kc, w.iters, om)
        assert_assign_equal(orc, xs, r.cent, om, out["assign"][h].cpu().numpy(), r.assign, f"{name}/{mode}/h{h}")
        np.testing.assert_array_equal(out["count"][h, :kc].cpu().numpy(), r.count)
        np.testing.assert_allclose(out["cent"][h, :kc].cpu().numpy(), r.cent, rtol=CENT_RTOL, atol=1e-7)
        if mode == "q":
            mn = orc.cluster_mean_norm(nrm, r.assign, kc)
            np.testing.assert_allclose(out["mean_norm"][h, :kc].cpu().numpy(), mn, rtol=CENT_RTOL)
        assert int(out["nclusters"][h]) == kc and int(out["dense_flag"][h]) == 0


@pytest.mark.parametrize("name", list(CASES))
def test_sort_bit_exact(orc, name):
    w = _case(name)
    rng = np.random.default_rng(0)
    ids = rng.integers(0, w.kk, (w.heads, w.n)).astype(np.int32)
    ids[ids == 3] = 4  # cluster 3 is empty
    ctx = _ctx(w)
    perm, off = ctx.ac_cluster_sort(torch.from_numpy(ids).cuda(), w.kk)
    torch.cuda.synchronize()
    for h in range(w.heads):
        p, o = orc.cluster_sort(ids[h], w.kk)
        np.testing.assert_array_equal(perm[h].cpu().numpy(), p)
        np.testing.assert_array_equal(off[h].cpu().numpy(), o)


def _oracle_clusters(orc, w, q, k):
    spec = orc.HeadSpec(kq=w.kq, kk=w.kk, iters=w.iters, top_p=w.top_p)
    res = []
    for h in range(w.heads):
        rq, qmn = orc.cluster_q(q[h], spec)
        rk = orc.cluster_k(k[h], spec)
        res.append((rq, qmn, rk))
    return res


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("top_p", [0.5, 0.9, 1.0])
def test_select_from_oracle_clusters(orc, name, top_p):
    w = _case(name)
    q, k, v = stack_heads(w)
    cl = _oracle_clusters(orc, w, q, k)
    ctx = _ctx(w, top_p=top_p)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(np.stack(a))).cuda()
    sel, cnt = ctx.ac_select(t([c[0].cent for c in cl]), t([c[1] for c in cl]), t([c[0].count for c in cl]),
                             t([c[2].cent for c in cl]), t([c[2].count for c in cl]))
    torch.cuda.synchronize()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for h, (rq, qmn, rk) in enumerate(cl):
        s, c = orc.select(rq.cent, qmn, rq.count, rk.cent, rk.count, top_p)
        np.testing.assert_array_equal(cnt[h], c)
        for a in range(w.kq):
            np.testing.assert_array_equal(sel[h, a, :c[a]], s[a, :c[a]])


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("top_p", [0.9, 1.0])
def test_sparse_attention_from_oracle_selection(orc, name, top_p):
    w = _case(name)
    q, k, v = stack_heads(w)
    cl = _oracle_clusters(orc, w, q, k)
    sels = [orc.select(rq.cent, qmn, rq.count, rk.cent, rk.count, top_p) for rq, qmn, rk in cl]
    ctx = _ctx(w, top_p=top_p)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(np.stack(a))).cuda()
    out, lse = ctx.ac_sparse_attn(to_dev(q, w.dtype), to_dev(k, w.dtype), to_dev(v, w.dtype),
                                  t([c[0].assign for c in cl]), t([c[2].assign for c in cl]),
                                  t([s[0] for s in sels]), t([s[1] for s in sels]), lse=True)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    got = out.float().cpu().numpy()
    rows = np.arange(w.n)
    for h, (rq, qmn, rk) in enumerate(cl):
        ref = orc.attention_rows(q[h], k[h], v[h], rq.assign, rk.assign, w.kk, sels[h][0], sels[h][1], 0, rows)
        attn_close(got[h], ref, f"{name}/p{top_p}/h{h}")


@pytest.mark.parametrize("name", ["bf16-d64-ragged", "bf16-d128-ragged"])
def test_sparse_attention_repeatable(orc, name):
    """Five calls on the same inputs give bit-identical outputs and lse: every
    reduction has a fixed order, so any difference would expose a race between
    the kernel's TMA, MMA and softmax roles."""
    w = _case(name)
    q, k, v = stack_heads(w)
    cl = _oracle_clusters(orc, w, q, k)
    sels = [orc.select(rq.cent, qmn, rq.count, rk.cent, rk.count, 1.0) for rq, qmn, rk in cl]
    ctx = _ctx(w, top_p=1.0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(np.stack(a))).cuda()
    args = (to_dev(q, w.dtype), to_dev(k, w.dtype), to_dev(v, w.dtype), t([c[0].assign for c in cl]),
            t([c[2].assign for c in cl]), t([s[0] for s in sels]), t([s[1] for s in sels]))
    first = None
    for _ in range(5):
        out, lse = ctx.ac_sparse_attn(*args, lse=True)
        torch.cuda.synchronize()
        got = (out.view(torch.int16).cpu().numpy(), lse.cpu().numpy())
        if first is None:
            first = got
        else:
            np.testing.assert_array_equal(got[0], first[0])
            np.testing.assert_array_equal(got[1], first[1])
    assert ctx.get_status() == 0


@pytest.mark.parametrize("name", ["f32-d64", "bf16-d128-ragged"])
def test_dense_flag_gives_dense_attention(orc, name):
    w = _case(name)
    q, k, v = stack_heads(w)
    ctx = _ctx(w)
    H, N = w.heads, w.n
    qa = torch.zeros(H, N, dtype=torch.int32, device="cuda")
    ka = torch.zeros(H, N, dtype=torch.int32, device="cuda")
    sel = torch.zeros(H, w.kq, w.kk, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(H, w.kq, dtype=torch.int32, device="cuda")
    dense = torch.ones(H, dtype=torch.uint8, device="cuda")
    out = ctx.ac_sparse_attn(to_dev(q, w.dtype), to_dev(k, w.dtype), to_dev(v, w.dtype), qa, ka, sel, cnt,
                             dense_flag=dense)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    rows = np.arange(0, N, 3)
    for h in range(H):
        ref = orc.attention_rows(q[h], k[h], v[h], None, None, 0, None, None, 1, rows)
        attn_close(got[h][rows], ref, f"{name}/dense/h{h}")


def test_forward_end_to_end_small(orc):
    """ac_forward on the 2048-token fp32 workload vs the oracle's Algorithm 3."""
    w = W.WORKLOADS["gmm16-n2048-d64-f32"]
    q, k, v = stack_heads(w)
    ctx = _ctx(w)
    out, st = ctx.ac_forward(to_dev(q, w.dtype), to_dev(k, w.dtype), to_dev(v, w.dtype), stats=True)
    assert ctx.get_status() == 0
    spec = orc.HeadSpec(kq=w.kq, kk=w.kk, iters=w.iters, top_p=w.top_p)
    r = orc.forward_head(q[0], k[0], v[0], spec)
    attn_close(out[0].float().cpu().numpy(), r.out_rows, "forward/f32")
    assert st["pairs"] == orc.pairs(r.q.count, r.k.count, r.sel_idx, r.sel_cnt)


ADAPTIVE = [
    # (mode, tau_rule, tau_value, m0, nmax)
    ("k", 1, 1.5, 16, 120),     # MEAN_X, the paper's 1.5 x mean distance
    ("k", 2, 0.5, 16, 64),      # MEDIAN_RADIUS_X 0.5: expected to hit N_max (F = 1)
    ("k", 0, 2.0, 12, 200),     # absolute tau
    ("q", 1, 1.5, 10, 80),      # Algorithm 1 on normalised queries
]


@pytest.mark.parametrize("mode,rule,val,m0,nmax", ADAPTIVE)
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_multistage_parity(orc, mode, rule, val, m0, nmax, dt):
    """Algorithm 1 (MultiStageClustering): |C|, F, the final assignment and the
    counts bit-exact, centroids within 1e-5 relative, against the oracle."""
    base = W.WORKLOADS["wan21-n75600-h40-d128"] if dt == "bf16" else W.WORKLOADS["gmm16-n2048-d64-f32"]
    w = W.small(base, 1999, heads=2, seed=9)
    q, k, v = stack_heads(w)
    x = q if mode == "q" else k
    om = orc.SPHERE if mode == "q" else orc.EUCLID
    over = dict(tau_rule=rule, tau_value=val, iters=5)
    if mode == "q":
        over.update(adaptive_q=True, kq=m0, nmax_q=nmax)
    else:
        over.update(adaptive_k=True, kk=m0, nmax_k=nmax)
    ctx = _ctx(w, **over)
    fn = ctx.ac_cluster_q if mode == "q" else ctx.ac_cluster_k
    out = fn(to_dev(x, w.dtype))
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    for h in range(w.heads):
        xs, _ = orc.prepare(x[h], om)
        r = orc.multistage(xs, m0, 5, rule, val, nmax, om)
        nc = int(out["nclusters"][h])
        print(f"{mode}/rule{rule}/h{h}: |C| {nc} (oracle {r.nclusters}), F {int(out['dense_flag'][h])} "
              f"(oracle {r.dense}), stages {r.nstages}, tau {r.tau:.4f}")
        assert nc == r.nclusters and int(out["dense_flag"][h]) == r.dense
        assert_assign_equal(orc, xs, r.cent, om, out["assign"][h].cpu().numpy(), r.assign, f"ms/{mode}/h{h}")
        np.testing.assert_array_equal(out["count"][h, :nc].cpu().numpy(), r.count)
        np.testing.assert_allclose(out["cent"][h, :nc].cpu().numpy(), r.cent, rtol=CENT_RTOL, atol=1e-7)


def test_forward_adaptive_dense_head(orc):
    """A head whose Algorithm 1 sets F takes dense attention inside ac_forward."""
    w = W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 1200, heads=2, seed=3, kq=10, kk=8, iters=3,
                adaptive_k=True, tau_rule=0, tau_value=0.0, nmax_k=16)
    q, k, v = stack_heads(w)
    ctx = _ctx(w)
    out, st = ctx.ac_forward(to_dev(q, w.dtype), to_dev(k, w.dtype), to_dev(v, w.dtype), stats=True)
    assert ctx.get_status() == 0
    assert st["dense_heads"] == 2
    got = out.float().cpu().numpy()
    rows = np.arange(0, w.n, 7)
    for h in range(w.heads):
        ref = orc.attention_rows(q[h], k[h], v[h], None, None, 0, None, None, 1, rows)
        attn_close(got[h][rows], ref, f"adaptive-dense/h{h}")


# --------------------------------------------------------------------------
# Quest page bounds, the Quest score and the argtopk cut
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["f32-d64", "bf16-d128-ragged"])
def test_key_bounds_bit_exact(orc, name):
    """Per key cluster and dimension max / min of the keys: exact."""
    w = _case(name)
    q, k, v = stack_heads(w)
    cl = _oracle_clusters(orc, w, q, k)
    ctx = _ctx(w)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(np.stack(a))).cuda()
    kmax, kmin = ctx.ac_key_bounds(to_dev(k, w.dtype), t([c[2].assign for c in cl]))
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    for h, (_, _, rk) in enumerate(cl):
        emax, emin = orc.key_bounds(k[h], rk.assign, w.kk)
        np.testing.assert_array_equal(kmax[h, :w.kk].cpu().numpy(), emax)
        np.testing.assert_array_equal(kmin[h, :w.kk].cpu().numpy(), emin)


SELECT_MODES = [
    # (score mode, top_k, top_p)
    (1, 0, 0.9),     # Quest score, top-p
    (1, 8, 0.9),     # Quest score, argtopk
    (0, 8, 0.9),     # centroid score, argtopk
    (1, 10000, 0.9), # argtopk with k above every cluster count
]


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("mode,top_k,top_p", SELECT_MODES)
def test_select_modes_from_oracle_clusters(orc, name, mode, top_k, top_p):
    """Selected sets bit-exact against the oracle for the Quest score (as
    TensorQuest's eq. (2) on the GPU, eq. (1) in the oracle) and argtopk."""
    w = _case(name)
    q, k, v = stack_heads(w)
    cl = _oracle_clusters(orc, w, q, k)
    ctx = _ctx(w, score_mode=mode, top_k=top_k, top_p=top_p)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(np.stack(a))).cuda()
    bounds = [orc.key_bounds(k[h], rk.assign, w.kk) for h, (_, _, rk) in enumerate(cl)]
    sel, cnt = ctx.ac_select(t([c[0].cent for c in cl]), t([c[1] for c in cl]), t([c[0].count for c in cl]),
                             t([c[2].cent for c in cl]), t([c[2].count for c in cl]),
                             k_max=t([b[0] for b in bounds]), k_min=t([b[1] for b in bounds]))
    torch.cuda.synchronize()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for h, (rq, qmn, rk) in enumerate(cl):
        s, c = orc.select2(rq.cent, qmn, rq.count, rk.cent, rk.count, top_p, mode, top_k, bounds[h][0], bounds[h][1])
        np.testing.assert_array_equal(cnt[h], c)
        for a in range(w.kq):
            np.testing.assert_array_equal(sel[h, a, :c[a]], s[a, :c[a]])
        if top_k:
            assert (c <= top_k).all()


def test_forward_quest_topk_end_to_end(orc):
    """ac_forward with the Quest score and argtopk (Algorithm 3 as the pages
    write it, with cluster-level pages) against the oracle's Algorithm 3."""
    w = W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 2777, heads=2, seed=6, kq=23, kk=41)
    q, k, v = stack_heads(w)
    ctx = _ctx(w, score_mode=1, top_k=12)
    out, st = ctx.ac_forward(to_dev(q, w.dtype), to_dev(k, w.dtype), to_dev(v, w.dtype), stats=True)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    spec = orc.HeadSpec(kq=w.kq, kk=w.kk, iters=w.iters, top_p=w.top_p, score_mode=1, top_k=12)
    pairs = 0
    got = out.float().cpu().numpy()
    for h in range(w.heads):
        r = orc.forward_head(q[h], k[h], v[h], spec)
        assert (r.sel_cnt <= 12).all()
        attn_close(got[h], r.out_rows, f"forward/quest-top12/h{h}")
        pairs += orc.pairs(r.q.count, r.k.count, r.sel_idx, r.sel_cnt)
    assert st["pairs"] == pairs
