"""The multi-step driver (ac_forward_step) against the oracle's forward_steps
on drifting seeded inputs (workloads.step_inputs), and the early stop of
fixed-count k-means.

Per step and head: cluster counts and dense flag F exact; query and key
centres within 1e-5 relative; attention rows within max-abs 2e-2 / mean-abs
2e-3.  Every head is compared at every step.  Only a head that fails the
comparison can be excused, and only when the oracle's own k-means of that
step meets a near-tie (two best scores within 1e-6 relative) on some rows:
the GPU may then take the other, equally valid branch there, which moves the
two clusters' centres and everything after.  Such a head is compared again
at the next step only through what does not depend on that branch (counts and
F); the excused heads and their near-tie rows are printed."""
import numpy as np
import pytest

from clustered_sparse_attention_head_b200 import workloads as W

from gpu_util import CENT_RTOL, TIE_REL, attn_close, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

NSTEPS = 4
DRIFT = 0.05


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
    "bf16-d128-fixed": (W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 2777, heads=2, seed=6, kq=23, kk=41), {}),
    # Algorithm 1 on the keys at step 0 (8-9 stages, 21 clusters per head)
    "bf16-d128-adaptive": (W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 1999, heads=2, seed=9, n_comp=12,
                                   outlier_frac=0.0),
                           dict(kq=10, adaptive_k=True, kk=6, nmax_k=200, tau_rule=1, tau_value=1.0, iters=5)),
    # Algorithm 1 reaches N_max at step 0: F = 1 for every step (dense attention)
    "bf16-d128-dense": (W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 1999, heads=2, seed=9),
                        dict(kq=10, adaptive_k=True, kk=16, nmax_k=40, tau_rule=1, tau_value=1.5, iters=5)),
    "f32-d64-fixed": (W.small(W.WORKLOADS["gmm16-n2048-d64-f32"], 1500, heads=1, seed=4, kq=12, kk=20), {}),
}


def _spec(orc, w, over):
    g = dict(kq=w.kq, kk=w.kk, iters=w.iters, top_p=w.top_p, adaptive_q=w.adaptive_q, adaptive_k=w.adaptive_k,
             tau_rule=w.tau_rule, tau_value=w.tau_value, nmax_q=w.nmax_q, nmax_k=w.nmax_k)
    g.update(over)
    return orc.HeadSpec(**g)


def _near_tie_rows(xs, cent, mode, orc):
    """Rows whose two best scores against `cent` are within TIE_REL."""
    x = np.asarray(xs, np.float64)
    c = np.asarray(cent, np.float64)
    if mode == orc.EUCLID:
        s = -((x * x).sum(1)[:, None] - 2 * x @ c.T + (c * c).sum(1)[None, :])
    else:
        s = x @ c.T
    top = np.sort(s, axis=1)[:, -2:]
    den = np.maximum(np.abs(top).max(1), 1e-300)
    return set(np.nonzero((top[:, 1] - top[:, 0]) / den < TIE_REL)[0].tolist())


def _kmeans_tie_rows(orc, x, k, iters, mode, init):
    """Replays fixed-count k-means with the oracle's steps; returns the rows
    that meet a near-tie in any of its assignment passes."""
    xs, _ = orc.prepare(x, mode)
    cent = np.asarray(init, np.float32)[:k].copy()
    rows = set()
    for _ in range(iters):
        rows |= _near_tie_rows(xs, cent, mode, orc)
        ids, _, _ = orc.assign(xs, cent, mode)
        cent, _ = orc.update(xs, ids, cent, mode)
    return rows | _near_tie_rows(xs, cent, mode, orc)


def _kmeans_has_tie(orc, x, k, iters, mode, init):
    return bool(_kmeans_tie_rows(orc, x, k, iters, mode, init))


def _compare_or_excuse(what, check, tie_rows, excused):
    """Runs `check`; a failure is excused only when the oracle's k-means of the
    step met near-ties (tie_rows() lists them), and is recorded in `excused`."""
    try:
        check()
        return True
    except AssertionError:
        rows = tie_rows()
        if not rows:
            raise
        excused.append((what, len(rows)))
        print(f"{what}: differs after {len(rows)} near-tie rows in the oracle's k-means; excused")
        return False


@pytest.mark.parametrize("name", list(CASES))
def test_forward_steps_parity(orc, name):
    w, over = CASES[name]
    ctx = _ctx(w, **over)
    spec = _spec(orc, w, over)
    H, N = w.heads, w.n
    rows = np.unique(np.concatenate([np.arange(0, N, max(1, N // 97)), [N - 1]])).astype(np.int32)
    inp = [[W.step_inputs(w, h, s, DRIFT) for s in range(NSTEPS)] for h in range(H)]
    ref = [orc.forward_steps([(x.q, x.k, x.v) for x in inp[h]], spec, rows=rows) for h in range(H)]
    state = ctx.step_state()
    diverged = [False] * H   # an excused branch earlier: centres follow the GPU's own branch
    excused = []
    for s in range(NSTEPS):
        q, k, v = (to_dev(np.stack([getattr(inp[h][s], a) for h in range(H)]), w.dtype) for a in "qkv")
        out, st = ctx.ac_forward_step(s, q, k, v, state, stats=True)
        torch.cuda.synchronize()
        assert ctx.get_status() == 0
        parts = {kk: t.cpu().numpy() for kk, t in ctx.step_state_parts(state).items()}
        got = out.float().cpu().numpy()
        print(f"{name}/step{s}: k-means rounds q {st['kmeans_rounds_q']} k {st['kmeans_rounds_k']}, "
              f"dense heads {st['dense_heads']}")
        for h in range(H):
            r = ref[h][s]
            # counts and F are fixed at step 0 and do not depend on later branches
            nq, nk = int(parts["nq"][h]), int(parts["nk"][h])
            assert nq == r.q.nclusters and nk == r.k.nclusters, f"{name}/step{s}/h{h}: counts"
            assert int(parts["dq"][h] | parts["dk"][h]) == r.dense, f"{name}/step{s}/h{h}: F"
            if r.dense:
                # dense attention does not depend on the clusters
                attn_close(got[h][rows], r.out_rows, f"{name}/step{s}/h{h}/attention (dense)")
                continue
            if diverged[h]:
                continue

            def check():
                np.testing.assert_allclose(parts["q_cent"][h, :nq], r.q.cent[:nq], rtol=CENT_RTOL, atol=1e-7)
                np.testing.assert_allclose(parts["k_cent"][h, :nk], r.k.cent[:nk], rtol=CENT_RTOL, atol=1e-7)
                attn_close(got[h][rows], r.out_rows, f"{name}/step{s}/h{h}/attention")

            def tie_rows():
                if s == 0:
                    return set()
                prev = ref[h][s - 1]
                return (_kmeans_tie_rows(orc, inp[h][s].q, r.q.nclusters, spec.iters, orc.SPHERE, prev.q.cent) |
                        _kmeans_tie_rows(orc, inp[h][s].k, r.k.nclusters, spec.iters, orc.EUCLID, prev.k.cent))

            if not _compare_or_excuse(f"{name}/step{s}/h{h}", check, tie_rows, excused):
                diverged[h] = True
    print(f"{name}: {len(excused)} head-steps excused ({sum(n for _, n in excused)} near-tie rows) "
          f"of {H * NSTEPS}")


def test_warm_steps_need_fewer_rounds(orc):
    """Warm-started steps stop after fewer k-means rounds than the cold step 0
    (same counts, inputs drifting by 0.05 per element and step)."""
    w, over = CASES["bf16-d128-fixed"]
    ctx = _ctx(w, iters=20)
    state = ctx.step_state()
    rounds = []
    for s in range(NSTEPS):
        q, k, v = (to_dev(np.stack([getattr(W.step_inputs(w, h, s, DRIFT), a) for h in range(w.heads)]), w.dtype)
                   for a in "qkv")
        _, st = ctx.ac_forward_step(s, q, k, v, state, stats=True)
        rounds.append((st["kmeans_rounds_q"], st["kmeans_rounds_k"]))
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    print("rounds per step (q, k):", rounds)
    cold_q, cold_k = rounds[0]
    assert all(1 <= a <= 20 and 1 <= b <= 20 for a, b in rounds)
    assert np.mean([a for a, _ in rounds[1:]]) < cold_q and np.mean([b for _, b in rounds[1:]]) < cold_k


def test_early_stop_matches_all_rounds(orc):
    """With a round budget far above what k-means needs, the GPU stops early and
    still returns the centres of the oracle's k-means run for every round."""
    w, _ = CASES["bf16-d128-fixed"]
    ctx = _ctx(w, iters=40)
    q, k, v = (to_dev(np.stack([getattr(W.head_inputs(w, h), a) for h in range(w.heads)]), w.dtype) for a in "qkv")
    state = ctx.step_state()
    _, st = ctx.ac_forward_step(0, q, k, v, state, stats=True)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    print("rounds:", st["kmeans_rounds_q"], st["kmeans_rounds_k"])
    assert st["kmeans_rounds_q"] < 40 and st["kmeans_rounds_k"] < 40
    parts = {kk: t.cpu().numpy() for kk, t in ctx.step_state_parts(state).items()}
    for h in range(w.heads):
        x = W.head_inputs(w, h)
        for mode, arr, kc, key in ((orc.SPHERE, x.q, w.kq, "q_cent"), (orc.EUCLID, x.k, w.kk, "k_cent")):
            xs, _ = orc.prepare(arr, mode)
            r = orc.kmeans(xs, kc, 40, mode)
            if _kmeans_has_tie(orc, arr, kc, 40, mode, orc.init_centroids(xs, kc)):
                print(f"h{h}/{key}: near-tie in the oracle's run; not compared")
                continue
            np.testing.assert_allclose(parts[key][h, :kc], r.cent, rtol=CENT_RTOL, atol=1e-7)


def test_forward_steps_with_text_keys(orc):
    """The driver with the text-key strip: the state counts the text group as
    one more key group, later steps cluster only the video keys with step 0's
    count and keep selecting the strip."""
    w0, _ = CASES["bf16-d128-fixed"]
    w = W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 2400, heads=2, seed=6, kq=23, kk=41, text=96)
    T = w.text
    ctx = _ctx(w, text_keys=T)
    spec = _spec(orc, w, dict(text_keys=T))
    H, N = w.heads, w.n
    rows = np.unique(np.concatenate([np.arange(0, N, max(1, N // 97)), [N - 1]])).astype(np.int32)
    inp = [[W.step_inputs(w, h, s, DRIFT) for s in range(3)] for h in range(H)]
    ref = [orc.forward_steps([(x.q, x.k, x.v) for x in inp[h]], spec, rows=rows) for h in range(H)]
    state = ctx.step_state()
    diverged = [False] * H
    excused = []
    for s in range(3):
        q, k, v = (to_dev(np.stack([getattr(inp[h][s], a) for h in range(H)]), w.dtype) for a in "qkv")
        out = ctx.ac_forward_step(s, q, k, v, state)
        torch.cuda.synchronize()
        assert ctx.get_status() == 0
        parts = {kk: t.cpu().numpy() for kk, t in ctx.step_state_parts(state).items()}
        got = out.float().cpu().numpy()
        for h in range(H):
            r = ref[h][s]
            nv = r.k.nclusters
            assert int(parts["nk"][h]) == nv + 1, f"step{s}/h{h}: key groups"
            if diverged[h]:
                continue

            def check():
                np.testing.assert_allclose(parts["k_cent"][h, :nv], r.k.cent[:nv], rtol=CENT_RTOL, atol=1e-7)
                attn_close(got[h][rows], r.out_rows, f"text/step{s}/h{h}/attention")

            def tie_rows():
                if s == 0:
                    return set()
                prev = ref[h][s - 1]
                return (_kmeans_tie_rows(orc, inp[h][s].q, r.q.nclusters, spec.iters, orc.SPHERE, prev.q.cent) |
                        _kmeans_tie_rows(orc, inp[h][s].k[:N - T], nv, spec.iters, orc.EUCLID, prev.k.cent))

            if not _compare_or_excuse(f"text/step{s}/h{h}", check, tie_rows, excused):
                diverged[h] = True
    print(f"text: {len(excused)} head-steps excused ({sum(n for _, n in excused)} near-tie rows) of {H * 3}")
