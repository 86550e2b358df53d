"""Per-query selection (Algorithm 3's argtopk along each row of S) on the GPU
against the oracle's per-query path.

  * ac_select_rows, fed the oracle's key clusters, gives every query row the
    oracle's set bit for bit (CENTROID and QUEST scores, ragged sizes; also
    from query and centroid buffers off the 16-byte grid, which take the
    element-wise score kernel instead of the tiled one);
  * ac_sparse_attn_rows, fed the oracle's clusters and row sets, matches the
    oracle's attention of each row over its own keys (max-abs 2e-2, mean-abs
    2e-3 on all rows);
  * ac_forward with per_query = 1 matches the oracle end to end on sampled
    rows, and its pair count equals the count the oracle's sets imply."""
import numpy as np
import pytest

from clustered_sparse_attention_head_b200 import workloads as W

from gpu_util import attn_close, stack_heads, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import build
    build()


CASES = {
    "centroid-top4": (W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 2777, heads=2, seed=6, kq=23, kk=41),
                      dict(score_mode=0, top_k=4)),
    "quest-top9": (W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 3001, heads=2, seed=7, kq=17, kk=53),
                   dict(score_mode=1, top_k=9)),
    "centroid-top1-d64": (W.small(W.WORKLOADS["cogvideox2b-n17776-h30-d64"], 2049, heads=3, seed=2, kq=11, kk=29),
                          dict(score_mode=0, top_k=1)),
}


def _ctx(w, over):
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    cfg = Config.from_workload(w)
    cfg.per_query = True
    for k, v in over.items():
        setattr(cfg, k, v)
    return AdaCluster(cfg)


def _bits(sel, cnt, W):
    out = np.zeros((sel.shape[0], W), np.uint32)
    for i in range(sel.shape[0]):
        for b in sel[i, :cnt[i]]:
            out[i, b >> 5] |= np.uint32(1) << np.uint32(b & 31)
    return out


@pytest.mark.parametrize("name", list(CASES))
def test_select_rows_and_attention_from_oracle_clusters(orc, name):
    w, over = CASES[name]
    ctx = _ctx(w, over)
    H, N, D = w.heads, w.n, w.d
    q, k, v = stack_heads(w)
    spec = orc.HeadSpec(kq=w.kq, kk=w.kk, iters=w.iters, top_p=w.top_p, **over, per_query=True)
    kk_cap = ctx.kk_cap
    Wd = (kk_cap + 31) // 32
    k_cent = np.zeros((H, kk_cap, D), np.float32)
    k_count = np.zeros((H, kk_cap), np.int32)
    k_max = np.zeros((H, kk_cap, D), np.float32)
    k_min = np.zeros((H, kk_cap, D), np.float32)
    qa = np.zeros((H, N), np.int32)
    ka = np.zeros((H, N), np.int32)
    want_bits = np.zeros((H, N, Wd), np.uint32)
    sets = []
    for h in range(H):
        rq, _ = orc.cluster_q(q[h], spec)
        rk = orc.cluster_k(k[h], spec)
        kc = rk.nclusters
        k_cent[h, :kc], k_count[h, :kc] = rk.cent, rk.count
        km, kn = orc.key_bounds(k[h], rk.assign, kc)
        k_max[h, :kc], k_min[h, :kc] = km, kn
        qa[h], ka[h] = rq.assign, rk.assign
        sel, cnt = orc.select_per_query(q[h], rk.cent, rk.count, spec.top_p, spec.score_mode, spec.top_k, km, kn)
        want_bits[h] = _bits(sel, cnt, Wd)
        sets.append((sel, cnt))
    dev = lambda a: torch.from_numpy(a).cuda()
    qd, kd, vd = (to_dev(a, w.dtype) for a in (q, k, v))
    bits = ctx.ac_select_rows(qd, dev(k_count), k_cent=dev(k_cent), k_max=dev(k_max), k_min=dev(k_min))
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    got_bits = bits.cpu().numpy().view(np.uint32)
    bad = np.nonzero((got_bits != want_bits).any(axis=2))
    assert len(bad[0]) == 0, f"{name}: {len(bad[0])} rows with a different set, e.g. {list(zip(*bad))[:5]}"
    if over["score_mode"] == 0:
        # queries and centroids at addresses off the 16-byte grid (the element-wise score kernel)
        def shifted(t):
            buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
            view = buf[1:].view(t.shape)
            view.copy_(t)
            assert view.data_ptr() % 16 != 0
            return view
        bits_u = ctx.ac_select_rows(shifted(qd), dev(k_count), k_cent=shifted(dev(k_cent)))
        torch.cuda.synchronize()
        assert ctx.get_status() == 0
        got_u = bits_u.cpu().numpy().view(np.uint32)
        assert np.array_equal(got_u, want_bits), f"{name}: unaligned operands give other sets"
    # attention from the oracle's clusters and sets, every row
    rb = torch.from_numpy(want_bits.view(np.int32)).cuda()
    nq = torch.full((H,), w.kq, dtype=torch.int32, device="cuda")
    nk = torch.full((H,), w.kk, dtype=torch.int32, device="cuda")
    out = ctx.ac_sparse_attn_rows(qd, kd, vd, dev(qa), dev(ka), rb, nq=nq, nk=nk)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    got = out.float().cpu().numpy()
    rows = np.arange(N, dtype=np.int32)
    for h in range(H):
        sel, cnt = sets[h]
        ref = orc.attend_per_query(q[h], k[h], v[h], ka[h], w.kk, sel, cnt, rows)
        attn_close(got[h], ref, f"{name}/h{h}/attention")


# hand-made key clusters for the per-row argtopk: duplicated centroids (exact
# score ties, broken towards the lower id), empty clusters (never chosen, also
# when they duplicate a chosen one), and cluster counts on both sides of 512
# (a register quickselect up to 512 clusters, the shared-memory scan beyond)
TIE_CASES = {
    "ties-kk40": (300, 40, 6),
    "ties-kk512": (600, 512, 5),
    "ties-kk600": (700, 600, 9),
}


@pytest.mark.parametrize("name", list(TIE_CASES))
def test_select_rows_ties_and_empty_clusters(orc, name):
    n, kk, top_k = TIE_CASES[name]
    w = W.small(W.WORKLOADS["wan21-n75600-h40-d128"], n, heads=1, seed=9, kq=4, kk=kk)
    ctx = _ctx(w, dict(score_mode=0, top_k=top_k))
    D = w.d
    q, _, _ = stack_heads(w)
    rng = np.random.default_rng(11)
    cent = (0.3 * rng.standard_normal((kk, D))).astype(np.float32)
    for a, b in ((5, 17), (20, 33), (3, 8), (1, kk - 1)):
        cent[b] = cent[a]
    count = rng.integers(1, 50, kk).astype(np.int32)
    count[[2, 11, 30, 33]] = 0
    kk_cap = ctx.kk_cap
    Wd = (kk_cap + 31) // 32
    k_cent = np.zeros((1, kk_cap, D), np.float32)
    k_count = np.zeros((1, kk_cap), np.int32)
    k_cent[0, :kk], k_count[0, :kk] = cent, count
    sel, cnt = orc.select_per_query(q[0], cent, count, w.top_p, 0, top_k, None, None)
    want = _bits(sel, cnt, Wd)
    bits = ctx.ac_select_rows(to_dev(q, w.dtype), torch.from_numpy(k_count).cuda(),
                              k_cent=torch.from_numpy(k_cent).cuda())
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    got = bits.cpu().numpy().view(np.uint32)[0]
    bad = np.nonzero((got != want).any(axis=1))[0]
    assert len(bad) == 0, f"{name}: {len(bad)} rows with a different set, e.g. rows {bad[:5].tolist()}"
    # the duplicated pairs tie exactly: wherever the higher id is chosen, so is the lower
    for a, b in ((5, 17), (3, 8), (1, kk - 1)):
        hi_on = ((got[:, b >> 5] >> np.uint32(b & 31)) & 1).astype(bool)
        lo_on = ((got[:, a >> 5] >> np.uint32(a & 31)) & 1).astype(bool)
        assert not np.any(hi_on & ~lo_on), f"{name}: tie between {a} and {b} broken upwards"


@pytest.mark.parametrize("name", list(CASES))
def test_forward_per_query_end_to_end(orc, name):
    w, over = CASES[name]
    ctx = _ctx(w, over)
    H, N = w.heads, w.n
    q, k, v = stack_heads(w)
    qd, kd, vd = (to_dev(a, w.dtype) for a in (q, k, v))
    out, st = ctx.ac_forward(qd, kd, vd, stats=True)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    got = out.float().cpu().numpy()
    spec = orc.HeadSpec(kq=w.kq, kk=w.kk, iters=w.iters, top_p=w.top_p, **over, per_query=True)
    rows = np.unique(np.concatenate([np.arange(0, N, 13), [N - 1]])).astype(np.int32)
    pairs = 0
    for h in range(H):
        r = orc.forward_head(q[h], k[h], v[h], spec, rows=np.arange(N, dtype=np.int32))
        sel, cnt = r.extra["sel_rows"], r.extra["cnt_rows"]
        pairs += int(sum(int(r.k.count[sel[i, :cnt[i]]].sum()) for i in range(N)))
        attn_close(got[h][rows], r.out_rows[rows], f"{name}/h{h}/forward")
    print(f"{name}: pairs {st['pairs']} (oracle {pairs}), computed {st['pairs_computed']}")
    assert st["pairs"] == pairs
    assert st["pairs_computed"] >= st["pairs"]


def test_per_query_needs_top_k_and_bf16():
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    w, _ = CASES["centroid-top4"]
    for over in (dict(top_k=0), dict(top_k=4, dtype="f32")):
        cfg = Config.from_workload(w)
        cfg.per_query = True
        for key, val in over.items():
            setattr(cfg, key, val)
        with pytest.raises(_abi.AcError) as e:
            AdaCluster(cfg)
        assert e.value.code == _abi.AC_ERR_UNSUPPORTED
