"""The text-key strip (ac_config.text_keys; a variant, not in the pages, that
checks their "no special treatment" of text tokens) through ac_forward against the oracle:
the last text_keys keys are not clustered and every non-empty query cluster
selects them.  Per head: key clusters and the dense flag exact, key centres
within 1e-5 relative, the selected lists bit-exact (text group last), attention
rows within max-abs 2e-2 / mean-abs 2e-3."""
import numpy as np
import pytest

from clustered_sparse_attention_head_b200 import workloads as W

from gpu_util import CENT_RTOL, assert_assign_equal, attn_close, stack_heads, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import build
    build()


CASES = {
    # CogVideoX-shaped: 226 text tokens after the video tokens, fixed counts
    "bf16-d64-text226": (W.small(W.WORKLOADS["cogvideox2b-n17776-h30-d64"], 2600, heads=2, seed=5, kq=20, kk=37,
                                 text=226), {}),
    # HunyuanVideo-shaped keys: 256 text tokens, Algorithm 1 on the video keys
    "bf16-d128-text256-adaptive": (W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 1999, heads=2, seed=9, n_comp=12,
                                           outlier_frac=0.0, text=256),
                                   dict(kq=10, adaptive_k=True, kk=6, nmax_k=200, tau_rule=1, tau_value=1.0,
                                        iters=5)),
    "f32-d64-text64": (W.small(W.WORKLOADS["gmm16-n2048-d64-f32"], 1500, heads=1, seed=4, kq=12, kk=20, text=64), {}),
}


@pytest.mark.parametrize("name", list(CASES))
def test_forward_text_keys(orc, name):
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    w, over = CASES[name]
    cfg = Config.from_workload(w)
    for k, v in over.items():
        setattr(cfg, k, v)
    cfg.text_keys = w.text
    ctx = AdaCluster(cfg)
    q, k, v = stack_heads(w)
    qd, kd, vd = (to_dev(a, w.dtype) for a in (q, k, v))
    out = ctx.ac_forward(qd, kd, vd)
    ck = ctx.ac_cluster_k(kd)
    cq = ctx.ac_cluster_q(qd)
    dense_t = (cq["dense_flag"] | ck["dense_flag"]).contiguous()
    sel_t, cnt_t = ctx.ac_select(cq["cent"], cq["mean_norm"], cq["count"], ck["cent"], ck["count"],
                                 nq=cq["nclusters"], nk=ck["nclusters"], dense_flag=dense_t)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    spec = orc.HeadSpec(kq=cfg.kq, kk=cfg.kk, iters=cfg.iters, top_p=cfg.top_p, adaptive_q=cfg.adaptive_q,
                        adaptive_k=cfg.adaptive_k, tau_rule=cfg.tau_rule, tau_value=cfg.tau_value,
                        nmax_q=cfg.nmax_q, nmax_k=cfg.nmax_k, text_keys=w.text)
    N, T = w.n, w.text
    rows = np.unique(np.concatenate([np.arange(0, N, max(1, N // 97)), np.arange(N - T, N, 13), [N - 1]])).astype(np.int32)
    got = out.float().cpu().numpy()
    ka, kn, kc = ck["assign"].cpu().numpy(), ck["nclusters"].cpu().numpy(), ck["cent"].cpu().numpy()
    sel, cnt = sel_t.cpu().numpy(), cnt_t.cpu().numpy()
    for h in range(w.heads):
        r = orc.forward_head(q[h], k[h], v[h], spec, rows=rows)
        nv = r.k.nclusters
        assert int(kn[h]) == nv + 1, f"{name}/h{h}: key groups {kn[h]} vs {nv} clusters + text"
        np.testing.assert_array_equal(ka[h, N - T:], nv)
        xs, _ = orc.prepare(k[h, :N - T], orc.EUCLID)
        assert_assign_equal(orc, xs, r.k.cent, orc.EUCLID, ka[h, :N - T], r.k.assign, f"{name}/h{h}/keys")
        if not np.array_equal(ka[h, :N - T], r.k.assign):
            print(f"{name}/h{h}: excused near-tie; downstream not compared")
            continue
        np.testing.assert_allclose(kc[h, :nv], r.k.cent[:nv], rtol=CENT_RTOL, atol=1e-7)
        assert int(dense_t[h]) == r.dense
        if not r.dense:
            nq = r.q.nclusters
            np.testing.assert_array_equal(cnt[h, :nq], r.sel_cnt)
            for a in range(nq):
                np.testing.assert_array_equal(sel[h, a, :cnt[h, a]], r.sel_idx[a, :r.sel_cnt[a]])
                if r.q.count[a] > 0:
                    assert sel[h, a, cnt[h, a] - 1] == nv, "text group last in every list"
        attn_close(got[h][rows], r.out_rows, f"{name}/h{h}/attention")
