"""Errors made on the host, without a GPU fault: each input below is one the
library must refuse or flag, and after it the same context must give, on its
next call, exactly what a fresh context gives.

  * a NaN in q with AC_FLAG_CHECK_FINITE: the norm pass flags it on the device
    and ac_get_status returns AC_ERR_NONFINITE;
  * a workspace one byte short: every call returns AC_ERR_WORKSPACE at once and
    launches nothing;
  * per-head counts beyond the capacities (nq, nk, ncl, sel_cnt in caller
    memory): the kernels clamp them and ac_get_status returns
    AC_ERR_INVALID_ARG;
  * Algorithm 1 whose last stage overshoots N_max by a whole first stage: the
    capacity N_max + m0 holds it, F is set and no AC_ERR_CAPACITY is raised
    (that code guards a bound the stage-size rule cannot break)."""
import ctypes

import numpy as np
import pytest

from clustered_sparse_attention_head_b200 import workloads as W

from gpu_util import stack_heads, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import build
    build()


def _case():
    w = W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 2777, heads=2, seed=6, kq=23, kk=41)
    return w, [to_dev(a, w.dtype) for a in stack_heads(w)]


def _fresh_forward(w, q, k, v, **over):
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    cfg = Config.from_workload(w)
    for key, val in over.items():
        setattr(cfg, key, val)
    ref = AdaCluster(cfg)
    out = ref.ac_forward(q, k, v)
    torch.cuda.synchronize()
    assert ref.get_status() == 0
    ref.close()
    return out


def _same(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_nonfinite_input_is_flagged_and_context_recovers():
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    w, (q, k, v) = _case()
    flags = _abi.AC_FLAG_CHECK_FINITE
    ref = _fresh_forward(w, q, k, v, flags=flags)
    cfg = Config.from_workload(w)
    cfg.flags = flags
    ctx = AdaCluster(cfg)
    bad = q.clone()
    bad[1, 1234, 77] = float("nan")
    ctx.ac_forward(bad, k, v)
    assert ctx.get_status() == _abi.AC_ERR_NONFINITE
    assert ctx.get_status() == _abi.AC_OK, "the status word is cleared by the read"
    bad_k = k.clone()
    bad_k[0, 5, 3] = float("inf")
    ctx.ac_forward(q, bad_k, v)
    assert ctx.get_status() == _abi.AC_ERR_NONFINITE
    out = ctx.ac_forward(q, k, v)
    torch.cuda.synchronize()
    assert ctx.get_status() == _abi.AC_OK
    assert _same(out, ref), "the next call differs from a fresh context's"


def test_workspace_one_byte_short_is_refused():
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200._abi import ptr
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    w, (q, k, v) = _case()
    ref = _fresh_forward(w, q, k, v)
    ctx = AdaCluster(Config.from_workload(w))
    out = torch.empty_like(q)
    ws, nb = ctx._args_ws()
    short = ctypes.c_size_t(nb.value - 1)
    lib = ctx.lib
    rc = lib.ac_forward(ctx._ctx, ptr(q), ptr(k), ptr(v), None, None, ptr(out), None, ws, short, None)
    assert rc == _abi.AC_ERR_WORKSPACE
    H, N, cap = w.heads, w.n, ctx.kk_cap
    ia = torch.zeros(H, N, dtype=torch.int32, device="cuda")
    perm = torch.empty(H, N, dtype=torch.int32, device="cuda")
    off = torch.empty(H, cap + 1, dtype=torch.int32, device="cuda")
    assert lib.ac_cluster_sort(ctx._ctx, ptr(ia), cap, None, ptr(perm), ptr(off), ws, short, None) == \
        _abi.AC_ERR_WORKSPACE
    assert lib.ac_forward(ctx._ctx, ptr(q), ptr(k), ptr(v), None, None, ptr(out), None, None, nb, None) == \
        _abi.AC_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert ctx.get_status() == _abi.AC_OK, "a refused call leaves no device-side error"
    out2 = ctx.ac_forward(q, k, v)
    torch.cuda.synchronize()
    assert ctx.get_status() == _abi.AC_OK
    assert _same(out2, ref)


def test_counts_beyond_capacity_are_clamped_and_flagged():
    """Caller-made per-head counts above the capacities: the selection, the
    sort and the attention stay inside their buffers, report
    AC_ERR_INVALID_ARG, and the context's next forward equals a fresh one."""
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    w, (q, k, v) = _case()
    ref = _fresh_forward(w, q, k, v)
    ctx = AdaCluster(Config.from_workload(w))
    cq = ctx.ac_cluster_q(q)
    ck = ctx.ac_cluster_k(k)
    torch.cuda.synchronize()
    assert ctx.get_status() == _abi.AC_OK
    big_q = torch.full_like(cq["nclusters"], ctx.kq_cap + 5)
    big_k = torch.full_like(ck["nclusters"], ctx.kk_cap + 7)
    sel, cnt = ctx.ac_select(cq["cent"], cq["mean_norm"], cq["count"], ck["cent"], ck["count"], nq=big_q, nk=big_k)
    assert ctx.get_status() == _abi.AC_ERR_INVALID_ARG
    # the clamped counts equal the capacities, which are the configured counts here
    sel_ok, cnt_ok = ctx.ac_select(cq["cent"], cq["mean_norm"], cq["count"], ck["cent"], ck["count"])
    torch.cuda.synchronize()
    assert ctx.get_status() == _abi.AC_OK
    assert torch.equal(cnt, cnt_ok) and torch.equal(sel, sel_ok)
    perm, off = ctx.ac_cluster_sort(ck["assign"], ctx.kk_cap, big_k)
    assert ctx.get_status() == _abi.AC_ERR_INVALID_ARG
    perm_ok, off_ok = ctx.ac_cluster_sort(ck["assign"], ctx.kk_cap)
    torch.cuda.synchronize()
    assert torch.equal(perm, perm_ok) and torch.equal(off, off_ok)
    bad_cnt = cnt_ok.clone()
    bad_cnt[0, 0] = ctx.kk_cap + 100
    out_bad = ctx.ac_sparse_attn(q, k, v, cq["assign"], ck["assign"], sel_ok, bad_cnt, nq=big_q, nk=big_k)
    assert ctx.get_status() == _abi.AC_ERR_INVALID_ARG
    assert bool(torch.isfinite(out_bad.float()).all())
    out = ctx.ac_forward(q, k, v)
    torch.cuda.synchronize()
    assert ctx.get_status() == _abi.AC_OK
    assert _same(out, ref)


def test_algorithm1_largest_overshoot_fits_capacity():
    """tau = 0 removes no token (the test is d < tau), so stage 1 again has all
    N tokens and m_1 = m0: |C| goes from m0 < N_max to 2 m0 >= N_max, the most
    the last stage can add.  The capacity N_max + m0 holds it, F = 1, and the
    status stays AC_OK; the context's next call equals a fresh one."""
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    w, (q, k, v) = _case()
    m0 = 12
    over = dict(kk=m0, adaptive_k=True, nmax_k=m0 + 1, tau_rule=_abi.AC_TAU_ABS, tau_value=0.0, iters=3)
    cfg = Config.from_workload(w)
    for key, val in over.items():
        setattr(cfg, key, val)
    ctx = AdaCluster(cfg)
    assert ctx.kk_cap == 2 * m0 + 1
    ck = ctx.ac_cluster_k(k)
    torch.cuda.synchronize()
    assert ctx.get_status() == _abi.AC_OK
    assert ck["nclusters"].cpu().tolist() == [2 * m0] * w.heads
    assert ck["dense_flag"].cpu().tolist() == [1] * w.heads
    ref = _fresh_forward(w, q, k, v, **over)
    out = ctx.ac_forward(q, k, v)
    torch.cuda.synchronize()
    assert ctx.get_status() == _abi.AC_OK
    assert _same(out, ref)
