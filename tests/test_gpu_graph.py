"""ac_forward replayed from a CUDA graph (AdaCluster.capture_forward) on the GPU.

  * a replay gives the output of a plain ac_forward call bit for bit (bf16 and
    fp32 inputs; every kernel of the path is deterministic, the dynamic item
    schedule of the attention kernel included);
  * after new values are copied into the same input buffers, a replay gives
    the plain call's output on those values (the graph holds the buffers'
    addresses, not their contents);
  * configurations whose call reads results on the host (Algorithm 1's
    adaptive counts, profiling) are refused."""
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


CASES = {
    "bf16-d128": W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 3000, heads=2, seed=4, kq=20, kk=37),
    "bf16-d64": W.small(W.WORKLOADS["cogvideox2b-n17776-h30-d64"], 2311, heads=3, seed=5, kq=13, kk=29),
    "f32-d64": W.small(W.WORKLOADS["gmm16-n2048-d64-f32"], 1500, heads=2, seed=6, kq=9, kk=11),
}


def _ctx(w):
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    return AdaCluster(Config.from_workload(w))


def _inputs(w):
    q, k, v = stack_heads(w)
    return tuple(to_dev(a, w.dtype) for a in (q, k, v))


@pytest.mark.parametrize("name", list(CASES))
def test_graph_replay_equals_plain_calls(name):
    w = CASES[name]
    ctx = _ctx(w)
    q, k, v = _inputs(w)
    plain = ctx.ac_forward(q, k, v).clone()
    graph, out = ctx.capture_forward(q, k, v)
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    assert torch.equal(out, plain), f"{name}: replay differs from the plain call"
    # new values in the same buffers
    from dataclasses import replace
    w2 = replace(w, seed=w.seed + 100)
    q2, k2, v2 = _inputs(w2)
    for dst, src in ((q, q2), (k, k2), (v, v2)):
        dst.copy_(src)
    graph.replay()
    torch.cuda.synchronize()
    plain2 = ctx.ac_forward(q2, k2, v2)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    assert not torch.equal(plain2, plain)
    assert torch.equal(out, plain2), f"{name}: replay on new inputs differs from the plain call"


def test_capture_refuses_host_reads():
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    adaptive = W.small(W.WORKLOADS["cogvideox2b720p-n70000-h30-d64-adaptive"], 2500, heads=1, seed=3)
    for w, over in ((adaptive, {}), (CASES["bf16-d128"], dict(flags=_abi.AC_FLAG_PROFILE))):
        assert w.adaptive_q or w.adaptive_k or over
        q, k, v = _inputs(w)
        cfg = Config.from_workload(w)
        for key, val in over.items():
            setattr(cfg, key, val)
        ctx = AdaCluster(cfg)
        with pytest.raises(ValueError):
            ctx.capture_forward(q, k, v)
