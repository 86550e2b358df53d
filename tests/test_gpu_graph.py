"""ac_forward replayed from CUDA graphs on the GPU: the library's own cache (a
fixed-count call on the same buffers as an earlier one replays that call's
captured launches) and AdaCluster.capture_forward (a graph the caller owns).

  * a replay gives the output of a plain ac_forward call bit for bit (bf16 and
    fp32 inputs; every kernel of the path is deterministic, the dynamic item
    schedule of the attention kernel included);
  * after new values are copied into the same input buffers, a replay gives
    the plain call's output on those values (the graph holds the buffers'
    addresses, not their contents);
  * configurations whose call reads results on the host (Algorithm 1's
    adaptive counts, profiling) are refused;
  * the library's cache: repeated calls, calls on new contents of the same
    buffers and calls that alternate two buffer sets give, bit for bit, what a
    context with AC_FLAG_NO_GRAPH (every call launch by launch) gives."""
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


def _ctx_flags(w, flags):
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    cfg = Config.from_workload(w)
    cfg.flags = flags
    return AdaCluster(cfg)


@pytest.mark.parametrize("name", list(CASES))
def test_library_graph_cache_equals_launch_by_launch(name):
    from dataclasses import replace
    from clustered_sparse_attention_head_b200 import _abi
    w = CASES[name]
    ctx, ref = _ctx_flags(w, 0), _ctx_flags(w, _abi.AC_FLAG_NO_GRAPH)
    sets = [_inputs(w), _inputs(replace(w, seed=w.seed + 7))]
    outs = [torch.empty_like(sets[0][0]), torch.empty_like(sets[0][0])]
    want = [ref.ac_forward(*sets[i]).clone() for i in range(2)]
    for rep in range(3):  # first call captures, later ones replay; two buffer sets alternate
        for i in range(2):
            outs[i].zero_()
            ctx.ac_forward(*sets[i], out=outs[i])
            torch.cuda.synchronize()
            assert ctx.get_status() == 0
            assert torch.equal(outs[i], want[i]), f"{name}: call {rep}/{i} differs"
    # new contents in the first buffer set: the replay reads them
    q2, k2, v2 = _inputs(replace(w, seed=w.seed + 13))
    for dst, src in zip(sets[0], (q2, k2, v2)):
        dst.copy_(src)
    ctx.ac_forward(*sets[0], out=outs[0])
    want2 = ref.ac_forward(q2, k2, v2)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0 and ref.get_status() == 0
    assert torch.equal(outs[0], want2), f"{name}: replay on new contents differs"
    # and the calls do replay: one graph launch costs the host far less than
    # the call's ~250 separate launches
    import time

    def host_s(c):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(10):
            c.ac_forward(*sets[1], out=outs[1])
        t1 = time.perf_counter()
        torch.cuda.synchronize()
        return t1 - t0
    t_graph, t_plain = host_s(ctx), host_s(ref)
    print(f"{name}: host time per call {1e6 * t_graph / 10:.0f} us replayed, {1e6 * t_plain / 10:.0f} us launch by launch")
    assert t_graph < 0.5 * t_plain, f"{name}: the calls were not replayed"

