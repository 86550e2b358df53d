"""The failure path without a GPU fault: a bounded device wait on a barrier
phase that nothing completes must give up after its limit, record
AC_ERR_TIMEOUT for the host, and leave the context usable (the next calls
return the same results as a fresh context)."""
import time

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


def test_bounded_wait_expires_and_context_stays_usable():
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    w = W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 2777, heads=2, seed=6, kq=23, kk=41)
    q, k, v = (to_dev(a, w.dtype) for a in stack_heads(w))
    ref = AdaCluster(Config.from_workload(w))
    out_ref = ref.ac_forward(q, k, v)
    torch.cuda.synchronize()
    assert ref.get_status() == 0

    ctx = AdaCluster(Config.from_workload(w))
    t0 = time.monotonic()
    ctx.selftest_wait(0.25)
    status = ctx.get_status()
    dt = time.monotonic() - t0
    print(f"selftest wait: status {status} after {dt:.3f} s")
    assert status == _abi.AC_ERR_TIMEOUT
    assert 0.2 <= dt < 5.0
    assert ctx.get_status() == 0, "the status word is cleared by the read"
    out = ctx.ac_forward(q, k, v)
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))


def test_selftest_rejects_bad_limits():
    from clustered_sparse_attention_head_b200 import _abi
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    w = W.small(W.WORKLOADS["wan21-n75600-h40-d128"], 512, heads=1, seed=1, kq=4, kk=8)
    ctx = AdaCluster(Config.from_workload(w))
    for bad in (0.0, -1.0, 11.0):
        assert ctx.lib.ac_selftest_wait(ctx._ctx, bad, None) == _abi.AC_ERR_INVALID_ARG
