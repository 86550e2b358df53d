"""The allocation-free cluster sort (ac_cluster_sort_static) against the
workspace-based ac_cluster_sort, through the C ABI.

ac_cluster_sort_static exists for callers that cannot allocate device memory
where they need the sort, such as an engine plugin limited to pre-reserved
memory or a loop with a fixed memory budget.  Its scratch is a fixed array
inside the library, so it must give the same permutation and offsets as the
entry point that takes a caller workspace, call after call.  The outputs are
integers, so the comparison is exact."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _ids(rng, heads, n, ncl):
    ids = np.stack([rng.integers(0, ncl[h], n) for h in range(heads)]).astype(np.int32)
    ids[0][ids[0] == 5] = 6  # an empty cluster in head 0
    return ids


def test_static_sort_matches_workspace_sort_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import _abi, build
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    build()
    lib = _abi.load()
    heads, n, cap = 3, 5003, 77
    ncl = np.array([77, 60, 1], np.int32)
    ref_ctx = AdaCluster(Config(heads=heads, n=n, d=64, kq=cap, kk=cap))
    ncl_t = torch.from_numpy(ncl).cuda()
    rng = np.random.default_rng(7)
    stream = torch.cuda.current_stream()
    for call in range(2):
        ids_t = torch.from_numpy(_ids(rng, heads, n, ncl)).cuda()
        perm_ref, off_ref = ref_ctx.ac_cluster_sort(ids_t, cap, ncl_t)
        perm = torch.full((heads, n), -1, dtype=torch.int32, device="cuda")
        off = torch.full((heads, cap + 1), -1, dtype=torch.int32, device="cuda")
        rc = lib.ac_cluster_sort_static(ctypes.c_void_p(ids_t.data_ptr()), heads, n, cap,
                                        ctypes.c_void_p(ncl_t.data_ptr()), ctypes.c_void_p(perm.data_ptr()),
                                        ctypes.c_void_p(off.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
        assert rc == _abi.AC_OK, _abi.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(perm, perm_ref), f"call {call}: permutation differs"
        assert torch.equal(off, off_ref), f"call {call}: offsets differ"
    ref_ctx.close()


def test_static_sort_rejects_oversize_without_launching():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import _abi
    lib = _abi.load()
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    # 64 heads x 1M tokens needs far more than the 16 MiB of static scratch
    rc = lib.ac_cluster_sort_static(p, 64, 1 << 20, 500, None, p, p, None)
    assert rc == _abi.AC_ERR_UNSUPPORTED
    assert lib.ac_cluster_sort_static(None, 1, 10, 4, None, p, p, None) == _abi.AC_ERR_INVALID_ARG
    torch.cuda.synchronize()
