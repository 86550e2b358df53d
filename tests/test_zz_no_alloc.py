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


def _static_sort(lib, ids_t, heads, n, cap, ncl_t, perm_fill=-1):
    from clustered_sparse_attention_head_b200 import _abi
    perm = torch.full((heads, n), perm_fill, dtype=torch.int32, device="cuda")
    off = torch.full((heads, cap + 1), -1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    rc = lib.ac_cluster_sort_static(ctypes.c_void_p(ids_t.data_ptr()), heads, n, cap,
                                    ctypes.c_void_p(ncl_t.data_ptr()) if ncl_t is not None else None,
                                    ctypes.c_void_p(perm.data_ptr()), ctypes.c_void_p(off.data_ptr()),
                                    ctypes.c_void_p(stream.cuda_stream))
    assert rc == _abi.AC_OK, _abi.status_string(rc)
    torch.cuda.synchronize()
    return perm.cpu().numpy(), off.cpu().numpy()


def _expected(ids, ncl_h, cap, n):
    """Stable sort of the tokens whose id lies in [0, min(ncl, cap)), and the
    cluster offsets; the perm slots past the valid tokens stay unwritten."""
    k = min(max(int(ncl_h), 0), cap)
    valid = np.nonzero((ids >= 0) & (ids < k))[0]
    order = valid[np.argsort(ids[valid], kind="stable")].astype(np.int32)
    cnt = np.bincount(ids[valid], minlength=cap)[:cap]
    off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    return order, off


def test_static_sort_large_cap_matches_workspace_sort():
    """cap = 4096 needs 64 KiB of shared memory per sorting block (above the
    48 KiB default), on a small n; two calls in a row."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import _abi, build
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    build()
    lib = _abi.load()
    heads, n, cap = 2, 4099, 4096  # a context needs n >= its cluster count
    ncl = np.array([4096, 3000], np.int32)
    ref_ctx = AdaCluster(Config(heads=heads, n=n, d=64, kq=cap, kk=cap))
    ncl_t = torch.from_numpy(ncl).cuda()
    rng = np.random.default_rng(11)
    for call in range(2):
        ids = _ids(rng, heads, n, ncl)
        ids_t = torch.from_numpy(ids).cuda()
        perm_ref, off_ref = ref_ctx.ac_cluster_sort(ids_t, cap, ncl_t)
        perm, off = _static_sort(lib, ids_t, heads, n, cap, ncl_t)
        np.testing.assert_array_equal(perm, perm_ref.cpu().numpy(), err_msg=f"call {call}")
        np.testing.assert_array_equal(off, off_ref.cpu().numpy(), err_msg=f"call {call}")
        for h in range(heads):
            order, eoff = _expected(ids[h], ncl[h], cap, n)
            np.testing.assert_array_equal(perm[h], order)
            np.testing.assert_array_equal(off[h], eoff)
    ref_ctx.close()


def test_static_sort_byte_limit_boundary():
    """One head with cap = 8192: n = 464,896 needs exactly 16,769,536 bytes of
    the 16 MiB (256 + 256 + 4n + 4 cap + 4 cap ceil(n/1024), each rounded up to
    256), the largest n that fits; n + 1 needs one more histogram tile and is
    refused without a launch."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import _abi, build
    build()
    lib = _abi.load()
    cap, n = 8192, 464896
    need = 256 + 256 + 4 * n + 4 * cap + 4 * cap * (-(-n // 1024))
    assert need <= 16 << 20
    assert 256 + 256 + 4 * (n + 1) + 4 * cap + 4 * cap * (-(-(n + 1) // 1024)) > 16 << 20
    rng = np.random.default_rng(3)
    ids = rng.integers(0, cap, (1, n)).astype(np.int32)
    ids_t = torch.from_numpy(ids).cuda()
    ncl_t = torch.tensor([cap], dtype=torch.int32, device="cuda")
    perm, off = _static_sort(lib, ids_t, 1, n, cap, ncl_t)
    order, eoff = _expected(ids[0], cap, cap, n)
    np.testing.assert_array_equal(perm[0], order)
    np.testing.assert_array_equal(off[0], eoff)
    big = torch.zeros((1, n + 1), dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(big.data_ptr())
    assert lib.ac_cluster_sort_static(p, 1, n + 1, cap, ctypes.c_void_p(ncl_t.data_ptr()), p, p, None) == \
        _abi.AC_ERR_UNSUPPORTED
    assert lib.ac_cluster_sort_static(p, 1, 16, 8193, None, p, p, None) == _abi.AC_ERR_UNSUPPORTED
    torch.cuda.synchronize()


def test_static_sort_ids_beyond_counts():
    """ids in [ncl[h], cap) and above cap are skipped: the sort covers only the
    valid ids and leaves the perm slots past them unwritten; a count above cap
    is clamped to cap.  Compared with a host stable sort, two calls in a row."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import _abi, build
    build()
    lib = _abi.load()
    heads, n, cap = 3, 2049, 64
    ncl = np.array([40, cap + 5, 0], np.int32)
    ncl_t = torch.from_numpy(ncl).cuda()
    rng = np.random.default_rng(19)
    for call in range(2):
        ids = rng.integers(0, cap + 5, (heads, n)).astype(np.int32)
        ids_t = torch.from_numpy(ids).cuda()
        perm, off = _static_sort(lib, ids_t, heads, n, cap, ncl_t, perm_fill=-7)
        for h in range(heads):
            order, eoff = _expected(ids[h], ncl[h], cap, n)
            nv = len(order)
            np.testing.assert_array_equal(perm[h, :nv], order, err_msg=f"call {call} head {h}")
            assert (perm[h, nv:] == -7).all(), f"call {call} head {h}: slots past the valid ids were written"
            np.testing.assert_array_equal(off[h], eoff, err_msg=f"call {call} head {h}")
