"""ctypes binding of libadacluster.so (include/adacluster.h).

Argument marshalling only: every step of the method runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors; their data pointers and the current
CUDA stream are passed through unchanged.  There is no CPU fallback: loading
fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_int, c_int64, c_size_t, c_uint, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libadacluster.so")

AC_OK, AC_ERR_INVALID_ARG, AC_ERR_UNSUPPORTED, AC_ERR_CUDA = 0, 1, 2, 3
AC_ERR_WORKSPACE, AC_ERR_TIMEOUT, AC_ERR_NONFINITE, AC_ERR_CAPACITY = 4, 5, 6, 7
AC_F32, AC_BF16 = 0, 1
AC_TAU_ABS, AC_TAU_MEAN_X, AC_TAU_MEDIAN_RADIUS_X = 0, 1, 2
AC_FLAG_WARM_START, AC_FLAG_CHECK_FINITE, AC_FLAG_PROFILE, AC_FLAG_NO_GRAPH = 1, 2, 4, 8
AC_SCORE_CENTROID, AC_SCORE_QUEST = 0, 1

# every entry point declared in include/adacluster.h
EXPORTS = ["ac_create", "ac_destroy", "ac_capacities", "ac_workspace_size", "ac_cluster_q", "ac_cluster_k",
           "ac_select", "ac_select_rows", "ac_sparse_attn_rows", "ac_key_bounds", "ac_cluster_sort", "ac_cluster_sort_static", "ac_sparse_attn", "ac_forward", "ac_step_state_size", "ac_step_state_parts", "ac_forward_step",
           "ac_profile_read", "ac_get_status", "ac_status_string", "ac_selftest_wait"]


class ac_config(ctypes.Structure):
    _fields_ = [("heads", c_int), ("n", c_int), ("d", c_int), ("dtype", c_int), ("kq", c_int), ("kk", c_int),
                ("iters", c_int), ("adaptive_q", c_int), ("adaptive_k", c_int), ("tau_rule", c_int),
                ("tau_value", c_double), ("nmax_q", c_int), ("nmax_k", c_int), ("top_p", c_double),
                ("flags", c_uint), ("score_mode", c_int), ("top_k", c_int), ("text_keys", c_int),
                ("per_query", c_int)]


class ac_stats(ctypes.Structure):
    _fields_ = [("ms_cluster_q", c_double), ("ms_cluster_k", c_double), ("ms_select", c_double),
                ("ms_sort", c_double), ("ms_attn", c_double), ("ms_total", c_double), ("pairs", c_int64),
                ("dense_heads", c_int), ("max_stages_q", c_int), ("max_stages_k", c_int),
                ("kmeans_rounds_q", c_int), ("kmeans_rounds_k", c_int), ("pairs_computed", c_int64)]


class ac_profile(ctypes.Structure):
    _fields_ = [("calls", c_int), ("ms_cluster_q", c_double), ("ms_cluster_k", c_double), ("ms_select", c_double),
                ("ms_prep", c_double), ("ms_attn_kernel", c_double), ("ms_total", c_double),
                ("launches", ctypes.c_longlong)]


class AcError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__(f"{fn}: {msg} (status {code})")
        self.code = code


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libadacluster.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libadacluster.so not found at {path}; run __graft_entry__.build() first")
    lib = ctypes.CDLL(path)
    P = c_void_p
    sig = {
        "ac_create": ([POINTER(ac_config), POINTER(c_void_p)], c_int),
        "ac_destroy": ([P], None),
        "ac_capacities": ([P, POINTER(c_int), POINTER(c_int)], c_int),
        "ac_workspace_size": ([P, POINTER(c_size_t)], c_int),
        "ac_cluster_q": ([P, P, P, P, P, P, P, P, P, P, c_size_t, P], c_int),
        "ac_cluster_k": ([P, P, P, P, P, P, P, P, P, c_size_t, P], c_int),
        "ac_select": ([P, P, P, P, P, P, P, P, P, P, P, P, P, P, c_size_t, P], c_int),
        "ac_key_bounds": ([P, P, P, P, P, P, P, c_size_t, P], c_int),
        "ac_select_rows": ([P, P, P, P, P, P, P, P, P, P, c_size_t, P], c_int),
        "ac_sparse_attn_rows": ([P, P, P, P, P, P, P, P, P, P, P, P, P, c_size_t, P], c_int),
        "ac_cluster_sort": ([P, P, c_int, P, P, P, P, c_size_t, P], c_int),
        "ac_cluster_sort_static": ([P, c_int, c_int, c_int, P, P, P, P], c_int),
        "ac_sparse_attn": ([P, P, P, P, P, P, P, P, P, P, P, P, P, P, c_size_t, P], c_int),
        "ac_forward": ([P, P, P, P, P, P, P, POINTER(ac_stats), P, c_size_t, P], c_int),
        "ac_step_state_size": ([P, POINTER(c_size_t)], c_int),
        "ac_step_state_parts": ([P, P, P], c_int),
        "ac_forward_step": ([P, c_int, P, P, P, P, P, POINTER(ac_stats), P, c_size_t, P], c_int),
        "ac_profile_read": ([P, POINTER(ac_profile)], c_int),
        "ac_get_status": ([P, P], c_int),
        "ac_selftest_wait": ([P, c_double, P], c_int),
        "ac_status_string": ([c_int], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().ac_status_string(code).decode()


def check(fn: str, code: int):
    if code != AC_OK:
        raise AcError(fn, code, status_string(code))


def ptr(t):
    """Device pointer of a torch tensor (or None)."""
    return None if t is None else c_void_p(t.data_ptr())


def stream_ptr(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)
