"""Python front end of the C ABI with the same call names (ac_cluster_q, ...).

``AdaCluster`` owns one ``ac_ctx`` and a workspace tensor.  Each method passes
torch CUDA tensors straight to the matching C call; outputs are allocated with
torch (device memory is torch's, the work is the library's kernels).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _abi
from ._abi import check, ptr, stream_ptr


@dataclass
class Config:
    heads: int
    n: int
    d: int
    dtype: str = "bf16"          # "bf16" | "f32"
    kq: int = 100
    kk: int = 200
    iters: int = 10
    adaptive_q: bool = False
    adaptive_k: bool = False
    tau_rule: int = _abi.AC_TAU_ABS
    tau_value: float = 0.0
    nmax_q: int = 0
    nmax_k: int = 0
    top_p: float = 0.9
    flags: int = 0
    score_mode: int = _abi.AC_SCORE_CENTROID   # or AC_SCORE_QUEST
    top_k: int = 0                             # > 0: argtopk instead of top-p
    text_keys: int = 0                         # > 0: last text_keys keys always attended, not clustered
    per_query: bool = False                    # selection per query row (argtopk along each row of S)

    def to_c(self) -> _abi.ac_config:
        return _abi.ac_config(self.heads, self.n, self.d, _abi.AC_BF16 if self.dtype == "bf16" else _abi.AC_F32,
                              self.kq, self.kk, self.iters, int(self.adaptive_q), int(self.adaptive_k),
                              self.tau_rule, float(self.tau_value), self.nmax_q, self.nmax_k, float(self.top_p),
                              self.flags, int(self.score_mode), int(self.top_k), int(self.text_keys),
                              int(self.per_query))

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @staticmethod
    def from_workload(w) -> "Config":
        return Config(heads=w.heads, n=w.n, d=w.d, dtype=w.dtype, kq=w.kq, kk=w.kk, iters=w.iters,
                      adaptive_q=w.adaptive_q, adaptive_k=w.adaptive_k, tau_rule=w.tau_rule,
                      tau_value=w.tau_value, nmax_q=w.nmax_q, nmax_k=w.nmax_k, top_p=w.top_p)


class AdaCluster:
    def __init__(self, cfg: Config, device="cuda", workspace: torch.Tensor | None = None):
        self.cfg = cfg
        self.lib = _abi.load()
        self._ctx = ctypes.c_void_p()
        c = cfg.to_c()
        check("ac_create", self.lib.ac_create(ctypes.byref(c), ctypes.byref(self._ctx)))
        kq, kk = ctypes.c_int(), ctypes.c_int()
        check("ac_capacities", self.lib.ac_capacities(self._ctx, ctypes.byref(kq), ctypes.byref(kk)))
        self.kq_cap, self.kk_cap = kq.value, kk.value
        nb = ctypes.c_size_t()
        check("ac_workspace_size", self.lib.ac_workspace_size(self._ctx, ctypes.byref(nb)))
        self.ws_bytes = nb.value
        self.device = torch.device(device)
        self.ws = workspace if workspace is not None else torch.empty(self.ws_bytes + 256, dtype=torch.uint8,
                                                                      device=self.device)
        off = (-self.ws.data_ptr()) % 256
        self._ws = self.ws[off:off + self.ws_bytes]

    def close(self):
        if self._ctx:
            self.lib.ac_destroy(self._ctx)
            self._ctx = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # --------------------------------------------------------------- helpers
    def _i32(self, *shape):
        return torch.empty(*shape, dtype=torch.int32, device=self.device)

    def _f32(self, *shape):
        return torch.empty(*shape, dtype=torch.float32, device=self.device)

    def _args_ws(self):
        return ptr(self._ws), ctypes.c_size_t(self.ws_bytes)

    def profile_read(self) -> dict:
        p = _abi.ac_profile()
        check("ac_profile_read", self.lib.ac_profile_read(self._ctx, ctypes.byref(p)))
        return {f: getattr(p, f) for f, _ in _abi.ac_profile._fields_}

    def get_status(self, stream=None) -> int:
        return self.lib.ac_get_status(self._ctx, stream_ptr(stream))

    # ------------------------------------------------------------ the calls
    def ac_cluster_q(self, q, init_cent=None, stream=None):
        H, N, D = self.cfg.heads, self.cfg.n, self.cfg.d
        out = dict(assign=self._i32(H, N), cent=self._f32(H, self.kq_cap, D).zero_(),
                   count=self._i32(H, self.kq_cap), mean_norm=self._f32(H, self.kq_cap), nclusters=self._i32(H),
                   dense_flag=torch.empty(H, dtype=torch.uint8, device=self.device))
        ws, nb = self._args_ws()
        check("ac_cluster_q", self.lib.ac_cluster_q(
            self._ctx, ptr(q), ptr(init_cent), ptr(out["assign"]), ptr(out["cent"]), ptr(out["count"]),
            ptr(out["mean_norm"]), ptr(out["nclusters"]), ptr(out["dense_flag"]), ws, nb, stream_ptr(stream)))
        return out

    def ac_cluster_k(self, k, init_cent=None, stream=None):
        H, N, D = self.cfg.heads, self.cfg.n, self.cfg.d
        out = dict(assign=self._i32(H, N), cent=self._f32(H, self.kk_cap, D).zero_(),
                   count=self._i32(H, self.kk_cap), nclusters=self._i32(H),
                   dense_flag=torch.empty(H, dtype=torch.uint8, device=self.device))
        ws, nb = self._args_ws()
        check("ac_cluster_k", self.lib.ac_cluster_k(
            self._ctx, ptr(k), ptr(init_cent), ptr(out["assign"]), ptr(out["cent"]), ptr(out["count"]),
            ptr(out["nclusters"]), ptr(out["dense_flag"]), ws, nb, stream_ptr(stream)))
        return out

    def ac_select(self, q_cent, q_mean_norm, q_count, k_cent, k_count, nq=None, nk=None, dense_flag=None,
                  k_max=None, k_min=None, stream=None):
        H = self.cfg.heads
        sel = torch.full((H, self.kq_cap, self.kk_cap), -1, dtype=torch.int32, device=self.device)
        cnt = self._i32(H, self.kq_cap)
        ws, nb = self._args_ws()
        check("ac_select", self.lib.ac_select(
            self._ctx, ptr(q_cent), ptr(q_mean_norm), ptr(q_count), ptr(k_cent), ptr(k_count), ptr(k_max),
            ptr(k_min), ptr(nq), ptr(nk), ptr(dense_flag), ptr(sel), ptr(cnt), ws, nb, stream_ptr(stream)))
        return sel, cnt

    def ac_key_bounds(self, k, k_assign, nk=None, stream=None):
        H, D = self.cfg.heads, self.cfg.d
        kmax, kmin = self._f32(H, self.kk_cap, D), self._f32(H, self.kk_cap, D)
        ws, nb = self._args_ws()
        check("ac_key_bounds", self.lib.ac_key_bounds(self._ctx, ptr(k), ptr(k_assign), ptr(nk), ptr(kmax),
                                                      ptr(kmin), ws, nb, stream_ptr(stream)))
        return kmax, kmin

    def ac_select_rows(self, q, k_count, k_cent=None, nk=None, dense_flag=None, k_max=None, k_min=None,
                       stream=None):
        """Per-query selection: each query row's top_k key clusters as a bit
        set [H, N, W] (int32 words, W = ceil(kk_cap / 32))."""
        H, N = self.cfg.heads, self.cfg.n
        bits = torch.zeros(H, N, (self.kk_cap + 31) // 32, dtype=torch.int32, device=self.device)
        ws, nb = self._args_ws()
        check("ac_select_rows", self.lib.ac_select_rows(
            self._ctx, ptr(q), ptr(k_cent), ptr(k_count), ptr(k_max), ptr(k_min), ptr(nk), ptr(dense_flag),
            ptr(bits), ws, nb, stream_ptr(stream)))
        return bits

    def ac_sparse_attn_rows(self, q, k, v, q_assign, k_assign, row_bits, nq=None, nk=None, dense_flag=None,
                            lse=False, out=None, stream=None):
        H, N, D = self.cfg.heads, self.cfg.n, self.cfg.d
        if out is None:
            out = torch.empty(H, N, D, dtype=self.cfg.torch_dtype, device=self.device)
        lse_t = self._f32(H, N) if lse else None
        ws, nb = self._args_ws()
        check("ac_sparse_attn_rows", self.lib.ac_sparse_attn_rows(
            self._ctx, ptr(q), ptr(k), ptr(v), ptr(q_assign), ptr(k_assign), ptr(row_bits), ptr(nq), ptr(nk),
            ptr(dense_flag), ptr(out), ptr(lse_t), ws, nb, stream_ptr(stream)))
        return (out, lse_t) if lse else out

    def ac_cluster_sort(self, assign, cap, ncl=None, stream=None):
        H, N = self.cfg.heads, self.cfg.n
        perm = self._i32(H, N)
        off = self._i32(H, cap + 1)
        ws, nb = self._args_ws()
        check("ac_cluster_sort", self.lib.ac_cluster_sort(self._ctx, ptr(assign), cap, ptr(ncl), ptr(perm),
                                                          ptr(off), ws, nb, stream_ptr(stream)))
        return perm, off

    def ac_sparse_attn(self, q, k, v, q_assign, k_assign, sel_idx, sel_cnt, nq=None, nk=None, dense_flag=None,
                       lse=False, out=None, stream=None):
        H, N, D = self.cfg.heads, self.cfg.n, self.cfg.d
        if out is None:
            out = torch.empty(H, N, D, dtype=self.cfg.torch_dtype, device=self.device)
        lse_t = self._f32(H, N) if lse else None
        ws, nb = self._args_ws()
        check("ac_sparse_attn", self.lib.ac_sparse_attn(
            self._ctx, ptr(q), ptr(k), ptr(v), ptr(q_assign), ptr(k_assign), ptr(sel_idx), ptr(sel_cnt), ptr(nq),
            ptr(nk), ptr(dense_flag), ptr(out), ptr(lse_t), ws, nb, stream_ptr(stream)))
        return (out, lse_t) if lse else out

    def ac_forward(self, q, k, v, q_cent_io=None, k_cent_io=None, out=None, stats=False, stream=None):
        H, N, D = self.cfg.heads, self.cfg.n, self.cfg.d
        if out is None:
            out = torch.empty(H, N, D, dtype=self.cfg.torch_dtype, device=self.device)
        st = _abi.ac_stats() if stats else None
        ws, nb = self._args_ws()
        check("ac_forward", self.lib.ac_forward(
            self._ctx, ptr(q), ptr(k), ptr(v), ptr(q_cent_io), ptr(k_cent_io), ptr(out),
            ctypes.byref(st) if st is not None else None, ws, nb, stream_ptr(stream)))
        if stats:
            return out, {f: getattr(st, f) for f, _ in _abi.ac_stats._fields_}
        return out

    def capture_forward(self, q, k, v, out=None):
        """One ac_forward call (q, k, v -> out) captured into a CUDA graph that
        the caller owns (to replay it inside a larger graph of its own, say).
        ac_forward itself already replays a cached graph of its launches when a
        call repeats the buffers of an earlier one (include/adacluster.h), so a
        plain loop needs none of this.  Returns (graph, out); graph.replay()
        recomputes out from the buffers' current contents.  The launches keep
        the buffers' addresses, so new inputs are copied into q, k and v.  Only
        for fixed cluster counts: Algorithm 1 (adaptive_q / adaptive_k) reads
        each stage's counts on the host, and neither stats nor profiling can
        run inside a graph."""
        if self.cfg.adaptive_q or self.cfg.adaptive_k:
            raise ValueError("capture_forward: Algorithm 1 (adaptive counts) synchronises with the host per stage")
        if self.cfg.flags & _abi.AC_FLAG_PROFILE:
            raise ValueError("capture_forward: profiling records host-side timings")
        H, N, D = self.cfg.heads, self.cfg.n, self.cfg.d
        if out is None:
            out = torch.empty(H, N, D, dtype=self.cfg.torch_dtype, device=self.device)
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            self.ac_forward(q, k, v, out=out)  # first-call work (attributes, tensor maps) outside the graph
        torch.cuda.current_stream(self.device).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.ac_forward(q, k, v, out=out)
        return graph, out

    def selftest_wait(self, seconds=0.2, stream=None):
        """Runs the bounded-wait diagnostic (a wait that must expire); the next
        get_status() returns AC_ERR_TIMEOUT."""
        check("ac_selftest_wait", self.lib.ac_selftest_wait(self._ctx, float(seconds), stream_ptr(stream)))

    def step_state(self):
        """A zeroed device buffer for ac_forward_step (counts, flags and centres
        carried from one denoising step to the next)."""
        n = ctypes.c_size_t(0)
        check("ac_step_state_size", self.lib.ac_step_state_size(self._ctx, ctypes.byref(n)))
        return torch.zeros(n.value, dtype=torch.uint8, device=self.device)

    def step_state_parts(self, state):
        """Views into a step state: nq, nk (int32 [H]), dq, dk (uint8 [H]),
        q_cent (fp32 [H, kq_cap, d]), k_cent (fp32 [H, kk_cap, d])."""
        parts = (ctypes.c_void_p * 6)()
        check("ac_step_state_parts", self.lib.ac_step_state_parts(self._ctx, ptr(state), parts))
        base = state.data_ptr()
        H, D = self.cfg.heads, self.cfg.d
        kq, kk = self.kq_cap, self.kk_cap
        spec = [("nq", torch.int32, (H,)), ("nk", torch.int32, (H,)), ("dq", torch.uint8, (H,)),
                ("dk", torch.uint8, (H,)), ("q_cent", torch.float32, (H, kq, D)), ("k_cent", torch.float32, (H, kk, D))]
        out = {}
        for (name, dt, shape), p in zip(spec, parts):
            off = p - base
            n = torch.Size(shape).numel() * torch.tensor([], dtype=dt).element_size()
            out[name] = state[off:off + n].view(dt).view(shape)
        return out

    def ac_forward_step(self, step, q, k, v, state, out=None, stats=False, stream=None):
        H, N, D = self.cfg.heads, self.cfg.n, self.cfg.d
        if out is None:
            out = torch.empty(H, N, D, dtype=self.cfg.torch_dtype, device=self.device)
        st = _abi.ac_stats() if stats else None
        ws, nb = self._args_ws()
        check("ac_forward_step", self.lib.ac_forward_step(
            self._ctx, int(step), ptr(q), ptr(k), ptr(v), ptr(state), ptr(out),
            ctypes.byref(st) if st is not None else None, ws, nb, stream_ptr(stream)))
        if stats:
            return out, {f: getattr(st, f) for f, _ in _abi.ac_stats._fields_}
        return out
