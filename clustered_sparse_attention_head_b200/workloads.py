"""Seeded synthetic attention inputs shaped like video-DiT attention layers.

This module only draws random inputs and names the clustering parameters of
each workload; it holds none of the method's arithmetic, so both the CUDA path
and the CPU oracle consume its output.

Recipe (numpy ``default_rng``; one spawned sub-stream per head, in head order):
  * Q, K and V of a token share one mixture-component id; Q and K (and V for the
    fp32 case) use independent component means ~ N(0, I_d) and add 0.3 * N(0, I_d).
  * Component ids follow spatio-temporal patches of the latent grid: token
    (t, y, x) lies in patch (t // e_t, y // e_y, x // e_x); the patch's
    component is perm[patch] mod n_comp for a seeded permutation perm.
  * Text tokens (appended after the video tokens) and V in the bf16 workloads
    are iid N(0, 1).  The 75.6K-token workload replaces 5% of tokens in Q and K
    by U(-3, 3)^d outliers.
  * bf16 workloads are rounded to bf16 (round to nearest even) and returned both
    as uint16 bit patterns and as the exactly equal float32 values.

The five workloads mirror CogVideoX-2B, Wan-2.1 and HunyuanVideo attention
shapes; the prompt sets and model weights the paper measured with are not
available, so these inputs stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# Clustering-rule ids shared with the C-ABI (ac_tau_rule).
TAU_ABS, TAU_MEAN_X, TAU_MEDIAN_RADIUS_X = 0, 1, 2


@dataclass(frozen=True)
class Workload:
    name: str
    heads: int
    grid: tuple | None      # (T, H, W) latent grid, or None for iid components
    text: int               # text tokens appended after the video tokens
    d: int
    dtype: str              # "f32" or "bf16"
    n_comp: int | tuple     # mixture components (tuple = per-head 2**u range)
    patch: tuple | None     # patch edges (e_t, e_y, e_x)
    outlier_frac: float
    kq: int
    kk: int
    iters: int
    top_p: float
    adaptive_q: bool = False
    adaptive_k: bool = False
    tau_rule: int = TAU_ABS
    tau_value: float = 0.0
    nmax_q: int = 0
    nmax_k: int = 0
    seed: int = 0
    n_iid: int = 2048        # video tokens when grid is None

    @property
    def n(self) -> int:
        base = int(np.prod(self.grid)) if self.grid is not None else self.n_iid
        return base + self.text

    def dense_flops(self) -> float:
        return 4.0 * self.d * float(self.n) ** 2 * self.heads


WORKLOADS = {
    "gmm16-n2048-d64-f32": Workload(
        "gmm16-n2048-d64-f32", 1, None, 0, 64, "f32", 16, None, 0.0, 32, 64, 10, 0.9, seed=0),
    "cogvideox2b-n17776-h30-d64": Workload(
        "cogvideox2b-n17776-h30-d64", 30, (13, 30, 45), 226, 64, "bf16", 256, (4, 4, 6), 0.0,
        100, 200, 10, 0.9, seed=1),
    "cogvideox2b720p-n70000-h30-d64-adaptive": Workload(
        "cogvideox2b720p-n70000-h30-d64-adaptive", 30, (25, 40, 70), 0, 64, "bf16", 256, (7, 5, 9), 0.0,
        100, 200, 10, 0.9, adaptive_k=True, tau_rule=TAU_MEDIAN_RADIUS_X, tau_value=0.5,
        nmax_k=1600, seed=2),
    "wan21-n75600-h40-d128": Workload(
        "wan21-n75600-h40-d128", 40, (21, 45, 80), 0, 128, "bf16", 512, (6, 6, 5), 0.05,
        250, 500, 10, 0.9, seed=3),
    "hunyuan720p-n119056-h24-d128-adaptive": Workload(
        "hunyuan720p-n119056-h24-d128-adaptive", 24, (33, 45, 80), 256, 128, "bf16", (6, 10), (3, 5, 5),
        0.0, 65, 256, 10, 0.9, adaptive_q=True, adaptive_k=True, tau_rule=TAU_MEAN_X, tau_value=1.5,
        nmax_q=520, nmax_k=2048, seed=4),
}
ORDER = list(WORKLOADS)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _components(w: Workload, rng: np.random.Generator, n_comp: int) -> np.ndarray:
    if w.grid is None:
        return rng.integers(0, n_comp, size=w.n - w.text)
    T, Hh, W = w.grid
    et, ey, ex = w.patch
    pt, py, px = -(-T // et), -(-Hh // ey), -(-W // ex)
    perm = rng.permutation(pt * py * px)
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(W), indexing="ij")
    patch = ((t // et) * py + (y // ey)) * px + (x // ex)
    return (perm[patch.reshape(-1)] % n_comp).astype(np.int64)


@dataclass
class HeadInputs:
    q: np.ndarray           # float32 [n, d] (bf16-exact for bf16 workloads)
    k: np.ndarray
    v: np.ndarray
    comp: np.ndarray        # component id per video token


def head_inputs(w: Workload, h: int) -> HeadInputs:
    """Inputs of head h (independent of which other heads are generated)."""
    root = np.random.default_rng(w.seed)
    hr = root.spawn(w.heads)[h]
    if isinstance(w.n_comp, tuple):
        lo, hi = w.n_comp
        n_comp = int(2 ** hr.integers(lo, hi + 1))
    else:
        n_comp = int(w.n_comp)
    d, nv = w.d, w.n - w.text
    comp = _components(w, hr, n_comp)
    mq = hr.standard_normal((n_comp, d), dtype=np.float32)
    mk = hr.standard_normal((n_comp, d), dtype=np.float32)
    q = mq[comp] + np.float32(0.3) * hr.standard_normal((nv, d), dtype=np.float32)
    k = mk[comp] + np.float32(0.3) * hr.standard_normal((nv, d), dtype=np.float32)
    if w.dtype == "f32":
        mv = hr.standard_normal((n_comp, d), dtype=np.float32)
        v = mv[comp] + np.float32(0.3) * hr.standard_normal((nv, d), dtype=np.float32)
    else:
        v = hr.standard_normal((nv, d), dtype=np.float32)
    if w.outlier_frac > 0:
        m = int(round(w.outlier_frac * nv))
        idx = hr.choice(nv, size=m, replace=False)
        q[idx] = hr.uniform(-3.0, 3.0, size=(m, d)).astype(np.float32)
        k[idx] = hr.uniform(-3.0, 3.0, size=(m, d)).astype(np.float32)
    if w.text:
        q = np.concatenate([q, hr.standard_normal((w.text, d), dtype=np.float32)])
        k = np.concatenate([k, hr.standard_normal((w.text, d), dtype=np.float32)])
        v = np.concatenate([v, hr.standard_normal((w.text, d), dtype=np.float32)])
    if w.dtype == "bf16":
        q, k, v = (bf16_bits_to_f32(to_bf16_bits(a)) for a in (q, k, v))
    return HeadInputs(np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v), comp)


def step_inputs(w: Workload, h: int, step: int, drift: float = 0.02) -> HeadInputs:
    """Inputs of head h at denoising step `step`, standing in for consecutive
    denoising steps, whose token distributions drift little.  Step 0 is
    head_inputs(w, h); each later step adds drift * N(0, I) to the previous
    step's q, k and v (one seeded stream per (workload seed, head, step)) and
    rounds to bf16 again for bf16 workloads."""
    base = head_inputs(w, h)
    q, k, v = base.q, base.k, base.v
    for s in range(1, step + 1):
        r = np.random.default_rng([w.seed, h, s, 7919])
        f = np.float32(drift)
        q = q + f * r.standard_normal(q.shape, dtype=np.float32)
        k = k + f * r.standard_normal(k.shape, dtype=np.float32)
        v = v + f * r.standard_normal(v.shape, dtype=np.float32)
        if w.dtype == "bf16":
            q, k, v = (bf16_bits_to_f32(to_bf16_bits(a)) for a in (q, k, v))
    return HeadInputs(np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v), base.comp)


def small(w: Workload, n: int, heads: int = 1, seed: int = 0, **over) -> Workload:
    """A reduced copy of workload w: n video tokens with iid mixture components
    and no text tokens, for tests that must finish in seconds."""
    from dataclasses import replace
    kw = dict(name=f"{w.name}-small{n}", heads=heads, grid=None, text=0, patch=None, seed=seed, n_iid=n)
    kw.update(over)
    return replace(w, **kw)
