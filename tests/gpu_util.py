"""Helpers for the GPU parity tests (inputs to the device, excused near-ties)."""
from __future__ import annotations

import numpy as np

from clustered_sparse_attention_head_b200 import workloads as W

# Tolerances for the attention output (bf16 or tf32 inputs, fp32 accumulation).
ATT_MAX_ABS = 2e-2
ATT_MEAN_ABS = 2e-3
CENT_RTOL = 1e-5
TIE_REL = 1e-6


def to_dev(a: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def stack_heads(w, heads=None):
    hs = [W.head_inputs(w, h) for h in (range(w.heads) if heads is None else heads)]
    q = np.stack([h.q for h in hs])
    k = np.stack([h.k for h in hs])
    v = np.stack([h.v for h in hs])
    return q, k, v


def excused_assign_mismatch(orc, xs, cent, mode, i, a_gpu, a_orc):
    """A mismatch is excused only when the two candidates' exact scores differ
    by less than TIE_REL relative (double precision, oracle arithmetic)."""
    _, _, _ = None, None, None
    s = []
    for j in (a_gpu, a_orc):
        c = cent[j].astype(np.float64)
        if mode == orc.EUCLID:
            s.append(float(((xs[i] - c) ** 2).sum()))
        else:
            s.append(float(xs[i] @ c))
    den = max(abs(s[0]), abs(s[1]), 1e-300)
    return abs(s[0] - s[1]) / den < TIE_REL


def assert_assign_equal(orc, xs, cent, mode, got, ref, what):
    bad = np.nonzero(got != ref)[0]
    unexcused = [i for i in bad if not excused_assign_mismatch(orc, xs, cent, mode, i, int(got[i]), int(ref[i]))]
    if len(bad):
        print(f"{what}: {len(bad)} mismatches, {len(bad) - len(unexcused)} excused near-ties")
    assert not unexcused, f"{what}: {len(unexcused)} unexcused assignment mismatches, e.g. rows {unexcused[:8]}"


def attn_close(got: np.ndarray, ref: np.ndarray, what: str):
    err = np.abs(got.astype(np.float64) - ref)
    print(f"{what}: max-abs {err.max():.3e} mean-abs {err.mean():.3e}")
    assert err.max() <= ATT_MAX_ABS, f"{what}: max-abs {err.max()}"
    assert err.mean() <= ATT_MEAN_ABS, f"{what}: mean-abs {err.mean()}"
