"""The seeded synthetic inputs follow their stated recipe (one head of every
workload, at full size): shapes, bf16 exactness, the patch structure of the
component ids on the latent grid, the iid text tokens, the outlier share, and
determinism per head."""
import numpy as np
import pytest

from clustered_sparse_attention_head_b200 import workloads as W


@pytest.fixture(scope="module", params=W.ORDER)
def wh(request):
    w = W.WORKLOADS[request.param]
    return w, W.head_inputs(w, w.heads - 1)


def test_shapes_and_dtype(wh):
    w, hi = wh
    for a in (hi.q, hi.k, hi.v):
        assert a.shape == (w.n, w.d) and a.dtype == np.float32 and np.isfinite(a).all()
    assert hi.comp.shape == (w.n - w.text,)
    if w.dtype == "bf16":
        for a in (hi.q, hi.k, hi.v):
            assert not (a.view(np.uint32) & np.uint32(0xFFFF)).any(), "not bf16-exact"


def test_components_follow_the_patches(wh):
    w, hi = wh
    if w.grid is None:
        return
    T, H, Wd = w.grid
    et, ey, ex = w.patch
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(Wd), indexing="ij")
    patch = (((t // et) * -(-H // ey) + (y // ey)) * -(-Wd // ex) + (x // ex)).reshape(-1)
    # every patch carries one component id
    first = np.full(patch.max() + 1, -1)
    first[patch[::-1]] = hi.comp[::-1]
    assert (first[patch] == hi.comp).all()


def test_text_tokens_are_iid_standard_normal(wh):
    w, hi = wh
    if not w.text:
        return
    txt = np.concatenate([hi.q[-w.text:], hi.k[-w.text:], hi.v[-w.text:]]).astype(np.float64)
    assert abs(txt.mean()) < 0.02 and abs(txt.std() - 1.0) < 0.02


def test_outlier_share(wh):
    """Outlier rows are U(-3, 3)^d: no element beyond 3 in magnitude, and a
    mean square of 3; mixture rows have a mean square near 1.09 (unit means
    plus 0.3 noise).  The share of rows with mean square above 2 matches the
    configured outlier fraction."""
    w, hi = wh
    nv = w.n - w.text
    ms = (hi.k[:nv].astype(np.float64) ** 2).mean(axis=1)
    share = (ms > 2.0).mean()
    assert abs(share - w.outlier_frac) < 0.005
    if w.outlier_frac > 0:
        assert np.abs(hi.k[:nv][ms > 2.0]).max() <= 3.0


def test_heads_are_deterministic_and_independent():
    w = W.WORKLOADS["cogvideox2b-n17776-h30-d64"]
    a = W.head_inputs(w, 7)
    W.head_inputs(w, 3)
    b = W.head_inputs(w, 7)
    c = W.head_inputs(w, 8)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k, b.k) and np.array_equal(a.v, b.v)
    assert not np.array_equal(a.q, c.q)


def test_bf16_rounding_is_nearest_even():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130, 0.0, -0.0])])
    ours = W.bf16_bits_to_f32(W.to_bf16_bits(x))
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
