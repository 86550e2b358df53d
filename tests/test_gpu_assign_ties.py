"""Assignment screen under adversarial near-ties (bf16 rows, tensor-core screen).

The screen scores rows against centroids in fp32 and sends every row whose two
best scores lie within its error bound to the exact double pass.  These inputs
put many rows on or next to that boundary:
* centroids that are exact duplicates of other centroids (exact ties, which the
  k-means of AdaCluster §3.1 breaks towards the lowest id),
* rows equal to a centroid (distance 0, cosine 1),
* rows at the bf16-rounded midpoint of two centroids,
* zero rows (every centroid ties in the query mode),
at centroid counts whose index needs 9 and 11 bits.  Every assignment must equal
the oracle's; a mismatch is excused only between two candidates whose exact
scores differ by less than 1e-6 relative, and not at all on an exact tie."""
import numpy as np
import pytest

from gpu_util import assert_assign_equal

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from clustered_sparse_attention_head_b200 import build
    build()


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def _inputs(n, d, k, seed):
    """Rows and centroids (float32 holding bf16 values), and the duplicate pairs."""
    rng = np.random.default_rng(seed)
    centres = rng.standard_normal((32, d)) * 2.0
    base = _bf16(centres[rng.integers(0, 32, k)] + rng.standard_normal((k, d)))
    dups = []
    for lo in rng.choice(k // 2, 24, replace=False):
        hi = int(rng.integers(k // 2, k))
        if hi not in [h for _, h in dups]:
            base[hi] = base[lo]
            dups.append((int(lo), hi))
    n4 = n // 4
    rows = np.empty((n, d), np.float32)
    rows[:n4] = _bf16(centres[rng.integers(0, 32, n4)] + rng.standard_normal((n4, d)))
    # copies of centroids, the duplicated ones first
    pick = np.concatenate([[lo for lo, _ in dups], rng.integers(0, k, n4 - len(dups))])
    rows[n4:2 * n4] = base[pick]
    # midpoints of random centroid pairs, rounded to bf16
    a, b = rng.integers(0, k, n4), rng.integers(0, k, n4)
    rows[2 * n4:3 * n4] = _bf16(0.5 * (base[a] + base[b]))
    # midpoints of the duplicated centroids and their nearest other centroid's
    # copy, and zero rows
    rest = n - 3 * n4
    rows[3 * n4:] = 0.0
    m = min(rest // 2, len(dups))
    for i in range(m):
        lo, _ = dups[i]
        other = (lo + 1) % k
        rows[3 * n4 + i] = _bf16(0.5 * (base[lo] + base[other]))
    copies = np.arange(n4, n4 + len(dups))
    return rows, base, dups, copies


@pytest.mark.parametrize("k", [300, 1500])
@pytest.mark.parametrize("mode", ["q", "k"])
def test_assign_near_ties(orc, k, mode):
    from clustered_sparse_attention_head_b200.api import AdaCluster, Config
    n, d = 4000, 128
    rows, base, dups, copies = _inputs(n, d, k, seed=21 + k)
    om = orc.SPHERE if mode == "q" else orc.EUCLID
    if mode == "q":
        cent = (base / np.linalg.norm(base.astype(np.float64), axis=1, keepdims=True)).astype(np.float32)
    else:
        cent = base.astype(np.float32)
    xs, _ = orc.prepare(rows, om)
    ref, _, _ = orc.assign(xs, cent, om)
    ctx = AdaCluster(Config(heads=1, n=n, d=d, dtype="bf16", kq=k, kk=k, iters=0))
    x_dev = torch.from_numpy(rows[None]).cuda().to(torch.bfloat16)
    fn = ctx.ac_cluster_q if mode == "q" else ctx.ac_cluster_k
    out = fn(x_dev, init_cent=torch.from_numpy(cent[None]).cuda())
    torch.cuda.synchronize()
    assert ctx.get_status() == 0
    got = out["assign"][0].cpu().numpy()
    # exact ties: the copies of duplicated centroids go to the lower id, on
    # both sides, with no excuse
    for (lo, hi), r in zip(dups, copies):
        assert ref[r] <= lo, (lo, hi, ref[r])
        assert got[r] == ref[r], f"row {r} (copy of centroids {lo} = {hi}): gpu {got[r]}, oracle {ref[r]}"
    if mode == "q":
        zero = np.nonzero(~rows.any(axis=1))[0]
        assert len(zero) > 0
        assert (ref[zero] == 0).all() and (got[zero] == 0).all()
    assert_assign_equal(orc, xs, cent, om, got, ref, f"ties/{mode}/k{k}")
    np.testing.assert_array_equal(out["count"][0, :k].cpu().numpy(), np.bincount(got, minlength=k))
    ctx.close()
