"""Host model of the tensor-core assignment screen's decision rule.

The bf16 screen (csrc/ac_assign_tc.cu) scores rows against split-bf16
centroids in fp32, shifts each score by a per-row constant, packs the column
index into the low mantissa bits, keeps the three smallest keys and decides a
row only when the best key is clear of the second by twice its error bound
plus the packing bound.  This test re-states that rule in numpy (fp32 products
and sums, the same shift, packing and margins) and checks, on adversarial
inputs, the property the exact pass relies on: every decided row has the exact
winner (AdaCluster §3.1 and §3.2.1: largest q_hat.mu, closest centroid, ties to
the lowest id), and a row sent on with two candidates has the exact winner among
them.  Inputs include scales where fp32 underflows (norms near 1e-20), which
only the absolute slack of the bound covers."""
import numpy as np
import pytest

EUCLID, SPHERE = 0, 1


def _bf16(a):
    """Round float32 to bf16 (nearest even), returned as float32."""
    b = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32)


def _screen(x, cent, mode, slack=True):
    """(decided, i1, i2, two) per row, following the kernel's arithmetic."""
    n, d = x.shape
    k = cent.shape[0]
    kpadc = ((k + 127) // 128) * 128
    kb = int(kpadc - 1).bit_length()
    imask = np.uint32((1 << kb) - 1)
    c_hi = _bf16(cent)
    c_lo = _bf16(cent - c_hi)
    # fp32 dot products of the two parts, accumulated in fp32
    dot = (x @ c_hi.T).astype(np.float32) + (x @ c_lo.T).astype(np.float32)
    xn = (np.sqrt((x.astype(np.float64) ** 2).sum(1)) * (1 + 1e-6)).astype(np.float32)
    cn2 = (cent.astype(np.float64) ** 2).sum(1).astype(np.float32)
    cm = np.float32(np.sqrt((cent.astype(np.float64) ** 2).sum(1)).max() * (1 + 1e-6))
    wv = -2.0 if mode == EUCLID else -1.0
    cc = cn2 if mode == EUCLID else np.zeros(k, np.float32)
    t = (wv * dot.astype(np.float64) + cc.astype(np.float64)).astype(np.float32)  # fma, one rounding
    sigma = (xn * xn) if mode == EUCLID else xn
    dd = (t + sigma[:, None]).astype(np.float32)
    cols = (np.float32(2.0 ** 23) + np.arange(k, dtype=np.float32)).view(np.uint32)
    key = ((dd.view(np.uint32) & ~imask) | (cols & imask)).view(np.float32)
    if k >= 3:
        part = np.partition(key, 2, axis=1)[:, :3]
    else:
        part = np.concatenate([key, np.full((n, 3 - k), np.float32(1e30))], axis=1)
    part = np.sort(part, axis=1)
    B1, B2, B3 = part[:, 0], part[:, 1], part[:, 2]
    i1 = (B1.view(np.uint32) & imask).astype(np.int64)
    i2 = (B2.view(np.uint32) & imask).astype(np.int64)
    edot = np.float32(2.0 ** -13) * xn * cm
    if mode == EUCLID:
        E = 2 * edot + np.float32(2.0 ** -22) * (cm * cm + 2 * xn * cm)
    else:
        E = edot
    if slack:
        E = E + np.float32(2.0 ** -100)
    rho = np.float32(2.0 ** (kb - 22))
    decided = (B2 - B1) > 2 * E + rho * (np.abs(B1) + np.abs(B2))
    two = (B3 - B1) > 2 * E + rho * (np.abs(B1) + np.abs(B3))
    if k <= 1:
        decided[:] = True
    return decided, i1, i2, two


def _exact(x, cent, mode):
    """Exact winner in double (ties to the lowest id) and the gap to the runner-up."""
    xd, cd = x.astype(np.float64), cent.astype(np.float64)
    if mode == EUCLID:
        s = (xd * xd).sum(1)[:, None] - 2 * xd @ cd.T + (cd * cd).sum(1)[None, :]
    else:
        s = -(xd @ cd.T)
    win = np.argmin(s, axis=1)
    srt = np.sort(s, axis=1)
    return win, srt[:, 1] - srt[:, 0], s


def _adversarial(n, d, k, seed, scale):
    rng = np.random.default_rng(seed)
    centres = rng.standard_normal((16, d)) * 2.0
    base = _bf16(centres[rng.integers(0, 16, k)] + rng.standard_normal((k, d)))
    for lo in range(0, 12):
        base[k - 1 - lo] = base[lo]          # exact duplicates
    near = np.arange(12, 44)
    for lo in near:                          # near-duplicates: one bf16 ulp apart in one element
        b = base[lo].copy().view(np.uint32)
        b[lo % d] += np.uint32(1 << 16)
        base[k - 1 - lo] = b.view(np.float32)
    q = n // 6
    # far rows: the higher-id centroid of a near-duplicate pair moved 3000
    # along another axis.  Both squared distances are large, so the packing
    # step exceeds 2E; when both keys fall in one step, the packed index puts
    # the lower id (the loser) first, and only the packing bound keeps the row
    # from being decided.
    far_lo = near[rng.integers(0, len(near), n - 5 * q)]
    far = base[k - 1 - far_lo].copy()
    far[np.arange(len(far_lo)), (far_lo % d + 1) % d] += 3000.0
    rows = np.concatenate([
        _bf16(centres[rng.integers(0, 16, q)] + rng.standard_normal((q, d))),   # ordinary rows first
        base[rng.integers(0, k, q)],                                       # copies of centroids
        _bf16(0.5 * (base[rng.integers(0, k, q)] + base[rng.integers(0, k, q)])),  # midpoints
        _bf16(base[rng.integers(0, k, q)] + 1e-3 * rng.standard_normal((q, d))),
        # rows right next to a near-duplicate pair: the exact gap is far below
        # the fp32 error of the scores
        _bf16(base[near[rng.integers(0, len(near), q)]] + 1e-2 * rng.standard_normal((q, d))),
        _bf16(far),
    ]).astype(np.float32)
    s = np.float32(scale)
    return _bf16(rows * s), (base * s).astype(np.float32)


@pytest.mark.parametrize("mode", [EUCLID, SPHERE])
@pytest.mark.parametrize("scale", [1.0, 2.0 ** 40, 2.0 ** -70])
@pytest.mark.parametrize("k", [200, 700])
def test_decided_rows_have_the_exact_winner(mode, scale, k):
    x, cent = _adversarial(2000, 64, k, seed=k + int(np.log2(scale)) + 7 * mode, scale=scale)
    if mode == SPHERE:
        nrm = np.sqrt((cent.astype(np.float64) ** 2).sum(1, keepdims=True))
        cent = (cent / nrm).astype(np.float32)
    decided, i1, i2, two = _screen(x, cent, mode)
    win, gap, _ = _exact(x, cent, mode)
    assert np.all(gap[decided] > 0), "a decided row has an exact tie"
    bad = np.nonzero(decided & (i1 != win))[0]
    assert len(bad) == 0, f"{len(bad)} decided rows with the wrong winner, e.g. {bad[:5]}"
    sent_two = ~decided & two
    assert np.all((win[sent_two] == i1[sent_two]) | (win[sent_two] == i2[sent_two]))
    # the screen still decides most ordinary rows (the first sixth)
    if scale == 1.0:
        assert decided[:len(x) // 6].mean() > 0.5


def test_underflow_needs_the_absolute_slack():
    """At norms near 1e-20 the fp32 products are subnormal; with the relative
    bound alone the model decides rows whose keys have lost their order, while
    the absolute 2^-100 sends them on."""
    x, cent = _adversarial(2000, 64, 200, seed=3, scale=2.0 ** -70)
    win, _, _ = _exact(x, cent, EUCLID)
    d0, i0, _, _ = _screen(x, cent, EUCLID, slack=False)
    d1, i1, _, _ = _screen(x, cent, EUCLID, slack=True)
    assert np.any(d0 & (i0 != win)), "the inputs no longer reach fp32 underflow"
    assert not np.any(d1 & (i1 != win))
