"""The eight-term e2m1 encoding of an activation row that the block-scaled
expert products read (the MoE-norm row for gate/up, the f16 SwiGLU row for
down), restated from its definition and checked against the bound the
design's precision reading states.

Encoding of a row v: f0 = 2^floor(log2(6 / max|v|)) brings the largest
magnitude into (3, 6]; term 0 is v f0 rounded to nearest (ties to the even
code) on the e2m1 grid {0, 0.5, 1, 1.5, 2, 3, 4, 6}, saturating at 6; term j
codes the residual the earlier terms left, times f0 4^j, the same way; the
row is sum_j t_j 4^-j / f0.

Bound: term 0 leaves at most one grid unit (spacing 2 near 6), so every
later term sees at most 4 in magnitude and leaves at most half a unit
(spacing 1 in [2, 4]); after eight terms the residual is at most
0.5 4^-7 / f0, i.e. at most 0.5 4^-7 / 3 (about 1.0e-5) of the row's
largest magnitude.  The tests use float64, where every step is exact for
f16 inputs, and also check that nothing is lost when the row is narrow (the
terms then reproduce every f16 value exactly).
"""
import numpy as np

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_rn(x):
    """Round to nearest on the e2m1 grid, ties to the even code, saturating."""
    a = np.minimum(np.abs(x), 6.0)
    d = np.abs(a[..., None] - GRID)
    best = d.min(axis=-1, keepdims=True)
    cand = np.isclose(d, best, rtol=0, atol=0)
    # among equally near grid points, the one with the even code index
    idx = np.where(cand & (np.arange(8) % 2 == 0), np.arange(8), 99).min(axis=-1)
    idx = np.where(idx == 99, np.argmin(d, axis=-1), idx)
    return np.sign(x) * GRID[idx]


def encode(v, n_terms=8):
    mx = np.abs(v).max()
    pe = 0 if mx == 0 else int(np.floor(np.log2(6.0 / mx)))
    f0 = 2.0 ** pe
    r = v.astype(np.float64).copy()
    terms = []
    for j in range(n_terms):
        t = e2m1_rn(r * f0 * 4.0 ** j)
        terms.append(t)
        r = r - t / (f0 * 4.0 ** j)
    approx = sum(t * 4.0 ** -j for j, t in enumerate(terms)) / f0
    return approx, f0, terms


def test_e2m1_rounding_ties_and_saturation():
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -5.0, -0.25, 100.0])
    # ties go to the even code: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2,
    # 2.5 -> 2, 3.5 -> 4, 5 -> 4; above 6 saturates
    want = np.array([0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, -4.0, -0.0, 6.0])
    assert np.array_equal(e2m1_rn(x), want)


def test_eight_terms_reach_the_stated_bound():
    rng = np.random.default_rng(0x5EED)
    worst = 0.0
    for trial in range(300):
        n = 1024
        spread = rng.uniform(0, 12)  # dynamic range of the row, in octaves
        v = rng.standard_normal(n) * 2.0 ** rng.uniform(-spread, 0, n) * 2.0 ** rng.uniform(-20, 12)
        v = v.astype(np.float16).astype(np.float64)
        if not np.isfinite(v).all() or np.abs(v).max() == 0:
            continue
        approx, f0, terms = encode(v)
        mx = np.abs(v).max()
        assert 3.0 < mx * f0 <= 6.0
        for j, t in enumerate(terms):
            assert np.abs(t).max() <= (6.0 if j == 0 else 4.0)
        err = np.abs(approx - v).max()
        assert err <= 0.5 * 4.0 ** -7 / f0 * (1 + 1e-12)
        worst = max(worst, err / mx)
    assert worst <= 0.5 * 4.0 ** -7 / 3.0 < 1.1e-5


def test_narrow_rows_are_exact():
    # values that are multiples of 2^-11 in a row whose largest magnitude is
    # about 1: the eight terms' finest unit is 0.5 4^-7 / f0 = 2^-17 there,
    # so every such value is reproduced exactly
    rng = np.random.default_rng(7)
    v = (rng.integers(-2048, 2048, 512) / 2048.0).astype(np.float16).astype(np.float64)
    approx, _, _ = encode(v)
    assert np.array_equal(approx, v)


def test_fewer_terms_miss_the_bound():
    # the bound needs all eight terms: with four the residual is ~4^4 larger
    rng = np.random.default_rng(3)
    v = rng.standard_normal(1024).astype(np.float16).astype(np.float64)
    approx4, f0, _ = encode(v, n_terms=4)
    assert np.abs(approx4 - v).max() > 0.5 * 4.0 ** -7 / f0
