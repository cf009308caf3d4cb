"""Pins for the oracle's rounding of quotients: eq. (1) of the devpress.csdn.net
SVDQuant walkthrough quantizes round(X / s), the real quotient, so every code
and scale the oracle emits must be the round-to-nearest-even (saturating) image
of the EXACT quotient. The reference here is Python's exact rational
arithmetic (fractions.Fraction), which shares nothing with the oracle's
midpoint comparisons.

Cases: every positive E4M3 scale x every E2M1 midpoint, exactly on the tie and
1..3 fp32 ulps to each side, both signs; random quotients over the whole code
range for every scale; every E4M3 midpoint of the scale rule amax / 6; and the
INT4 variant's fp16 scales (amax / 7) and integer codes (v / s).
"""
from bisect import bisect_right
from fractions import Fraction

import numpy as np
import pytest

import oracle as O


def _fracs(grid):
    return [Fraction(float(g)) for g in grid]


E2M1_F = _fracs(O.E2M1_VALUES)
E4M3_F = _fracs(O.E4M3_GRID)
INT4_F = _fracs(O.INT4_GRID)


def exact_rne_index(num: float, den: float, G) -> int:
    """Index of the grid value nearest to |num| / den (exact), ties to the even
    index, quotients past the last value saturating to it."""
    q = Fraction(abs(float(num))) / Fraction(float(den))
    if q >= G[-1]:
        return len(G) - 1
    i = bisect_right(G, q) - 1
    lo, hi = q - G[i], G[i + 1] - q
    if lo < hi:
        return i
    if hi < lo:
        return i + 1
    return i if i % 2 == 0 else i + 1


def f32_steps(x: np.ndarray, k: int) -> np.ndarray:
    """x moved k fp32 ulps (k may be negative)."""
    x = np.asarray(x, dtype=np.float32).copy()
    direction = np.float32(np.inf) if k > 0 else np.float32(-np.inf)
    for _ in range(abs(k)):
        x = np.nextafter(x, direction)
    return x


def _nvfp4_groups_with_scale(s: np.ndarray, vals: np.ndarray) -> np.ndarray:
    """Groups of 16 fp32 values whose first element is 6 s (so amax / 6 = s
    exactly and the group's scale is s) and whose other 15 are ``vals``."""
    n = vals.shape[0]
    g = np.empty((n, 16), dtype=np.float32)
    g[:, 0] = (6.0 * s).astype(np.float32)
    g[:, 1:] = vals
    return g


def test_e2m1_codes_every_scale_every_midpoint_and_neighbours():
    scales = O.E4M3_GRID[1:]                                  # 126 positive scales
    mids = (O.E2M1_VALUES[:-1] + O.E2M1_VALUES[1:]) / 2       # 0.25 .. 5
    rows_s, rows_v = [], []
    for s in scales:
        base = (mids * s).astype(np.float32)                  # exact: <= 7 significant bits
        assert np.array_equal(base.astype(np.float64), mids * s)
        cand = np.concatenate([f32_steps(base, k) for k in range(-3, 4)])
        cand = np.concatenate([cand, -cand])                  # 98 values
        cand = np.concatenate([cand, np.zeros(-cand.size % 15, np.float32)])
        for chunk in cand.reshape(-1, 15):
            rows_s.append(s)
            rows_v.append(chunk)
    s_arr = np.array(rows_s)
    g = _nvfp4_groups_with_scale(s_arr, np.array(rows_v))
    codes, sbytes = O.quantize_nvfp4(g.reshape(-1, 16))
    assert np.array_equal(O.e4m3_decode(sbytes[:, 0]), s_arr)
    for r in range(g.shape[0]):
        for i in range(16):
            v = float(g[r, i])
            want = exact_rne_index(v, s_arr[r], E2M1_F) | (8 if np.signbit(v) else 0)
            assert codes[r, i] == want, (s_arr[r], v)


def test_e2m1_codes_random_quotients_every_scale():
    rng = np.random.default_rng(11)
    scales = O.E4M3_GRID[1:]
    s_arr = np.repeat(scales, 16)
    u = rng.uniform(-6.0, 6.0, size=(s_arr.size, 15))
    vals = (u * s_arr[:, None]).astype(np.float32)            # one fp32 rounding: generic, off-grid values
    g = _nvfp4_groups_with_scale(s_arr, vals)
    codes, sbytes = O.quantize_nvfp4(g)
    assert np.array_equal(O.e4m3_decode(sbytes[:, 0]), s_arr)
    for r in range(g.shape[0]):
        for i in range(1, 16):
            v = float(g[r, i])
            assert codes[r, i] == exact_rne_index(v, s_arr[r], E2M1_F) | (8 if np.signbit(v) else 0)


def test_exact_quotient_differs_from_the_rounded_reciprocal_recipe():
    """The reading matters: s = 1.875 * 2^-3 and v = 1.25 s is an exact tie
    (code 2, value 1.0, ties to even), while fp32(v * fp32(1 / s)) lands just
    above 1.25 and would give code 3. Over all 882 exact ties the two recipes
    disagree somewhere, so the pins above can tell them apart."""
    s = np.float32(0.234375)
    v = np.float32(1.25) * s
    assert float(v) == 1.25 * 0.234375
    codes, sb = O.quantize_nvfp4(np.array([[6 * s, v] + [0.0] * 14], dtype=np.float32))
    assert O.e4m3_decode(sb[0, 0]) == 0.234375 and codes[0, 1] == 2
    recip = np.float32(v * (np.float32(1.0) / s))
    assert recip > np.float32(1.25) and O.e2m1_encode(np.array([recip]))[0] == 3
    mids = (O.E2M1_VALUES[:-1] + O.E2M1_VALUES[1:]) / 2
    s_all = O.E4M3_GRID[1:].astype(np.float32)
    ties = (mids[None, :] * s_all[:, None]).astype(np.float32)
    recipe = ties * (np.float32(1.0) / s_all)[:, None]
    exact = np.array([[exact_rne_index(float(ties[a, b]), float(s_all[a]), E2M1_F) for b in range(7)]
                      for a in range(s_all.size)])
    assert (O.e2m1_encode(recipe.astype(np.float64)) != exact).sum() > 0


def test_e4m3_scale_every_midpoint_and_neighbours():
    """s = RNE_E4M3(amax / 6) of the exact quotient at and around every
    midpoint 6 mu of adjacent E4M3 values; and the fp32 recipe
    E4M3(fp32(amax / 6)) agrees on all of them (a midpoint times 6 is exact
    in fp32, so the fp32 quotient can only land on a midpoint when the exact
    quotient is that midpoint)."""
    grid = O.E4M3_GRID
    mids = (grid[:-1] + grid[1:]) / 2
    base = (6.0 * mids).astype(np.float32)
    assert np.array_equal(base.astype(np.float64), 6.0 * mids)
    amax = np.concatenate([f32_steps(base, k) for k in range(-3, 4)] +
                          [np.float32([0.0, 6 * 448.0, 6 * 464.0, 1e30, 6 * 2.0 ** -10])])
    got = O.rne_quotient_index(amax, 6.0, grid)
    want = np.array([exact_rne_index(float(a), 6.0, E4M3_F) for a in amax])
    assert np.array_equal(got, want)
    fp32_recipe = O.e4m3_encode((amax / np.float32(6.0)).astype(np.float64))
    assert np.array_equal(fp32_recipe, want.astype(np.uint8))
    # through the group quantizer: a group holding only amax
    g = np.zeros((amax.size, 16), dtype=np.float32)
    g[:, 5] = -amax
    _, sb = O.quantize_nvfp4(g)
    assert np.array_equal(sb[:, 0], want.astype(np.uint8))


def test_e4m3_scale_random_amax():
    rng = np.random.default_rng(12)
    amax = np.exp(rng.uniform(np.log(2.0 ** -14), np.log(3000.0), 20000)).astype(np.float32)
    want = np.array([exact_rne_index(float(a), 6.0, E4M3_F) for a in amax])
    assert np.array_equal(O.rne_quotient_index(amax, 6.0, O.E4M3_GRID), want)


# ---------------------------------------------------------------------------
# INT4 variant: fp16 scale of amax / 7, integer codes of v / s
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def fp16_fracs():
    return _fracs(O.FP16_GRID)


def test_int4_fp16_scale_at_midpoints(fp16_fracs):
    grid = O.FP16_GRID
    rng = np.random.default_rng(13)
    pick = np.unique(np.concatenate([np.arange(0, 40), rng.integers(0, grid.size - 1, 400),
                                     np.arange(grid.size - 40, grid.size - 1)]))
    mids = (grid[pick] + grid[pick + 1]) / 2
    base = (7.0 * mids).astype(np.float32)
    assert np.array_equal(base.astype(np.float64), 7.0 * mids)      # <= 15 significant bits
    amax = np.concatenate([f32_steps(base, k) for k in range(-2, 3)] + [np.float32([7 * 65504.0, 1e30])])
    want = np.array([exact_rne_index(float(a), 7.0, fp16_fracs) for a in amax])
    assert np.array_equal(O.rne_quotient_index(amax, 7.0, grid), want)
    # the fp32 recipe fp16(fp32(amax / 7)), saturating at 65504, agrees
    recipe = np.minimum((amax / np.float32(7.0)).astype(np.float32), np.float32(65504.0)).astype(np.float16)
    assert np.array_equal(recipe.astype(np.float64), grid[want])


def test_int4_codes_at_midpoints_and_neighbours():
    rng = np.random.default_rng(14)
    s_vals = np.concatenate([O.FP16_GRID[rng.integers(1, 1024, 8)],            # fp16 subnormals
                             O.FP16_GRID[rng.integers(1024, 0x7800, 120)]])    # normals
    s_vals = s_vals[s_vals * 7 < 3e38]
    mids = np.arange(7) + 0.5
    rows = []
    for s in s_vals:
        base = (mids * s).astype(np.float32)
        assert np.array_equal(base.astype(np.float64), mids * s)
        cand = np.concatenate([f32_steps(base, k) for k in range(-3, 4)])
        cand = np.concatenate([cand, -cand, np.zeros(63 * 2 - 2 * cand.size, np.float32)])
        for chunk in cand.reshape(-1, 63):
            rows.append((s, chunk))
    g = np.array([np.concatenate([[7.0 * s], c]) for s, c in rows], dtype=np.float32)
    codes, sc = O.quantize_int4(g)
    s_arr = np.array([s for s, _ in rows])
    assert np.array_equal(sc[:, 0], s_arr)
    for r in range(g.shape[0]):
        for i in range(64):
            v = float(g[r, i])
            m = exact_rne_index(v, s_arr[r], INT4_F)
            assert codes[r, i] == (-m if v < 0 else m), (s_arr[r], v)


def test_rne_quotient_index_per_group_divisors_match_scalar_path():
    rng = np.random.default_rng(15)
    num = rng.standard_normal((50, 16)).astype(np.float32).astype(np.float64)
    den = O.E4M3_GRID[rng.integers(1, 127, 50)]
    per_group = O.rne_quotient_index(num, den, O.E2M1_VALUES)
    for r in range(50):
        assert np.array_equal(per_group[r], O.rne_quotient_index(num[r], float(den[r]), O.E2M1_VALUES))
