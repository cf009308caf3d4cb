"""Pins for the oracle's number formats and NVFP4 group codec.

Each check ties the oracle to something other than itself: IEEE binary32 and
bfloat16 conversions done by numpy/torch, torch's float8_e4m3fn decoder and
rounding, the FP4 grid with q_max = 6 (devpress.csdn.net SVDQuant walkthrough,
eq. (1)), exhaustive tie cases, and exact round trips on grid-aligned groups.
"""
import numpy as np
import pytest
import torch

import oracle as O


def test_round_to_format_matches_ieee_binary32():
    rng = np.random.default_rng(1)
    v = rng.standard_normal(200_000) * np.exp(rng.uniform(-80, 80, 200_000))
    got = O.round_to_format(v, 23, -126, float(np.finfo(np.float32).max))
    want = v.astype(np.float32).astype(np.float64)
    assert np.array_equal(got, want)


def test_round_to_format_subnormal_binary32():
    rng = np.random.default_rng(2)
    v = rng.uniform(-1, 1, 50_000) * 2.0 ** -130
    got = O.round_to_format(v, 23, -126, float(np.finfo(np.float32).max))
    assert np.array_equal(got, v.astype(np.float32).astype(np.float64))


def test_bf16_matches_torch_from_fp32():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(100_000) * np.exp(rng.uniform(-30, 30, 100_000))).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16(v.astype(np.float64)), want)


def test_e4m3_decode_all_codes_match_torch():
    b = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(b)
    theirs = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(theirs)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2                       # 0x7f and 0xff
    assert np.array_equal(ours[~nan], theirs[~nan])
    assert np.nanmax(ours) == 448.0 and ours[1] == 2.0 ** -9


def test_e4m3_encode_roundtrip_and_ties():
    vals = O.e4m3_decode(np.arange(127, dtype=np.uint8))      # all non-negative finite
    assert np.array_equal(O.e4m3_encode(vals), np.arange(127, dtype=np.uint8))
    lo, hi = vals[:-1], vals[1:]
    mid = (lo + hi) / 2                                       # exact in fp64
    enc = O.e4m3_encode(mid)
    even = np.where(np.arange(126) % 2 == 0, np.arange(126), np.arange(1, 127))
    assert np.array_equal(enc, even.astype(np.uint8))         # ties go to the even code
    # saturation (satfinite): anything above the largest finite maps to 448
    assert np.all(O.e4m3_decode(O.e4m3_encode(np.array([448.0, 460.0, 464.0, 1e9]))) == 448.0)
    # below half the smallest subnormal rounds to zero; exactly half is a tie to 0
    assert np.all(O.e4m3_encode(np.array([0.0, 2.0 ** -11, 2.0 ** -10])) == 0)
    assert O.e4m3_encode(np.array([2.0 ** -10 * 1.0000001]))[0] == 1


def test_e4m3_rounding_matches_torch_cast_in_range():
    rng = np.random.default_rng(4)
    v = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 200_000)).astype(np.float32)
    theirs = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v.astype(np.float64)), theirs)


def test_e2m1_grid_is_the_fp4_grid_with_qmax_6():
    # eq. (1): q_max = 6 for 4-bit floating point
    assert list(O.E2M1_VALUES) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    codes = np.arange(16, dtype=np.uint8)
    dec = O.e2m1_decode(codes)
    assert np.array_equal(O.e2m1_encode(dec[:8]), codes[:8])
    assert np.array_equal(np.abs(dec[8:]), O.E2M1_VALUES)
    assert np.all(np.signbit(dec[8:]))


@pytest.mark.parametrize("x,code", [
    (0.25, 0), (0.2500001, 1), (0.75, 2), (0.7499999, 1), (1.25, 2), (1.2500001, 3),
    (1.75, 4), (2.5, 4), (2.5000002, 5), (3.5, 6), (3.4999998, 5), (5.0, 6), (5.0000005, 7),
    (6.0, 7), (6.5, 7), (1e30, 7),
])
def test_e2m1_ties_to_even_and_saturation(x, code):
    assert O.e2m1_encode(np.array([x]))[0] == code
    assert O.e2m1_encode(np.array([-x]))[0] == code | 8


def test_e2m1_sign_of_zero():
    enc = O.e2m1_encode(np.array([0.0, -0.0, -0.1, 0.1, -0.25]))
    assert list(enc) == [0, 8, 8, 0, 8]


def test_quantize_exact_grid_groups_roundtrip():
    """Groups built as e * s (e on the FP4 grid, s an E4M3 value) with one
    element at +-6 s quantize to exactly s and e: deq == input."""
    rng = np.random.default_rng(5)
    s_bytes = rng.integers(8, 120, size=(64, 8))               # normal E4M3 scales
    s = O.e4m3_decode(s_bytes)
    e = rng.choice(np.concatenate([O.E2M1_VALUES, -O.E2M1_VALUES]), size=(64, 8, 16))
    e[..., 3] = np.where(rng.random((64, 8)) < 0.5, 6.0, -6.0)
    v = (e * s[..., None]).reshape(64, 128)
    assert np.array_equal(v.astype(np.float32).astype(np.float64), v)   # exact in fp32
    codes, scales = O.quantize_nvfp4(v.astype(np.float32))
    assert np.array_equal(scales, s_bytes.astype(np.uint8))
    assert np.array_equal(O.dequantize_nvfp4(codes, scales), v)


def test_quantize_scale_rule_and_error_bound():
    rng = np.random.default_rng(6)
    v = (rng.standard_normal((32, 256)) * np.exp(rng.uniform(-6, 6, (32, 1)))).astype(np.float32)
    codes, scales = O.quantize_nvfp4(v)
    g = v.reshape(32, 16, 16).astype(np.float64)
    amax = np.abs(g).max(axis=2)
    sval = O.e4m3_decode(scales)
    # the scale is the E4M3 value nearest to amax / 6
    grid = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    nearest = np.abs(grid[None, None, :] - (amax / 6)[..., None]).min(axis=2)
    assert np.allclose(np.abs(sval - amax / 6), nearest, rtol=0, atol=1e-12 * amax.max())
    # with a normal (not subnormal) scale, every element is reconstructed within
    # one grid half-gap (<= 1 * s); below 4 s within half a gap (0.5 s)
    err = np.abs(O.dequantize_nvfp4(codes, scales).reshape(32, 16, 16) - g)
    S = np.broadcast_to(sval[..., None], g.shape)
    normal = np.broadcast_to((sval >= 2.0 ** -6)[..., None], g.shape)
    assert normal.mean() > 0.5
    assert np.all(err[normal] <= S[normal] + 1e-12)
    small = normal & (np.abs(g) <= 4 * S)
    assert np.all(err[small] <= 0.5 * S[small] + 1e-12)
    # with any scale, the element is the saturated RNE of v / s on the grid
    pos = S > 0
    y = np.clip(np.abs(g[pos]) / S[pos], 0, 6)
    q = np.abs(O.dequantize_nvfp4(codes, scales).reshape(32, 16, 16)[pos]) / S[pos]
    nearest_grid = O.E2M1_VALUES[np.abs(O.E2M1_VALUES[None, :] - y[:, None]).argmin(axis=1)]
    assert np.all(np.abs(q - y) <= np.abs(nearest_grid - y) + 1e-6)


def test_quantize_zero_and_underflow_groups_encode_plus_zero():
    v = np.zeros((2, 32), dtype=np.float32)
    v[1, 16:] = -1e-6                        # amax/6 underflows E4M3
    v[1, :16] = -0.0
    codes, scales = O.quantize_nvfp4(v)
    assert np.all(scales == 0) and np.all(codes == 0)


def test_pack_nibble_order():
    codes = np.array([[1, 2, 15, 0]], dtype=np.uint8)
    assert list(O.pack_nibbles(codes)[0]) == [0x21, 0x0F]
    assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(codes)), codes)


def test_native_scale_layout_is_a_bijection_with_atoms():
    rng = np.random.default_rng(7)
    rows, K = 300, 192                       # ragged last row block, 3 k-blocks
    s = rng.integers(0, 255, size=(rows, K // 16), dtype=np.uint8)
    nat = O.scales_to_native(s)
    assert nat.size == 3 * 3 * 512
    assert np.array_equal(O.native_to_scales(nat, rows, K), s)
    # one atom: rows 0..127, k-block 1 -> bytes 512..1023
    atom = nat[512:1024].reshape(32, 4, 4)   # [i][q][j]
    assert np.array_equal(atom[5, 2, 3], s[2 * 32 + 5, 4 + 3])
    # padded rows (300..383) of the last block are zero
    pad = O.scales_to_native(np.zeros((rows, K // 16), dtype=np.uint8) + 1)
    assert pad.sum() == rows * K // 16
