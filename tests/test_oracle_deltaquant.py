"""Pins of the oracle's DeltaQuant-style core + delta activation codec
(libaedu.com article on 4-bit diffusion-model quantization, DeltaQuant
paragraphs: local 3-D spatio-temporal blocks, the block's mean token kept in
FP8, 4-bit differences to it). Anchors outside the oracle: torch's
float8_e4m3fn conversion, plain-Python loops over blocks and tokens, exact
special cases, the E2M1 grid's half-step bound, and the method's premise on
spatio-temporally smooth inputs."""
import numpy as np
import torch

import oracle as O
from w4a4_diffusion_model_b200 import synth


def test_e4m3_encode_signed_matches_torch():
    rng = np.random.default_rng(41)
    v = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-4, 3, 4000),
                        [0.0, -0.0, 448.0, -448.0, 2.0 ** -9, -(2.0 ** -9), 2.0 ** -10]])
    v = v[np.abs(v) <= 448.0].astype(np.float32).astype(np.float64)
    lib = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode_signed(v), lib)


def test_video_blocks_brute_force_with_ragged_edges():
    for dims, block in (((4, 4, 4), (2, 2, 2)), ((3, 5, 3), (2, 2, 2)), ((2, 6, 4), (1, 3, 2))):
        F, H, Wd = dims
        blk = O.video_blocks(F, H, Wd, block)
        nbh, nbw = -(-H // block[1]), -(-Wd // block[2])
        t = 0
        for f in range(F):
            for h in range(H):
                for w in range(Wd):
                    assert blk[t] == (f // block[0]) * nbh * nbw + (h // block[1]) * nbw + w // block[2]
                    t += 1
        counts = np.bincount(blk)
        assert counts.min() >= 1 and counts.max() <= block[0] * block[1] * block[2]


def test_core_is_the_rounded_block_mean_and_delta_is_relative_to_it():
    """Brute force: per block and channel the exact mean in Python floats, its
    E4M3 byte from torch; the delta codes are the NVFP4 codes of
    fp32(x - decode(core))."""
    F, H, Wd, C = 3, 3, 4, 32
    X = synth.smooth_video(F, H, Wd, C, seed=7).float().numpy().astype(np.float64)
    enc = O.deltaquant_encode(X, (F, H, Wd))
    blk = enc["block_of_token"]
    for b in range(int(blk.max()) + 1):
        rows = [t for t in range(F * H * Wd) if blk[t] == b]
        for c in range(C):
            mean = sum(float(X[t, c]) for t in rows) / len(rows)
            byte = torch.tensor([mean], dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8).item()
            assert enc["core_codes"][b, c] == byte
    core = torch.from_numpy(enc["core_codes"]).view(torch.float8_e4m3fn).double().numpy()
    delta = (X - core[blk]).astype(np.float32)
    codes, scales = O.quantize_nvfp4(delta)
    assert np.array_equal(enc["delta_codes"], codes) and np.array_equal(enc["delta_scales"], scales)


def test_block_constant_input_reconstructs_exactly():
    """Every token of a block equal to one E4M3-exact value: the core is that
    value, every delta is zero (zero scale bytes, +0 codes) and decoding is
    exact."""
    rng = np.random.default_rng(43)
    F, H, Wd, C = 4, 4, 6, 48
    blk = O.video_blocks(F, H, Wd)
    grid = O.e4m3_decode(np.arange(256))
    grid = grid[np.isfinite(grid)]
    vals = rng.choice(grid, size=(int(blk.max()) + 1, C))
    X = vals[blk]
    enc = O.deltaquant_encode(X, (F, H, Wd))
    assert not enc["delta_scales"].any() and not enc["delta_codes"].any()
    assert np.array_equal(O.deltaquant_decode(enc), X)


def test_reconstruction_error_within_the_e2m1_half_step():
    """|x - x~| <= s_g (the decoded delta scale of its 16-group): the E2M1
    grid's largest gap is 2 s (between 4 s and 6 s), and a scale rounded down
    by E4M3 leaves at most amax / 16 above 6 s."""
    F, H, Wd, C = 4, 6, 6, 64
    X = synth.smooth_video(F, H, Wd, C, seed=11, noise=0.3).float().numpy().astype(np.float64)
    enc = O.deltaquant_encode(X, (F, H, Wd))
    err = np.abs(O.deltaquant_decode(enc) - X)
    s = np.repeat(enc["delta_scales"], 16, axis=1)
    assert np.all(err <= s * (1 + 1e-6) + 1e-7 * np.abs(X))


def test_smooth_video_premise():
    """On a spatio-temporally smooth input the core + delta code is clearly
    more accurate than NVFP4 of the raw tokens (the deltas are smaller than
    the tokens); on i.i.d. noise it gains little."""
    F, H, Wd, C = 4, 8, 8, 64
    X = synth.smooth_video(F, H, Wd, C, seed=5).float().numpy().astype(np.float64)
    err_dq = O.rel_fro(O.deltaquant_decode(O.deltaquant_encode(X, (F, H, Wd))), X)
    c, s = O.quantize_nvfp4(X.astype(np.float32))
    err_fp4 = O.rel_fro(O.dequantize_nvfp4(c, s), X)
    assert err_dq < 0.7 * err_fp4
    N = np.random.default_rng(1).standard_normal((F * H * Wd, C))
    err_dq_n = O.rel_fro(O.deltaquant_decode(O.deltaquant_encode(N, (F, H, Wd))), N)
    c, s = O.quantize_nvfp4(N.astype(np.float32))
    err_fp4_n = O.rel_fro(O.dequantize_nvfp4(c, s), N)
    assert err_dq_n > 0.8 * err_fp4_n


def test_core_rounds_the_exact_mean_ties_and_double_rounding_cases():
    """The core is one RNE rounding of the exact block mean: a mean exactly on
    an E4M3 midpoint goes to the even code; a mean a hair above it (2^-28
    relative, lost if the mean were first rounded to fp32) goes up; a mean
    above 448 saturates; a negative mean that rounds to zero keeps the sign."""
    F, H, Wd, C = 2, 2, 2, 16
    X = np.zeros((8, C))
    X[0, 0] = 8.5                      # mean 1.0625: midpoint of 1.0 and 1.125 -> even code 1.0
    X[0, 1], X[3, 1] = 8.5, 2.0 ** -25  # mean 1.0625 + 2^-28 -> 1.125
    X[:, 2] = 500.0                    # mean 500 -> 448
    X[5, 3] = -(2.0 ** -14)            # mean -2^-17 rounds to -0
    X[:, 4] = -3.0                     # block-constant
    X[0, 5], X[1, 5] = 1.0, -1.0       # zero sum -> +0
    assert np.array_equal(O.bf16(X), X)
    enc = O.deltaquant_encode(X, (F, H, Wd))
    core = enc["core_codes"][0]
    assert O.e4m3_decode(core[0]) == 1.0 and O.e4m3_decode(core[1]) == 1.125
    assert O.e4m3_decode(core[2]) == 448.0 and core[3] == 0x80 and O.e4m3_decode(core[4]) == -3.0
    assert core[5] == 0x00
