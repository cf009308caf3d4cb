"""Parity of the DeltaQuant-style core + delta encoder (libaedu.com article on
4-bit diffusion-model quantization, DeltaQuant paragraphs) with the oracle's
deltaquant_encode: core bytes, delta codes and delta scales bit-exact, through
the C ABI. Inputs: smooth synthetic video latents with ragged block grids
(odd F, H, W), i.i.d. noise, and hand-built blocks for the edge cases (block
means on E4M3 midpoints and a hair above them, saturating and underflowing
means, zero and -0 blocks, block-constant tokens)."""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

from gpu_helpers import np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


def _compare(X: torch.Tensor, dims):
    F, H, W = dims
    C = X.shape[1]
    enc = O.deltaquant_encode(np64(X), dims)
    core, Qd, Sd = S.svdq_deltaquant_encode(X.cuda(), dims)
    S.svdq_check()
    assert np.array_equal(core.cpu().numpy(), enc["core_codes"])
    assert np.array_equal(Qd.cpu().numpy(), O.pack_nibbles(enc["delta_codes"]))
    assert np.array_equal(Sd.cpu().numpy(), O.scales_to_native(enc["delta_scales"]))
    return enc


@pytest.mark.parametrize("dims,C", [((2, 2, 2), 64), ((3, 5, 7), 64), ((4, 6, 6), 192), ((5, 9, 11), 128),
                                    ((1, 1, 1), 64), ((7, 3, 40), 256), ((16, 12, 18), 1024)])
def test_smooth_video_bit_exact(dims, C):
    F, H, W = dims
    X = synth.smooth_video(F, H, W, C, seed=F * 100 + H * 10 + W)
    enc = _compare(X, dims)
    # the codec reconstructs within the delta scale (the oracle's own bound)
    err = np.abs(O.deltaquant_decode(enc) - np64(X))
    assert np.all(err <= np.repeat(O.e4m3_decode(enc["delta_scales"]), 16, axis=1) * (1 + 1e-6) + 1e-7 * np.abs(np64(X)))


def test_noise_and_wide_range_bit_exact():
    rng = np.random.default_rng(61)
    F, H, W, C = 3, 10, 13, 320
    X = rng.standard_normal((F * H * W, C)) * np.exp(rng.uniform(-8, 6, (F * H * W, 1)))
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    _compare(Xt, (F, H, W))


def test_edge_blocks_bit_exact():
    """One 2 x 2 x 2 block per channel group of special values."""
    F, H, W, C = 2, 2, 2, 128
    X = np.zeros((8, C))
    rng = np.random.default_rng(62)
    grid = O.E4M3_GRID[1:]
    mids = (grid[:-1] + grid[1:]) / 2
    for c in range(16):                        # means exactly on E4M3 midpoints: 8 mu in one token
        X[c % 8, c] = 8 * rng.choice(mids[:80]) * rng.choice([-1, 1])
    above = rng.choice(np.arange(40, 80), 16)
    for c in range(16, 32):                    # a hair above a midpoint (2^-28 relative)
        mu = mids[above[c - 16]]
        X[0, c], X[3, c] = 8 * mu, 8 * mu * 2.0 ** -28
    X[:, 32:40] = 500.0 * rng.choice([-1, 1], (8, 8))      # saturating means (some cancel)
    X[5, 40:48] = -(2.0 ** -14)                              # means rounding to -0
    X[:, 48:56] = -0.0                                       # -0 block: core +0, delta codes
    X[:, 56:64] = rng.choice(grid, 8)[None, :]               # block-constant, E4M3-exact
    X[:, 64:] = rng.standard_normal((8, C - 64)) * 3
    X = O.bf16(X)
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    assert np.array_equal(np64(Xt), X)
    enc = _compare(Xt, (F, H, W))
    core = enc["core_codes"][0]
    # a hair above midpoint i goes to grid value i + 1 (rounding the mean to
    # fp32 first would have made it a tie and picked the even neighbour)
    assert np.array_equal(O.e4m3_decode(core[16:32]), grid[above + 1])
    assert np.all(core[40:48] == 0x80) and np.all(core[48:56] == 0x00)
