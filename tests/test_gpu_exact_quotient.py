"""Every encoder of the CUDA path rounds the EXACT quotient v / s (walkthrough
eq. (1), round(X / s)): the activation quantizer (NVFP4 and INT4), the
residual encoders of the weight preparation, and the next-layer quantization in
the GEMM epilogue. The inputs put v / s exactly on code midpoints and 1..3 fp32
ulps to either side of them, where a product with a rounded reciprocal picks
the wrong code; each case first checks on the CPU that it has such elements.
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S

from gpu_helpers import np64

pytestmark = pytest.mark.gpu

E2M1_MIDS = (O.E2M1_VALUES[:-1] + O.E2M1_VALUES[1:]) / 2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


def _ulp_factors(K: int, rng) -> np.ndarray:
    """Per-column multipliers 1 + k 2^-23, k in -3..3 (fp32-exact), so that
    fp32(x * f) lies 0..3 ulps from x."""
    return (1.0 + rng.integers(-3, 4, K) * 2.0 ** -23).astype(np.float32)


def _recipe_disagreements_nvfp4(xhat: np.ndarray, scales: np.ndarray) -> int:
    """How many codes the rounded-reciprocal product fp32(v * fp32(1/s)) would
    get wrong on these inputs (the exact rule is the oracle's)."""
    rows, K = xhat.shape
    s = np.repeat(O.e4m3_decode(scales).astype(np.float32), 16, axis=1)
    live = s > 0
    with np.errstate(divide="ignore", invalid="ignore"):
        prod = xhat.astype(np.float32) * (np.float32(1.0) / np.where(live, s, 1)).astype(np.float32)
    recipe = np.where(live, O.e2m1_encode(prod.astype(np.float64)), 0)
    exact, _ = O.quantize_nvfp4(xhat.astype(np.float32))
    return int((recipe != exact).sum())


def _nvfp4_tie_rows(M: int, K: int, rng) -> np.ndarray:
    """Rows of 16-groups whose elements are +-(E2M1 midpoint) * s or +-6 s
    (one per group, fixing the scale at s), s = (1 + j/8) 2^e."""
    X = np.zeros((M, K))
    for r in range(M):
        for g in range(K // 16):
            s = (1 + rng.integers(0, 8) / 8) * 2.0 ** rng.integers(-10, 6)
            grp = rng.choice(np.concatenate([E2M1_MIDS, -E2M1_MIDS]), 16) * s
            grp[rng.integers(0, 16)] = 6 * s * rng.choice([-1, 1])
            X[r, 16 * g:16 * g + 16] = grp
    assert np.array_equal(O.bf16(X), X)
    return X


def test_quantize_act_near_midpoints_bit_exact():
    rng = np.random.default_rng(21)
    M, K = 200, 512
    X = _nvfp4_tie_rows(M, K, rng)
    inv = _ulp_factors(K, rng)
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    codes, scales, _ = O.quantize_act(np64(Xt), inv, np.zeros((K, 0)))
    xhat = np64(Xt).astype(np.float32) * inv[None, :]
    assert _recipe_disagreements_nvfp4(xhat, scales) > 100
    Qx, Sx, _ = S.svdq_quantize_act(Xt.cuda(), torch.from_numpy(inv).cuda(), None, 0, 128)
    S.svdq_check()
    assert np.array_equal(Sx.cpu().numpy(), O.scales_to_native(scales))
    assert np.array_equal(Qx.cpu().numpy(), O.pack_nibbles(codes))


@pytest.mark.parametrize("rank", [0, 32])
def test_quantize_act_with_branch_near_midpoints_bit_exact(rank):
    """The same inputs through the fused quantizer with a low-rank branch (its
    down-projection shares the shared-memory tiles)."""
    rng = np.random.default_rng(22 + rank)
    M, K = 256, 1024
    X = _nvfp4_tie_rows(M, K, rng)
    inv = _ulp_factors(K, rng)
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    L1p = O.bf16(rng.standard_normal((K, rank)) / np.sqrt(K))
    codes, scales, T = O.quantize_act(np64(Xt), inv, L1p)
    L1d = torch.from_numpy(np.ascontiguousarray(L1p.T)).float().to(torch.bfloat16).cuda() if rank else None
    Qx, Sx, Td = S.svdq_quantize_act(Xt.cuda(), torch.from_numpy(inv).cuda(), L1d, rank, 256)
    S.svdq_check()
    assert np.array_equal(Sx.cpu().numpy(), O.scales_to_native(scales))
    assert np.array_equal(Qx.cpu().numpy(), O.pack_nibbles(codes))
    if rank:
        assert O.rel_fro(np64(Td), T) < 4e-3


def test_residual_encoder_ties_and_near_midpoints_bit_exact():
    """Rank 0 with act_amax chosen so that lambda_j = sqrt(ax_j) / sqrt(aw_j)
    is 1 or within a few ulps of it: R = fp32(lambda W) puts the residual's
    quotients on and next to the midpoints."""
    rng = np.random.default_rng(23)
    N, K = 256, 512
    W = _nvfp4_tie_rows(N, K, rng)
    aw = np.abs(W).max(axis=0)
    ax = (aw * (1.0 + rng.integers(-3, 4, K) * 2.0 ** -22)).astype(np.float32)
    ax[: K // 4] = aw[: K // 4]                     # lambda exactly 1: exact ties
    lam32, inv32 = O.smoothing_lambda(ax, W, 0.5)
    assert (lam32 == 1).sum() >= K // 4 and (lam32 != 1).sum() > K // 4
    R32, qr, sr = O.residual_quantize(W, lam32, np.zeros((K, 0)), np.zeros((0, N)))
    assert _recipe_disagreements_nvfp4(R32.T.astype(np.float32), sr) > 50
    Wd = torch.from_numpy(W).to(torch.float32).to(torch.bfloat16).cuda()
    P = S.svdq_prepare_weights(Wd, torch.from_numpy(ax).cuda(), 0.5, 0)
    S.svdq_check()
    assert np.array_equal(P.lam.cpu().numpy(), lam32)
    assert np.array_equal(P.Sr.cpu().numpy(), O.scales_to_native(sr))
    assert np.array_equal(P.Qr.cpu().numpy(), O.pack_nibbles(qr))


def test_int4_quantize_act_near_midpoints_bit_exact():
    """INT4: quotients on and next to k + 1/2 with scales that are not powers
    of two (their reciprocals are inexact)."""
    rng = np.random.default_rng(24)
    M, K = 160, 512
    X = np.zeros((M, K))
    for r in range(M):
        for g in range(K // 64):
            s = (1 + rng.integers(1, 8) / 8) * 2.0 ** rng.integers(-8, 6)
            grp = (rng.integers(0, 7, 64) + 0.5) * rng.choice([-1, 1], 64) * s
            grp[rng.integers(0, 64)] = 7 * s * rng.choice([-1, 1])
            X[r, 64 * g:64 * g + 64] = grp
    assert np.array_equal(O.bf16(X), X)
    inv = _ulp_factors(K, rng)
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    xhat = np64(Xt).astype(np.float32) * inv[None, :]
    q_ref, s_ref = O.quantize_int4(xhat)
    sv = np.repeat(s_ref.astype(np.float32), 64, axis=1)
    recipe = np.clip(np.rint(xhat * (np.float32(1.0) / sv).astype(np.float32)), -7, 7)
    assert (recipe != q_ref).sum() > 100
    Qx, Sx, _ = S.svdq_int4_quantize_act(Xt.cuda(), torch.from_numpy(inv).cuda(), None, 0, 128)
    S.svdq_check()
    got = Qx.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.int64)
    assert np.array_equal(got, q_ref.astype(np.int64))
    assert np.array_equal(Sx.cpu().numpy().astype(np.float64).T[:M], s_ref)


def _next_layer_case(rng, M: int, K: int):
    """X on the E2M1 grid and next-layer factors f for the epilogue case.

    Group g's column 0 holds 6 s_x with factor f0 = 1.25 (g even) or 0.75
    (g odd), so that the next scale is s' = 1.5 s_x f0 (E4M3 mantissas 1.875
    and 1.125, whose reciprocals are inexact); the other columns cycle through
    (factor, grid values e) with e f / f0 an E2M1 midpoint and e f < 6 f0."""
    classes = {1.25: [(0.9375, [1.0]), (1.5625, [1.0, 2.0, 4.0]), (2.1875, [1.0, 2.0]), (0.625, [0.5, 1.5])],
               0.75: [(0.9375, [1.0, 2.0, 4.0]), (1.3125, [1.0, 2.0]), (0.375, [0.5, 1.5]), (1.875, [0.5, 1.0, 2.0])]}
    f = np.ones(K)
    X = np.zeros((M, K))
    for g in range(K // 16):
        f0 = 1.25 if g % 2 == 0 else 0.75
        f[16 * g] = f0
        for c in range(1, 16):
            f[16 * g + c] = classes[f0][(c + g) % 4][0]
        for r in range(M):
            sx = 2.0 ** rng.integers(-6, 3)
            X[r, 16 * g] = 6 * sx * rng.choice([-1, 1])
            for c in range(1, 16):
                X[r, 16 * g + c] = rng.choice(classes[f0][(c + g) % 4][1]) * sx * rng.choice([-1, 1])
    k = rng.integers(-3, 4, K)
    k[::16] = 0
    return X, (f * (1.0 + k * 2.0 ** -23)).astype(np.float32)


def test_next_layer_epilogue_ties_and_near_midpoints_bit_exact():
    """The next-layer quantization in the GEMM epilogue on a Y built to be
    tie-dense: W = 1.5 I (its residual encodes exactly, lambda = 1), X on the
    E2M1 grid, so Y = 1.5 X exactly; the next layer's per-column factors (times
    1 + k 2^-23) put y f / s' on and next to midpoints."""
    rng = np.random.default_rng(25)
    M, K = 256, 512
    N = K
    X, f = _next_layer_case(rng, M, K)
    assert np.array_equal(O.bf16(X), X)
    W = 1.5 * np.eye(N, K)
    Wd = torch.from_numpy(W).to(torch.float32).to(torch.bfloat16).cuda()
    P = S.svdq_prepare_weights(Wd, torch.full((K,), 1.5, device="cuda"), 0.5, 0)
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    ones = torch.ones(K, dtype=torch.float32, device="cuda")
    Qx, Sx, _ = S.svdq_quantize_act(Xt.cuda(), ones, None, 0, N)
    Y_exact = 1.5 * X
    codes, scales, _ = O.quantize_act(Y_exact, f, np.zeros((N, 0)))
    xhat = Y_exact.astype(np.float32) * f[None, :]
    assert _recipe_disagreements_nvfp4(xhat, scales) > 100
    Qn, Sn, _, Y = S.svdq_linear_quantize_next(Qx, Sx, None, P, torch.from_numpy(f).cuda(), None, 0, store_y=True)
    S.svdq_check()
    assert np.array_equal(P.lam.cpu().numpy(), np.ones(K, np.float32))
    assert np.array_equal(np64(Y), Y_exact)
    assert np.array_equal(Sn.cpu().numpy(), O.scales_to_native(scales))
    assert np.array_equal(Qn.cpu().numpy(), O.pack_nibbles(codes))
