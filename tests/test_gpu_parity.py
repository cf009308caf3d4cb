"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar: bit-exact packed E2M1 codes, native E4M3 scale bytes (including the zero
padding rows), smoothing factors (alpha = 0.5) and channel maxima; Y within a
relative Frobenius error of 5e-3 (fused and unfused); T within 4e-3.
Shapes span several tiles, ragged M, K with a half-filled last 256-element
stage, rank 0 and the maximum rank 128.
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

from gpu_helpers import TOL_T, TOL_Y, gpu_layer, gpu_prepare, np64, oracle_factors_to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


def _inputs(M, K, N, rank, seed, outliers="first4"):
    w = synth.Workload(f"t{M}x{K}x{N}r{rank}", M, K, N, rank, seed=seed, outliers=outliers,
                       outlier_lo=50.0, outlier_hi=50.0, spikes=2)
    X, W = synth.generate(w)
    return w, X, W


CASES = [
    # M, K, N, rank        N % 256 == 0 runs the CTA-pair GEMM on 256 x 256 tiles, N % 384 == 0
    # (not % 256) on 256 x 384 tiles, otherwise the single-CTA one; small M takes the single-CTA
    # kernel when it keeps 1.5x as many SMs busy
    (256, 512, 512, 16),      # the tiny layer
    (200, 384, 256, 32),      # ragged M, K % 256 == 128
    (1, 128, 128, 0),         # one row, no branch
    (1, 256, 256, 16),        # one row on a CTA pair: the second CTA's rows are all past M
    (130, 256, 384, 128),     # maximum rank, ragged M
    (130, 256, 512, 128),     # maximum rank, ragged M, CTA pair
    (300, 384, 768, 32),      # ragged M and K on a CTA pair
    (512, 1024, 640, 48),
    (3000, 256, 1920, 32),    # ragged M on 256 x 384 pair tiles (two MMAs per K block, scale buffers in turn)
]


@pytest.mark.parametrize("M,K,N,rank", CASES)
def test_layer_parity_given_factors(M, K, N, rank):
    w, X, W = _inputs(M, K, N, rank, seed=1000 + M + K + rank)
    Xn, Wn = np64(X), np64(W)
    ref = O.layer_reference(Xn, Wn, 0.5, rank)

    Xd, Wd = X.cuda(), W.cuda()
    amax = S.svdq_channel_amax(Xd)
    assert np.array_equal(amax.cpu().numpy(), O.channel_amax(Xn))
    P = gpu_prepare(Wd, amax, 0.5, rank, oracle_factors_to_device(ref) if rank else None)
    assert np.array_equal(P.lam.cpu().numpy(), ref["lam32"])
    assert np.array_equal(P.inv_lam.cpu().numpy(), ref["inv32"])
    assert np.array_equal(P.Qr.cpu().numpy(), O.pack_nibbles(ref["Qr"]))
    assert np.array_equal(P.Sr.cpu().numpy(), O.scales_to_native(ref["Sr"]))

    for variant in (S.SVDQ_FUSED, S.SVDQ_UNFUSED):
        Qx, Sx, T, Y = gpu_layer(Xd, P, variant)
        assert np.array_equal(Qx.cpu().numpy(), O.pack_nibbles(ref["Qx"])), variant
        assert np.array_equal(Sx.cpu().numpy(), O.scales_to_native(ref["Sx"])), variant
        if rank:
            assert O.rel_fro(np64(T), ref["T"]) < TOL_T
        Yn = np64(Y)
        assert np.all(np.isfinite(Yn))
        err = O.rel_fro(Yn, ref["Y"])
        assert err < TOL_Y, (variant, err)


def test_codec_ties_saturation_and_signed_zero():
    """Groups built so that x_hat / s hits every E2M1 midpoint exactly, plus
    -0, zero groups, tiny (subnormal / underflowing) scales and huge values
    that saturate the E4M3 scale."""
    K, M = 128, 128
    rng = np.random.default_rng(7)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rows = []
    for r in range(M):
        s = (1 + rng.integers(0, 8) / 8) * 2.0 ** rng.integers(-8, 4)
        row = np.zeros(K)
        for g in range(K // 16):
            grp = rng.choice(np.concatenate([mids, -mids, [0.0, 1.0, -3.0]]), 16) * s
            grp[rng.integers(0, 16)] = 6 * s * rng.choice([-1, 1])
            row[16 * g:16 * g + 16] = grp
        rows.append(row)
    X = np.array(rows)
    assert np.array_equal(O.bf16(X), X)            # the tie rows are exact in bf16
    X[5] = 0.0
    X[6, :16] = -0.0
    X[7] = O.bf16(rng.standard_normal(K) * 1e-4)   # scales underflow / subnormal
    X[8] = O.bf16(rng.standard_normal(K) * 1e4)    # E4M3 scale saturates at 448
    X[9, ::2] = -1e-30
    X[9] = O.bf16(X[9])
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    assert np.array_equal(np64(Xt), X)
    inv = np.ones(K, dtype=np.float32)
    codes, scales, _ = O.quantize_act(np64(Xt), inv, np.zeros((K, 0)))
    Qx, Sx, _ = S.svdq_quantize_act(Xt.cuda(), torch.from_numpy(inv).cuda(), None, 0, 128)
    torch.cuda.synchronize()
    assert np.array_equal(Sx.cpu().numpy(), O.scales_to_native(scales))
    assert np.array_equal(Qx.cpu().numpy(), O.pack_nibbles(codes))


def test_codec_random_inv_lambda_bit_exact():
    rng = np.random.default_rng(8)
    M, K = 384, 1024
    X = rng.standard_normal((M, K)) * np.exp(rng.uniform(-12, 8, (M, 1)))
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    inv = np.exp(rng.uniform(-5, 5, K)).astype(np.float32)
    codes, scales, _ = O.quantize_act(np64(Xt), inv, np.zeros((K, 0)))
    Qx, Sx, _ = S.svdq_quantize_act(Xt.cuda(), torch.from_numpy(inv).cuda(), None, 0, 128)
    torch.cuda.synchronize()
    assert np.array_equal(Sx.cpu().numpy(), O.scales_to_native(scales))
    assert np.array_equal(Qx.cpu().numpy(), O.pack_nibbles(codes))
    can = S.svdq_scales_to_canonical(Sx, M, K)
    assert np.array_equal(can.cpu().numpy(), scales)


def test_empty_M_is_a_noop():
    lib = S.load()
    assert lib.svdq_quantize_act(S.Shape(0, 256, 128, 0), None, None, None, None, None, None, 0, None) == 0
    assert lib.svdq_linear(S.Shape(0, 256, 128, 0), None, None, None, None, None, None, None, 0, None) == 0


@pytest.mark.parametrize("w", [synth.FLUX_QKV, synth.FLUX_MLP_UP, synth.FLUX_MLP_DOWN], ids=lambda w: w.name)
def test_full_size_parity_sampled(w):
    """Full FLUX-shaped layer on the GPU, in the launch configuration the
    benchmark times; the oracle checks sampled rows / columns one by one."""
    X, W = synth.generate(w)
    Xn, Wn = np64(X), np64(W)
    amax_ref = O.channel_amax(Xn)
    # the oracle's split, restricted to what the sampled checks need
    lam32, inv32 = O.smoothing_lambda(amax_ref, Wn, w.alpha)
    What = lam32.astype(np.float64)[:, None] * Wn.T
    U, Sg, Vt = np.linalg.svd(What, full_matrices=False)
    L1p = O.bf16(U[:, :w.rank] * Sg[:w.rank] / lam32.astype(np.float64)[:, None])
    L2 = O.bf16(Vt[:w.rank])
    del U, Vt, What

    Xd, Wd = X.cuda(), W.cuda()
    amax = S.svdq_channel_amax(Xd)
    P = gpu_prepare(Wd, amax, w.alpha, w.rank, oracle_factors_to_device(dict(L1p=L1p, L2=L2)))
    Qx, Sx, T, Y = gpu_layer(Xd, P, S.SVDQ_FUSED)
    assert np.array_equal(amax.cpu().numpy(), amax_ref)
    assert np.array_equal(P.lam.cpu().numpy(), lam32)

    rng = np.random.default_rng(w.seed)
    rows = np.sort(rng.choice(w.M, 48, replace=False))
    cols = np.sort(rng.choice(w.N, 96, replace=False))
    rows = np.unique(np.concatenate([rows, [0, w.M - 1]]))
    cols = np.unique(np.concatenate([cols, [0, w.N - 1]]))
    # weights: sampled output channels
    _, qr_c, sr_c = O.residual_quantize(Wn[cols], lam32, L1p, L2[:, cols])
    Qr = P.Qr.cpu().numpy()
    Sr_can = S.svdq_scales_to_canonical(P.Sr, w.N, w.K).cpu().numpy()
    assert np.array_equal(Qr[cols], O.pack_nibbles(qr_c))
    assert np.array_equal(Sr_can[cols], sr_c)
    # activations: sampled rows
    qx_r, sx_r, T_r = O.quantize_act(Xn[rows], inv32, L1p)
    Sx_can = S.svdq_scales_to_canonical(Sx, w.M, w.K).cpu().numpy()
    assert np.array_equal(Qx.cpu().numpy()[rows], O.pack_nibbles(qx_r))
    assert np.array_equal(Sx_can[rows], sx_r)
    assert O.rel_fro(np64(T)[rows], T_r) < TOL_T
    # output block
    Y_ref = O.linear(qx_r, sx_r, T_r, qr_c, sr_c, L2[:, cols])
    Y_blk = np64(Y)[np.ix_(rows, cols)]
    assert O.rel_fro(Y_blk, Y_ref) < TOL_Y
    assert torch.isfinite(Y).all().item()
