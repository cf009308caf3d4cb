"""Parity of the INT4 W4A4 variant (through the C ABI) with the oracle's INT4
functions (walkthrough eq. (1) with q_max = 7; handbook: one fp16 scale per 64
elements).

Bar: the activation's and the residual's INT4 codes bit-exact -- as integers
(the E4M3 bytes decoded) and as bytes (against the E4M3 encoding of the
oracle's integers) -- and their scales bit-exact as fp32 values; T within
4e-3 and Y within 5e-3 relative Frobenius error of the oracle's fp64 layer;
and every element of Y within bf16 rounding of the fp64 sum of the codes the
GPU produced (the GEMM alone, element by element). Shapes span several tiles,
ragged M, a last column tile that is half outside N, rank 0 and 128, more
tiles than SMs (the persistent loop wraps), and the full FLUX QKV layer on
sampled rows and columns.
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

from gpu_helpers import TOL_T, TOL_Y, gpu_prepare, np64, oracle_factors_to_device

pytestmark = pytest.mark.gpu


def e4m3_bytes(codes: np.ndarray) -> np.ndarray:
    """The E4M3 bytes of integer codes (the oracle's encoder on |c|, sign bit 0x80)."""
    c = np.asarray(codes, dtype=np.int64)
    return (O.e4m3_encode(np.abs(c).astype(np.float64)) | np.where(c < 0, 0x80, 0x00)).astype(np.uint8)


def decode(q: torch.Tensor) -> np.ndarray:
    return q.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.int64)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


def _check_y_elementwise(Y, Qx, Sx, T, W4, M):
    """Y against the fp64 sum of the GPU's own codes and scales, element by
    element: only the final bf16 rounding (half an ulp, 2^-9 relative) and the
    fp32 accumulation separate them."""
    K, N = W4.shape.K, W4.shape.N
    qx = decode(Qx).astype(np.float64)
    qr = decode(W4.Qr).astype(np.float64)
    sx = Sx.cpu().numpy().astype(np.float64)[:, :M].T
    sr = W4.Sr.cpu().numpy().astype(np.float64).T
    ref = O.dequantize_int4(qx, sx) @ O.dequantize_int4(qr, sr).T
    if T is not None:
        ref = ref + np64(T) @ np64(W4.L2t).T
    Yn = np64(Y)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.abs(ref).max()
    bad = np.abs(Yn - ref) > bound
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5])


CASES = [
    # M, K, N, rank
    (256, 512, 512, 16),      # the tiny layer
    (200, 384, 256, 32),      # ragged M, three k-tiles
    (1, 128, 128, 0),         # one row; the only column tile is half outside N
    (130, 256, 384, 128),     # maximum rank (two low-rank k-tiles), ragged M, half last tile
    (300, 384, 768, 32),
    (512, 1024, 640, 48),     # half last column tile
    (2100, 512, 4096, 32),    # 17 x 16 = 272 tiles: more than one per SM, ragged M
]


@pytest.mark.parametrize("M,K,N,rank", CASES)
def test_int4_layer_parity(M, K, N, rank):
    w = synth.Workload(f"i{M}x{K}x{N}r{rank}", M, K, N, rank, seed=3000 + M + K + rank, outliers="first4",
                       outlier_lo=50.0, outlier_hi=50.0, spikes=2)
    X, W = synth.generate(w)
    Xn, Wn = np64(X), np64(W)
    ref = O.layer_reference_int4(Xn, Wn, 0.5, rank)

    Xd, Wd = X.cuda(), W.cuda()
    amax = S.svdq_channel_amax(Xd)
    P = gpu_prepare(Wd, amax, 0.5, rank, oracle_factors_to_device(ref) if rank else None)
    W4 = S.svdq_int4_prepare_weights(Wd, P)
    Qx, Sx, T = S.svdq_int4_quantize_act(Xd, P.inv_lam, P.L1p, rank, N)
    Y = S.svdq_int4_linear(Qx, Sx, T, W4)
    S.svdq_check()

    assert np.array_equal(P.lam.cpu().numpy(), ref["lam32"])
    # residual: [N][K] codes, [K/64][N] scales
    assert np.array_equal(W4.Qr.cpu().numpy(), e4m3_bytes(ref["Qr4"]))
    assert np.array_equal(decode(W4.Qr), ref["Qr4"])
    assert np.array_equal(W4.Sr.cpu().numpy().astype(np.float64).T, ref["Sr4"])
    # activation: rows past M (up to the 128-row padding) hold zero scales
    assert np.array_equal(Qx.cpu().numpy(), e4m3_bytes(ref["Qx4"]))
    sx = Sx.cpu().numpy().astype(np.float64)
    assert np.array_equal(sx[:, :M].T, ref["Sx4"])
    assert not sx[:, M:].any()
    if rank:
        assert O.rel_fro(np64(T), ref["T"]) < TOL_T
    Yn = np64(Y)
    assert np.all(np.isfinite(Yn))
    assert O.rel_fro(Yn, ref["Y"]) < TOL_Y
    _check_y_elementwise(Y, Qx, Sx, T, W4, M)


def test_int4_codec_edge_cases():
    """Exact ties (power-of-two scales), zero groups and -0, fp16-subnormal
    scales, scales that underflow to 0 and scales that saturate at 65504."""
    M, K = 128, 256
    rng = np.random.default_rng(17)
    X = np.zeros((M, K))
    for r in range(M):
        s = 2.0 ** rng.integers(-6, 6)
        for g in range(K // 64):
            grp = (rng.integers(-7, 7, 64) + rng.choice([0.0, 0.5], 64)) * s
            grp[rng.integers(0, 64)] = 7 * s * rng.choice([-1, 1])
            X[r, 64 * g:64 * g + 64] = grp
    assert np.array_equal(O.bf16(X), X)            # ties exact in bf16
    X[5] = 0.0
    X[6, :64] = -0.0
    X[7] = O.bf16(rng.standard_normal(K) * 3e-5)   # fp16-subnormal scales
    X[8] = O.bf16(rng.standard_normal(K) * 1e-8)   # scales underflow to 0
    X[9] = O.bf16(rng.standard_normal(K) * 1e6)    # scales saturate at 65504
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    assert np.array_equal(np64(Xt), X)
    inv = np.ones(K, dtype=np.float32)
    q_ref, s_ref = O.quantize_int4(np64(Xt).astype(np.float32))
    Qx, Sx, _ = S.svdq_int4_quantize_act(Xt.cuda(), torch.from_numpy(inv).cuda(), None, 0, 128)
    S.svdq_check()
    assert np.array_equal(Qx.cpu().numpy(), e4m3_bytes(q_ref))
    assert np.array_equal(Sx.cpu().numpy().astype(np.float64).T, s_ref)
    assert s_ref[9].max() == 65504.0 and s_ref[8].max() == 0.0 and 0 < s_ref[7].max() < 2.0 ** -14


def test_int4_random_inv_lambda_bit_exact():
    rng = np.random.default_rng(18)
    M, K = 384, 1024
    X = rng.standard_normal((M, K)) * np.exp(rng.uniform(-10, 8, (M, 1)))
    Xt = torch.from_numpy(X).to(torch.float32).to(torch.bfloat16)
    inv = np.exp(rng.uniform(-5, 5, K)).astype(np.float32)
    xhat = np64(Xt).astype(np.float32) * inv[None, :]
    q_ref, s_ref = O.quantize_int4(xhat)
    Qx, Sx, _ = S.svdq_int4_quantize_act(Xt.cuda(), torch.from_numpy(inv).cuda(), None, 0, 128)
    S.svdq_check()
    assert np.array_equal(Qx.cpu().numpy(), e4m3_bytes(q_ref))
    assert np.array_equal(Sx.cpu().numpy().astype(np.float64).T, s_ref)


def test_int4_empty_M_is_a_noop():
    lib = S.load()
    assert lib.svdq_int4_quantize_act(S.Shape(0, 256, 128, 0), None, None, None, None, None, None, None) == 0
    assert lib.svdq_int4_linear(S.Shape(0, 256, 128, 0), None, None, None, None, None, None, None, None) == 0


def test_int4_full_size_qkv_sampled():
    """The FLUX QKV layer at full size (1296 tiles), in the launch configuration
    the benchmark times; the oracle checks sampled rows and columns."""
    w = synth.FLUX_QKV
    X, W = synth.generate(w)
    Xn, Wn = np64(X), np64(W)
    Xd, Wd = X.cuda(), W.cuda()
    amax = S.svdq_channel_amax(Xd)
    P = S.svdq_prepare_weights(Wd, amax, w.alpha, w.rank)   # device SVD
    W4 = S.svdq_int4_prepare_weights(Wd, P)
    Qx, Sx, T = S.svdq_int4_quantize_act(Xd, P.inv_lam, P.L1p, w.rank, w.N)
    Y = S.svdq_int4_linear(Qx, Sx, T, W4)
    S.svdq_check()
    lam32 = P.lam.cpu().numpy()
    inv32 = P.inv_lam.cpu().numpy()
    L1p = np64(P.L1p).T          # [K][r]
    L2 = np64(P.L2t).T           # [r][N]

    rng = np.random.default_rng(w.seed)
    rows = np.unique(np.concatenate([rng.choice(w.M, 48, replace=False), [0, w.M - 1]]))
    cols = np.unique(np.concatenate([rng.choice(w.N, 96, replace=False), [0, w.N - 1]]))
    R32, _, _ = O.residual_quantize(Wn[cols], lam32, L1p, L2[:, cols])
    qr_c, sr_c = O.quantize_int4(R32.T)
    assert np.array_equal(W4.Qr.cpu().numpy()[cols], e4m3_bytes(qr_c))
    assert np.array_equal(W4.Sr.cpu().numpy().astype(np.float64).T[cols], sr_c)
    xhat = Xn[rows].astype(np.float32) * inv32[None, :]
    qx_r, sx_r = O.quantize_int4(xhat)
    assert np.array_equal(Qx.cpu().numpy()[rows], e4m3_bytes(qx_r))
    assert np.array_equal(Sx.cpu().numpy().astype(np.float64).T[rows], sx_r)
    T_r = Xn[rows] @ L1p
    assert O.rel_fro(np64(T)[rows], T_r) < TOL_T
    Y_ref = O.dequantize_int4(qx_r, sx_r) @ O.dequantize_int4(qr_c, sr_c).T + T_r @ L2[:, cols]
    assert O.rel_fro(np64(Y)[np.ix_(rows, cols)], Y_ref) < TOL_Y
    assert torch.isfinite(Y).all().item()
