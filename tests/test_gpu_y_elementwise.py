"""Every element of the NVFP4 layer's Y against the fp64 sum of the GPU's own
operands (devpress.csdn.net SVDQuant walkthrough, eq. (2) and eq. (5)):

    ref[m][n] = sum_k deq(Qx)[m][k] deq(Qr)[n][k] + sum_j T[m][j] L2t[n][j]

decoded from the codes, scales, T and L2t the library produced. Only the
GEMM's fp32 accumulation and the final bf16 rounding separate Y from ref, so
each element must satisfy

    |Y - ref| <= 2^-8 |ref| + 2^-14 * sum of |terms|

(bf16 rounding is at most 2^-8 relative; the fp32 accumulator takes at most
one rounding per 64-element MMA, K/64 * 2^-24 <= 2^-16.4 of the absolute sum
at K = 12288). A wrong scale, a dropped low-rank term or a misplaced tile
moves an element by far more. Unlike the relative-Frobenius parity bar this
checks every row: all rows of tiny and ragged shapes, and every row of a few
256-column blocks of the full FLUX QKV and MLP-down layers, rank 32 included.
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

from gpu_helpers import gpu_layer, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


def _deq_rows(Q: torch.Tensor, Sn: torch.Tensor, rows_total: int, K: int, rows=None) -> np.ndarray:
    codes = O.unpack_nibbles(Q.cpu().numpy().reshape(rows_total, K // 2))
    scales = O.native_to_scales(Sn.cpu().numpy(), rows_total, K)
    if rows is not None:
        codes, scales = codes[rows], scales[rows]
    return O.dequantize_nvfp4(codes, scales)


def _check(Y, Qx, Sx, T, P, M, K, N, cols=None, unfused=False):
    """unfused: Y of the 4-bit GEMM is rounded to bf16 before the separate
    up-projection adds T L2t^T: one more bf16 rounding, up to 2^-8 of
    |deq(Qx) deq(Qr)^T| (the unit roundoff of an 8-bit significand)."""
    cols = np.arange(N) if cols is None else cols
    A = _deq_rows(Qx, Sx, M, K)
    B = _deq_rows(P.Qr, P.Sr, N, K, cols)
    ref = A @ B.T
    first = np.abs(ref) if unfused else 0.0
    absum = np.abs(A) @ np.abs(B).T
    if T is not None:
        Tn, Ln = np64(T), np64(P.L2t)[cols]
        ref += Tn @ Ln.T
        absum += np.abs(Tn) @ np.abs(Ln).T
    Yn = np64(Y)[:, cols]
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -8 * first + 2.0 ** -14 * absum
    bad = np.abs(Yn - ref) > bound
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5], float(np.abs(Yn - ref).max()))
    # the bound is not vacuous: it stays below 0.4 % of the absolute sum, so a
    # dropped low-rank term or a misplaced tile shows (single scales are pinned
    # bit for bit by the parity tests; at K = 12288 one 16-group is 1/768 of
    # the sum, below Y's own bf16 rounding)
    assert float(np.median(bound / np.maximum(absum, 1e-30))) < 4e-3


@pytest.mark.parametrize("M,K,N,rank", [
    (256, 512, 512, 16),      # tiny layer, CTA pairs
    (200, 384, 256, 32),      # ragged M, K % 256 == 128
    (130, 256, 512, 128),     # maximum rank, ragged M
    (300, 384, 768, 32),      # ragged M and K on 256 x 256 pair tiles
    (3000, 256, 1920, 32),    # 256 x 384 pair tiles
    (96, 512, 640, 48),       # single-CTA kernel
])
def test_y_elementwise_all_rows(M, K, N, rank):
    w = synth.Workload(f"e{M}x{K}x{N}r{rank}", M, K, N, rank, seed=4000 + M + N, outliers="first4",
                       outlier_lo=50.0, outlier_hi=50.0, spikes=2)
    X, W = synth.generate(w)
    Xd, Wd = X.cuda(), W.cuda()
    P = S.svdq_prepare_weights(Wd, S.svdq_channel_amax(Xd), 0.5, rank)
    Qx, Sx, T, Y = gpu_layer(Xd, P, S.SVDQ_FUSED)
    _check(Y, Qx, Sx, T, P, M, K, N)
    Qx2, Sx2, T2, Y2 = gpu_layer(Xd, P, S.SVDQ_UNFUSED)
    _check(Y2, Qx2, Sx2, T2, P, M, K, N, unfused=True)


@pytest.mark.parametrize("w", [synth.FLUX_QKV, synth.FLUX_MLP_DOWN], ids=lambda w: w.name)
def test_y_elementwise_full_flux_column_blocks(w):
    X, W = synth.generate(w)
    Xd, Wd = X.cuda(), W.cuda()
    P = S.svdq_prepare_weights(Wd, S.svdq_channel_amax(Xd), w.alpha, w.rank)   # device SVD
    del Wd
    Qx, Sx, T, Y = gpu_layer(Xd, P, S.SVDQ_FUSED)
    blocks = [0, w.N // 256 // 2, w.N // 256 - 1]
    cols = np.concatenate([np.arange(256 * b, 256 * b + 256) for b in blocks])
    _check(Y, Qx, Sx, T, P, w.M, w.K, w.N, cols)
