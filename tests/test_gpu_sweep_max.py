"""The sweep's largest layers at full size (M = 18432, K = N = 3072; rank 0,
32 and the maximum rank 128), in the launch configuration the benchmark times
(the library chooses it: 128-row quantizer CTAs without a K split at this M,
256 x 256 CTA-pair GEMM tiles). Checked on outputs the oracle computes row by
row (devpress.csdn.net SVDQuant walkthrough, eq. (1), eq. (2), eq. (5)):

  * packed codes and native scale bytes of sampled rows, bit for bit against
    the oracle quantizer applied to those rows with the GPU's own inverse
    smoothing factors;
  * T of the sampled rows within 4e-3 (relative Frobenius) of fp64 X L1p^T;
  * every sampled row of Y in two 256-column blocks against the fp64 sum of
    the GPU's own operands, within bf16 rounding plus the fp32 accumulation
    bound (2^-8 |ref| + 2^-14 sum |terms|).
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

from gpu_helpers import TOL_T, gpu_layer, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


@pytest.mark.parametrize("rank", [0, 32, 128])
def test_sweep_max_rows_sampled(rank):
    w = next(x for x in synth.sweep() if x.M == 18432 and x.rank == rank)
    M, K, N = w.M, w.K, w.N
    X, W = synth.generate(w)
    Xd, Wd = X.cuda(), W.cuda()
    P = S.svdq_prepare_weights(Wd, S.svdq_channel_amax(Xd), w.alpha, rank)
    del Wd
    Qx, Sx, T, Y = gpu_layer(Xd, P, S.SVDQ_FUSED)

    rng = np.random.default_rng(18432 + rank)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, M // 2, M - 129, M - 128, M - 1],
                                     rng.choice(M, 1016, replace=False)]))
    ri = torch.from_numpy(rows)
    Xn = np64(X[ri])
    inv32 = P.inv_lam.cpu().numpy()
    L1p = np64(P.L1p).T if rank else np.zeros((K, 0))
    codes, scales, Tref = O.quantize_act(Xn, inv32, L1p)

    Qn = Qx.cpu().numpy().reshape(M, K // 2)[rows]
    assert np.array_equal(Qn, O.pack_nibbles(codes))
    Sn = O.native_to_scales(Sx.cpu().numpy(), M, K)[rows]
    assert np.array_equal(Sn, scales)
    if rank:
        assert O.rel_fro(np64(T[ri.cuda()]), Tref) < TOL_T

    cols = np.concatenate([np.arange(0, 256), np.arange(N - 256, N)])
    A = O.dequantize_nvfp4(O.unpack_nibbles(Qn), Sn)
    Bc = O.dequantize_nvfp4(O.unpack_nibbles(P.Qr.cpu().numpy().reshape(N, K // 2))[cols],
                            O.native_to_scales(P.Sr.cpu().numpy(), N, K)[cols])
    ref = A @ Bc.T
    absum = np.abs(A) @ np.abs(Bc).T
    if rank:
        Tn, Ln = np64(T[ri.cuda()]), np64(P.L2t)[cols]
        ref += Tn @ Ln.T
        absum += np.abs(Tn) @ np.abs(Ln).T
    Yn = np64(Y[ri.cuda()][:, torch.from_numpy(cols).cuda()])
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -14 * absum
    bad = np.abs(Yn - ref) > bound
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[:5])
    assert float(np.median(bound / np.maximum(absum, 1e-30))) < 4e-3
