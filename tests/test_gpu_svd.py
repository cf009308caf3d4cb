"""The device-side top-rank split of svdq_prepare_weights (no given factors).

The SVD factors have sign and rotation freedom, so they are not compared
element by element. What is fixed (devpress.csdn.net SVDQuant walkthrough,
eq. (3)-(4) and the Eckart-Young remark on the residual's energy):
  * ||W_hat - L1 L2||_F^2 is within (1 + 1e-3) of the optimal tail energy
    sum_{i>r} sigma_i^2 (fp64 LAPACK on the oracle side), plus the slack of
    storing both factors in bf16 (relative rounding 2^-9 per factor);
  * given the factors the library stored, the residual R and its NVFP4
    encoding are bit-exact with the oracle's residual step;
  * the whole layer then matches the oracle within the layer tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

from gpu_helpers import TOL_Y, gpu_layer, np64

pytestmark = pytest.mark.gpu

ENERGY_TOL = 1e-3
BF16_SLACK = 2.0 * 2.0 ** -16     # (2 u)^2 with u = 2^-9, times ||L1 L2||^2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


CASES = [
    # workload template, M (calibration rows), K, N, rank
    (synth.TINY, 256, 512, 512, 16),
    (synth.FLUX_QKV, 256, 3072, 1024, 32),
    (synth.FLUX_QKV, 128, 128, 256, 128),     # rank == K: the split is exact up to bf16
    (synth.FLUX_MLP_DOWN, 128, 1536, 384, 48),
    (synth.FLUX_QKV, 64, 384, 640, 112),
]


def _case(tmpl, M, K, N, rank):
    w = tmpl.with_(name=f"svd_{M}x{K}x{N}_r{rank}", M=M, K=K, N=N, rank=rank, seed=tmpl.seed + 17 * K + N)
    X, W = synth.generate(w)
    return w, X, W


def _device_prepare(X, W, rank):
    Xd, Wd = X.cuda(), W.cuda()
    amax = S.svdq_channel_amax(Xd)
    P = S.svdq_prepare_weights(Wd, amax, 0.5, rank)
    S.svdq_check()
    return Xd, P


@pytest.mark.parametrize("tmpl,M,K,N,rank", CASES, ids=[f"{c[2]}x{c[3]}r{c[4]}" for c in CASES])
def test_device_split_near_optimal_and_residual_exact(tmpl, M, K, N, rank):
    w, X, W = _case(tmpl, M, K, N, rank)
    Xn, Wn = np64(X), np64(W)
    Xd, P = _device_prepare(X, W, rank)
    lam32, inv32 = O.smoothing_lambda(O.channel_amax(Xn), Wn, 0.5)
    assert np.array_equal(P.lam.cpu().numpy(), lam32)

    What = lam32.astype(np.float64)[:, None] * Wn.T
    sig = np.linalg.svd(What, compute_uv=False)
    tail = float(np.sum(sig[rank:] ** 2))
    L1p = np64(P.L1p)            # [r][K]
    L2t = np64(P.L2t)            # [N][r]
    assert np.all(np.isfinite(L1p)) and np.all(np.isfinite(L2t))
    approx = (lam32.astype(np.float64)[:, None] * L1p.T) @ L2t.T
    err = float(np.sum((What - approx) ** 2))
    bound = (1.0 + ENERGY_TOL) * tail + BF16_SLACK * float(np.sum(approx ** 2))
    assert err <= bound, (err, tail, err / max(tail, 1e-300) - 1.0)

    _, codes, scales = O.residual_quantize(Wn, lam32, L1p.T, L2t.T)
    assert np.array_equal(P.Qr.cpu().numpy(), O.pack_nibbles(codes))
    assert np.array_equal(P.Sr.cpu().numpy(), O.scales_to_native(scales))

    cx, sx, T = O.quantize_act(Xn, inv32, L1p.T)
    Y_ref = O.linear(cx, sx, T, codes, scales, L2t.T)
    _, _, _, Y = gpu_layer(Xd, P)
    assert O.rel_fro(np64(Y), Y_ref) < TOL_Y


def test_device_split_is_deterministic():
    w, X, W = _case(synth.FLUX_QKV, 128, 1024, 768, 32)
    _, P1 = _device_prepare(X, W, 32)
    _, P2 = _device_prepare(X, W, 32)
    assert torch.equal(P1.L1p, P2.L1p) and torch.equal(P1.L2t, P2.L2t)
    assert torch.equal(P1.Qr, P2.Qr) and torch.equal(P1.Sr, P2.Sr)


def test_device_split_of_an_exactly_low_rank_weight():
    """W_hat of exact rank r (integer factors): the split captures all of it,
    so the residual is only the bf16 rounding of the stored factors."""
    K, N, r = 256, 384, 16
    rng = np.random.default_rng(7)
    A = rng.integers(-3, 4, size=(N, r)).astype(np.float64)
    B = rng.integers(-3, 4, size=(r, K)).astype(np.float64)
    Wn = (A @ B) / 64.0                           # small integers / 64: exact in bf16
    W = torch.from_numpy(Wn).to(torch.bfloat16)
    assert np.array_equal(np64(W), Wn)
    X = torch.ones(8, K, dtype=torch.bfloat16)    # amax 1: lambda_j = 1 / sqrt(max|W_j|)
    _, P = _device_prepare(X, W, r)
    lam32 = P.lam.cpu().numpy().astype(np.float64)
    What = lam32[:, None] * Wn.T
    approx = (lam32[:, None] * np64(P.L1p).T) @ np64(P.L2t).T
    rel = float(np.sum((What - approx) ** 2) / np.sum(What ** 2))
    assert rel <= BF16_SLACK, rel
