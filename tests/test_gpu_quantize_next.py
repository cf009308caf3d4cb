"""Parity of svdq_linear_quantize_next: Y of one layer, quantized for the next.

The reference is the two-call sequence on the same device data (svdq_linear,
then svdq_quantize_act on its Y) and the oracle's quantizer applied to that Y
(the oracle is fed the library's tolerance-checked Y, as in the other
conditional parity checks). Bar: next_Qx, the native next_Sx (padding rows
included) and Y (when it is stored) bit-exact against the two calls. next_T
(for a next layer with a low-rank branch) within the T tolerance of the fp64
product Y L1p'^T; on the two-call route it is also bit-exact against the two
calls, on the fused route (next rank 16 or 32 on 256 x 256 pair tiles: the
epilogue's tcgen05 partials, added in tile order) within the T tolerance of
them and identical from call to call. Shapes cover the fused epilogue (next
ranks 0, 16, 32, with ragged M, rows past the padded end of the last row
block, and several tiles per CTA pair) and the two-call route (next ranks 48,
128; the single-CTA kernel), and full-size FLUX projections for both.
"""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

from gpu_helpers import TOL_T, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


def _layer(M, K, N, rank, seed):
    w = synth.Workload(f"q{M}x{K}x{N}r{rank}", M, K, N, rank, seed=seed, outliers="frac", outlier_frac=0.01,
                       spikes=4)
    X, W = synth.generate(w)
    Xd, Wd = X.cuda(), W.cuda()
    P = S.svdq_prepare_weights(Wd, S.svdq_channel_amax(Xd), 0.5, rank)
    Qx, Sx, T = S.svdq_quantize_act(Xd, P.inv_lam, P.L1p, rank, N)
    return P, Qx, Sx, T


def _next_layer(N, next_rank, seed):
    """The next layer's smoothing and down-projection factors (K' = N)."""
    rng = np.random.default_rng(seed)
    inv = np.exp(rng.uniform(-1.5, 1.5, N)).astype(np.float32)
    L1p = rng.standard_normal((next_rank, N)) / np.sqrt(N)
    L1p_t = torch.from_numpy(L1p).to(torch.float32).to(torch.bfloat16)
    return torch.from_numpy(inv).cuda(), L1p_t.cuda() if next_rank else None


def _fused(M, K, N, rank, next_rank, flags=S.SVDQ_NEXT_FUSE_LOWRANK) -> bool:
    """Whether the library takes the low-rank fused route: its workspace then
    holds the fp32 partials of T' ([N/256][M][next_rank]) instead of Y."""
    ws = S.svdq_linear_quantize_next_workspace(S.LayerShape(M, K, N, rank), next_rank, flags)
    return next_rank > 0 and ws == (N // 256) * M * next_rank * 4


def _two_calls(Qx, Sx, T, P, inv_n, L1p_n, next_rank):
    Y = S.svdq_linear(Qx, Sx, T, P)
    Qn, Sn, Tn = S.svdq_quantize_act(Y, inv_n, L1p_n, next_rank, 128)
    S.svdq_check()
    return Y, Qn, Sn, Tn


@pytest.mark.parametrize("M,K,N,rank,next_rank", [
    (256, 512, 512, 16, 0),       # fused epilogue on pair tiles
    (300, 384, 768, 32, 0),       # fused, ragged M, K % 256 == 128
    (4400, 1024, 2048, 32, 0),    # fused; the last pair tile has rows past the padded end of the scales
    (1000, 256, 1024, 0, 0),      # fused, no branch in the producer
    (256, 512, 512, 16, 32),      # a low-rank next layer: T' partials in the epilogue
    (300, 384, 768, 32, 16),      # ... ragged M
    (4400, 1024, 2048, 32, 32),   # ... 144 tiles: two tiles on most CTA pairs
    (4608, 256, 4096, 16, 16),    # ... 288 tiles: four tiles per CTA pair
    (1000, 256, 1024, 0, 128),    # the largest next rank: Y, then the quantizer
    (4400, 1024, 2048, 32, 48),   # next rank 48: Y, then the quantizer
    (512, 1024, 640, 32, 0),      # N % 256 != 0: single-CTA GEMM, then the quantizer
    (130, 256, 384, 16, 0),       # small M and N % 256 != 0
])
@pytest.mark.parametrize("flags", [0, S.SVDQ_NEXT_FUSE_LOWRANK], ids=["default", "fuse_lowrank"])
def test_fused_next_quantization_matches_two_calls_and_oracle(M, K, N, rank, next_rank, flags):
    if flags and not _fused(M, K, N, rank, next_rank):
        pytest.skip("the low-rank fused route does not serve this shape / next rank")
    P, Qx, Sx, T = _layer(M, K, N, rank, seed=500 + M + N)
    inv_n, L1p_n = _next_layer(N, next_rank, seed=900 + N)
    Y, Qn2, Sn2, Tn2 = _two_calls(Qx, Sx, T, P, inv_n, L1p_n, next_rank)

    Qn, Sn, Tn, Yf = S.svdq_linear_quantize_next(Qx, Sx, T, P, inv_n, L1p_n, next_rank, store_y=True, flags=flags)
    Qn0, Sn0, Tn0, Y0 = S.svdq_linear_quantize_next(Qx, Sx, T, P, inv_n, L1p_n, next_rank, store_y=False, flags=flags)
    S.svdq_check()
    assert Y0 is None
    assert torch.equal(Yf, Y)
    for q, s in ((Qn, Sn), (Qn0, Sn0)):
        assert torch.equal(q, Qn2)
        assert torch.equal(s, Sn2)

    # the oracle's quantizer on the same Y
    Yn = np64(Y)
    L1p_o = np64(L1p_n).T if next_rank else np.zeros((N, 0))
    codes, scales, T_ref = O.quantize_act(Yn, inv_n.cpu().numpy(), L1p_o)
    assert np.array_equal(Qn.cpu().numpy(), O.pack_nibbles(codes))
    assert np.array_equal(Sn.cpu().numpy(), O.scales_to_native(scales))
    if next_rank:
        assert O.rel_fro(np64(Tn), T_ref) < TOL_T
        if flags and _fused(M, K, N, rank, next_rank):
            assert O.rel_fro(np64(Tn), np64(Tn2)) < TOL_T
            assert torch.equal(Tn0, Tn)                       # the same order of additions every call
        else:
            assert torch.equal(Tn, Tn2) and torch.equal(Tn0, Tn2)
    else:
        assert Tn is None and Tn0 is None


@pytest.mark.parametrize("w,next_rank,flags", [(synth.FLUX_MLP_UP, 32, S.SVDQ_NEXT_FUSE_LOWRANK),
                                               (synth.FLUX_MLP_UP, 32, 0), (synth.FLUX_QKV, 0, 0)],
                         ids=["mlp_up_r32_fused", "mlp_up_r32_two_calls", "qkv_r0"])
def test_flux_projection_full_size(w, next_rank, flags):
    """A full-size FLUX projection quantizing its output for a next layer of
    the given rank (MLP-up -> MLP-down at rank 32 and a rank-0 next layer both
    run in the fused epilogue): against the two calls on the GPU, the oracle on
    sampled rows."""
    P, Qx, Sx, T = _layer(w.M, w.K, w.N, w.rank, seed=w.seed)
    inv_n, L1p_n = _next_layer(w.N, next_rank, seed=w.seed + 1)
    Y, Qn2, Sn2, Tn2 = _two_calls(Qx, Sx, T, P, inv_n, L1p_n, next_rank)
    Qn, Sn, Tn, _ = S.svdq_linear_quantize_next(Qx, Sx, T, P, inv_n, L1p_n, next_rank, flags=flags)
    S.svdq_check()
    assert torch.equal(Qn, Qn2)
    assert torch.equal(Sn, Sn2)
    if next_rank and flags:
        assert _fused(w.M, w.K, w.N, w.rank, next_rank, flags)
        assert O.rel_fro(np64(Tn), np64(Tn2)) < TOL_T
    elif next_rank:
        assert torch.equal(Tn, Tn2)
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(w.M, 32, replace=False), [0, w.M - 1]]))
    Yr = np64(Y[torch.from_numpy(rows).cuda()])
    L1p_o = np64(L1p_n).T if next_rank else np.zeros((w.N, 0))
    codes, scales, T_ref = O.quantize_act(Yr, inv_n.cpu().numpy(), L1p_o)
    assert np.array_equal(Qn.cpu().numpy()[rows], O.pack_nibbles(codes))
    can = S.svdq_scales_to_canonical(Sn, w.M, w.N).cpu().numpy()
    assert np.array_equal(can[rows], scales)
    if next_rank:
        assert O.rel_fro(np64(Tn)[rows], T_ref) < TOL_T
