"""LoRA through the low-rank branch (walkthrough, Figure 9 and Figure 16: the
branch runs a LoRA with no re-quantization of the residual), and the failure
path of the bounded waits (a wait that nothing completes gives up, the host
reads SVDQ_ERR_TIMEOUT, the context stays usable)."""
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

from gpu_helpers import TOL_Y, gpu_layer, gpu_prepare, np64, oracle_factors_to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


@pytest.mark.parametrize("M,K,N,rank,extra", [(256, 512, 512, 16, 16), (200, 384, 768, 32, 32), (130, 256, 384, 0, 48)])
def test_lora_appended_to_the_branch(M, K, N, rank, extra):
    w = synth.TINY.with_(name="lora", M=M, K=K, N=N, rank=rank, seed=4000 + K + extra)
    X, W = synth.generate(w)
    Xn, Wn = np64(X), np64(W)
    ref = O.layer_reference(Xn, Wn, 0.5, rank)
    rng = np.random.default_rng(5)
    A = O.bf16(rng.standard_normal((extra, K)) * 0.2)        # LoRA down [extra][K]
    B = O.bf16(rng.standard_normal((N, extra)) * 0.2)        # LoRA up   [N][extra]
    Xd = X.cuda()
    amax = S.svdq_channel_amax(Xd)
    P = gpu_prepare(W.cuda(), amax, 0.5, rank, oracle_factors_to_device(ref) if rank else None)
    Ad = torch.from_numpy(A).float().to(torch.bfloat16).cuda()
    Bd = torch.from_numpy(B).float().to(torch.bfloat16).cuda()
    PL = S.svdq_append_lowrank(P, Ad, Bd)
    assert PL.shape.rank == rank + extra
    if rank:
        assert torch.equal(PL.L1p[:rank], P.L1p) and torch.equal(PL.L2t[:, :rank], P.L2t)
    assert torch.equal(PL.L1p[rank:], Ad) and torch.equal(PL.L2t[:, rank:], Bd)

    # oracle: the same layer with the concatenated branch, residual untouched
    L1p_cat = np.concatenate([ref["L1p"], A.T], axis=1) if rank else A.T.copy()
    L2_cat = np.concatenate([ref["L2"], B.T], axis=0) if rank else B.T.copy()
    cx, sx, T = O.quantize_act(Xn, ref["inv32"], L1p_cat)
    Y_ref = O.linear(cx, sx, T, ref["Qr"], ref["Sr"], L2_cat)
    for variant in (S.SVDQ_FUSED, S.SVDQ_UNFUSED):
        _, _, _, Y = gpu_layer(Xd, PL, variant)
        assert O.rel_fro(np64(Y), Y_ref) < TOL_Y, variant
    # the LoRA update itself: Y_lora - Y_base == X A^T B^T up to the bf16 roundings
    _, _, _, Y0 = gpu_layer(Xd, P)
    delta = Xn @ A.T @ B.T
    assert O.rel_fro(np64(Y) - np64(Y0), delta) < 1e-2


def test_bounded_wait_reports_timeout_and_context_survives():
    S.svdq_check()                                   # start from a clear error word
    S.svdq_selftest_timeout()
    with pytest.raises(S.SvdqError) as e:
        S.svdq_check()
    assert e.value.status == 7 and "device error 6" in str(e.value)   # SVDQ_ERR_TIMEOUT, kDevErrSelfTest
    S.svdq_check()                                   # cleared
    # the context still runs the layer correctly
    w = synth.TINY
    X, W = synth.generate(w)
    ref = O.layer_reference(np64(X), np64(W), 0.5, w.rank)
    Xd = X.cuda()
    P = gpu_prepare(W.cuda(), S.svdq_channel_amax(Xd), 0.5, w.rank, oracle_factors_to_device(ref))
    Qx, _, _, Y = gpu_layer(Xd, P)
    assert np.array_equal(Qx.cpu().numpy(), O.pack_nibbles(ref["Qx"]))
    assert O.rel_fro(np64(Y), ref["Y"]) < TOL_Y
