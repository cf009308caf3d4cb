"""svdq_prepare_weights_static: the weight preparation that runs its device
SVD in the library's fixed scratch instead of a caller workspace. Called
through the C ABI and compared with svdq_prepare_weights (caller workspace) on
the same inputs, for two calls in a row (the second one must leave the
device's free memory and torch's allocation count unchanged); shapes beyond
the scratch are refused.

This file is collected last and also passes on its own in a fresh process."""
import ctypes

import pytest
import torch

from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20     # SVDQ_STATIC_SCRATCH_BYTES


def _p(t):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _static_prepare(lib, W, amax, alpha, rank, check_no_alloc=False):
    N, K = W.shape
    qr, sr, l1, l2, _ = S.svdq_weight_sizes(S.LayerShape(0, K, N, rank))
    dev = W.device
    out = {
        "L1p": torch.empty(rank, K, dtype=torch.bfloat16, device=dev),
        "L2t": torch.empty(N, rank, dtype=torch.bfloat16, device=dev),
        "Qr": torch.empty(qr, dtype=torch.uint8, device=dev),
        "Sr": torch.empty(sr, dtype=torch.uint8, device=dev),
        "lam": torch.empty(K, dtype=torch.float32, device=dev),
        "inv_lam": torch.empty(K, dtype=torch.float32, device=dev),
    }
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    st = lib.svdq_prepare_weights_static(
        S.Shape(0, K, N, rank), _p(W), _p(amax), ctypes.c_float(alpha), 0, _p(out["L1p"]), _p(out["L2t"]),
        _p(out["Qr"]), _p(out["Sr"]), _p(out["lam"]), _p(out["inv_lam"]),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.svdq_last_error().decode()
    assert lib.svdq_check(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    if check_no_alloc:
        # after a first call has loaded the kernels, a call takes no device
        # memory: neither from the driver nor from torch's allocator
        assert torch.cuda.mem_get_info()[0] == free0
        assert torch.cuda.memory_allocated() == alloc0
    return out


@pytest.mark.parametrize("tmpl,K,N,rank", [(synth.TINY, 512, 512, 16), (synth.FLUX_QKV, 3072, 1024, 32),
                                           (synth.FLUX_MLP_DOWN, 1536, 384, 48),
                                           (synth.FLUX_QKV, 3072, 9216, 32)])   # the full QKV weight
def test_static_scratch_prepare_matches_workspace_prepare(tmpl, K, N, rank):
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    lib = S.load()
    w = tmpl.with_(name=f"noalloc_{K}x{N}_r{rank}", M=128, K=K, N=N, rank=rank, seed=tmpl.seed + 3 * K + N)
    X, W = synth.generate(w)
    Xd, Wd = X.cuda(), W.cuda()
    amax = S.svdq_channel_amax(Xd)
    *_, ws = S.svdq_weight_sizes(S.LayerShape(0, K, N, rank))
    assert 0 < ws <= SCRATCH_BYTES
    ref = S.svdq_prepare_weights(Wd, amax, 0.5, rank)
    torch.cuda.synchronize()
    for call in range(2):
        got = _static_prepare(lib, Wd, amax, 0.5, rank, check_no_alloc=call > 0)
        for name in ("lam", "inv_lam", "Qr", "Sr"):
            assert torch.equal(got[name], getattr(ref, name).reshape(got[name].shape)), (call, name)
        for name in ("L1p", "L2t"):
            a, b = got[name].float(), getattr(ref, name).float()
            assert torch.allclose(a, b, rtol=0.0, atol=0.0), (call, name, (a - b).abs().max().item())
        Qx, Sx, T = S.svdq_quantize_act(Xd, got["inv_lam"], got["L1p"], rank, N)
        P = S.PreparedWeights(S.LayerShape(0, K, N, rank), got["Qr"].view(N, K // 2), got["Sr"], got["L1p"],
                              got["L2t"], got["lam"], got["inv_lam"])
        Y = S.svdq_linear(Qx, Sx, T, P)
        Y_ref = S.svdq_linear(Qx, Sx, T, ref)
        assert torch.equal(Y, Y_ref), call


def test_static_scratch_refuses_shapes_beyond_it():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    lib = S.load()
    sh = S.LayerShape(0, 8192, 16384, 128)
    *_, ws = S.svdq_weight_sizes(sh)
    assert ws > SCRATCH_BYTES
    good = ctypes.c_void_p(1 << 20)
    st = lib.svdq_prepare_weights_static(sh.c(), good, good, ctypes.c_float(0.5), 0, good, good, good, good, good,
                                         good, None)
    assert st == 4                       # SVDQ_ERR_BUFFER_TOO_SMALL, before any device work
    msg = lib.svdq_last_error().decode()
    assert "static scratch" in msg and str(ws) in msg
