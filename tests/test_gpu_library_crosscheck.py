"""Cross-check of the FP4 GEMM against an independent implementation.

cuBLASLt's NVFP4 GEMM (reached through torch's scaled_mm) consumes E2M1 codes
with one E4M3 scale per 16 K-elements in the 128 x 4 tiled scale layout, which
is the layout this library writes natively. Fed the codes and scales that
svdq_quantize_act and svdq_prepare_weights produced, it must return the same
bf16 Y as svdq_linear without a low-rank branch, element for element: both
evaluate sum_k deq(Qx)[m,k] deq(Qr)[n,k] on the tensor cores in the same
block-scaled MMA arithmetic. A mismatch would point at the nibble order, the
scale layout, the scale-to-MMA mapping or a tile/edge error of the GEMM.
The library GEMM is test infrastructure here only; the product path never
calls it.
"""
import pytest
import torch

from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


def _library_nvfp4_gemm(Qx, Sx, Qr, Sr):
    a = Qx.view(torch.float4_e2m1fn_x2)
    b = Qr.view(torch.float4_e2m1fn_x2).t()
    return torch._scaled_mm(a, b, Sx.view(torch.float8_e4m3fn), Sr.view(torch.float8_e4m3fn),
                            out_dtype=torch.bfloat16)


@pytest.mark.parametrize("M,K,N", [
    (256, 512, 512),      # the tiny layer's shape
    (200, 384, 256),      # ragged M, K % 256 == 128
    (300, 384, 768),      # ragged M and K on 256 x 256 pair tiles
    (512, 1024, 640),     # N % 256 != 0: the single-CTA GEMM
    (3000, 256, 1920),    # 256 x 384 pair tiles
    (4608, 3072, 9216),   # the FLUX QKV projection, 256 x 256 pair tiles
])
def test_rank0_gemm_equals_library_nvfp4_gemm(M, K, N):
    w = synth.Workload(f"x{M}x{K}x{N}", M, K, N, 0, seed=4242 + M + N, outliers="frac",
                       outlier_frac=0.01, spikes=4)
    X, W = synth.generate(w)
    Xd, Wd = X.cuda(), W.cuda()
    amax = S.svdq_channel_amax(Xd)
    P = S.svdq_prepare_weights(Wd, amax, 0.5, 0)
    Qx, Sx, _ = S.svdq_quantize_act(Xd, P.inv_lam, None, 0, N)
    Y = S.svdq_linear(Qx, Sx, None, P)
    S.svdq_check()
    try:
        Yc = _library_nvfp4_gemm(Qx, Sx, P.Qr, P.Sr)
    except (RuntimeError, NotImplementedError) as e:   # a torch build without the NVFP4 GEMM
        pytest.skip(f"library NVFP4 GEMM unavailable: {e}")
    torch.cuda.synchronize()
    assert Y.shape == Yc.shape
    assert torch.isfinite(Y).all().item()
    diff = (Y != Yc).sum().item()
    assert diff == 0, f"{diff} of {Y.numel()} outputs differ from the library NVFP4 GEMM"
