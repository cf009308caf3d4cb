"""Back-to-back launches: the kernels run their prologue while the previous
kernel of the stream finishes and wait for it before touching global memory.
A kernel that read its inputs or wrote its outputs too early would race with
its neighbours; these tests chain many dependent calls with no host
synchronization in between and compare every result with the same call run
in isolation (synchronized before and after), bit for bit.
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


def _layer(M, K, N, rank, seed):
    w = synth.Workload(f"d{M}x{K}x{N}r{rank}", M, K, N, rank, seed=seed, outliers="frac", outlier_frac=0.01,
                       spikes=4)
    X, W = synth.generate(w)
    Xd, Wd = X.cuda(), W.cuda()
    P = S.svdq_prepare_weights(Wd, S.svdq_channel_amax(Xd), 0.5, rank)
    torch.cuda.synchronize()
    return Xd, P


@pytest.mark.parametrize("M,K,N,rank", [(4608, 3072, 9216, 32), (300, 384, 768, 32), (512, 1024, 640, 16)])
def test_back_to_back_steps_match_isolated_calls(M, K, N, rank):
    """Quantize + GEMM of several layers' inputs in a row, sharing the Qx / Sx / T
    buffers (each step overwrites what the previous GEMM is reading)."""
    X0, P = _layer(M, K, N, rank, seed=77 + M)
    xs = [X0] + [(X0 * (1.0 + 0.25 * i)).to(torch.bfloat16) for i in range(1, 4)]
    ref = []
    for X in xs:
        torch.cuda.synchronize()
        Qx, Sx, T = S.svdq_quantize_act(X, P.inv_lam, P.L1p, rank, N)
        torch.cuda.synchronize()
        ref.append(S.svdq_linear(Qx, Sx, T, P).clone())
        torch.cuda.synchronize()
    Qx, Sx, T = S.svdq_quantize_act(xs[0], P.inv_lam, P.L1p, rank, N)
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for _ in xs]
    for rep in range(3):
        for X, Y in zip(xs, Ys):
            S.svdq_quantize_act(X, P.inv_lam, P.L1p, rank, N, out=(Qx, Sx, T))
            S.svdq_linear(Qx, Sx, T, P, out=Y)
    S.svdq_check()
    for Y, R in zip(Ys, ref):
        assert torch.equal(Y, R)


def test_chained_layers_match_isolated_calls():
    """Layer 1's Y is layer 2's X: GEMM -> quantize -> GEMM with no sync, twice."""
    M, K, N1, N2 = 1024, 1024, 2048, 512
    X, P1 = _layer(M, K, N1, 32, seed=5)
    w2 = synth.Workload("d2", M, N1, N2, 16, seed=6, outliers="frac", outlier_frac=0.01, spikes=4)
    _, W2 = synth.generate(w2)
    Y1_probe = torch.empty(M, N1, dtype=torch.bfloat16, device="cuda")
    Qx, Sx, T = S.svdq_quantize_act(X, P1.inv_lam, P1.L1p, 32, N1)
    S.svdq_linear(Qx, Sx, T, P1, out=Y1_probe)
    P2 = S.svdq_prepare_weights(W2.cuda(), S.svdq_channel_amax(Y1_probe), 0.5, 16)
    torch.cuda.synchronize()

    def run(sync):
        def barrier():
            if sync:
                torch.cuda.synchronize()
        Qa, Sa, Ta = S.svdq_quantize_act(X, P1.inv_lam, P1.L1p, 32, N1)
        barrier()
        Y1 = S.svdq_linear(Qa, Sa, Ta, P1)
        barrier()
        Qb, Sb, Tb = S.svdq_quantize_act(Y1, P2.inv_lam, P2.L1p, 16, N2)
        barrier()
        Y2 = S.svdq_linear(Qb, Sb, Tb, P2)
        barrier()
        return Y1, Y2
    r1, r2 = run(True)
    for _ in range(2):
        y1, y2 = run(False)
        S.svdq_check()
        assert torch.equal(y1, r1)
        assert torch.equal(y2, r2)
