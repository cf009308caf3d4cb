"""Guard regions around every output buffer of the GPU path.

Each output is a view into the middle of a larger device buffer whose head and
tail (4 KB each) hold a byte pattern; after the calls the pattern must be
intact, i.e. no kernel writes outside the documented extent of its outputs.
Shapes are ragged: partial last row tiles, column tiles half outside N, the
padding rows of the scale layouts, one-row inputs, rank 0 and 128.
"""
import ctypes

import pytest
import torch

from w4a4_diffusion_model_b200 import svdq as S
from w4a4_diffusion_model_b200 import synth

pytestmark = pytest.mark.gpu

PAT = 0xA5
GUARD = 4096


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    S.load()


class Guarded:
    """A device buffer of `nbytes` (viewed as dtype/shape) between two guards."""

    def __init__(self, nbytes, dtype=torch.uint8, shape=None):
        self.nbytes = nbytes
        self.buf = torch.full((GUARD + nbytes + GUARD,), PAT, dtype=torch.uint8, device="cuda")
        v = self.buf[GUARD:GUARD + nbytes].view(dtype)
        self.t = v.view(shape) if shape is not None else v

    def intact(self) -> bool:
        return bool((self.buf[:GUARD] == PAT).all()) and bool((self.buf[GUARD + self.nbytes:] == PAT).all())


def ptr(g):
    return ctypes.c_void_p(g.t.data_ptr()) if g is not None else None


def stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


SHAPES = [
    # M, K, N, rank
    (300, 384, 768, 32),      # CTA pairs, ragged M, K % 256 == 128
    (130, 256, 384, 128),     # single-CTA GEMM, maximum rank, INT4 tile partly past N
    (1, 128, 128, 0),         # one row, no branch
    (200, 512, 640, 48),      # N % 256 != 0, INT4 last tile 64 wide
    (2100, 512, 1024, 16),    # several row blocks, pair tiles
]


@pytest.mark.parametrize("M,K,N,rank", SHAPES)
def test_outputs_stay_inside_their_buffers(M, K, N, rank):
    lib = S.load()
    w = synth.Workload(f"g{M}x{K}x{N}r{rank}", M, K, N, rank, seed=4000 + M + N, outliers="frac",
                       outlier_frac=0.01, spikes=2)
    X, W = synth.generate(w)
    Xd, Wd = X.cuda(), W.cuda()
    shape = S.LayerShape(M, K, N, rank)
    guards = {}

    # channel maxima
    amax = guards["amax"] = Guarded(4 * K, torch.float32)
    amax.t.zero_()
    assert lib.svdq_channel_amax(M, K, ctypes.c_void_p(Xd.data_ptr()), ptr(amax), stream()) == 0

    # prepare (device SVD in a workspace)
    qr_b, sr_b, l1_b, l2_b, ws_b = S.svdq_weight_sizes(shape)
    Qr = guards["Qr"] = Guarded(qr_b)
    Sr = guards["Sr"] = Guarded(sr_b)
    L1p = guards["L1p"] = Guarded(l1_b, torch.bfloat16, (rank, K)) if rank else None
    L2t = guards["L2t"] = Guarded(l2_b, torch.bfloat16, (N, rank)) if rank else None
    lam = guards["lam"] = Guarded(4 * K, torch.float32)
    inv = guards["inv"] = Guarded(4 * K, torch.float32)
    work = torch.empty(max(ws_b, 16), dtype=torch.uint8, device="cuda")
    assert lib.svdq_prepare_weights(shape.c(), ctypes.c_void_p(Wd.data_ptr()), ptr(amax), ctypes.c_float(0.5), 0,
                                    ptr(L1p), ptr(L2t), ptr(Qr), ptr(Sr), ptr(lam), ptr(inv),
                                    ctypes.c_void_p(work.data_ptr()), ws_b, stream()) == 0, lib.svdq_last_error()
    P = S.PreparedWeights(S.LayerShape(0, K, N, rank), Qr.t.view(N, K // 2), Sr.t, L1p.t if rank else None,
                          L2t.t if rank else None, lam.t, inv.t)

    # NVFP4 per-call path, fused and unfused
    qx_b, sx_b, t_b = S.svdq_act_sizes(shape)
    for variant in (S.SVDQ_FUSED, S.SVDQ_UNFUSED):
        Qx = guards[f"Qx{variant}"] = Guarded(qx_b, torch.uint8, (M, K // 2))
        Sx = guards[f"Sx{variant}"] = Guarded(sx_b)
        T = guards[f"T{variant}"] = Guarded(t_b, torch.bfloat16, (M, rank)) if rank else None
        Y = guards[f"Y{variant}"] = Guarded(2 * M * N, torch.bfloat16, (M, N))
        S.svdq_quantize_act(Xd, inv.t, P.L1p, rank, N, variant, out=(Qx.t, Sx.t, T.t if rank else None))
        S.svdq_linear(Qx.t, Sx.t, T.t if rank else None, P, variant, out=Y.t)

    # next-layer quantization (rank-0 next layer: the fused epilogue where it applies)
    Qx, Sx, T = guards["Qx0"], guards["Sx0"], guards.get("T0")
    _, snb, _ = S.svdq_act_sizes(S.LayerShape(M, N, 128, 0))
    Qn = guards["Qn"] = Guarded(M * N // 2, torch.uint8, (M, N // 2))
    Sn = guards["Sn"] = Guarded(snb)
    Yn = guards["Yn"] = Guarded(2 * M * N, torch.bfloat16, (M, N))
    inv_n = torch.ones(N, dtype=torch.float32, device="cuda")
    S.svdq_linear_quantize_next(Qx.t, Sx.t, T.t if rank else None, P, inv_n, None, 0, out=(Qn.t, Sn.t, None, Yn.t))

    # INT4 variant
    q4_b, s4_b = S.svdq_int4_weight_sizes(shape)
    Qr4 = guards["Qr4"] = Guarded(q4_b, torch.uint8, (N, K))
    Sr4 = guards["Sr4"] = Guarded(s4_b, torch.float32, (K // 64, N))
    assert lib.svdq_int4_quantize_residual(shape.c(), ctypes.c_void_p(Wd.data_ptr()), ptr(lam), ptr(L1p), ptr(L2t),
                                           ptr(Qr4), ptr(Sr4), stream()) == 0
    W4 = S.Int4Weights(S.LayerShape(0, K, N, rank), Qr4.t, Sr4.t, P.L2t, P.L1p, inv.t)
    a4, s4, t4 = S.svdq_int4_act_sizes(shape)
    Qx4 = guards["Qx4"] = Guarded(a4, torch.uint8, (M, K))
    Sx4 = guards["Sx4"] = Guarded(s4, torch.float32, (K // 64, (M + 127) // 128 * 128))
    T4 = guards["T4"] = Guarded(t4, torch.bfloat16, (M, rank)) if rank else None
    Y4 = guards["Y4"] = Guarded(2 * M * N, torch.bfloat16, (M, N))
    S.svdq_int4_quantize_act(Xd, inv.t, P.L1p, rank, N, out=(Qx4.t, Sx4.t, T4.t if rank else None))
    S.svdq_int4_linear(Qx4.t, Sx4.t, T4.t if rank else None, W4, out=Y4.t)

    S.svdq_check()
    bad = [name for name, g in guards.items() if g is not None and not g.intact()]
    assert not bad, bad
    assert torch.isfinite(guards["Y0"].t.float()).all() and torch.isfinite(Y4.t.float()).all()
