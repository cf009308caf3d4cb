"""Python binding of the SVDQuant W4A4 C ABI (include/svdq.h).

Argument marshalling only: every step of the layer runs in the CUDA library
``libsvdq.so`` built in this directory. Tensors are torch CUDA tensors; calls
are issued on torch's current CUDA stream. There is no CPU fallback: if the
library is missing or the device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

SVDQ_FUSED = 0
SVDQ_UNFUSED = 1
SVDQ_PREPARE_GIVEN_FACTORS = 1
SVDQ_NEXT_FUSE_LOWRANK = 1

STATUS = {
    0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_UNSUPPORTED_SHAPE", 3: "SVDQ_ERR_MISALIGNED",
    4: "SVDQ_ERR_BUFFER_TOO_SMALL", 5: "SVDQ_ERR_NO_DEVICE", 6: "SVDQ_ERR_CUDA", 7: "SVDQ_ERR_TIMEOUT",
    8: "SVDQ_ERR_INTERNAL",
}

# Every symbol the header declares, with its ctypes signature.
EXPORTS = [
    "svdq_status_string", "svdq_last_error", "svdq_version", "svdq_act_sizes", "svdq_weight_sizes",
    "svdq_channel_amax", "svdq_prepare_weights", "svdq_prepare_weights_static", "svdq_quantize_act",
    "svdq_linear", "svdq_linear_quantize_next", "svdq_linear_quantize_next_workspace", "svdq_append_lowrank",
    "svdq_selftest_timeout", "svdq_scales_to_canonical", "svdq_check",
    "svdq_int4_act_sizes", "svdq_int4_weight_sizes", "svdq_int4_quantize_residual", "svdq_int4_quantize_act",
    "svdq_int4_linear", "svdq_deltaquant_sizes", "svdq_deltaquant_encode",
]


class Shape(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("K", ctypes.c_int64), ("N", ctypes.c_int64), ("rank", ctypes.c_int32)]


class SvdqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m w4a4_diffusion_model_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i64, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int
    P = ctypes.POINTER
    lib.svdq_status_string.argtypes, lib.svdq_status_string.restype = [ctypes.c_int], ctypes.c_char_p
    lib.svdq_last_error.argtypes, lib.svdq_last_error.restype = [], ctypes.c_char_p
    lib.svdq_version.argtypes, lib.svdq_version.restype = [], ctypes.c_int
    lib.svdq_act_sizes.argtypes, lib.svdq_act_sizes.restype = [Shape, P(sz), P(sz), P(sz)], st
    lib.svdq_weight_sizes.argtypes = [Shape, P(sz), P(sz), P(sz), P(sz), P(sz)]
    lib.svdq_weight_sizes.restype = st
    lib.svdq_channel_amax.argtypes, lib.svdq_channel_amax.restype = [i64, i64, vp, vp, vp], st
    lib.svdq_prepare_weights.argtypes = [Shape, vp, vp, ctypes.c_float, ctypes.c_uint, vp, vp, vp, vp, vp, vp,
                                         vp, sz, vp]
    lib.svdq_prepare_weights.restype = st
    lib.svdq_prepare_weights_static.argtypes = [Shape, vp, vp, ctypes.c_float, ctypes.c_uint, vp, vp, vp, vp, vp,
                                                vp, vp]
    lib.svdq_prepare_weights_static.restype = st
    lib.svdq_append_lowrank.argtypes = [Shape, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp]
    lib.svdq_append_lowrank.restype = st
    lib.svdq_selftest_timeout.argtypes = [vp]
    lib.svdq_selftest_timeout.restype = st
    lib.svdq_quantize_act.argtypes = [Shape, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp]
    lib.svdq_quantize_act.restype = st
    lib.svdq_linear.argtypes = [Shape, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp]
    lib.svdq_linear.restype = st
    lib.svdq_scales_to_canonical.argtypes, lib.svdq_scales_to_canonical.restype = [i64, i64, vp, vp, vp], st
    lib.svdq_check.argtypes, lib.svdq_check.restype = [vp], st
    lib.svdq_linear_quantize_next.argtypes = [Shape, vp, vp, vp, vp, vp, vp, ctypes.c_int32, vp, vp, vp, vp, vp, vp,
                                              vp, sz, ctypes.c_uint, vp]
    lib.svdq_linear_quantize_next.restype = st
    lib.svdq_linear_quantize_next_workspace.argtypes = [Shape, ctypes.c_int32, ctypes.c_uint, P(sz)]
    lib.svdq_linear_quantize_next_workspace.restype = st
    lib.svdq_int4_act_sizes.argtypes, lib.svdq_int4_act_sizes.restype = [Shape, P(sz), P(sz), P(sz)], st
    lib.svdq_int4_weight_sizes.argtypes, lib.svdq_int4_weight_sizes.restype = [Shape, P(sz), P(sz)], st
    lib.svdq_int4_quantize_residual.argtypes = [Shape, vp, vp, vp, vp, vp, vp, vp]
    lib.svdq_int4_quantize_residual.restype = st
    lib.svdq_int4_quantize_act.argtypes, lib.svdq_int4_quantize_act.restype = [Shape, vp, vp, vp, vp, vp, vp, vp], st
    lib.svdq_int4_linear.argtypes, lib.svdq_int4_linear.restype = [Shape, vp, vp, vp, vp, vp, vp, vp, vp], st
    lib.svdq_deltaquant_sizes.argtypes = [i64, i64, i64, i64, P(sz), P(sz), P(sz)]
    lib.svdq_deltaquant_sizes.restype = st
    lib.svdq_deltaquant_encode.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp, vp]
    lib.svdq_deltaquant_encode.restype = st
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        raise SvdqError(status, load().svdq_last_error().decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@dataclass(frozen=True)
class LayerShape:
    M: int
    K: int
    N: int
    rank: int

    def c(self) -> Shape:
        return Shape(self.M, self.K, self.N, self.rank)


def svdq_act_sizes(shape: LayerShape) -> tuple[int, int, int]:
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().svdq_act_sizes(shape.c(), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def svdq_weight_sizes(shape: LayerShape) -> tuple[int, int, int, int, int]:
    v = [ctypes.c_size_t() for _ in range(5)]
    _check(load().svdq_weight_sizes(shape.c(), *[ctypes.byref(x) for x in v]))
    return tuple(x.value for x in v)


def svdq_channel_amax(X: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    M, K = X.shape
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=X.device)
    _check(load().svdq_channel_amax(M, K, _ptr(X), _ptr(out), _stream()))
    return out


@dataclass
class PreparedWeights:
    shape: LayerShape          # M is unused (0)
    Qr: torch.Tensor
    Sr: torch.Tensor
    L1p: torch.Tensor | None
    L2t: torch.Tensor | None
    lam: torch.Tensor
    inv_lam: torch.Tensor


def svdq_prepare_weights(W_lin: torch.Tensor, act_amax: torch.Tensor, alpha: float, rank: int,
                         L1p: torch.Tensor | None = None, L2t: torch.Tensor | None = None) -> PreparedWeights:
    """Smoothing, top-rank split and residual NVFP4 encoding of W_lin [N][K].
    Pass both L1p [rank][K] and L2t [N][rank] (bf16) to use given factors."""
    N, K = W_lin.shape
    shape = LayerShape(0, K, N, rank)
    qr, sr, l1, l2, ws = svdq_weight_sizes(shape)
    dev = W_lin.device
    given = L1p is not None and L2t is not None
    if not given:
        L1p = torch.empty(rank, K, dtype=torch.bfloat16, device=dev) if rank else None
        L2t = torch.empty(N, rank, dtype=torch.bfloat16, device=dev) if rank else None
    Qr = torch.empty(qr, dtype=torch.uint8, device=dev)
    Sr = torch.empty(sr, dtype=torch.uint8, device=dev)
    lam = torch.empty(K, dtype=torch.float32, device=dev)
    inv = torch.empty(K, dtype=torch.float32, device=dev)
    work = torch.empty(ws, dtype=torch.uint8, device=dev) if (ws and not given) else None
    _check(load().svdq_prepare_weights(
        shape.c(), _ptr(W_lin), _ptr(act_amax), ctypes.c_float(alpha),
        SVDQ_PREPARE_GIVEN_FACTORS if given else 0, _ptr(L1p), _ptr(L2t), _ptr(Qr), _ptr(Sr), _ptr(lam), _ptr(inv),
        _ptr(work), ws if work is not None else 0, _stream()))
    return PreparedWeights(shape, Qr.view(N, K // 2), Sr, L1p, L2t, lam, inv)


def svdq_quantize_act(X: torch.Tensor, inv_lambda: torch.Tensor, L1p: torch.Tensor | None, rank: int, N: int = 128,
                      variant: int = SVDQ_FUSED, out: tuple | None = None):
    """Returns (Qx [M][K/2] uint8, Sx native uint8, T [M][rank] bf16 or None)."""
    M, K = X.shape
    shape = LayerShape(M, K, N, rank)
    if out is None:
        qx, sx, _ = svdq_act_sizes(shape)
        Qx = torch.empty(M, K // 2, dtype=torch.uint8, device=X.device)
        Sx = torch.empty(sx, dtype=torch.uint8, device=X.device)
        T = torch.empty(M, rank, dtype=torch.bfloat16, device=X.device) if rank else None
    else:
        Qx, Sx, T = out
    _check(load().svdq_quantize_act(shape.c(), _ptr(X), _ptr(inv_lambda), _ptr(L1p), _ptr(Qx), _ptr(Sx), _ptr(T),
                                    variant, _stream()))
    return Qx, Sx, T


def svdq_linear(Qx: torch.Tensor, Sx: torch.Tensor, T: torch.Tensor | None, W: PreparedWeights,
                variant: int = SVDQ_FUSED, out: torch.Tensor | None = None) -> torch.Tensor:
    M = Qx.shape[0]
    K, N, rank = W.shape.K, W.shape.N, W.shape.rank
    shape = LayerShape(M, K, N, rank)
    Y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=Qx.device)
    _check(load().svdq_linear(shape.c(), _ptr(Qx), _ptr(Sx), _ptr(T), _ptr(W.Qr), _ptr(W.Sr), _ptr(W.L2t), _ptr(Y),
                              variant, _stream()))
    return Y


def svdq_linear_quantize_next_workspace(shape: LayerShape, next_rank: int, flags: int = 0) -> int:
    v = ctypes.c_size_t()
    _check(load().svdq_linear_quantize_next_workspace(shape.c(), next_rank, flags, ctypes.byref(v)))
    return v.value


def svdq_linear_quantize_next(Qx: torch.Tensor, Sx: torch.Tensor, T: torch.Tensor | None, W: PreparedWeights,
                              next_inv_lambda: torch.Tensor, next_L1p: torch.Tensor | None, next_rank: int,
                              store_y: bool = False, out: tuple | None = None, workspace: torch.Tensor | None = None,
                              flags: int = 0):
    """svdq_linear whose epilogue also quantizes Y for the next layer (K' = N).
    Returns (next_Qx [M][N/2] uint8, next_Sx native uint8, next_T [M][next_rank] bf16 or None,
    Y [M][N] bf16 or None)."""
    M = Qx.shape[0]
    K, N, rank = W.shape.K, W.shape.N, W.shape.rank
    shape = LayerShape(M, K, N, rank)
    dev = Qx.device
    if out is None:
        _, sxb, _ = svdq_act_sizes(LayerShape(M, N, 128, next_rank))
        Qn = torch.empty(M, N // 2, dtype=torch.uint8, device=dev)
        Sn = torch.empty(sxb, dtype=torch.uint8, device=dev)
        Tn = torch.empty(M, next_rank, dtype=torch.bfloat16, device=dev) if next_rank else None
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev) if store_y else None
    else:
        Qn, Sn, Tn, Y = out
    need = svdq_linear_quantize_next_workspace(shape, next_rank, flags)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(load().svdq_linear_quantize_next(
        shape.c(), _ptr(Qx), _ptr(Sx), _ptr(T), _ptr(W.Qr), _ptr(W.Sr), _ptr(W.L2t), next_rank, _ptr(next_inv_lambda),
        _ptr(next_L1p), _ptr(Qn), _ptr(Sn), _ptr(Tn), _ptr(Y), _ptr(workspace), workspace.numel(), flags, _stream()))
    return Qn, Sn, Tn, Y


def svdq_scales_to_canonical(native: torch.Tensor, rows: int, K: int) -> torch.Tensor:
    out = torch.empty(rows, K // 16, dtype=torch.uint8, device=native.device)
    _check(load().svdq_scales_to_canonical(rows, K, _ptr(native), _ptr(out), _stream()))
    return out


def svdq_append_lowrank(W: PreparedWeights, A: torch.Tensor, B: torch.Tensor) -> PreparedWeights:
    """Prepared weights whose low-rank branch also carries the LoRA update
    X A^T B^T: A bf16 [extra][K], B bf16 [N][extra]. Qr/Sr are shared."""
    K, N, r = W.shape.K, W.shape.N, W.shape.rank
    extra = A.shape[0]
    L1p = torch.empty(r + extra, K, dtype=torch.bfloat16, device=A.device)
    L2t = torch.empty(N, r + extra, dtype=torch.bfloat16, device=A.device)
    _check(load().svdq_append_lowrank(W.shape.c(), extra, _ptr(W.L1p), _ptr(W.L2t), _ptr(A), _ptr(B), _ptr(L1p),
                                      _ptr(L2t), _stream()))
    return PreparedWeights(LayerShape(0, K, N, r + extra), W.Qr, W.Sr, L1p, L2t, W.lam, W.inv_lam)


# ---------------------------------------------------------------- INT4 variant

def svdq_int4_act_sizes(shape: LayerShape) -> tuple[int, int, int]:
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().svdq_int4_act_sizes(shape.c(), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def svdq_int4_weight_sizes(shape: LayerShape) -> tuple[int, int]:
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().svdq_int4_weight_sizes(shape.c(), ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


@dataclass
class Int4Weights:
    shape: LayerShape          # M is unused (0)
    Qr: torch.Tensor           # uint8 [N][K]: E4M3 bytes of the INT4 codes
    Sr: torch.Tensor           # fp32 [K/64][N]
    L2t: torch.Tensor | None   # shared with the NVFP4 preparation
    L1p: torch.Tensor | None
    inv_lam: torch.Tensor


def svdq_int4_prepare_weights(W_lin: torch.Tensor, P: PreparedWeights) -> Int4Weights:
    """INT4 encoding of the residual of an NVFP4-prepared layer (same smoothing
    and low-rank factors)."""
    N, K = W_lin.shape
    shape = LayerShape(0, K, N, P.shape.rank)
    qr, sr = svdq_int4_weight_sizes(shape)
    Qr = torch.empty(N, K, dtype=torch.uint8, device=W_lin.device)
    Sr = torch.empty(K // 64, N, dtype=torch.float32, device=W_lin.device)
    assert Qr.numel() == qr and Sr.numel() * 4 == sr
    _check(load().svdq_int4_quantize_residual(shape.c(), _ptr(W_lin), _ptr(P.lam), _ptr(P.L1p), _ptr(P.L2t), _ptr(Qr),
                                              _ptr(Sr), _stream()))
    return Int4Weights(shape, Qr, Sr, P.L2t, P.L1p, P.inv_lam)


def svdq_int4_quantize_act(X: torch.Tensor, inv_lambda: torch.Tensor, L1p: torch.Tensor | None, rank: int,
                           N: int = 128, out: tuple | None = None):
    """Returns (Qx [M][K] uint8 E4M3 bytes, Sx fp32 [K/64][ceil(M/128)*128], T [M][rank] bf16 or None)."""
    M, K = X.shape
    shape = LayerShape(M, K, N, rank)
    if out is None:
        Qx = torch.empty(M, K, dtype=torch.uint8, device=X.device)
        Sx = torch.empty(K // 64, (M + 127) // 128 * 128, dtype=torch.float32, device=X.device)
        T = torch.empty(M, rank, dtype=torch.bfloat16, device=X.device) if rank else None
    else:
        Qx, Sx, T = out
    _check(load().svdq_int4_quantize_act(shape.c(), _ptr(X), _ptr(inv_lambda), _ptr(L1p), _ptr(Qx), _ptr(Sx), _ptr(T),
                                         _stream()))
    return Qx, Sx, T


def svdq_int4_linear(Qx: torch.Tensor, Sx: torch.Tensor, T: torch.Tensor | None, W: Int4Weights,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    M = Qx.shape[0]
    K, N, rank = W.shape.K, W.shape.N, W.shape.rank
    shape = LayerShape(M, K, N, rank)
    Y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=Qx.device)
    _check(load().svdq_int4_linear(shape.c(), _ptr(Qx), _ptr(Sx), _ptr(T), _ptr(W.Qr), _ptr(W.Sr), _ptr(W.L2t),
                                   _ptr(Y), _stream()))
    return Y


# ---------------------------------------------------------------- DeltaQuant

def svdq_deltaquant_sizes(F: int, H: int, W: int, C: int) -> tuple[int, int, int]:
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().svdq_deltaquant_sizes(F, H, W, C, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def svdq_deltaquant_encode(X: torch.Tensor, dims: tuple[int, int, int], out: tuple | None = None):
    """Core + delta encoding of video tokens X bf16 [F*H*W][C] (2 x 2 x 2 blocks).
    Returns (core uint8 [blocks][C], delta codes uint8 [F*H*W][C/2], delta scales native uint8)."""
    F, H, W = dims
    C = X.shape[1]
    if out is None:
        cb, _, sb = svdq_deltaquant_sizes(F, H, W, C)
        core = torch.empty(cb // C, C, dtype=torch.uint8, device=X.device)
        Qd = torch.empty(F * H * W, C // 2, dtype=torch.uint8, device=X.device)
        Sd = torch.empty(sb, dtype=torch.uint8, device=X.device)
    else:
        core, Qd, Sd = out
    _check(load().svdq_deltaquant_encode(F, H, W, C, _ptr(X), _ptr(core), _ptr(Qd), _ptr(Sd), _stream()))
    return core, Qd, Sd


def svdq_selftest_timeout() -> None:
    """Launch the failure-path diagnostic (a bounded wait that gives up after 2 s)."""
    _check(load().svdq_selftest_timeout(_stream()))


def svdq_check() -> None:
    _check(load().svdq_check(_stream()))
