"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/svdq.h declares, answers size queries, and rejects bad
shapes, null and misaligned pointers with the documented status codes before
touching a device."""
import ctypes
import os
import re

import pytest
import torch

from w4a4_diffusion_model_b200 import build as B
from w4a4_diffusion_model_b200 import svdq as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return S.load()


def header_symbols():
    with open(os.path.join(ROOT, "include", "svdq.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"SVDQ_API\s+[\w\s\*]+?\b(svdq_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    syms = header_symbols()
    assert len(syms) >= 11
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(S.EXPORTS)


def test_status_strings_and_version(lib):
    assert lib.svdq_version() == 100
    for code, name in S.STATUS.items():
        assert lib.svdq_status_string(code).decode() == name
    assert lib.svdq_status_string(99).decode() == "SVDQ_ERR_UNKNOWN"


def test_size_queries():
    qx, sx, t = S.svdq_act_sizes(S.LayerShape(4608, 3072, 12288, 32))
    assert qx == 4608 * 1536 and sx == 36 * 48 * 512 and t == 4608 * 32 * 2
    qx, sx, t = S.svdq_act_sizes(S.LayerShape(130, 384, 128, 0))
    assert qx == 130 * 192 and sx == 2 * 6 * 512 and t == 0
    qr, sr, l1, l2, ws = S.svdq_weight_sizes(S.LayerShape(0, 12288, 3072, 32))
    assert qr == 3072 * 6144 and sr == 24 * 192 * 512 and l1 == 32 * 12288 * 2 and l2 == 3072 * 32 * 2
    assert ws > 0
    *_, ws0 = S.svdq_weight_sizes(S.LayerShape(0, 12288, 3072, 0))
    assert ws0 == 0                                   # no branch, no SVD
    *_, ws128 = S.svdq_weight_sizes(S.LayerShape(0, 3072, 3072, 128))
    assert ws128 > ws


def test_prepare_without_factors_needs_the_workspace(lib):
    """The device SVD runs in the caller's workspace: a missing or short one is
    refused before any device work (rank 0 needs none)."""
    sh = S.Shape(0, 512, 256, 16)
    good = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_size_t()
    assert lib.svdq_weight_sizes(sh, None, None, None, None, ctypes.byref(ws)) == 0
    args = (good, good, ctypes.c_float(0.5), 0, good, good, good, good, good, good)
    assert lib.svdq_prepare_weights(sh, *args, None, 0, None) == 4
    assert lib.svdq_prepare_weights(sh, *args, good, ws.value - 256, None) == 4
    assert b"workspace" in lib.svdq_last_error()


@pytest.mark.parametrize("M,K,N,r", [(-1, 128, 128, 0), (1, 100, 128, 0), (1, 128, 100, 0), (1, 128, 128, 8),
                                     (1, 128, 128, 144), (1, 64, 128, 16), (1, 128, 128, -16)])
def test_bad_shapes_rejected(lib, M, K, N, r):
    sh = S.Shape(M, K, N, r)
    a = ctypes.c_size_t()
    assert lib.svdq_act_sizes(sh, ctypes.byref(a), None, None) == 2
    assert lib.svdq_quantize_act(sh, None, None, None, None, None, None, 0, None) == 2
    assert lib.svdq_linear(sh, None, None, None, None, None, None, None, 0, None) == 2


def test_null_misaligned_and_variant_rejected(lib):
    sh = S.Shape(128, 256, 128, 16)
    good = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    assert lib.svdq_quantize_act(sh, good, good, good, good, good, None, 0, None) == 1          # T missing
    assert lib.svdq_quantize_act(sh, good, good, good, good, good, good, 7, None) == 1         # variant
    assert lib.svdq_quantize_act(sh, good, good, good, bad, good, good, 0, None) == 3          # misaligned
    assert lib.svdq_linear(sh, good, good, good, good, good, bad, good, 0, None) == 3
    assert lib.svdq_linear(sh, good, good, None, good, good, good, good, 0, None) == 1
    assert lib.svdq_prepare_weights(sh, good, good, ctypes.c_float(1.5), 0, good, good, good, good, good, good,
                                    None, 0, None) == 1                                         # alpha
    assert lib.svdq_prepare_weights(sh, good, good, ctypes.c_float(0.5), 4, good, good, good, good, good, good,
                                    None, 0, None) == 1                                         # flags
    assert lib.svdq_channel_amax(0, 128, good, good, None) == 2
    assert lib.svdq_channel_amax(4, 128, good, bad, None) == 3
    assert b"aligned" in lib.svdq_last_error()


def test_append_lowrank_argument_checks(lib):
    good = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    sh = S.Shape(0, 256, 128, 32)
    assert lib.svdq_append_lowrank(sh, 8, good, good, good, good, good, good, None) == 2      # not a multiple of 16
    assert lib.svdq_append_lowrank(sh, 112, good, good, good, good, good, good, None) == 2    # 32 + 112 > 128
    assert lib.svdq_append_lowrank(sh, 0, good, good, good, good, good, good, None) == 2
    assert lib.svdq_append_lowrank(sh, 16, None, good, good, good, good, good, None) == 1     # L1p missing (r > 0)
    assert lib.svdq_append_lowrank(sh, 16, good, good, bad, good, good, good, None) == 3
    if not torch.cuda.is_available():   # r == 0: factors may be NULL; only the device check remains
        assert lib.svdq_append_lowrank(S.Shape(0, 256, 128, 0), 16, None, None, good, good, good, good, None) == 5


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_is_reported_not_emulated(lib):
    sh = S.Shape(128, 256, 128, 0)
    good = ctypes.c_void_p(1 << 20)
    assert lib.svdq_quantize_act(sh, good, good, None, good, good, None, 0, None) == 5
    assert lib.svdq_linear(sh, good, good, None, good, good, None, good, 0, None) == 5
    assert lib.svdq_check(None) == 5


def test_linear_quantize_next_argument_checks(lib):
    """The next-layer quantization validates the next layer's rank, its
    pointers and their alignment before any device work."""
    good = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    sh = S.Shape(256, 512, 768, 16)
    ws = ctypes.c_size_t()
    assert lib.svdq_linear_quantize_next_workspace(sh, 20, 0, ctypes.byref(ws)) == 2    # next rank not a multiple of 16
    assert lib.svdq_linear_quantize_next_workspace(sh, 144, 0, ctypes.byref(ws)) == 2
    assert lib.svdq_linear_quantize_next_workspace(sh, 32, 0, None) == 1
    assert lib.svdq_linear_quantize_next_workspace(sh, 32, 2, ctypes.byref(ws)) == 1   # unknown flag
    assert lib.svdq_linear_quantize_next_workspace(S.Shape(0, 512, 768, 16), 32, 1, ctypes.byref(ws)) == 0
    assert ws.value == 0                                                                   # M == 0 needs none
    args = [good] * 6   # Qx, Sx, T, Qr, Sr, L2t
    nxt = [good] * 6    # next_inv_lambda, next_L1p, next_Qx, next_Sx, next_T, Y
    assert lib.svdq_linear_quantize_next(sh, *args, 48, *nxt, good, 1 << 20, 0, None) not in (0, 1, 3)  # device / shape only
    assert lib.svdq_linear_quantize_next(sh, *args, 24, *nxt, good, 1 << 20, 0, None) == 2
    assert lib.svdq_linear_quantize_next(sh, *args, 32, *nxt, good, 1 << 20, 4, None) == 1              # unknown flag
    assert lib.svdq_linear_quantize_next(S.Shape(256, 512, 100, 16), *args, 16, *nxt, good, 1 << 20, 0, None) == 2
    assert lib.svdq_linear_quantize_next(sh, *args, 32, good, None, good, good, good, good, good, 1 << 20, 0, None) == 1
    assert lib.svdq_linear_quantize_next(sh, *args, 0, good, None, good, good, None, None, good, 1 << 20, 0, None) != 1
    assert lib.svdq_linear_quantize_next(sh, *args, 32, good, good, good, bad, good, good, good, 1 << 20, 0, None) == 3
    assert lib.svdq_linear_quantize_next(S.Shape(0, 512, 768, 16), None, None, None, None, None, None, 32, None, None,
                                         None, None, None, None, None, 0, 0, None) == 0   # M == 0: a no-op
    if not torch.cuda.is_available():
        assert lib.svdq_linear_quantize_next(sh, *args, 32, *nxt, good, 1 << 20, 0, None) == 5
        assert lib.svdq_linear_quantize_next_workspace(sh, 32, 0, ctypes.byref(ws)) == 5


def test_int4_sizes_and_argument_checks(lib):
    """The INT4 entry points: byte sizes of the one-byte codes and the
    group-major fp32 scales, and argument errors reported before any device
    work."""
    qx, sx, t = S.svdq_int4_act_sizes(S.LayerShape(4608, 3072, 9216, 32))
    assert qx == 4608 * 3072 and sx == 48 * 4608 * 4 and t == 4608 * 32 * 2
    qx, sx, t = S.svdq_int4_act_sizes(S.LayerShape(130, 384, 128, 0))
    assert qx == 130 * 384 and sx == 6 * 256 * 4 and t == 0          # rows padded to 128
    qr, sr = S.svdq_int4_weight_sizes(S.LayerShape(0, 12288, 3072, 32))
    assert qr == 3072 * 12288 and sr == 192 * 3072 * 4
    good = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    sh = S.Shape(128, 256, 128, 16)
    assert lib.svdq_int4_quantize_act(S.Shape(128, 200, 128, 16), good, good, good, good, good, good, None) == 2
    assert lib.svdq_int4_quantize_act(sh, good, good, good, good, good, None, None) == 1      # T missing
    assert lib.svdq_int4_quantize_act(sh, good, good, good, bad, good, good, None) == 3
    assert lib.svdq_int4_linear(sh, good, good, good, good, good, None, good, None) == 1      # L2t missing
    assert lib.svdq_int4_linear(sh, good, good, good, good, bad, good, good, None) == 3
    assert lib.svdq_int4_linear(S.Shape(128, 256, 100, 0), good, good, None, good, good, None, good, None) == 2
    assert lib.svdq_int4_quantize_residual(sh, good, good, None, good, good, good, None) == 1  # L1p missing
    assert lib.svdq_int4_quantize_residual(sh, good, good, good, good, good, bad, None) == 3
    assert lib.svdq_int4_quantize_act(S.Shape(0, 256, 128, 0), None, None, None, None, None, None, None) == 0
    if not torch.cuda.is_available():
        sh0 = S.Shape(128, 256, 128, 0)
        assert lib.svdq_int4_linear(sh0, good, good, None, good, good, None, good, None) == 5
        assert lib.svdq_int4_quantize_residual(sh0, good, good, None, None, good, good, None) == 5


def test_deltaquant_sizes_and_argument_checks(lib):
    core, qd, sd = S.svdq_deltaquant_sizes(5, 7, 9, 192)      # 3 x 4 x 5 blocks, 315 tokens
    assert core == 60 * 192 and qd == 315 * 96 and sd == 3 * 3 * 512
    for F, H, W, C in ((0, 4, 4, 64), (2, 2, 2, 48), (2, 2, 2, 0), (2, 2, 2, (1 << 20) + 64), (1 << 20, 1 << 11, 1, 64)):
        a = ctypes.c_size_t()
        assert lib.svdq_deltaquant_sizes(F, H, W, C, ctypes.byref(a), None, None) == 2, (F, H, W, C)
    good, bad = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    assert lib.svdq_deltaquant_encode(2, 2, 2, 64, None, good, good, good, None) == 1
    assert lib.svdq_deltaquant_encode(2, 2, 2, 64, good, good, bad, good, None) == 3
    assert lib.svdq_deltaquant_encode(2, 2, 2, 96, good, good, good, good, None) == 2
