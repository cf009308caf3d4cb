"""Shared helpers of the GPU tests: run the layer through the C ABI and run
the oracle on the same seeded inputs. The oracle never sees a value produced by
the CUDA path; the CUDA path may receive oracle-computed inputs (the low-rank
factors in "given factors" mode)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from w4a4_diffusion_model_b200 import svdq as S

TOL_Y = 5e-3      # relative Frobenius error of Y (fused and unfused)
TOL_T = 4e-3      # relative Frobenius error of the bf16 down-projection T


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_factors_to_device(P: dict, dev="cuda"):
    """Oracle L1p [K][r] / L2 [r][N] (bf16 values) -> device bf16 L1p [r][K], L2t [N][r]."""
    L1p = torch.from_numpy(np.ascontiguousarray(P["L1p"].T)).to(torch.float32).to(torch.bfloat16).to(dev)
    L2t = torch.from_numpy(np.ascontiguousarray(P["L2"].T)).to(torch.float32).to(torch.bfloat16).to(dev)
    return L1p, L2t


def gpu_prepare(W: torch.Tensor, act_amax: torch.Tensor, alpha: float, rank: int, factors=None):
    L1p, L2t = factors if factors is not None else (None, None)
    return S.svdq_prepare_weights(W, act_amax, alpha, rank, L1p, L2t)


def gpu_layer(X: torch.Tensor, P: S.PreparedWeights, variant=S.SVDQ_FUSED):
    Qx, Sx, T = S.svdq_quantize_act(X, P.inv_lam, P.L1p, P.shape.rank, P.shape.N, variant)
    Y = S.svdq_linear(Qx, Sx, T, P, variant)
    S.svdq_check()
    return Qx, Sx, T, Y


def packed_oracle_codes(codes: np.ndarray) -> np.ndarray:
    return O.pack_nibbles(codes)


def rel_fro(a, b) -> float:
    return O.rel_fro(a, b)
