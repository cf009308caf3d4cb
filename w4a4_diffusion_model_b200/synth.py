"""Seeded synthetic workloads for the SVDQuant W4A4 linear layer.

This module is the only code shared by the CUDA path's tests/benchmark and the
CPU oracle's tests. It draws random inputs and nothing else: it holds none of
the method's arithmetic (no smoothing, no SVD, no quantization).

Recipe (one numpy PCG64 stream per workload, draws taken in the order below):

* activation X [M][K]: i.i.d. N(0,1) in fp64 (or |N(0,1)| - 0.3 for the
  post-GELU-like down-projection input); a set of outlier input channels is
  multiplied by a per-channel factor (fixed x50, or log-uniform in [lo, hi]).
  The outlier channels are channels 0..3 for the tiny layer, otherwise
  ``round(frac*K)`` channels chosen by a seeded permutation.
* weight W_lin [N][K] (nn.Linear orientation, W = W_lin^T in the paper's
  ``X W`` notation): i.i.d. N(0, 1/K) plus ``spikes`` rank-1 terms
  ``a * u v^T`` with Rademacher u in {+-1}^N, v in {+-1}^K and amplitude
  ``a = 10/sqrt(K)``, so that every entry of a spike has magnitude a.
* both are rounded fp64 -> fp32 (round-to-nearest) -> bf16 (round-to-nearest-
  even) by torch's dtype conversion; every consumer sees the bf16 values.

These stand in for FLUX.1 activations and weights (the workloads the SVDQuant
paper measures), which are not available offline. ``smooth_video`` draws a
spatio-temporally smooth activation for the core + delta video codec.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    rank: int
    seed: int
    alpha: float = 0.5
    x_kind: str = "gauss"            # "gauss" | "gelu"
    outliers: str = "frac"           # "first4" | "frac"
    outlier_frac: float = 0.01
    outlier_lo: float = 20.0         # factor range; lo == hi means a fixed factor
    outlier_hi: float = 100.0
    spikes: int = 8

    def flops(self) -> int:
        """Effective FLOPs of one layer call: 2MNK + 2Mr(K+N)."""
        return 2 * self.M * self.N * self.K + 2 * self.M * self.rank * (self.K + self.N)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The workloads of the FLUX-shaped study: a tiny layer, the fused QKV
# projection, the MLP up- and down-projections, and the M x rank sweep.
TINY = Workload("tiny_256x512x512_r16", 256, 512, 512, 16, seed=0,
                outliers="first4", outlier_lo=50.0, outlier_hi=50.0, spikes=2)
FLUX_QKV = Workload("flux_qkv_4608x3072x9216_r32", 4608, 3072, 9216, 32, seed=1)
FLUX_MLP_UP = Workload("flux_mlp_up_4608x3072x12288_r32", 4608, 3072, 12288, 32, seed=2)
FLUX_MLP_DOWN = Workload("flux_mlp_down_4608x12288x3072_r32", 4608, 12288, 3072, 32, seed=3,
                         x_kind="gelu", outlier_frac=0.005, outlier_lo=50.0, outlier_hi=50.0)


def sweep() -> list[Workload]:
    out = []
    i = 0
    for M in (256, 1024, 4608, 18432):
        for r in (0, 16, 32, 64, 128):
            out.append(Workload(f"sweep_{M}x3072x3072_r{r}", M, 3072, 3072, r, seed=100 + i))
            i += 1
    return out


WORKLOADS = {w.name: w for w in (TINY, FLUX_QKV, FLUX_MLP_UP, FLUX_MLP_DOWN, *sweep())}


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.float32).to(torch.bfloat16)


def outlier_channels(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.outliers == "first4":
        return np.arange(min(4, w.K))
    n = int(round(w.outlier_frac * w.K))
    return np.sort(rng.permutation(w.K)[:n])


def make_activation(w: Workload, rng: np.random.Generator, M: int | None = None) -> torch.Tensor:
    M = w.M if M is None else M
    x = rng.standard_normal((M, w.K))
    if w.x_kind == "gelu":
        x = np.abs(x) - 0.3
    ch = outlier_channels(w, rng)
    if w.outlier_lo == w.outlier_hi:
        fac = np.full(len(ch), w.outlier_lo)
    else:
        fac = np.exp(rng.uniform(math.log(w.outlier_lo), math.log(w.outlier_hi), size=len(ch)))
    x[:, ch] *= fac[None, :]
    return _to_bf16(x)


def make_weight(w: Workload, rng: np.random.Generator) -> torch.Tensor:
    W = rng.standard_normal((w.N, w.K)) * (1.0 / math.sqrt(w.K))
    a = 10.0 / math.sqrt(w.K)
    for _ in range(w.spikes):
        u = rng.choice(np.array([-1.0, 1.0]), size=w.N)
        v = rng.choice(np.array([-1.0, 1.0]), size=w.K)
        W += a * np.outer(u, v)
    return _to_bf16(W)


def generate(w: Workload, M: int | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Return (X bf16 [M][K], W_lin bf16 [N][K]) on the CPU for workload ``w``.

    ``M`` overrides the row count (same K, N and distributions); rows are drawn
    first, so a smaller M is not a prefix of a larger one.
    """
    rng = np.random.default_rng(w.seed)
    X = make_activation(w, rng, M)
    W = make_weight(w, rng)
    return X, W


def smooth_video(F: int, H: int, Wd: int, C: int, seed: int, noise: float = 0.05,
                 outlier_channels: int = 2) -> torch.Tensor:
    """A video-latent-like activation, tokens as rows in frame, row, column
    order ([F*H*Wd][C] bf16): per channel, a sum of four low-frequency
    separable cosines over (frame, row, column) with random frequencies below
    a quarter cycle per token and random phases, plus i.i.d. N(0, noise^2);
    the first ``outlier_channels`` channels are scaled by 20."""
    rng = np.random.default_rng(seed)
    f = np.arange(F)[:, None, None, None]
    h = np.arange(H)[None, :, None, None]
    w = np.arange(Wd)[None, None, :, None]
    x = np.zeros((F, H, Wd, C))
    for _ in range(4):
        kf, kh, kw = (rng.uniform(0.0, 0.25, C) * 2 * np.pi for _ in range(3))
        ph = rng.uniform(0.0, 2 * np.pi, C)
        x += rng.standard_normal(C) * np.cos(kf * f + kh * h + kw * w + ph)
    x += noise * rng.standard_normal(x.shape)
    x[..., :outlier_channels] *= 20.0
    return _to_bf16(x.reshape(F * H * Wd, C))
