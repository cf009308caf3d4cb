"""CPU oracle for the SVDQuant W4A4 linear layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code with the CUDA library and imports nothing from it.

It restates, slowly and in plain numpy (fp64 unless a step fixes another
precision), what the layer computes:

    Y ~= Q(X_hat) Q(R) + (X_hat L1) L2,   X_hat = X diag(lambda)^-1,
    W_hat = diag(lambda) W = L1 L2 + R

Sources (web pages on SVDQuant):
  [P1] libaedu.com, article on 4-bit diffusion-model quantization (smoothing,
       kernel fusion, and the DeltaQuant core + delta outline for video).
  [P2] devpress.csdn.net, SVDQuant paper walkthrough: eq. (1) symmetric
       quantization with q_max = 6 for 4-bit float, eq. (2) the factored W4A4
       product, eq. (3) the error E, eq. (4)/(9) Proposition 4.1, eq. (5) the
       low-rank + 4-bit split, eq. (6) the residual-error identity, the SVD as
       optimal rank-r approximation (text after eq. (8), Fig. 5), Fig. 6 kernel
       fusion, Table 3 (NVFP4's small microscaling group).
  [P3] anrans.github.io AI-infra handbook, "Quantization" chapter: the
       SmoothQuant section (lambda_j = max|X_j|^alpha / max|W_j|^(1-alpha),
       X_hat = X / lambda, W_hat = W * lambda per input channel) and the
       SVDQuant section (L1 = U_r diag(S_r), L2 = V_r^T, R = W_hat - L1 L2).

Readings where the pages leave a step open (each one is also listed in the
design notes of the repository):
  * NVFP4 = one E4M3 scale per 16 consecutive elements along the reduction
    dimension, scale s = E4M3_RNE_satfinite(amax / 6); no second-level
    per-tensor scale.
  * codes: q = E2M1_RNE_satfinite(v / s) of the exact real quotient ([P2]
    eq. (1), round(X / s)), sign-preserving (a negative value that rounds to
    zero keeps the sign bit); a group whose scale is zero encodes all +0.
  * "round to nearest, ties to even" of an exact quotient num / den onto a
    grid is taken by comparing |num| with each grid midpoint times den; those
    products are exact in fp64 for every grid and divisor used here, so no
    intermediate rounding of the quotient enters any decision.
  * smoothing: lambda64 = ax^alpha / aw^(1-alpha) (alpha = 0.5 uses sqrt on
    both sides), lambda = 1 where ax or aw is zero; lambda32 = fp32(lambda64),
    inv_lambda32 = fp32(1 / lambda32).
  * stored low-rank factors are bf16: L1' = bf16(L1 / lambda32) so the
    down-projection consumes raw X (X L1' == X_hat L1), L2 = bf16(V_r^T).
  * residual: R = fp32(W_hat - sum_k (lambda32 L1'_k) L2_k), evaluated in fp64
    in increasing k without fused multiply-add, so that R absorbs the rounding
    of the stored factors and X_hat (lambda L1') L2 + X_hat R == X_hat W_hat.
  * the packed FP4 byte holds element 2i in its low nibble, 2i+1 in the high.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "round_to_format", "bf16", "fp32", "E2M1_VALUES",
    "e2m1_encode", "e2m1_decode", "e4m3_encode", "e4m3_decode",
    "quantize_nvfp4", "dequantize_nvfp4", "pack_nibbles", "unpack_nibbles",
    "scales_to_native", "native_to_scales",
    "channel_amax", "smoothing_lambda", "prepare_weights", "residual_quantize",
    "quantize_act", "linear", "layer_reference",
    "int_quant_dequant", "smoothed_pair", "fakequant_output", "lambda64", "svd_split",
    "rne_quotient_index", "E4M3_GRID", "FP16_GRID", "INT4_GRID",
    "quant_error", "prop41_bound", "rel_fro", "fro",
    "INT4_QMAX", "INT4_GROUP", "fp16", "quantize_int4", "dequantize_int4", "pack_int4", "unpack_int4",
    "layer_reference_int4",
    "e4m3_encode_signed", "video_blocks", "deltaquant_encode", "deltaquant_decode",
]

# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def round_to_format(v, man_bits: int, emin: int, max_finite: float) -> np.ndarray:
    """Round real values to nearest, ties to even, in a binary floating-point
    format with ``man_bits`` explicit mantissa bits, smallest normal exponent
    ``emin`` (gradual underflow below it) and saturation to +-``max_finite``.

    ``v`` must be exactly representable in fp64 (it is: every caller passes
    fp32/bf16 values or exact fp64 products), so this is a single rounding.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, e = np.frexp(a)                 # a = m * 2**e with m in [0.5, 1)
    e = np.maximum(e - 1, emin)        # exponent of the leading bit, floored at emin
    quantum = np.ldexp(1.0, e - man_bits)
    r = np.rint(a / quantum) * quantum  # a / quantum is exact; rint = half-to-even
    r = np.minimum(r, max_finite)
    return np.copysign(r, v)


def bf16(v) -> np.ndarray:
    """bfloat16 round-to-nearest-even (8-bit significand, fp32 exponent range)."""
    return round_to_format(v, 7, -126, float(np.ldexp(2.0 - 2.0 ** -7, 127)))


def fp32(v) -> np.ndarray:
    """IEEE binary32 round-to-nearest-even, returned as fp64 values."""
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


# E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit. Magnitude codes 0..7.
def _e2m1_magnitude(code: int) -> float:
    e, m = (code >> 1) & 3, code & 1
    if e == 0:
        return m * 0.5                       # subnormal: m * 2^(1-1) * 2^-1
    return (1.0 + 0.5 * m) * 2.0 ** (e - 1)


E2M1_VALUES = np.array([_e2m1_magnitude(c) for c in range(8)])  # 0,.5,1,1.5,2,3,4,6
E2M1_QMAX = 6.0                                                  # q_max of 4-bit float


def e2m1_encode(y) -> np.ndarray:
    """E2M1 code (uint8 nibble) of RNE_satfinite(y); sign bit kept for -0 and
    for negative values that round to zero."""
    y = np.asarray(y, dtype=np.float64)
    mag = np.abs(round_to_format(y, 1, 0, E2M1_QMAX))
    code = np.searchsorted(E2M1_VALUES, mag).astype(np.uint8)   # exact match
    return code | (np.signbit(y).astype(np.uint8) << 3)


def e2m1_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_VALUES[code & 7]
    return np.where(code & 8, -mag, mag)


# E4M3 (fn variant): 1 sign, 4 exponent (bias 7), 3 mantissa; S.1111.111 is NaN,
# no infinities, largest finite 448.
E4M3_MAX = 448.0


def e4m3_decode(byte) -> np.ndarray:
    b = np.asarray(byte, dtype=np.int64)
    s, e, m = (b >> 7) & 1, (b >> 3) & 15, b & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e4m3_encode(v) -> np.ndarray:
    """E4M3 byte of RNE_satfinite(v) for v >= 0 (scales are non-negative)."""
    r = round_to_format(v, 3, -6, E4M3_MAX)
    if np.any(r < 0):
        raise ValueError("e4m3_encode: scales are non-negative")
    _, e = np.frexp(r)
    e = e - 1
    normal = r >= 2.0 ** -6
    ebits = np.where(normal, e + 7, 0)
    mbits = np.where(normal, np.rint((r / np.ldexp(1.0, e) - 1.0) * 8.0),
                     np.rint(r / 2.0 ** -9))
    return (ebits.astype(np.int64) << 3 | mbits.astype(np.int64)).astype(np.uint8)


E4M3_BYTES_FINITE = np.arange(127, dtype=np.uint8)            # 0x00..0x7e: every finite value >= 0


# ---------------------------------------------------------------------------
# NVFP4 group quantization ([P2] eq. (1) with q_max = 6, Table 3's microscaling)
# ---------------------------------------------------------------------------

GROUP = 16


def rne_quotient_index(num, den, grid: np.ndarray) -> np.ndarray:
    """Index into ``grid`` of RNE_satfinite(|num| / den), the quotient taken
    exactly.

    ``grid`` holds the non-negative values of a format in ascending order, so
    that an even index is an even code. Midpoint i lies between grid[i] and
    grid[i + 1]; |num| passes it when |num| > mid_i * den, and on a tie
    (|num| == mid_i * den) exactly when i + 1 is even. Quotients above the
    last midpoint take the last grid value (saturation). ``den`` is a positive
    scalar or an array broadcasting against ``num`` on all but its last axis
    (one divisor per group of the last axis). Each product mid_i * den must be
    exact in fp64, which the callers guarantee (few significant bits on both
    sides).
    """
    a = np.abs(np.asarray(num, dtype=np.float64))
    grid = np.asarray(grid, dtype=np.float64)
    mids = (grid[:-1] + grid[1:]) / 2                       # exact in fp64
    if np.ndim(den) == 0:
        t = mids * float(den)
        i = np.searchsorted(t, a, side="left")              # midpoints strictly below |num|
        j = np.minimum(i, t.size - 1)
        tie_up = (i < t.size) & (t[j] == a) & ((i + 1) % 2 == 0)
        return (i + tie_up).astype(np.int64)
    d = np.asarray(den, dtype=np.float64)[..., None]
    idx = np.zeros(a.shape, dtype=np.int64)
    for i, mu in enumerate(mids):                           # thresholds ascend with i
        t = mu * d
        passed = a > t
        if (i + 1) % 2 == 0:
            passed |= a == t
        idx += passed
    return idx


E4M3_GRID = e4m3_decode(E4M3_BYTES_FINITE)                     # ascending; index = byte


def quantize_nvfp4(v32: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Quantize rows of fp32 values, grouped by 16 along the last axis.

    Returns (codes uint8 [rows][K] one nibble per element, scales uint8
    [rows][K/16] E4M3 bytes). Per group ([P2] eq. (1) with q_max = 6):
    a = max|v|; s = E4M3_RNE_satfinite(a / 6); q = E2M1_RNE_satfinite(v / s),
    both quotients exact; all codes +0 if s == 0.
    """
    v = np.asarray(v32, dtype=np.float32).astype(np.float64)
    rows, K = v.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 16")
    g = v.reshape(rows, K // GROUP, GROUP)
    amax = np.max(np.abs(g), axis=2)                                 # exact
    sbyte = rne_quotient_index(amax, E2M1_QMAX, E4M3_GRID).astype(np.uint8)
    sval = e4m3_decode(sbyte)
    live = sval > 0
    mag = rne_quotient_index(g, np.where(live, sval, 1.0), E2M1_VALUES).astype(np.uint8)
    codes = mag | (np.signbit(g).astype(np.uint8) << 3)
    codes = np.where(live[..., None], codes, np.uint8(0))
    return codes.reshape(rows, K).astype(np.uint8), sbyte


def dequantize_nvfp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    rows, K = codes.shape
    d = e2m1_decode(codes).reshape(rows, K // GROUP, GROUP) * e4m3_decode(scales)[..., None]
    return d.reshape(rows, K)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[rows][K] nibbles -> [rows][K/2] bytes; element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 15
    out[:, 1::2] = p >> 4
    return out


# Native scale layout (the tcgen05 block-scaled MMA's scale-factor tile, one
# 512-byte atom per 128 rows x 64 reduction elements): atom (rb, kb) sits at
# byte (rb * (K/64) + kb) * 512; inside it, row r = 32*q + i and scale j (0..3)
# of the 64-element block sit at byte 16*i + 4*q + j. Rows past the end of the
# matrix (last partial block) hold zero.

def _native_index(rows: int, G: int) -> np.ndarray:
    """Byte offset in the native layout of scale (r, g), as an [rows][G] array."""
    r = np.arange(rows)[:, None]
    g = np.arange(G)[None, :]
    rb, rr = r // 128, r % 128
    q, i = rr // 32, rr % 32
    kb, j = g // 4, g % 4
    return (rb * (G // 4) + kb) * 512 + 16 * i + 4 * q + j


def scales_to_native(scales: np.ndarray) -> np.ndarray:
    rows, G = scales.shape
    if G % 4:
        raise ValueError("K must be a multiple of 64")
    RB = -(-rows // 128)
    out = np.zeros(RB * (G // 4) * 512, dtype=np.uint8)
    out[_native_index(rows, G)] = scales
    return out


def native_to_scales(native: np.ndarray, rows: int, K: int) -> np.ndarray:
    return np.asarray(native, dtype=np.uint8)[_native_index(rows, K // GROUP)]


# ---------------------------------------------------------------------------
# Smoothing ([P3] SmoothQuant section; [P2] Fig. 3)
# ---------------------------------------------------------------------------

def channel_amax(X: np.ndarray) -> np.ndarray:
    """Per input channel j: max_m |X[m][j]| (fp32, exact)."""
    return np.max(np.abs(np.asarray(X, dtype=np.float64)), axis=0).astype(np.float32)


def lambda64(ax, aw, alpha: float) -> np.ndarray:
    """lambda_j = ax_j^alpha / aw_j^(1-alpha) in fp64 ([P3] SmoothQuant
    section), 1 where either channel maximum is 0. alpha = 0.5 takes a square
    root on each side."""
    ax = np.asarray(ax, dtype=np.float64)
    aw = np.asarray(aw, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        if alpha == 0.5:
            lam = np.sqrt(ax) / np.sqrt(aw)
        else:
            lam = np.power(ax, alpha) / np.power(aw, 1.0 - alpha)
    return np.where((ax == 0) | (aw == 0), 1.0, lam)


def smoothing_lambda(act_amax: np.ndarray, W_lin: np.ndarray, alpha: float):
    """lambda_j = max|X_j|^alpha / max|W_j|^(1-alpha), W_j = input channel j.

    W_lin is [N][K] (nn.Linear); the paper's W = W_lin^T, so channel j of the
    weight is column j of W_lin. Returns (lambda32, inv_lambda32) as float32.
    """
    aw = np.max(np.abs(np.asarray(W_lin, dtype=np.float64)), axis=0)
    lam32 = lambda64(act_amax, aw, alpha).astype(np.float32)
    inv32 = np.float32(1.0) / lam32
    return lam32, inv32


# ---------------------------------------------------------------------------
# Weight preparation ([P2] eq. (5), SVD paragraph; [P3] SVDQuant section)
# ---------------------------------------------------------------------------

def residual_quantize(W_lin: np.ndarray, lam32: np.ndarray, L1p: np.ndarray, L2: np.ndarray):
    """R = fp32(W_hat - sum_k (lambda32 L1'_k) L2_k) and its NVFP4 encoding.

    W_lin [N][K] (bf16 values), lam32 [K], L1p [K][r] and L2 [r][N] (bf16
    values). The sum runs over k = 0..r-1 in order, each product exact and each
    addition rounded once in fp64 (no fused multiply-add). Returns
    (R32 [K][N] float32, codes [N][K], scales [N][K/16]).
    """
    W = np.asarray(W_lin, dtype=np.float64)
    lam = np.asarray(lam32, dtype=np.float64)
    What = lam[:, None] * W.T                       # [K][N], exact (24b x 8b)
    K, N = What.shape
    r = L1p.shape[1]
    acc = np.zeros((K, N))
    for k in range(r):
        a = lam * L1p[:, k]                          # exact (24b x 8b)
        acc = acc + a[:, None] * L2[k][None, :]      # product exact (32b x 8b), one rounding per add
    R32 = (What - acc).astype(np.float32)
    codes, scales = quantize_nvfp4(R32.T.copy())
    return R32, codes, scales


def svd_split(What: np.ndarray, rank: int):
    """Top-rank split of W_hat [K][N] by the SVD ([P2] text after eq. (8):
    the optimal rank-r approximation; [P3] SVDQuant section): L1 = U_r
    diag(S_r) [K][r], L2 = V_r^T [r][N], and all singular values (descending)."""
    U, S, Vt = np.linalg.svd(What, full_matrices=False)
    return U[:, :rank] * S[:rank], Vt[:rank], S


def prepare_weights(W_lin: np.ndarray, act_amax: np.ndarray, alpha: float, rank: int) -> dict:
    """Offline preparation: smoothing, top-r SVD split, residual quantization.

    Returns a dict with lam32, inv32 [K]; L1p [K][r], L2 [r][N] (bf16 values in
    fp64); S (singular values of W_hat, descending); R32 [K][N]; Qr codes
    [N][K]; Sr scales [N][K/16]; What [K][N].
    """
    W = np.asarray(W_lin, dtype=np.float64)
    lam32, inv32 = smoothing_lambda(act_amax, W, alpha)
    What = lam32.astype(np.float64)[:, None] * W.T
    L1, L2_64, S = svd_split(What, rank)
    L1p = bf16(L1 / lam32.astype(np.float64)[:, None])
    L2 = bf16(L2_64)
    R32, codes, scales = residual_quantize(W, lam32, L1p, L2)
    return dict(lam32=lam32, inv32=inv32, L1p=L1p, L2=L2, S=S, R32=R32,
                Qr=codes, Sr=scales, What=What)


# ---------------------------------------------------------------------------
# Per-call path ([P2] eq. (5) and Fig. 6: quantize + down-projection, then the
# 4-bit GEMM with the up-projection added to the same output)
# ---------------------------------------------------------------------------

def quantize_act(X: np.ndarray, inv32: np.ndarray, L1p: np.ndarray):
    """x_hat = fp32(fp32(x) * inv_lambda32); NVFP4 codes/scales of x_hat; and
    T = X L1' in fp64 (== X_hat L1 for the stored factors). Returns
    (codes [M][K], scales [M][K/16], T [M][r])."""
    X32 = np.asarray(X, dtype=np.float32)
    xhat = X32 * np.asarray(inv32, dtype=np.float32)[None, :]     # fp32 multiply
    codes, scales = quantize_nvfp4(xhat)
    T = np.asarray(X, dtype=np.float64) @ np.asarray(L1p, dtype=np.float64)
    return codes, scales, T


def linear(Qx, Sx, T, Qr, Sr, L2, rows=None) -> np.ndarray:
    """Y = deq(Qx) deq(Qr)^T + T L2 in fp64 ([P2] eq. (2) and eq. (5)).
    ``rows`` optionally restricts the output to a subset of rows."""
    if rows is not None:
        Qx, Sx, T = Qx[rows], Sx[rows], T[rows]
    A = dequantize_nvfp4(Qx, Sx)
    B = dequantize_nvfp4(Qr, Sr)
    return A @ B.T + np.asarray(T, dtype=np.float64) @ np.asarray(L2, dtype=np.float64)


def layer_reference(X, W_lin, alpha: float, rank: int, act_amax=None) -> dict:
    """The whole layer on the oracle: prepare from (W, amax), then quantize X
    and evaluate Y. Also returns the exact product X W_lin^T."""
    X = np.asarray(X, dtype=np.float64)
    if act_amax is None:
        act_amax = channel_amax(X)
    P = prepare_weights(W_lin, act_amax, alpha, rank)
    Qx, Sx, T = quantize_act(X, P["inv32"], P["L1p"])
    Y = linear(Qx, Sx, T, P["Qr"], P["Sr"], P["L2"])
    return dict(P, Qx=Qx, Sx=Sx, T=T, Y=Y, Y_exact=X @ np.asarray(W_lin, dtype=np.float64).T)


# ---------------------------------------------------------------------------
# The handbook's per-tensor INT fake-quant flow ([P3] "outliers", SmoothQuant
# and SVDQuant sections), used to pin the smoothing orientation and the SVD
# split against the printed error tables.
# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# INT4 W4A4 variant (the pages' path for GPUs without NVFP4: [P2] eq. (1) with
# q_max = 2^(k-1) - 1 = 7 for signed 4-bit integers; [P3] "one scale per 64
# elements"). Readings: fp16 scales, s = fp16_RNE(amax / 7) saturating at
# 65504; q = clamp(RNE(v / s), -7, 7), both quotients exact (eq. (1)'s
# round(X / s)); a zero scale gives zero codes.

INT4_QMAX = 7
INT4_GROUP = 64
FP16_GRID = np.arange(0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)   # 0 .. 65504, index = bits
INT4_GRID = np.arange(INT4_QMAX + 1, dtype=np.float64)                                  # 0 .. 7


def fp16(v) -> np.ndarray:
    """IEEE binary16 round-to-nearest-even (10-bit fraction, emin -14), saturating at 65504."""
    return round_to_format(v, 10, -14, 65504.0)


def quantize_int4(v32: np.ndarray, group: int = INT4_GROUP) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric INT4 group quantization along the last axis of fp32 values.

    Returns (codes int8 in [-7, 7], scales as fp16 values in float64 [.., K/group])."""
    v = np.asarray(v32, dtype=np.float32).astype(np.float64)
    rows, K = v.shape
    assert K % group == 0
    g = v.reshape(rows, K // group, group)
    amax = np.max(np.abs(g), axis=2)
    s = FP16_GRID[rne_quotient_index(amax, INT4_QMAX, FP16_GRID)]   # products mid * 7: <= 15 bits
    live = s > 0
    mag = rne_quotient_index(g, np.where(live, s, 1.0), INT4_GRID)  # products (k + 1/2) s: <= 15 bits
    q = np.where(np.signbit(g), -mag, mag)
    q = np.where(live[..., None], q, 0)
    return q.reshape(rows, K).astype(np.int8), s


def dequantize_int4(codes: np.ndarray, scales: np.ndarray, group: int = INT4_GROUP) -> np.ndarray:
    c = np.asarray(codes, dtype=np.float64)
    rows, K = c.shape
    return (c.reshape(rows, K // group, group) * np.asarray(scales, np.float64)[:, :, None]).reshape(rows, K)


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Two's-complement nibbles, element 2i in the low nibble of byte i."""
    u = (np.asarray(codes, dtype=np.int16) & 0xF).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((p.shape[0], 2 * p.shape[1]), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def layer_reference_int4(X, W_lin, alpha: float, rank: int, act_amax=None) -> dict:
    """The same layer with INT4 (g = 64, fp16 scales) in place of NVFP4: the
    smoothing and the stored low-rank factors are those of prepare_weights; the
    residual R and the smoothed activation are INT4-quantized along K."""
    X = np.asarray(X, dtype=np.float64)
    if act_amax is None:
        act_amax = channel_amax(X)
    P = prepare_weights(W_lin, act_amax, alpha, rank)
    Qr, Sr = quantize_int4(P["R32"].T)                        # [N][K], grouped along K
    X32 = np.asarray(X, dtype=np.float32)
    xhat = X32 * np.asarray(P["inv32"], dtype=np.float32)[None, :]
    Qx, Sx = quantize_int4(xhat)
    T = X @ P["L1p"] if rank else np.zeros((X.shape[0], 0))
    Y = dequantize_int4(Qx, Sx) @ dequantize_int4(Qr, Sr).T
    if rank:
        Y = Y + T @ P["L2"]
    return {**P, "Qx4": Qx, "Sx4": Sx, "Qr4": Qr, "Sr4": Sr, "T": T, "Y": Y, "Y_exact": X @ np.asarray(W_lin, np.float64).T}


# ---------------------------------------------------------------------------
# DeltaQuant-style core + delta activations ([P1] libaedu.com article on
# 4-bit diffusion-model quantization, DeltaQuant paragraphs: video
# activations are split into local 3-D spatio-temporal blocks; each block's
# mean token is the core token, kept in FP8; the differences to it are
# quantized to 4 bits). The page gives the method in outline only. Readings:
#   * tokens of a video latent [F][H][Wd] are rows in frame, row, column
#     order; blocks are bf x bh x bw tokens (default 2 x 2 x 2), tiled from
#     the origin; blocks at a ragged edge hold the tokens that exist;
#   * core = E4M3_RNE_satfinite of the block's exact mean (the fp64 sum of its
#     tokens in token order, divided by the token count, rounded once), per
#     channel, with no scale (the page names FP8 and nothing else);
#   * delta = fp32(x - decode(core)), the exact difference rounded once to
#     fp32, i.e. relative to the stored core, so the core's rounding is
#     absorbed by the delta; deltas are NVFP4 (groups of 16 channels, the codec
#     above);
#   * reconstruction x~ = decode(core) + deq(delta).
# Oracle only: no kernel consumes this encoding yet.

def e4m3_encode_signed(v) -> np.ndarray:
    """E4M3 byte of RNE_satfinite(v) for any sign (sign bit 0x80; a negative
    value that rounds to zero keeps it)."""
    v = np.asarray(v, dtype=np.float64)
    mag = e4m3_encode(np.abs(v)).astype(np.int64)
    return (mag | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def video_blocks(F: int, H: int, Wd: int, block=(2, 2, 2)) -> np.ndarray:
    """Block index of every token (rows in frame, row, column order)."""
    bf, bh, bw = block
    nbh, nbw = -(-H // bh), -(-Wd // bw)
    f, h, w = np.meshgrid(np.arange(F), np.arange(H), np.arange(Wd), indexing="ij")
    return ((f // bf) * nbh * nbw + (h // bh) * nbw + (w // bw)).reshape(-1)


def deltaquant_encode(X: np.ndarray, dims, block=(2, 2, 2)) -> dict:
    """Core tokens (E4M3 bytes, [blocks][C]) and NVFP4 deltas of X [F*H*Wd][C]."""
    X = np.asarray(X, dtype=np.float64)
    F, H, Wd = dims
    assert X.shape[0] == F * H * Wd and X.shape[1] % 16 == 0
    blk = video_blocks(F, H, Wd, block)
    nb = int(blk.max()) + 1
    sums = np.zeros((nb, X.shape[1]))
    np.add.at(sums, blk, X)
    counts = np.bincount(blk, minlength=nb).astype(np.float64)
    # E4M3 RNE (satfinite) of the exact quotient sum / count; a negative mean
    # that rounds to zero keeps the sign bit, a zero sum encodes +0
    mag = rne_quotient_index(sums, counts, E4M3_GRID)
    core_codes = (mag | np.where(np.signbit(sums) & (sums != 0), 0x80, 0)).astype(np.uint8)
    core = e4m3_decode(core_codes)
    # one rounding of the exact difference (bf16 and E4M3 values are exact in fp32)
    delta = X.astype(np.float32) - core[blk].astype(np.float32)
    codes, scales = quantize_nvfp4(delta)
    return dict(block_of_token=blk, core_codes=core_codes, delta_codes=codes, delta_scales=scales)


def deltaquant_decode(enc: dict) -> np.ndarray:
    core = e4m3_decode(enc["core_codes"])
    return core[enc["block_of_token"]] + dequantize_nvfp4(enc["delta_codes"], enc["delta_scales"])


# ---------------------------------------------------------------------------
# The method in real arithmetic with per-tensor integer quantization: the
# setting of the handbook's printed error tables ([P3] outlier, SmoothQuant and
# SVDQuant sections). Composed from eq. (1), the smoothing rule and the SVD
# split above, in fp64 and with no storage format.
# ---------------------------------------------------------------------------

def int_quant_dequant(t: np.ndarray, bits: int, axis=None) -> np.ndarray:
    """s * Q(t) of eq. (1) for signed ``bits``-bit integers: one scale
    s = max|t| / q_max for the whole tensor (axis None) or per slice along
    ``axis``; Q = round(t / s) half to even, clipped to +-q_max. An all-zero
    tensor or slice stays zero."""
    q_max = 2 ** (bits - 1) - 1
    t = np.asarray(t, dtype=np.float64)
    amax = np.abs(t).max(axis=axis, keepdims=axis is not None)
    s = np.where(amax > 0, amax / q_max, 1.0)
    return s * np.clip(np.rint(t / s), -q_max, q_max)


def smoothed_pair(x: np.ndarray, W_io: np.ndarray, alpha: float = 0.5):
    """(X_hat, W_hat) = (X diag(lambda)^-1, diag(lambda) W) for W_io in the
    paper's (in x out) orientation, lambda64 of the fp64 channel maxima."""
    x = np.asarray(x, dtype=np.float64)
    W_io = np.asarray(W_io, dtype=np.float64)
    lam = lambda64(np.abs(x).max(axis=0), np.abs(W_io).max(axis=1), alpha)
    return x / lam, lam[:, None] * W_io


def fakequant_output(x: np.ndarray, W_io: np.ndarray, rank: int, q, alpha: float = 0.5) -> np.ndarray:
    """Eq. (5) in real arithmetic: X_hat L1 L2 + q(X_hat) q(R) with
    R = W_hat - L1 L2 (rank 0: q(X_hat) q(W_hat)); ``q`` is a quantize-
    dequantize function."""
    xh, Wh = smoothed_pair(x, W_io, alpha)
    L1, L2, _ = svd_split(Wh, rank)
    return q(xh) @ q(Wh - L1 @ L2) + (xh @ L1) @ L2


# ---------------------------------------------------------------------------
# Error measures ([P2] eq. (3), eq. (4)/(9))
# ---------------------------------------------------------------------------

def fro(a) -> float:
    return float(np.linalg.norm(np.asarray(a, dtype=np.float64)))


def rel_fro(a, b) -> float:
    """||a - b||_F / ||b||_F."""
    return fro(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64)) / fro(b)


def quant_error(X, W, QX, QW) -> float:
    """E(X, W) = ||X W - Q(X) Q(W)||_F."""
    return fro(np.asarray(X) @ np.asarray(W) - np.asarray(QX) @ np.asarray(QW))


def prop41_bound(X, W, QX, QW) -> float:
    """||X|| ||W - Q(W)|| + ||X - Q(X)|| (||W|| + ||W - Q(W)||)."""
    dW = fro(np.asarray(W) - np.asarray(QW))
    return fro(X) * dW + fro(np.asarray(X) - np.asarray(QX)) * (fro(W) + dW)
