"""Pins for the oracle's method steps: smoothing, SVD split, residual,
activation quantization with the fused down-projection, and the layer output.

Anchors outside the oracle itself:
  * the handbook's printed error tables (anrans.github.io AI-infra handbook,
    Quantization chapter: outlier, SmoothQuant and SVDQuant sections),
    regenerated from torch's seeded CPU RNG, to their printed 4 decimals;
  * identities and bounds of the devpress.csdn.net SVDQuant walkthrough:
    X_hat W_hat = X W (smoothing), eq. (6), Proposition 4.1 (eq. (4)/(9)),
    Eckart-Young optimality of the SVD split;
  * brute-force per-element loops in plain Python floats on tiny inputs;
  * special cases: rank 0, exactly rank-r weights, lambda = 1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O


# ---------------------------------------------------------------------------
# Handbook tables
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def handbook(golden_dir):
    with open(os.path.join(golden_dir, "handbook_quant_tables.json")) as f:
        tab = json.load(f)
    torch.manual_seed(0)
    base = torch.randn(1024, 512).double().numpy()
    W = (torch.randn(512, 512) * 0.02).double().numpy()
    return tab, base, W


def _r4(x):
    return round(float(x), 4)


def test_handbook_outlier_table(handbook):
    tab, base, _ = handbook
    for scale, row in tab["outlier_table"]["rows"].items():
        x = base.copy()
        x[:, :4] *= float(scale)
        got = [O.rel_fro(O.int_quant_dequant(x, b, ax)[:, 4:], x[:, 4:])
               for b, ax in ((8, None), (8, 0), (4, None), (4, 0))]
        assert [_r4(g) for g in got] == row, scale


def test_handbook_smoothquant_table(handbook):
    tab, base, W = handbook
    t = tab["smoothquant_table"]
    x = base.copy()
    x[:, :4] *= 50
    y = x @ W
    q8 = lambda a: O.int_quant_dequant(a, 8)  # noqa: E731
    q4 = lambda a: O.int_quant_dequant(a, 4)  # noqa: E731
    xs, Ws = O.smoothed_pair(x, W)
    assert _r4(O.rel_fro(q8(x) @ q8(W), y)) == t["w8a8"]
    assert _r4(O.rel_fro(q8(xs) @ q8(Ws), y)) == t["w8a8_smooth"]
    assert _r4(O.rel_fro(q4(x) @ q4(W), y)) == t["w4a4"]
    assert _r4(O.rel_fro(q4(xs) @ q4(Ws), y)) == t["w4a4_smooth"]


def test_handbook_svdquant_table(handbook):
    tab, base, W = handbook
    t = tab["svdquant_table"]
    x = base.copy()
    x[:, :4] *= 50
    y = x @ W
    q4 = lambda a: O.int_quant_dequant(a, 4)  # noqa: E731
    for r, want in t["rank"].items():
        got = O.rel_fro(O.fakequant_output(x, W, int(r), q4), y)
        assert _r4(got) == want, r
    assert _r4(O.rel_fro(q4(base) @ q4(W), base @ W)) == t["no_outlier_w4a4_floor"]


def test_prepare_weights_matches_handbook_flow(handbook):
    """The NVFP4-path preparation (lambda32, bf16 factors folded with 1/lambda,
    fp32 residual) applies the same smoothing and SVD split as the handbook
    flow: with the handbook's INT4 per-tensor quantizer on its residual, the
    output error matches the printed rank-32 entry to ~1e-3."""
    tab, base, W = handbook
    x = base.copy()
    x[:, :4] *= 50
    y = x @ W
    W_lin = W.T.copy()
    P = O.prepare_weights(W_lin, O.channel_amax(x), 0.5, 32)
    lam = P["lam32"].astype(np.float64)
    xs = x / lam
    q4 = lambda a: O.int_quant_dequant(a, 4)  # noqa: E731
    yq = q4(xs) @ q4(P["R32"].astype(np.float64)) + xs @ (lam[:, None] * P["L1p"]) @ P["L2"]
    assert abs(O.rel_fro(yq, y) - tab["svdquant_table"]["rank"]["32"]) < 2e-3


# ---------------------------------------------------------------------------
# Smoothing
# ---------------------------------------------------------------------------

def test_smoothing_identity_and_lambda_rule():
    rng = np.random.default_rng(10)
    X = rng.standard_normal((64, 48))
    X[:, 3] *= 40
    W_lin = rng.standard_normal((32, 48)) * 0.1
    ax = O.channel_amax(X)
    lam, inv = O.smoothing_lambda(ax, W_lin, 0.5)
    # the smoothed product equals the original product (only rounding of lambda
    # to fp32 enters, and it cancels exactly in exact arithmetic)
    lam64 = lam.astype(np.float64)
    Xh, Wh = X / lam64, lam64[:, None] * W_lin.T
    assert O.rel_fro(Xh @ Wh, X @ W_lin.T) < 1e-13
    # alpha = 0.5 (sqrt form) agrees with the generic power form to 1 ulp of fp32
    lam_pow, _ = O.smoothing_lambda(ax, W_lin, 0.5000000000000001)
    assert np.all(np.abs(lam.view(np.int32) - lam_pow.view(np.int32)) <= 1)
    # alpha = 1: lambda = max|X_j| ; alpha = 0: lambda = 1 / max|W_j|
    l1, _ = O.smoothing_lambda(ax, W_lin, 1.0)
    assert np.array_equal(l1, ax)
    l0, _ = O.smoothing_lambda(ax, W_lin, 0.0)
    assert np.allclose(l0, 1.0 / np.abs(W_lin).max(axis=0), rtol=1e-7)
    # smoothing flattens the activation channel maxima: max|X_hat_j| = sqrt(ax_j aw_j)
    aw = np.abs(W_lin).max(axis=0)
    assert np.allclose(np.abs(Xh).max(axis=0), np.sqrt(ax * aw), rtol=1e-6)
    # inv is the fp32-rounded reciprocal
    assert np.array_equal(inv, (np.float32(1) / lam).astype(np.float32))


def test_smoothing_zero_channels_give_unit_lambda():
    X = np.ones((4, 32))
    X[:, 5] = 0
    W_lin = np.ones((8, 32))
    W_lin[:, 7] = 0
    lam, inv = O.smoothing_lambda(O.channel_amax(X), W_lin, 0.5)
    assert lam[5] == 1 and lam[7] == 1 and inv[5] == 1


# ---------------------------------------------------------------------------
# Weight preparation
# ---------------------------------------------------------------------------

def test_residual_brute_force_tiny():
    """Each R[j][n] evaluated with Python floats (IEEE fp64, no FMA) in the
    stated order equals the vectorized residual."""
    rng = np.random.default_rng(11)
    K, N, r = 32, 4, 3
    W_lin = O.bf16(rng.standard_normal((N, K)))
    lam = rng.uniform(0.5, 3, K).astype(np.float32)
    L1p = O.bf16(rng.standard_normal((K, r)))
    L2 = O.bf16(rng.standard_normal((r, N)))
    R32, codes, scales = O.residual_quantize(W_lin, lam, L1p, L2)
    for j in range(K):
        for n in range(N):
            acc = 0.0
            for k in range(r):
                acc = acc + (float(lam[j]) * float(L1p[j, k])) * float(L2[k, n])
            want = np.float32(float(lam[j]) * float(W_lin[n, j]) - acc)
            assert R32[j, n] == want
    assert codes.shape == (N, K) and scales.shape == (N, K // 16)


def test_rank0_residual_is_the_smoothed_weight():
    rng = np.random.default_rng(12)
    W_lin = O.bf16(rng.standard_normal((16, 64)))
    lam = rng.uniform(0.5, 3, 64).astype(np.float32)
    R32, codes, scales = O.residual_quantize(W_lin, lam, np.zeros((64, 0)), np.zeros((0, 16)))
    assert np.array_equal(R32, (lam.astype(np.float64)[:, None] * W_lin.T).astype(np.float32))
    c2, s2 = O.quantize_nvfp4(R32.T.copy())
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2)


def test_svd_split_is_eckart_young_optimal():
    """||W_hat - (lambda L1') L2||^2 with the stored bf16 factors is the tail
    energy sum_{i>r} sigma_i^2 up to the factors' bf16 rounding."""
    rng = np.random.default_rng(13)
    K, N, r = 96, 80, 8
    X = rng.standard_normal((40, K))
    X[:, :3] *= 30
    W_lin = O.bf16(rng.standard_normal((N, K)) / math.sqrt(K)
                   + 0.5 * np.outer(rng.choice([-1, 1], N), rng.choice([-1, 1], K)) / math.sqrt(K))
    P = O.prepare_weights(W_lin, O.channel_amax(X), 0.5, r)
    lam = P["lam32"].astype(np.float64)
    resid = P["What"] - (lam[:, None] * P["L1p"]) @ P["L2"]
    tail = np.sum(P["S"][r:] ** 2)
    assert np.sum(resid ** 2) <= tail * (1 + 1e-2) + 1e-4 * np.sum(P["S"][:r] ** 2) * 2.0 ** -14
    assert np.sum(resid ** 2) >= tail * (1 - 1e-9)
    # R32 is that residual rounded to fp32
    assert np.array_equal(P["R32"], resid.astype(np.float32)) or \
        np.max(np.abs(P["R32"] - resid)) <= np.max(np.abs(resid)) * 2.0 ** -23


def test_exactly_rank_r_weight_leaves_small_residual():
    rng = np.random.default_rng(14)
    K, N, r = 64, 48, 4
    # small-integer factors: W_lin is exactly representable in bf16 and exactly rank r
    W_lin = (rng.integers(-2, 3, (N, r)) @ rng.integers(-2, 3, (r, K))).astype(np.float64) / 8
    assert np.array_equal(O.bf16(W_lin), W_lin) and np.linalg.matrix_rank(W_lin) == r
    X = rng.standard_normal((16, K))
    P = O.prepare_weights(W_lin, O.channel_amax(X), 0.5, r)
    assert P["S"][r] < 1e-12 * P["S"][0]
    # only the bf16 rounding of the stored factors remains (relative ~2^-8)
    assert np.linalg.norm(P["R32"]) <= 2.0 ** -7 * np.linalg.norm(P["What"])
    # and the layer output is then dominated by the exact low-rank branch
    Qx, Sx, T = O.quantize_act(X, P["inv32"], P["L1p"])
    Y = O.linear(Qx, Sx, T, P["Qr"], P["Sr"], P["L2"])
    assert O.rel_fro(Y, X @ W_lin.T) < 2.0 ** -6


# ---------------------------------------------------------------------------
# Per-call path
# ---------------------------------------------------------------------------

def test_quantize_act_grid_inputs_exact():
    """lambda = 1 and grid-aligned X: codes/scales recover X exactly and T is
    the exact product."""
    rng = np.random.default_rng(15)
    s_bytes = rng.integers(40, 110, size=(8, 4))
    e = rng.choice(np.concatenate([O.E2M1_VALUES, -O.E2M1_VALUES]), size=(8, 4, 16))
    e[..., 0] = 6.0
    X = (e * O.e4m3_decode(s_bytes)[..., None]).reshape(8, 64)
    L1p = O.bf16(rng.standard_normal((64, 16)))
    codes, scales, T = O.quantize_act(X, np.ones(64, dtype=np.float32), L1p)
    assert np.array_equal(scales, s_bytes.astype(np.uint8))
    assert np.array_equal(O.dequantize_nvfp4(codes, scales), X)
    assert np.array_equal(T, X @ L1p)


def test_linear_brute_force_tiny():
    """8 x 32 x 16 layer: per-element Python loop (decode each nibble and
    scale byte by index) equals the vectorized dequantize + matmul."""
    rng = np.random.default_rng(16)
    M, K, N, r = 8, 32, 16, 2
    Qx = rng.integers(0, 16, (M, K)).astype(np.uint8)
    Sx = rng.integers(0, 120, (M, K // 16)).astype(np.uint8)
    Qr = rng.integers(0, 16, (N, K)).astype(np.uint8)
    Sr = rng.integers(0, 120, (N, K // 16)).astype(np.uint8)
    T = rng.standard_normal((M, r))
    L2 = rng.standard_normal((r, N))
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]

    def fp4(c):
        c = int(c)
        return (-1.0 if c & 8 else 1.0) * grid[c & 7]

    def e4m3(b):
        b = int(b)
        e, m = (b >> 3) & 15, b & 7
        return (m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)

    Y = O.linear(Qx, Sx, T, Qr, Sr, L2)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += fp4(Qx[m, k]) * e4m3(Sx[m, k // 16]) * fp4(Qr[n, k]) * e4m3(Sr[n, k // 16])
            for k in range(r):
                acc += T[m, k] * L2[k, n]
            assert abs(Y[m, n] - acc) <= 1e-12 * (1 + abs(acc))


def _tiny_layer():
    rng = np.random.default_rng(17)
    M, K, N, r = 64, 128, 96, 8
    X = rng.standard_normal((M, K))
    X[:, :4] *= 50
    X = O.bf16(X)
    W_lin = O.bf16(rng.standard_normal((N, K)) / math.sqrt(K)
                   + 2 * np.outer(rng.choice([-1, 1], N), rng.choice([-1, 1], K)) / math.sqrt(K))
    return X, W_lin, r


def test_eq6_identity_and_prop41_bound():
    X, W_lin, r = _tiny_layer()
    L = O.layer_reference(X, W_lin, 0.5, r)
    lam = L["lam32"].astype(np.float64)
    Xh = X / lam
    What = L["What"]
    L1L2 = (lam[:, None] * L["L1p"]) @ L["L2"]
    R = L["R32"].astype(np.float64)
    QX = O.dequantize_nvfp4(L["Qx"], L["Sx"])
    QR = O.dequantize_nvfp4(L["Qr"], L["Sr"]).T
    # eq. (6): error of the split layer == E(X_hat, R) (R exact up to fp32 rounding)
    lhs = O.fro(Xh @ What - (Xh @ L1L2 + QX @ QR))
    rhs = O.quant_error(Xh, R, QX, QR)
    assert abs(lhs - rhs) <= 1e-6 * rhs
    # the oracle's linear() is that split layer: T L2 == X_hat L1 L2
    assert O.rel_fro(L["Y"], Xh @ L1L2 + QX @ QR) < 1e-12
    # Proposition 4.1 on (X_hat, R) and on the unsplit smoothed layer
    assert rhs <= O.prop41_bound(Xh, R, QX, QR)
    c, s = O.quantize_nvfp4(What.T.astype(np.float32).copy())
    QW = O.dequantize_nvfp4(c, s).T
    assert O.quant_error(Xh, What, QX, QW) <= O.prop41_bound(Xh, What, QX, QW)


def test_low_rank_branch_reduces_error_and_rank_trend():
    """The printed trend: smoothing alone < low-rank branch; error falls as r
    grows (handbook SVDQuant table; walkthrough Fig. 18 text)."""
    X, W_lin, _ = _tiny_layer()
    errs = []
    for r in (0, 4, 8, 16):
        L = O.layer_reference(X, W_lin, 0.5, r)
        errs.append(O.rel_fro(L["Y"], L["Y_exact"]))
    assert errs[0] > errs[1] > errs[2] > errs[3]
    Lr = O.layer_reference(X, W_lin, 0.5, 0)
    # rank 0 reduces to plain smoothed NVFP4 W4A4 with no branch
    c, s = O.quantize_nvfp4((Lr["What"].T).astype(np.float32).copy())
    assert np.array_equal(c, Lr["Qr"]) and np.array_equal(s, Lr["Sr"])
    assert Lr["T"].shape == (X.shape[0], 0)


def test_native_scales_of_quantized_activation_roundtrip():
    X, W_lin, r = _tiny_layer()
    L = O.layer_reference(X, W_lin, 0.5, r)
    nat = O.scales_to_native(L["Sx"])
    assert np.array_equal(O.native_to_scales(nat, X.shape[0], X.shape[1]), L["Sx"])


def test_eq7_eq8_gaussian_residual_monte_carlo():
    """Walkthrough eq. (7)/(8) with its Gaussian constant
    c = sqrt(pi log(size) / size) (Gaussian maximal inequality and the
    half-normal mean): on iid normal matrices E[max|R|] <= c E[||R||_F], and
    each of the oracle's 4-bit quantizers keeps
    E[||R - Q(R)||_F] <= c sqrt(size) / q_max E[||R||_F] (per-tensor INT4,
    NVFP4 groups of 16 with q_max = 6, INT4 groups of 64 with q_max = 7).
    The two uniform quantizers also match the uniform-rounding error
    E||R - Q(R)||^2 = sum over elements of step^2 / 12 within 5 %, which pins
    their step sizes (max/7 per tensor, the fp16 group scale per 64)."""
    rng = np.random.default_rng(21)
    for shape in ((64, 64), (128, 512), (512, 1024)):
        size = shape[0] * shape[1]
        c = math.sqrt(math.pi * math.log(size) / size)
        Rs = [(rng.standard_normal(shape) * 0.37).astype(np.float32).astype(np.float64) for _ in range(12)]
        m_max = np.mean([np.abs(R).max() for R in Rs])
        m_fro = np.mean([O.fro(R) for R in Rs])
        assert m_max <= c * m_fro
        quantizers = {
            "int4 per tensor": (7, lambda R: O.int_quant_dequant(R, 4)),
            "nvfp4 g16": (6, lambda R: O.dequantize_nvfp4(*O.quantize_nvfp4(R))),
            "int4 g64": (7, lambda R: O.dequantize_int4(*O.quantize_int4(R))),
        }
        for name, (qmax, q) in quantizers.items():
            m_err = np.mean([O.fro(R - q(R)) for R in Rs])
            assert m_err <= c * math.sqrt(size) / qmax * m_fro, name
        # uniform rounding: error variance step^2 / 12 per element
        for R in Rs[:4]:
            err2 = O.fro(R - O.int_quant_dequant(R, 4)) ** 2
            step = np.abs(R).max() / 7
            assert abs(err2 / (size * step ** 2 / 12) - 1) < 0.05
            _, s = O.quantize_int4(R)
            err2 = O.fro(R - O.dequantize_int4(*O.quantize_int4(R))) ** 2
            assert abs(err2 / (64 * np.sum(s ** 2) / 12) - 1) < 0.05
