"""Pins of the oracle's INT4 W4A4 variant (walkthrough eq. (1): q = round(x / s),
s = max|x| / q_max with q_max = 2^(k-1) - 1 = 7 for signed 4-bit; handbook:
one scale per 64 elements; fp16 scales). Each pin checks the oracle against
something other than itself: numpy's float16 conversion, exactly representable
grids, hand-enumerated ties, a brute-force loop, and error trends."""
import numpy as np

import oracle as O
from w4a4_diffusion_model_b200 import synth


def test_fp16_matches_numpy_below_overflow():
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 5, 20000), [0.0, 65504.0, 65519.0]])
    assert np.array_equal(O.fp16(v), v.astype(np.float16).astype(np.float64))


def test_int4_exact_grid_round_trips():
    """x = e * s with integer e in [-7, 7], one element per group equal to 7 s
    and s an fp16 value: the codes are e and the product is exact."""
    rng = np.random.default_rng(12)
    rows, K = 6, 256
    s = np.float16(rng.uniform(0.01, 3.0, (rows, K // 64))).astype(np.float64)
    e = rng.integers(-7, 8, (rows, K // 64, 64)).astype(np.float64)
    e[:, :, 5] = 7 * np.sign(rng.standard_normal((rows, K // 64))) + 0.0
    x = (e * s[:, :, None]).reshape(rows, K)
    assert np.array_equal(O.fp32(x), x)
    q, sc = O.quantize_int4(x.astype(np.float32))
    assert np.array_equal(sc, s)
    assert np.array_equal(q.astype(np.float64), e.reshape(rows, K))
    assert np.array_equal(O.dequantize_int4(q, sc), x)


def test_int4_ties_to_even_clamp_and_zero_groups():
    row = np.zeros(64)
    row[:10] = [0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 6.5, -6.5, 7.0]   # amax 7: s = 1
    q, s = O.quantize_int4(row[None, :].astype(np.float32))
    assert s[0, 0] == 1.0
    assert list(q[0, :10]) == [0, 2, 2, 4, 0, -2, -2, 6, -6, 7]
    zero, sz = O.quantize_int4(np.zeros((1, 64), np.float32))
    assert sz[0, 0] == 0.0 and not zero.any()
    tiny, st = O.quantize_int4(np.full((1, 64), 1e-9, np.float32))       # scale underflows to 0
    assert st[0, 0] == 0.0 and not tiny.any()
    huge, sh = O.quantize_int4(np.full((1, 64), 3e38, np.float32))       # scale saturates at 65504
    assert sh[0, 0] == 65504.0 and np.all(huge == 7)


def test_int4_pack_round_trip_and_nibble_order():
    codes = np.array([[1, -1, -7, 7, 0, 3]], dtype=np.int8)
    p = O.pack_int4(codes)
    assert list(p[0]) == [0xF1, 0x79, 0x30]          # element 2i in the low nibble, two's complement
    assert np.array_equal(O.unpack_int4(p), codes)


def test_int4_quantizer_brute_force():
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((3, 128)) * 2.0).astype(np.float32)
    q, s = O.quantize_int4(x)
    for r in range(3):
        for g in range(2):
            v = x[r, 64 * g:64 * g + 64].astype(np.float64)
            amax = max(abs(float(t)) for t in v)
            sc = float(np.float16(np.float32(amax / 7.0)))
            assert s[r, g] == sc
            inv = float(np.float32(1.0 / sc))
            for j in range(64):
                y = float(np.float32(v[j] * inv))
                k = max(-7, min(7, int(round(y))))                     # Python round: half to even
                assert q[r, 64 * g + j] == k


def test_int4_layer_error_trends():
    """Smoothing + the low-rank branch lower the INT4 layer's error the way they
    lower the NVFP4 layer's (walkthrough: the branch absorbs the outliers); the
    64-element groups leave INT4 coarser than 16-element NVFP4."""
    w = synth.TINY
    X, W = synth.generate(w)
    Xn = X.float().numpy().astype(np.float64)
    Wn = W.float().numpy().astype(np.float64)
    exact = Xn @ Wn.T
    e4_r0 = O.rel_fro(O.layer_reference_int4(Xn, Wn, 0.5, 0)["Y"], exact)
    e4_r16 = O.rel_fro(O.layer_reference_int4(Xn, Wn, 0.5, 16)["Y"], exact)
    ef_r16 = O.rel_fro(O.layer_reference(Xn, Wn, 0.5, 16)["Y"], exact)
    assert e4_r16 < e4_r0 < 0.5
    assert ef_r16 < e4_r16 < 4 * ef_r16


def test_int4_codes_as_e4m3_bytes_match_torch():
    """The byte form of INT4 codes used by the B200 kernels: the E4M3 encoding
    of the integers -7..7 is exact, and the oracle's encoder (with the sign bit)
    agrees with torch's float8_e4m3fn conversion."""
    import torch
    ints = np.arange(-7, 8)
    ours = (O.e4m3_encode(np.abs(ints).astype(np.float64)) | np.where(ints < 0, 0x80, 0)).astype(np.uint8)
    lib = torch.tensor(ints, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)
    assert np.array_equal(O.e4m3_decode(ours), ints.astype(np.float64))


def test_int4_layer_output_brute_force_tiny():
    """layer_reference_int4's Y against a plain-Python loop over its own codes,
    scales and factors: Y[m][n] = sum_k qx sx(m, k/64) qr sr(n, k/64)
    + sum_j T[m][j] L2[j][n]."""
    rng = np.random.default_rng(31)
    M, K, N, r = 3, 128, 4, 2
    X = O.bf16(rng.standard_normal((M, K)) * np.exp(rng.uniform(-1, 1, K)))
    W = O.bf16(rng.standard_normal((N, K)) / np.sqrt(K))
    ref = O.layer_reference_int4(X, W, 0.5, r)
    qx, sx, qr, sr, T, L2 = ref["Qx4"], ref["Sx4"], ref["Qr4"], ref["Sr4"], ref["T"], ref["L2"]
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(qx[m, k]) * float(sx[m, k // 64]) * float(qr[n, k]) * float(sr[n, k // 64])
            for j in range(r):
                acc += float(T[m, j]) * float(L2[j, n])
            assert abs(acc - ref["Y"][m, n]) <= 1e-12 * max(1.0, abs(acc))
