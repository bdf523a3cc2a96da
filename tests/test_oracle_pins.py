"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Quantization ("Joy-face_change_optimized" model card, files table and tools
row: RTN, int8 per output channel, int4 grouped along K with gs 64 / 16):
  * brute force: on tiny groups, every code equals the argmin over all
    q in [-qmax, qmax] of |W - q s| (ties to the even q), computed with exact
    rationals; every scale equals the fp32 nearest to absmax / qmax, found by
    exact comparison with its fp32 neighbours;
  * closed form: |W - q s| <= s / 2 for every element;
  * invariants: the absmax element of a nonzero group gets +-qmax with its
    sign; re-quantizing the dequantized weights returns the same codes;
  * special cases: exact ties go to the even code; all-zero groups give
    s = 0 and q = 0; non-finite weights are rejected.
Linear ("Joy-face_change_optimized", files table: weight-only Linear;
"Nunchaku Lite", why it matters: 16-bit low-rank correction):
  * brute force with exact rationals on tiny shapes;
  * special cases reducing to numpy fp64 matmul, to s * (x q^T) for int8
    per-channel, to the pure low-rank product when the codes are zero, and to
    a scaled identity when W = c I.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import wlq_inputs as wi

QMAX = {8: 127, 4: 7}


# --------------------------------------------------------------------------
# exact helpers (independent of the oracle)
# --------------------------------------------------------------------------

def nearest_f32(fr: Fraction) -> np.float32:
    """The fp32 nearest to a non-negative rational, ties to even mantissa."""
    c = np.float32(float(fr))
    cands = {float(c), float(np.nextafter(c, np.float32(np.inf))),
             float(np.nextafter(c, np.float32(0)))}
    best = None
    for v in sorted(cands):
        d = abs(Fraction(v) - fr)
        key = (d, int(np.float32(v).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, v)
    return np.float32(best[1])


def brute_codes(w: np.ndarray, s: np.float32, qmax: int) -> np.ndarray:
    if s == 0:
        return np.zeros(len(w), np.int8)
    S = Fraction(float(s))
    out = []
    for v in w:
        V = Fraction(float(v))
        best = None
        for q in range(-qmax, qmax + 1):
            key = (abs(V - q * S), q & 1)  # nearest, then even
            if best is None or key < best[0]:
                best = (key, q)
        out.append(best[1])
    return np.array(out, np.int8)


def brute_group(w: np.ndarray, bits: int):
    qmax = QMAX[bits]
    a = max((abs(Fraction(float(v))) for v in w), default=Fraction(0))
    s = nearest_f32(a / qmax)
    return brute_codes(w, s, qmax), s


def adversarial_groups(g, size):
    f32 = np.float32
    out = [
        np.zeros(size, f32),
        np.full(size, f32(0.25)),
        np.full(size, f32(-3.0e38)),
        (g.standard_normal(size) * 1e-40).astype(f32),   # subnormal inputs
        (g.standard_normal(size) * 1e30).astype(f32),
        g.integers(-9, 10, size).astype(f32) * f32(0.5),  # many exact halves
    ]
    w = g.standard_normal(size).astype(f32)
    w[0] = -np.abs(w).max() * f32(1.0)  # negative absmax
    out.append(w)
    return out


# --------------------------------------------------------------------------
# quantization
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [8, 4])
def test_quantize_matches_brute_force(bits):
    g = np.random.default_rng(1234 + bits)
    for size in (1, 2, 3, 5, 8, 16):
        groups = [g.standard_normal(size).astype(np.float32) * np.float32(s)
                  for s in (1e-3, 0.02, 1.0, 7.0)]
        groups += adversarial_groups(g, size)
        for w in groups:
            codes, scales = oracle.quantize(w[None, :], bits, 0)
            bq, bs = brute_group(w, bits)
            assert scales[0, 0].view(np.uint32) == bs.view(np.uint32), (w, scales, bs)
            np.testing.assert_array_equal(codes[0], bq, err_msg=str(w))


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
def test_grouping_matches_brute_force(bits, group):
    g = np.random.default_rng(7)
    K = 128
    W = wi.weight(5, 1, 6, K, outlier_frac=0.05)
    W[2, :] = 0.0
    W[3, 5] = g.standard_normal() * 50
    codes, scales = oracle.quantize(W, bits, group)
    gs = K if group == 0 else group
    for n in range(W.shape[0]):
        for gi in range(K // gs):
            bq, bs = brute_group(W[n, gi * gs:(gi + 1) * gs], bits)
            assert scales[n, gi].view(np.uint32) == bs.view(np.uint32)
            np.testing.assert_array_equal(codes[n, gi * gs:(gi + 1) * gs], bq)


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
def test_rtn_error_bound(bits, group):
    W = wi.weight(6, 1, 257, 1024, outlier_frac=0.01)
    codes, scales = oracle.quantize(W, bits, group)
    gs = W.shape[1] if group == 0 else group
    s = np.repeat(scales.astype(np.float64), gs, axis=1)
    err = np.abs(W.astype(np.float64) - codes.astype(np.float64) * s)
    assert np.all(err <= s / 2)
    assert np.all(np.abs(codes) <= QMAX[bits])


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
def test_absmax_maps_to_qmax(bits, group):
    W = wi.weight(7, 1, 64, 512)
    codes, _ = oracle.quantize(W, bits, group)
    gs = W.shape[1] if group == 0 else group
    Wg = W.reshape(64, -1, gs)
    Cg = codes.reshape(64, -1, gs)
    idx = np.abs(Wg).argmax(axis=2)
    at = np.take_along_axis(Cg, idx[..., None], axis=2)[..., 0]
    sign = np.sign(np.take_along_axis(Wg, idx[..., None], axis=2)[..., 0])
    np.testing.assert_array_equal(at, (sign * QMAX[bits]).astype(np.int8))


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
def test_requantize_is_idempotent(bits, group):
    W = wi.weight(8, 1, 96, 256, outlier_frac=0.02)
    codes, scales = oracle.quantize(W, bits, group)
    gs = W.shape[1] if group == 0 else group
    W2 = (codes.astype(np.float64) *
          np.repeat(scales.astype(np.float64), gs, axis=1)).astype(np.float32)
    codes2, scales2 = oracle.quantize(W2, bits, group)
    np.testing.assert_array_equal(codes2, codes)
    ulp = np.abs(np.spacing(scales))
    assert np.all(np.abs(scales2.astype(np.float64) - scales) <= ulp)


def test_exact_ties_round_to_even():
    # absmax 127 -> s = 1 exactly; every half-integer is an exact tie
    w = np.array([127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -126.5, 3.49999], np.float32)
    codes, scales = oracle.quantize(w[None, :], 8, 0)
    assert scales[0, 0] == 1.0
    np.testing.assert_array_equal(codes[0], [127, 0, 2, 2, 0, -2, -2, 126, -126, 3])
    # int4: absmax 7 -> s = 1
    w4 = np.array([7, 0.5, 1.5, 2.5, 3.5, -4.5, 5.5, -6.5] * 2, np.float32)
    c4, s4 = oracle.quantize(w4[None, :], 4, 16)
    assert s4[0, 0] == 1.0
    np.testing.assert_array_equal(c4[0], [7, 0, 2, 2, 4, -4, 6, -6] * 2)


def test_zero_group_and_nonfinite():
    W = np.zeros((2, 64), np.float32)
    W[1, :16] = 1.0
    codes, scales = oracle.quantize(W, 4, 16)
    np.testing.assert_array_equal(scales[0], 0)
    np.testing.assert_array_equal(scales[1, 1:], 0)
    np.testing.assert_array_equal(codes[0], 0)
    for bad in (np.nan, np.inf, -np.inf):
        W2 = W.copy()
        W2[1, 3] = bad
        with pytest.raises(oracle.OracleError):
            oracle.quantize(W2, 8, 0)


def test_dequantize_within_half_step():
    W = wi.weight(9, 1, 33, 128)
    codes, scales = oracle.quantize(W, 4, 64)
    deq = oracle.dequantize(codes, scales, 64)
    s = np.repeat(scales.astype(np.float64), 64, axis=1)
    assert np.all(np.abs(deq - W) <= s / 2)
    assert np.all(deq / np.where(s == 0, 1, s) == codes)


# --------------------------------------------------------------------------
# linear
# --------------------------------------------------------------------------

def test_linear_exact_rationals_tiny():
    g = np.random.default_rng(3)
    M, N, K, r = 2, 3, 8, 2
    x = wi.normal_bf16(g, (M, K), 1.0)
    W = wi.normal_f32(g, (N, K), 0.1)
    b = wi.normal_bf16(g, (N,), 0.1)
    L1 = wi.normal_bf16(g, (K, r), 0.5)
    L2 = wi.normal_bf16(g, (r, N), 0.5)
    codes, scales = oracle.quantize(W, 4, 4)
    y = oracle.linear(x, codes, scales, 4, b, L1, L2)
    X = [[Fraction(float(v)) for v in row] for row in wi.bf16_to_f32(x)]
    A = [[Fraction(float(v)) for v in row] for row in wi.bf16_to_f32(L1)]
    B = [[Fraction(float(v)) for v in row] for row in wi.bf16_to_f32(L2)]
    bb = [Fraction(float(v)) for v in wi.bf16_to_f32(b)]
    for m in range(M):
        T = [sum(X[m][k] * A[k][j] for k in range(K)) for j in range(r)]
        for n in range(N):
            exact = sum(X[m][k] * int(codes[n, k]) * Fraction(float(scales[n, k // 4]))
                        for k in range(K))
            exact += sum(T[j] * B[j][n] for j in range(r)) + bb[n]
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2**50) + Fraction(1, 2**60)


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
def test_linear_matches_numpy_matmul(bits, group):
    M, N, K = 9, 70, 256
    x = wi.activations(11, 1, M, K)
    W = wi.weight(11, 2, N, K, outlier_frac=0.02)
    b = wi.bias(11, 3, N)
    codes, scales = oracle.quantize(W, bits, group)
    y = oracle.linear(x, codes, scales, group, b)
    gs = K if group == 0 else group
    deq = codes.astype(np.float64) * np.repeat(scales.astype(np.float64), gs, axis=1)
    xf = wi.bf16_to_f32(x).astype(np.float64)
    ref = xf @ deq.T + wi.bf16_to_f32(b).astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12 * np.sqrt(np.mean(ref ** 2)))


def test_linear_int8_per_channel_is_row_scaled_integer_gemm():
    M, N, K = 5, 40, 512
    x = wi.activations(12, 1, M, K)
    W = wi.weight(12, 2, N, K)
    codes, scales = oracle.quantize(W, 8, 0)
    y = oracle.linear(x, codes, scales, 0)
    xq = wi.bf16_to_f32(x).astype(np.float64) @ codes.astype(np.float64).T
    ref = xq * scales[:, 0].astype(np.float64)[None, :]
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-300)


def test_linear_low_rank_only_and_plain_only():
    M, N, K, r = 4, 48, 128, 32
    x = wi.activations(13, 1, M, K)
    L1 = wi.normal_bf16(wi.rng(13, 2), (K, r), 0.05)
    L2 = wi.normal_bf16(wi.rng(13, 3), (r, N), 0.05)
    zero_codes = np.zeros((N, K), np.int8)
    scales = np.ones((N, K // 64), np.float32)
    y = oracle.linear(x, zero_codes, scales, 64, None, L1, L2)
    xf = wi.bf16_to_f32(x).astype(np.float64)
    ref = (xf @ wi.bf16_to_f32(L1).astype(np.float64)) @ wi.bf16_to_f32(L2).astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12 * np.sqrt(np.mean(ref ** 2)))
    # zero low-rank factors reduce to the plain path
    W = wi.weight(13, 4, N, K)
    codes, sc = oracle.quantize(W, 4, 64)
    y1 = oracle.linear(x, codes, sc, 64, None, np.zeros_like(L1), np.zeros_like(L2))
    y0 = oracle.linear(x, codes, sc, 64)
    np.testing.assert_array_equal(y1, y0)


def test_linear_scaled_identity():
    N = K = 64
    c = np.float32(0.37)
    W = np.eye(N, dtype=np.float32) * c
    codes, scales = oracle.quantize(W, 8, 0)
    np.testing.assert_array_equal(codes, np.eye(N, dtype=np.int8) * 127)
    s = np.float32(np.float64(c) / 127)
    assert np.all(scales == s)
    x = wi.activations(14, 1, 3, K)
    b = wi.bias(14, 2, N)
    y = oracle.linear(x, codes, scales, 0, b)
    ref = wi.bf16_to_f32(x).astype(np.float64) * (127 * np.float64(s)) + wi.bf16_to_f32(b)
    np.testing.assert_allclose(y, ref, rtol=1e-15, atol=0)


def test_linear_gemv_and_empty():
    x = wi.activations(15, 1, 1, 128)
    W = wi.weight(15, 2, 30, 128)
    codes, scales = oracle.quantize(W, 4, 16)
    y = oracle.linear(x, codes, scales, 16)
    deq = oracle.dequantize(codes, scales, 16)
    ref = wi.bf16_to_f32(x).astype(np.float64)[0] @ deq.T
    np.testing.assert_allclose(y[0], ref, rtol=0, atol=1e-13)
    y0 = oracle.linear(x[:0], codes, scales, 16)
    assert y0.shape == (0, 30)
