"""Pins for the oracle's NVFP4 quantizer and W4A4 Linear ("Nunchaku Lite"
article: the svdq_w4a4 kernels, NVFP4 variant on Blackwell; section "why it
matters": 4-bit weights and activations plus a 16-bit low-rank correction).

Nothing here re-uses the oracle's arithmetic: E2M1 values are decoded from
the bit fields (sign, 2 exponent bits, 1 mantissa bit), E4M3 values through
torch's float8_e4m3fn type, nearest codes found by enumerating every code,
and the Linear reduced to numpy matmuls of independently decoded values.
"""
import numpy as np
import pytest
import torch

import oracle


def e2m1_value(code):
    """The 16 E2M1 codes from their fields: exponent bits e, mantissa bit m;
    e = 0 is subnormal (m * 0.5), else (1 + m / 2) * 2^(e - 1)."""
    code = np.asarray(code, np.int64)
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.ldexp(1.0, e - 1))
    return np.where(s == 1, -mag, mag)


def e4m3_value(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


ALL_E2M1 = e2m1_value(np.arange(16))
POS_E4M3_BITS = np.arange(0, 127, dtype=np.uint8)          # 0x7f is NaN
POS_E4M3 = e4m3_value(POS_E4M3_BITS)


def nearest_e2m1(t):
    """Brute force: the magnitude code nearest |t| (ties: even mantissa bit;
    above 6: 6), sign bit from t."""
    out = np.empty(np.shape(t), np.uint8)
    for i, v in np.ndenumerate(np.asarray(t, np.float64)):
        a = abs(v)
        dist = np.abs(ALL_E2M1[:8] - a)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:
            best = [b for b in best if (b & 1) == 0]
        out[i] = best[0] | (8 if np.signbit(v) else 0)
    return out


def nearest_e4m3(t):
    """Brute force over the 127 non-negative E4M3 values; ties to an even
    mantissa bit; above 448: 448."""
    dist = np.abs(POS_E4M3 - t)
    best = np.flatnonzero(dist == dist.min())
    if len(best) > 1:
        best = [b for b in best if (POS_E4M3_BITS[b] & 1) == 0]
    return np.uint8(POS_E4M3_BITS[best[0]])


def _tensor_with_unit_g(block):
    """Row 0: the block under test (16 values, |values| <= 6); row 1: one
    value 2688 (so amax = 2688 and g = 1 exactly)."""
    X = np.zeros((2, 16), np.float32)
    X[0] = block
    X[1, 0] = 2688.0
    return X


def test_every_e2m1_code_and_midpoint_with_unit_scales():
    """g = 1 and s_b = 1 (block amax 6): every code's value must come back as
    itself, every midpoint must go to the even neighbour, and points just
    either side of each midpoint to the nearer neighbour."""
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mids = (mags[:-1] + mags[1:]) / 2
    vals = np.concatenate([mags, -mags, mids, -mids,
                           np.nextafter(mids.astype(np.float32), np.float32(0)),
                           np.nextafter(mids.astype(np.float32), np.float32(7)),
                           [6.0, 6.0001, -5.99, 0.1, -0.1, 6.0]])
    for i in range(0, len(vals), 15):
        blk = np.zeros(16, np.float32)
        chunk = vals[i:i + 15]
        blk[:len(chunk)] = chunk
        blk[15] = 6.0                                       # block amax 6 -> s_b = 1
        X = _tensor_with_unit_g(blk)
        codes, scales, g = oracle.nvfp4_quantize(X)
        assert g == 1.0
        assert scales[0, 0] == 0x38                           # E4M3 1.0
        want = nearest_e2m1(blk.astype(np.float64))
        np.testing.assert_array_equal(codes[0], want)


def test_e2m1_code_table_values_round_trip():
    """All 16 codes decode to the values the fields define, and each value
    (times a block scale) quantizes back to its own code (-0 to 8)."""
    for s_bits in (0x38, 0x30, 0x45, 0x01, 0x7e):
        s = float(e4m3_value(np.array([s_bits], np.uint8))[0])
        blk = (ALL_E2M1 * s).astype(np.float32)
        X = np.zeros((2, 16), np.float32)
        X[0] = blk
        X[1, 0] = 2688.0
        if 6 * s <= 2688:
            codes, scales, g = oracle.nvfp4_quantize(X)
            assert scales[0, 0] == s_bits
            back = e2m1_value(codes[0]) * s
            np.testing.assert_array_equal(back, blk.astype(np.float64))


def test_block_scales_are_the_nearest_e4m3_with_ties_to_even():
    g_rng = np.random.default_rng(11)
    rows, K = 48, 64
    X = (g_rng.standard_normal((rows, K)) * np.exp(g_rng.uniform(-6, 4, (rows, 1)))).astype(np.float32)
    X[0, 0] = 2688.0                                         # g = 1
    # exact E4M3 midpoints (in units of 6 g): 1.0625 (between 1 and 1.125, even: 1),
    # 1.1875 (between 1.125 and 1.25, even: 1.25), 464 is above 448 (saturates)
    X[1, :16] = 0.0
    X[1, 3] = 6.0 * 1.0625
    X[2, :16] = 0.0
    X[2, 5] = -6.0 * 1.1875
    X[3, 16:32] = 0.0
    X[3, 20] = 6.0 * 0.001953125 * 1.5                     # 1.5 subnormal steps: between 1 and 2 -> 2
    codes, scales, g = oracle.nvfp4_quantize(X)
    assert g == np.float32(np.abs(X).max() / 2688.0)
    for r in range(rows):
        for b in range(K // 16):
            a = np.abs(X[r, 16 * b:16 * b + 16].astype(np.float64)).max()
            assert scales[r, b] == nearest_e4m3(a / (6.0 * g)), (r, b)
    assert scales[1, 0] == 0x38 and scales[2, 0] == 0x3a and scales[3, 1] == 0x02


def test_codes_are_the_brute_force_nearest_for_random_tensors():
    g_rng = np.random.default_rng(12)
    for rows, K, spread in ((8, 128, 1.0), (5, 256, 8.0), (16, 32, 0.01)):
        X = (g_rng.standard_normal((rows, K)) * np.exp(spread * g_rng.standard_normal((rows, K)))).astype(np.float32)
        codes, scales, g = oracle.nvfp4_quantize(X)
        assert g == np.float32(np.abs(X).max() / 2688.0)
        d = e4m3_value(scales).repeat(16, axis=1) * g
        want = np.where(d > 0, nearest_e2m1(np.where(d > 0, X / np.where(d > 0, d, 1), 0.0)), 0)
        np.testing.assert_array_equal(codes, want)


def test_bf16_input_equals_the_same_values_in_fp32():
    g_rng = np.random.default_rng(13)
    X = g_rng.standard_normal((6, 96)).astype(np.float32)
    bits = (X.view(np.uint32) >> 16).astype(np.uint16)          # truncation gives exact bf16 values
    Xb = (bits.astype(np.uint32) << 16).view(np.float32)
    a = oracle.nvfp4_quantize(bits)
    b = oracle.nvfp4_quantize(Xb)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_power_of_two_and_sign_invariance():
    g_rng = np.random.default_rng(14)
    X = g_rng.standard_normal((7, 64)).astype(np.float32)
    c0, s0, g0 = oracle.nvfp4_quantize(X)
    for k in (-20, -3, 5, 30):
        c, s, g = oracle.nvfp4_quantize(np.ldexp(X, k).astype(np.float32))
        np.testing.assert_array_equal(c, c0)
        np.testing.assert_array_equal(s, s0)
        assert g == np.ldexp(np.float32(g0), k)
    c, s, g = oracle.nvfp4_quantize(-X)
    np.testing.assert_array_equal(c, c0 ^ 8)
    np.testing.assert_array_equal(s, s0)


def test_zero_tensor_zero_block_and_reconstruction_bound():
    c, s, g = oracle.nvfp4_quantize(np.zeros((3, 32), np.float32))
    assert g == 0.0 and not s.any() and not (c & 7).any()
    g_rng = np.random.default_rng(15)
    X = g_rng.standard_normal((9, 160)).astype(np.float32)
    X[4, 32:48] = 0.0
    X[5, 64:80] = 1e-30                                       # block scale underflows to 0
    c, s, g = oracle.nvfp4_quantize(X)
    assert s[4, 2] == 0 and not (c[4, 32:48] & 7).any()
    assert s[5, 4] == 0 and not (c[5, 64:80] & 7).any()
    xh = oracle.nvfp4_dequantize(c, s, g)
    d = e4m3_value(s).repeat(16, axis=1) * g
    # nearest-code error: at most half the spacing (1 above 4), saturation at
    # most 6 / (1 - 2^-4) - 6 = 0.4 in units of d
    assert np.all(np.abs(X - xh) <= d * 1.0 + (d == 0) * np.abs(X))


def test_dequantize_decodes_the_fields():
    g_rng = np.random.default_rng(16)
    c = g_rng.integers(0, 16, (5, 48)).astype(np.uint8)
    s = g_rng.integers(0, 127, (5, 3)).astype(np.uint8)
    g = np.float32(0.0173)
    out = oracle.nvfp4_dequantize(c, s, float(g))
    want = e2m1_value(c) * e4m3_value(s).repeat(16, axis=1) * np.float64(g)
    np.testing.assert_array_equal(out, want)


def _bf16(x):
    return oracle._bf16_rne_bits(x)


@pytest.mark.parametrize("r,bias", [(0, False), (0, True), (16, True), (8, False)])
def test_w4a4_linear_matches_numpy_matmul(r, bias):
    g_rng = np.random.default_rng(17 + r)
    M, N, K = 7, 24, 96
    x_bits = _bf16(g_rng.standard_normal((M, K)))
    W = g_rng.standard_normal((N, K)).astype(np.float32)
    xq, xs, xg = oracle.nvfp4_quantize(x_bits)
    wq, ws, wg = oracle.nvfp4_quantize(W)
    b = _bf16(g_rng.standard_normal(N)) if bias else None
    L1 = _bf16(0.1 * g_rng.standard_normal((K, r))) if r else None
    L2 = _bf16(0.1 * g_rng.standard_normal((r, N))) if r else None
    y = oracle.nvfp4_linear(xq, xs, xg, x_bits, wq, ws, wg, b, L1, L2)
    xd = e2m1_value(xq) * e4m3_value(xs).repeat(16, axis=1) * np.float64(xg)
    wd = e2m1_value(wq) * e4m3_value(ws).repeat(16, axis=1) * np.float64(wg)
    want = xd @ wd.T
    if r:
        want = want + (oracle._bf16_value(x_bits) @ oracle._bf16_value(L1)) @ oracle._bf16_value(L2)
    if bias:
        want = want + oracle._bf16_value(b)[None, :]
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_w4a4_linear_exact_small_case():
    """Every product and partial sum exact: codes chosen so that the result is
    a small dyadic rational computed by hand.  x = [1, 0.5, ..] in block 0,
    w = [2, -3, ..]; scales 1 and g = 1."""
    K = 16
    xq = np.zeros((1, K), np.uint8)
    wq = np.zeros((2, K), np.uint8)
    xq[0, 0], xq[0, 1], xq[0, 15] = 2, 1, 15                   # 1, 0.5, -6
    wq[0, 0], wq[0, 1], wq[0, 15] = 4, 13, 7                    # 2, -3, 6
    wq[1, 1], wq[1, 15] = 6, 9                                  # 4, -0.5
    xs = np.full((1, 1), 0x38, np.uint8)                        # 1.0
    ws = np.array([[0x38], [0x40]], np.uint8)                   # 1.0, 2.0
    y = oracle.nvfp4_linear(xq, xs, 1.0, None, wq, ws, 1.0)
    # row 0: 1*2 + 0.5*(-3) + (-6)*6 = -35.5 ; row 1: (0.5*4 + (-6)(-0.5)) * 2 = 10
    np.testing.assert_array_equal(y, [[-35.5, 10.0]])
    y = oracle.nvfp4_linear(xq, xs, 0.25, None, wq, ws, 2.0)
    np.testing.assert_array_equal(y, [[-17.75, 5.0]])
