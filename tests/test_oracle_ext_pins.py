"""Pins of the oracle's wider quantizers (other bit widths, bf16 input, 16-bit
scales, fp8 e4m3 blocks), each checked against something other than the
oracle's own arithmetic: brute-force enumeration of the codes, the nearest
representable value found by stepping through the format's neighbours, a
library conversion (torch's float8_e4m3fn), and the already-pinned int8/int4
quantizer for the cases that coincide."""
import numpy as np
import pytest
import torch

import oracle


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (numpy only)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF
    return r.astype(np.uint16)


def _bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def _neighbours(v: float, fmt: int):
    """The representable values of the scale format around v (v itself one of them)."""
    if fmt == oracle.SCALE_F32:
        f = np.float32(v)
        return [float(np.nextafter(f, np.float32(-np.inf))), float(f), float(np.nextafter(f, np.float32(np.inf)))]
    if fmt == oracle.SCALE_F16:
        h = np.float16(v)
        return [float(np.nextafter(h, np.float16(-np.inf))), float(h), float(np.nextafter(h, np.float16(np.inf)))]
    b = int(_bf16_bits(np.array([v], np.float32))[0])
    out = []
    for bb in (b - 1, b, b + 1):
        if 0 <= bb < 0x7F80:
            out.append(float(_bf16_to_f32(np.array([bb], np.uint16))[0]))
    return out


def _is_nearest(s: float, exact: float, fmt: int) -> bool:
    """s is a value of the format, and one nearest to `exact` (any tie is
    accepted here)."""
    if fmt == oracle.SCALE_F16 and float(np.float16(s)) != s:
        return False
    if fmt == oracle.SCALE_BF16 and (np.array([s], np.float32).view(np.uint32)[0] & 0xFFFF):
        return False
    cands = _neighbours(s, fmt)
    return all(abs(s - exact) <= abs(c - exact) for c in cands)


def _brute_codes(w: np.ndarray, s: float, qmax: int) -> np.ndarray:
    """argmin over q in [-qmax, qmax] of |w - q s|, ties to even q (exact, via fractions of fp64 products)."""
    qs = np.arange(-qmax, qmax + 1, dtype=np.float64)
    out = np.empty(w.shape, np.int8)
    for i, x in enumerate(w.astype(np.float64)):
        if s == 0.0:
            out[i] = 0
            continue
        err = np.abs(x - qs * s)  # q*s exact in fp64 (q <= 127, s fp32); x - q*s exact enough to compare
        best = err.min()
        tied = qs[err == best]
        even = tied[np.mod(tied, 2) == 0]
        out[i] = int(even[0] if len(even) else tied[0])
    return out


@pytest.mark.parametrize("bits", [2, 3, 5, 6, 7, 8])
@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_F16, oracle.SCALE_BF16])
def test_codes_are_the_brute_force_nearest_with_the_stored_scale(bits, fmt):
    g = np.random.default_rng(bits * 7 + fmt)
    qmax = (1 << (bits - 1)) - 1
    W = (g.standard_normal((6, 32)) * np.exp(g.uniform(-3, 3, (6, 1)))).astype(np.float32)
    W[1, :8] = (g.integers(-qmax, qmax + 1, 8) + 0.5).astype(np.float32) * 0.25  # many exact halves
    codes, scales = oracle.quantize_ex(W, bits, 8, fmt)
    for n in range(6):
        for gi in range(4):
            w = W[n, gi * 8:(gi + 1) * 8]
            s = float(scales[n, gi])
            a = float(np.max(np.abs(w.astype(np.float64))))
            assert _is_nearest(s, a / qmax, fmt)
            np.testing.assert_array_equal(codes[n, gi * 8:(gi + 1) * 8], _brute_codes(w, s, qmax))


def test_sixteen_bit_scale_may_round_down_and_codes_clamp():
    """a / qmax just above an fp16 value rounds down: the absmax weight's
    quotient exceeds qmax + 1/2 is impossible, but exceeds qmax, so its code is
    the clamp qmax."""
    qmax = 127
    s16 = float(np.float16(0.0123))
    a = np.float32(s16 * qmax * (1 + 2.0 ** -12))  # a / qmax a hair above s16
    W = np.full((1, 8), 0.001, np.float32)
    W[0, 3] = a
    codes, scales = oracle.quantize_ex(W, 8, 0, oracle.SCALE_F16)
    assert float(scales[0, 0]) == s16
    assert a / s16 > qmax
    assert codes[0, 3] == qmax


@pytest.mark.parametrize("group", [16, 32, 128, 256, 512])
@pytest.mark.parametrize("bits,fmt", [(8, oracle.SCALE_F16), (4, oracle.SCALE_F32), (5, oracle.SCALE_BF16)])
def test_groups_are_independent_row_problems(group, bits, fmt):
    """Grouping is only a partition of each row: the codes and scales of
    group g equal those of its g-wide slice quantized as rows of their own
    (group 0), for bf16 input too; a group's scale follows its own maximum."""
    g = np.random.default_rng(group + 10 * bits + fmt)
    K = 1024
    W = (g.standard_normal((5, K)) * np.exp(g.uniform(-3, 3, (5, K // group))).repeat(group, 1)).astype(np.float32)
    W[2, group:2 * group] = 0.0  # one all-zero group
    for x in (W, _bf16_bits(W)):
        codes, scales = oracle.quantize_ex(x, bits, group, fmt)
        assert codes.shape == (5, K) and scales.shape == (5, K // group)
        for gi in range(K // group):
            sl = np.ascontiguousarray(x[:, gi * group:(gi + 1) * group])
            c1, s1 = oracle.quantize_ex(sl, bits, 0, fmt)
            np.testing.assert_array_equal(codes[:, gi * group:(gi + 1) * group], c1)
            np.testing.assert_array_equal(scales[:, gi], s1[:, 0])
    assert not codes[2, group:2 * group].any() and scales[2, 1] == 0.0


@pytest.mark.parametrize("bits,group", [(8, 0), (8, 64), (4, 64), (4, 16)])
def test_fp32_scales_reduce_to_the_int8_int4_quantizer(bits, group):
    g = np.random.default_rng(11 + bits + group)
    W = (g.standard_normal((9, 128)) * 0.05).astype(np.float32)
    c0, s0 = oracle.quantize(W, bits, group)
    c1, s1 = oracle.quantize_ex(W, bits, group, oracle.SCALE_F32)
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_array_equal(s0, s1)


@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_F16, oracle.SCALE_BF16])
def test_bf16_input_equals_its_fp32_values(fmt):
    g = np.random.default_rng(3)
    b = _bf16_bits((g.standard_normal((12, 128)) * 0.7).astype(np.float32))
    c_b, s_b = oracle.quantize_ex(b, 8, 128, fmt)
    c_f, s_f = oracle.quantize_ex(_bf16_to_f32(b), 8, 128, fmt)
    np.testing.assert_array_equal(c_b, c_f)
    np.testing.assert_array_equal(s_b, s_f)


def test_fp16_scale_overflow_is_rejected():
    W = np.full((1, 8), 1e7, np.float32)  # 1e7 / 127 > 65504
    with pytest.raises(oracle.OracleError):
        oracle.quantize_ex(W, 8, 0, oracle.SCALE_F16)


def _e4m3_value(c: int) -> float:
    sgn = -1.0 if c & 0x80 else 1.0
    e, m = (c >> 3) & 15, c & 7
    if e == 15 and m == 7:
        return float("nan")
    return sgn * (2.0 ** -6 * m / 8 if e == 0 else 2.0 ** (e - 7) * (1 + m / 8))


def test_fp8_codes_are_the_nearest_e4m3_ties_to_even_saturated():
    g = np.random.default_rng(5)
    W = (g.standard_normal((8, 64)) * np.exp(g.uniform(-6, 6, (8, 1)))).astype(np.float32)
    codes, scales = oracle.quantize_fp8(W, 16)
    vals = np.array([_e4m3_value(c) for c in range(256)])
    finite = ~np.isnan(vals)
    for n in range(8):
        for k in range(64):
            s = float(scales[n, k // 16])
            t = float(np.float32(np.float64(W[n, k]) / np.float64(s)))
            if abs(t) >= 448.0:
                assert _e4m3_value(int(codes[n, k])) == np.copysign(448.0, t)
                continue
            err = np.where(finite, np.abs(vals - t), np.inf)
            best = err.min()
            tied = [c for c in range(256) if err[c] == best and (np.signbit(vals[c]) == np.signbit(t) or vals[c] != 0)]
            even = [c for c in tied if (c & 1) == 0]
            assert int(codes[n, k]) in (even if even else tied)
        # the scale is fp32(a / 448)
        for gi in range(4):
            a = float(np.max(np.abs(W[n, gi * 16:(gi + 1) * 16].astype(np.float64))))
            assert float(scales[n, gi]) == float(np.float32(a / 448.0))


def test_fp8_codes_match_torch_e4m3fn_conversion():
    """Within range the code is torch's float8_e4m3fn of the fp32 quotient."""
    g = np.random.default_rng(9)
    W = (g.standard_normal((32, 256)) * np.exp(g.uniform(-8, 8, (32, 1)))).astype(np.float32)
    codes, scales = oracle.quantize_fp8(W, 32)
    t = (W.astype(np.float64) / np.repeat(scales, 32, axis=1).astype(np.float64)).astype(np.float32)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mask = np.abs(t) <= 448.0
    np.testing.assert_array_equal(codes[mask], ref[mask])


def test_fp8_all_zero_group_and_bf16_input():
    W = np.zeros((2, 32), np.float32)
    W[1, 5] = -3.0
    codes, scales = oracle.quantize_fp8(W, 16)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and not codes[0].any()
    assert codes[1, 5] == 0xFE  # -448: the group's absmax maps to the largest code
    b = _bf16_bits(np.random.default_rng(1).standard_normal((4, 64)).astype(np.float32))
    c_b, s_b = oracle.quantize_fp8(b, 32)
    c_f, s_f = oracle.quantize_fp8(_bf16_to_f32(b), 32)
    np.testing.assert_array_equal(c_b, c_f)
    np.testing.assert_array_equal(s_b, s_f)
