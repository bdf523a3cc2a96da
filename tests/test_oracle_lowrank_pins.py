"""Pins of the oracle's low-rank split (top-r SVD of W before quantizing the
residual), against constructions whose answer is known without an SVD:
orthogonal factors from QR with chosen singular values, exact low rank, and
bf16 storage checked through torch's own conversion."""
import numpy as np
import pytest
import torch

import oracle


def _orthonormal(g, n, k):
    q, r = np.linalg.qr(g.standard_normal((n, k)))
    return q * np.sign(np.diag(r))[None, :]


@pytest.mark.parametrize("N,K,r", [(96, 64, 8), (64, 128, 16), (40, 40, 1)])
def test_known_singular_values_give_the_eckart_young_split(N, K, r):
    g = np.random.default_rng(N + K + r)
    k = min(N, K)
    d = np.sort(g.uniform(0.1, 10.0, k))[::-1]           # distinct, descending
    P, Q = _orthonormal(g, K, k), _orthonormal(g, N, k)  # W^T = P diag(d) Q^T
    W = (P * d[None, :]) @ Q.T
    W = W.T                                              # [N, K]
    out = oracle.lowrank_split(W, r)
    np.testing.assert_allclose(out["sigma"], d, rtol=1e-12, atol=1e-12)
    best = (P[:, :r] * d[None, :r]) @ Q[:, :r].T         # the unique best rank-r part of W^T
    np.testing.assert_allclose(out["L1"] @ out["L2"], best, rtol=0, atol=1e-10 * d[0])
    resid = np.linalg.norm(W.T - out["L1"] @ out["L2"])
    assert resid == pytest.approx(np.sqrt(np.sum(d[r:] ** 2)), rel=1e-10)


def test_factors_split_the_singular_values_evenly():
    g = np.random.default_rng(2)
    W = g.standard_normal((80, 48))
    out = oracle.lowrank_split(W, 6)
    s = out["sigma"][:6]
    np.testing.assert_allclose(out["L1"].T @ out["L1"], np.diag(s), atol=1e-10 * s[0])
    np.testing.assert_allclose(out["L2"] @ out["L2"].T, np.diag(s), atol=1e-10 * s[0])


def test_exact_low_rank_leaves_only_the_bf16_storage_error():
    g = np.random.default_rng(4)
    A, B = g.standard_normal((64, 4)), g.standard_normal((4, 96))
    W = (A @ B).astype(np.float32)                       # rank 4
    out = oracle.lowrank_split(W, 4)
    assert out["sigma"][4] < 2.0 ** -20 * out["sigma"][0]  # rank 4 up to the fp32 rounding of W
    # the residual is what bf16 rounding of the factors left: well under bf16's 2^-8 relative
    assert np.linalg.norm(out["R"]) < 2.0 ** -7 * np.linalg.norm(W)
    np.testing.assert_allclose(out["R"], W - (oracle._bf16_value(out["L1_bits"]) @
                                              oracle._bf16_value(out["L2_bits"])).T, atol=1e-6)


def test_bf16_storage_is_round_to_nearest_even():
    g = np.random.default_rng(6)
    x = g.standard_normal(4000) * np.exp(g.uniform(-20, 20, 4000))
    x = np.concatenate([x, [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 2.0 ** -130]])
    bits = oracle._bf16_rne_bits(x)
    # torch rounds fp32 to bf16 to nearest even; these values are exact in fp32
    # only where they have <= 24 bits, so compare on fp32-representable inputs
    x32 = x.astype(np.float32)
    exact = x32.astype(np.float64) == x
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits[exact], ref[exact])


def test_bf16_rounding_of_fp64_values_is_nearest_with_ties_to_even():
    """fp64 values that fp32 cannot hold (where rounding through fp32 first
    could differ): the chosen bf16 is at least as near as both neighbours,
    and an exact midpoint goes to the even significand."""
    g = np.random.default_rng(8)
    x = g.standard_normal(20000) * np.exp(g.uniform(-30, 30, 20000))
    # exact midpoints between bf16 neighbours, and values just off them
    base = (g.integers(128, 256, 2000) * 2.0 ** g.integers(-20, 20, 2000)).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(base)) - 7)
    mids = base + ulp / 2
    x = np.concatenate([x, mids, -mids, mids + ulp * 2.0 ** -30, mids - ulp * 2.0 ** -30])
    bits = oracle._bf16_rne_bits(x)
    v = oracle._bf16_value(bits)
    up = oracle._bf16_value((bits.astype(np.int64) + 1).astype(np.uint16))
    dn = oracle._bf16_value((bits.astype(np.int64) - 1).astype(np.uint16))
    d0, d1, d2 = np.abs(x - v), np.abs(x - up), np.abs(x - dn)
    assert np.all(d0 <= d1) and np.all(d0 <= d2)
    tie = (d0 == d1) | (d0 == d2)
    assert tie.sum() >= 4000
    assert np.all(bits[tie] % 2 == 0)
    assert np.all(np.sign(v[x != 0]) == np.sign(x[x != 0]))


def _bf16_of(x):
    return oracle._bf16_rne_bits(np.asarray(x, np.float64))


def test_residual_with_zero_factors_is_w():
    g = np.random.default_rng(11)
    W = g.standard_normal((37, 24)).astype(np.float32)
    R = oracle.lowrank_residual(W, np.zeros((24, 8), np.uint16), np.zeros((8, 37), np.uint16))
    np.testing.assert_array_equal(R, W)


def test_residual_equals_fp64_matmul_when_every_sum_is_exact():
    """Small-integer factors and weights: every product and partial sum is an
    exact integer, so the result must equal numpy's fp64 matmul bit for bit,
    whatever order it sums in.  N != K != r, so a transposed or swapped index
    changes the answer."""
    g = np.random.default_rng(12)
    N, K, r = 23, 17, 5
    L1 = g.integers(-8, 9, (K, r)).astype(np.float64)
    L2 = g.integers(-8, 9, (r, N)).astype(np.float64)
    W = g.integers(-500, 501, (N, K)).astype(np.float32)
    R = oracle.lowrank_residual(W, _bf16_of(L1), _bf16_of(L2))
    np.testing.assert_array_equal(R, (W.astype(np.float64) - (L1 @ L2).T).astype(np.float32))


def test_residual_rounds_once_to_fp32():
    """W - p with p exact in fp64 but W - p not representable in fp32: one
    rounding of the exact difference (not of an fp32 product)."""
    W = np.array([[1.0]], np.float32)
    L1 = _bf16_of([[2.0 ** -30]])
    L2 = _bf16_of([[1.0 + 2.0 ** -7]])
    R = oracle.lowrank_residual(W, L1, L2)
    exact = 1.0 - 2.0 ** -30 * (1.0 + 2.0 ** -7)
    assert R[0, 0] == np.float32(exact)
    assert R[0, 0] == np.float32(1.0)  # the difference is far below fp32's half ulp of 1


def test_split_residual_is_the_split_formula():
    g = np.random.default_rng(13)
    W = g.standard_normal((40, 30)).astype(np.float32)
    out = oracle.lowrank_split(W, 6)
    R = oracle.lowrank_residual(W, out["L1_bits"], out["L2_bits"])
    np.testing.assert_allclose(R, out["R"], rtol=0, atol=1e-6)
