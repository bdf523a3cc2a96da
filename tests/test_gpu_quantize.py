"""GPU quantization and packing against the oracle: codes and fp32 scales
bit-exact on the weights of all five workloads and on edge cases; pack/unpack
round trip; device-side error reporting."""
import numpy as np
import pytest
import torch

import oracle
import wlq_inputs as wi
from tests.gpu_helpers import assert_codes_equal, dev_f32, quantize_both

pytestmark = pytest.mark.gpu


def wlq():
    import weight_only_quantized_rtn_b200 as m
    return m


def _workload_weights():
    yield "tiny", wi.tiny_w8()["W"], 8, 0
    yield "attn", wi.attn_w8(1)["W"], 8, 0
    yield "mlp_up", wi.mlp_w4(1, "up")["W"], 4, 64
    yield "mlp_down", wi.mlp_w4(1, "down")["W"], 4, 64
    blk = wi.mixed_block(1)
    for name, layer in blk["layers"].items():
        yield "mixed_" + name, layer["W"], layer["bits"], layer["group"]
    yield "svdq_residual", wi.svdq_w4_lr(1)["W"], 4, 64


@pytest.mark.parametrize("case", list(range(11)))
def test_quantize_bit_exact_on_workload_weights(case):
    name, W, bits, group = list(_workload_weights())[case]
    cg, sg, co, so = quantize_both(W, bits, group)
    assert_codes_equal(cg, sg, co, so)


@pytest.mark.parametrize("case", list(range(11)))
def test_quantize_pack_bit_exact_on_workload_weights(case):
    """The fused quantize-pack pass (the benchmark's first launch) against the
    oracle on every workload weight: unpacked codes and fp32 scales bit-exact."""
    name, W, bits, group = list(_workload_weights())[case]
    m = wlq()
    s_f, p_f = m.quantize_pack(dev_f32(W), bits, group)
    m.check_status()
    co, so = oracle.quantize(W, bits, group)
    assert_codes_equal(m.unpack(p_f, W.shape[0], W.shape[1], bits, group), s_f, co, so)


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16), (8, 64), (4, 0), (8, 16), (4, 32), (4, 128)])
def test_quantize_edge_cases(bits, group):
    g = np.random.default_rng(99)
    K = 384
    W = (g.standard_normal((37, K)) * 0.02).astype(np.float32)
    W[0] = 0.0                                            # all-zero row
    W[1] = g.integers(-9, 10, K).astype(np.float32) * 0.5  # many exact halves (ties)
    W[1, ::16] = 7.0 if bits == 4 else 127.0               # absmax sets s = 1
    W[2] *= 1e-38                                         # tiny / subnormal range
    W[3] *= 1e36                                          # huge
    W[4, 5] = -50.0                                       # a single outlier, negative
    W[5, :] = 3.0                                         # constant row
    cg, sg, co, so = quantize_both(W, bits, group)
    assert_codes_equal(cg, sg, co, so)


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
def test_quantize_quotients_near_half_integers(bits, group):
    """Weights at (k + 1/2 + d) * s for small d, on both sides of the tie and on
    it: the estimate W * (1/s) may round either way there, so the exact
    residual decides (both the fast and the corrected branch run)."""
    g = np.random.default_rng(123 + bits + group)
    qmax = 127 if bits == 8 else 7
    N, K = 64, 256
    gsz = K if group == 0 else group
    W = np.zeros((N, K), dtype=np.float32)
    deltas = np.array([0.0, 2.0**-12, -2.0**-12, 2.0**-14, -2.0**-14, 2.0**-17, -2.0**-17, 2.0**-21, -2.0**-21, 1e-3])
    for n in range(N):
        for g0 in range(0, K, gsz):
            a = np.float32(g.uniform(0.01, 3.0))
            s = np.float32(a / np.float32(qmax))  # the group's fp32 scale (division correctly rounded)
            k = g.integers(-qmax, qmax, gsz)
            d = deltas[g.integers(0, len(deltas), gsz)]
            w = ((k + 0.5 + d) * np.float64(s)).astype(np.float32)
            w = np.clip(w, -a, a)
            w[0] = a  # the group's absmax
            W[n, g0:g0 + gsz] = w
    cg, sg, co, so = quantize_both(W, bits, group)
    assert_codes_equal(cg, sg, co, so)


def test_quantize_ragged_and_single_row():
    for N, K in [(1, 8), (3, 24), (129, 1000), (257, 4104)]:
        W = wi.weight(21, N, N, K)
        for bits, group in [(8, 0), (4, 0)]:
            cg, sg, co, so = quantize_both(W, bits, group)
            assert_codes_equal(cg, sg, co, so)


def test_nonfinite_weight_is_reported():
    m = wlq()
    W = wi.weight(22, 1, 64, 128)
    W[7, 3] = np.nan
    m.quantize(dev_f32(W), 8, 0)
    assert m.get_status() == m.ERR_NONFINITE
    assert m.get_status() == m.OK  # the word is cleared once read
    W[7, 3] = np.inf
    m.quantize(dev_f32(W), 4, 16)
    assert m.get_status() == m.ERR_NONFINITE
    W[7, 3] = 0.0
    m.quantize(dev_f32(W), 4, 16)
    assert m.get_status() == m.OK


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
@pytest.mark.parametrize("N,K", [(128, 64), (300, 320), (1, 64), (257, 4160)])
def test_pack_unpack_roundtrip(bits, group, N, K):
    m = wlq()
    W = wi.weight(23, N + K, N, K, outlier_frac=0.02)
    codes, scales = m.quantize(dev_f32(W), bits, group)
    packed = m.pack(codes, scales, bits, group)
    assert packed.numel() == m.packed_bytes(N, K, bits, group)
    back = m.unpack(packed, N, K, bits, group)
    assert torch.equal(back, codes)


def test_wait_probe_times_out_and_device_stays_usable():
    m = wlq()
    m.probe_wait_timeout(2_000_000)  # 2 ms on a barrier nothing arrives at
    assert m.get_status() == m.ERR_TIMEOUT
    assert m.get_status() == m.OK
    W = wi.weight(24, 1, 16, 64)
    cg, sg, co, so = quantize_both(W, 8, 0)
    assert_codes_equal(cg, sg, co, so)


def _pack_reference(W, bits, group):
    """quantize then pack, the two-kernel path, on the device."""
    m = wlq()
    codes, scales = m.quantize(dev_f32(W), bits, group)
    return scales, m.pack(codes, scales, bits, group)


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
@pytest.mark.parametrize("N,K", [(37, 384), (300, 448), (129, 2112), (1, 64), (256, 4096), (70, 12288)])
def test_quantize_pack_equals_quantize_then_pack(bits, group, N, K):
    """The fused pass writes the same packed bytes and scales as quantize
    followed by pack, on edge-case rows (zero, ties, subnormal, huge, a lone
    outlier, constant) and ragged N; ragged K for the recipes that allow it."""
    g = np.random.default_rng(7 * N + K + bits)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    if N > 6:
        W[0] = 0.0
        W[1] = g.integers(-9, 10, K).astype(np.float32) * 0.5
        W[2] *= 1e-38
        W[3] *= 1e36
        W[4, 5] = -50.0
        W[5, :] = 3.0
    m = wlq()
    s_ref, p_ref = _pack_reference(W, bits, group)
    s_f, p_f = m.quantize_pack(dev_f32(W), bits, group)
    torch.cuda.synchronize()
    m.check_status()
    assert torch.equal(s_f, s_ref)
    assert p_f.numel() == p_ref.numel()
    assert torch.equal(p_f, p_ref)
    # and against the oracle directly: the packed codes and the scales
    co, so = oracle.quantize(W, bits, group)
    assert_codes_equal(m.unpack(p_f, N, K, bits, group), s_f, co, so)


@pytest.mark.parametrize("bits,group,K", [(8, 0, 200), (8, 0, 4040), (4, 16, 1232)])
def test_quantize_pack_ragged_k(bits, group, K):
    """K not a multiple of 64: the last tile's inputs beyond K are code 0 (and
    their int4 group scales 0), as pack writes them."""
    g = np.random.default_rng(K)
    W = (g.standard_normal((150, K)) * 0.05).astype(np.float32)
    m = wlq()
    s_ref, p_ref = _pack_reference(W, bits, group)
    s_f, p_f = m.quantize_pack(dev_f32(W), bits, group)
    torch.cuda.synchronize()
    assert torch.equal(s_f, s_ref)
    assert torch.equal(p_f, p_ref)
    co, so = oracle.quantize(W, bits, group)
    assert_codes_equal(m.unpack(p_f, W.shape[0], K, bits, group), s_f, co, so)


@pytest.mark.parametrize("bits,group", [(8, 0), (4, 64), (4, 16)])
def test_quantize_pack_nonfinite_flags_and_zeroes(bits, group):
    """A NaN or infinity sets the non-finite error bit; its group (row) gets
    scale 0 and codes 0, exactly as the two-kernel path."""
    g = np.random.default_rng(5)
    W = (g.standard_normal((140, 256)) * 0.02).astype(np.float32)
    W[3, 17] = np.nan
    W[130, 200] = np.inf
    m = wlq()
    m.check_status()
    s_f, p_f = m.quantize_pack(dev_f32(W), bits, group)
    torch.cuda.synchronize()
    assert m.get_status() == m.ERR_NONFINITE
    s_ref, p_ref = _pack_reference(W, bits, group)
    assert m.get_status() == m.ERR_NONFINITE  # the two-kernel path flags it too (and clears the word)
    assert torch.equal(s_f, s_ref)
    assert torch.equal(p_f, p_ref)
