"""GPU RTN at other widths / inputs / scale formats and fp8 e4m3 block
quantization against the oracle: codes and stored scales bit-exact; the
int8 KV-cache shape (one group per token and head) timed."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import dev_f32

pytestmark = pytest.mark.gpu


def wlq():
    import weight_only_quantized_rtn_b200 as m
    return m


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF).astype(np.uint16)


def _dev(W: np.ndarray, bf16: bool) -> torch.Tensor:
    if bf16:
        return torch.from_numpy(_bf16_bits(W).view(np.int16)).cuda().view(torch.bfloat16)
    return dev_f32(W)


def _host_in(W: np.ndarray, bf16: bool) -> np.ndarray:
    return _bf16_bits(W) if bf16 else W


def _edge_weights(seed, N, K):
    g = np.random.default_rng(seed)
    W = (g.standard_normal((N, K)) * np.exp(g.uniform(-4, 4, (N, 1)))).astype(np.float32)
    W[0] = 0.0                                            # all-zero row
    W[1] = g.integers(-9, 10, K).astype(np.float32) * 0.5  # many halves
    W[2] *= 1e-36                                         # tiny
    W[3, 7] = -40.0                                       # a lone outlier
    W[4] = 3.0                                            # constant
    return W


@pytest.mark.parametrize("bits", [2, 3, 5, 8])
@pytest.mark.parametrize("group", [0, 16, 128])
@pytest.mark.parametrize("scale_dtype", [0, 1, 2])
@pytest.mark.parametrize("bf16", [False, True])
def test_quantize_ex_bit_exact(bits, group, scale_dtype, bf16):
    m = wlq()
    W = _edge_weights(bits * 31 + group + scale_dtype, 37, 384)
    if scale_dtype == 1:
        W[2] = 0.001  # keep fp16 scales inside their range (the tiny row would be 0 there anyway)
    co, so = oracle.quantize_ex(_host_in(W, bf16), bits, group, scale_dtype)
    cg, sg = m.quantize_ex(_dev(W, bf16), bits, group, scale_dtype)
    torch.cuda.synchronize()
    m.check_status()
    np.testing.assert_array_equal(cg.cpu().numpy(), co)
    np.testing.assert_array_equal(sg.float().cpu().numpy(), so)


def test_quantize_ex_eight_bit_fp32_equals_quantize():
    m = wlq()
    W = _edge_weights(3, 64, 512)
    for group, bits in ((0, 8), (64, 4), (16, 4)):
        c0, s0 = m.quantize(dev_f32(W), bits, group)
        c1, s1 = m.quantize_ex(dev_f32(W), bits, group, 0)
        torch.cuda.synchronize()
        assert torch.equal(c0, c1) and torch.equal(s0, s1)


def test_quantize_ex_nonfinite_and_fp16_overflow_flag():
    m = wlq()
    m.check_status()
    W = (np.random.default_rng(1).standard_normal((8, 64)) * 0.1).astype(np.float32)
    W[2, 3] = np.nan
    c, s = m.quantize_ex(dev_f32(W), 8, 32, 0)
    assert m.get_status() == m.ERR_NONFINITE
    assert float(s[2, 0]) == 0.0 and not c[2, :32].any()
    W[2, 3] = 0.0
    W[5, 40] = 1e7  # 1e7 / 127 overflows fp16
    c, s = m.quantize_ex(dev_f32(W), 8, 32, 1)
    assert m.get_status() == m.ERR_NONFINITE
    assert float(s[5, 1]) == 0.0 and not c[5, 32:].any()
    c, s = m.quantize_ex(dev_f32(W), 8, 32, 2)  # bf16 holds it
    assert m.get_status() == m.OK


@pytest.mark.parametrize("group", [0, 32, 128])
@pytest.mark.parametrize("bf16", [False, True])
def test_quantize_fp8_bit_exact(group, bf16):
    m = wlq()
    W = _edge_weights(77 + group, 41, 512)
    co, so = oracle.quantize_fp8(_host_in(W, bf16), group)
    cg, sg = m.quantize_fp8(_dev(W, bf16), group)
    torch.cuda.synchronize()
    m.check_status()
    np.testing.assert_array_equal(sg.cpu().numpy(), so)
    np.testing.assert_array_equal(cg.cpu().numpy(), co)


def test_kv_cache_int8_per_token_head_timed():
    """K/V of 4096 tokens x 32 heads x head_dim 128 in bf16, one int8 scale
    group per (token, head), fp16 scales: bit-exact on a slice, and timed
    (HBM-bound: 2 B read + 1 B + 2/128 B written per element)."""
    m = wlq()
    T, H, D = 4096, 32, 128
    g = np.random.default_rng(12)
    kv = (g.standard_normal((T * H, D)) * 0.5).astype(np.float32)
    x = _dev(kv, True)
    codes, scales = m.quantize_ex(x, 8, D, 1)
    torch.cuda.synchronize()
    co, so = oracle.quantize_ex(_bf16_bits(kv[:2048]), 8, D, 1)
    np.testing.assert_array_equal(codes[:2048].cpu().numpy(), co)
    np.testing.assert_array_equal(scales[:2048].float().cpu().numpy(), so)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ts = []
    for _ in range(10):
        flush.zero_()
        flush.view(torch.float32).sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        m.quantize_ex(x, 8, D, 1)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    us = sorted(ts)[len(ts) // 2]
    nbytes = T * H * D * (2 + 1) + T * H * 2
    print("\nKV int8 per (token, head): %d x %d x %d bf16 -> %.1f us, %.0f GB/s" % (T, H, D, us, nbytes / us / 1e3))


def _scale_edge_weights(scale_dtype, qmax, seed):
    """Groups of 16 whose absmax a makes a / qmax land exactly on, or one fp32
    step beside, the midpoint of two neighbouring 16-bit values (where rounding
    the fp32 quotient again would be wrong), plus, for fp16, absmaxes whose
    scale is subnormal in fp16 (where the scale can round far below a / qmax
    and the clamp to +-qmax acts)."""
    g = np.random.default_rng(seed)
    if scale_dtype == 1:
        lo = g.integers(0x1000, 0x5000, 200).astype(np.uint16)          # normal fp16 values
        v = lo.view(np.float16).astype(np.float64)
        nxt = (lo + 1).view(np.float16).astype(np.float64)
    else:
        lo = g.integers(0x3000, 0x4300, 200).astype(np.uint16)          # bf16 values
        v = (lo.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        nxt = ((lo.astype(np.uint32) + 1) << 16).view(np.float32).astype(np.float64)
    mids = (v + nxt) / 2                                                 # exact in fp64
    a0 = (mids * qmax).astype(np.float32)                                # exact: <= 19 significant bits
    a = np.concatenate([a0, np.nextafter(a0, np.float32(np.inf)), np.nextafter(a0, np.float32(0))])
    if scale_dtype == 1:
        sub = (g.integers(1, 1024, 150) * 2.0 ** -24 * qmax * g.uniform(0.9, 1.1, 150)).astype(np.float32)
        a = np.concatenate([a, sub])
    a = a[np.isfinite(a) & (a > 0)]
    a = a[: len(a) // 4 * 4]  # four groups of 16 per row of 64
    G = len(a)
    W = (g.uniform(-1, 1, (G, 16)) * a[:, None]).astype(np.float32)
    W[np.arange(G), g.integers(0, 16, G)] = a * np.where(g.random(G) < 0.5, -1, 1)
    return W.reshape(-1, 64)


@pytest.mark.parametrize("bits", [2, 4, 5, 8])
@pytest.mark.parametrize("scale_dtype", [1, 2])
def test_quantize_ex_scale_midpoints_and_subnormal_scales(bits, scale_dtype):
    m = wlq()
    qmax = (1 << (bits - 1)) - 1
    W = _scale_edge_weights(scale_dtype, qmax, 17 * bits + scale_dtype)
    co, so = oracle.quantize_ex(W, bits, 16, scale_dtype)
    cg, sg = m.quantize_ex(dev_f32(W), bits, 16, scale_dtype)
    torch.cuda.synchronize()
    m.check_status()
    np.testing.assert_array_equal(sg.float().cpu().numpy(), so)
    np.testing.assert_array_equal(cg.cpu().numpy(), co)


@pytest.mark.parametrize("group,N,K", [(8, 29, 1024), (16, 29, 1024), (32, 29, 1024), (64, 29, 1024),
                                       (256, 29, 1024), (512, 29, 1024), (16, 7, 80), (128, 5, 384)])
@pytest.mark.parametrize("bits,scale_dtype", [(8, 1), (4, 0), (5, 2)])
def test_quantize_ex_bf16_power_of_two_groups_bit_exact(group, N, K, bits, scale_dtype):
    """bf16 input with groups of 8..512 (8 or 16 inputs a lane, groups across
    1..32 lanes, a last warp-round only partly filled) against the oracle."""
    m = wlq()
    W = _edge_weights(group + bits + scale_dtype, N, K)
    if scale_dtype == 1:
        W[2] = 0.001
    co, so = oracle.quantize_ex(_host_in(W, True), bits, group, scale_dtype)
    cg, sg = m.quantize_ex(_dev(W, True), bits, group, scale_dtype)
    torch.cuda.synchronize()
    m.check_status()
    np.testing.assert_array_equal(cg.cpu().numpy(), co)
    np.testing.assert_array_equal(sg.float().cpu().numpy(), so)


def test_quantize_ex_bf16_nonfinite_group_and_unaligned_codes():
    """A NaN zeroes its group and raises the flag; codes that are only 8-byte
    aligned (8 inputs a lane) or 4-byte aligned (the general path) give the
    same bytes."""
    m = wlq()
    m.check_status()
    W = (np.random.default_rng(5).standard_normal((16, 256)) * 0.3).astype(np.float32)
    W[3, 70] = np.nan
    x = _dev(W, True)
    c, s = m.quantize_ex(x, 8, 64, 1)
    assert m.get_status() == m.ERR_NONFINITE
    assert float(s[3, 1]) == 0.0 and not c[3, 64:128].any()
    W[3, 70] = 0.25
    x = _dev(W, True)
    c, s = m.quantize_ex(x, 8, 64, 1)
    m.check_status()
    buf = torch.empty(16 * 256 + 16, dtype=torch.int8, device="cuda")
    for off in (4, 8):
        c_mis = buf[off:off + 16 * 256].view(16, 256)
        s2 = torch.empty_like(s)
        m.lib.wlq_quantize_ex(m._ptr(x), 1, 16, 256, 8, 64, 1, m._ptr(c_mis), m._ptr(s2), m._stream())
        m.check_status()
        assert torch.equal(c, c_mis) and torch.equal(s, s2)
