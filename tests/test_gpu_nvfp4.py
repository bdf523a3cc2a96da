"""NVFP4 quantizer and W4A4 Linear on the GPU against the oracle ("Nunchaku
Lite" article: svdq_w4a4, NVFP4 variant on Blackwell; section "why it
matters": 4-bit weights and activations plus a 16-bit low-rank branch).

Codes, block scales and the tensor scale are compared bit for bit (the GPU's
scale atoms are read back through the documented layout).  The Linear is
compared with the oracle's fp64 sum over the oracle's own codes: the tensor
cores multiply E2M1 x E2M1 x E4M3 x E4M3 exactly (at most 12 significant
bits) and accumulate in fp32, so with K <= 16384 the error stays far below
1e-3 * rms(y) for fp32 output; bf16 output adds the rounding of each value
(at most 2^-9 of it, bounded here by 2^-8 |y_ref|); the low-rank term's bf16
hi/lo split costs ~2^-16 relative.
"""
import numpy as np
import pytest
import torch

import oracle
import wlq_inputs as wi
from tests.gpu_helpers import dev_bf16, dev_f32, rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-3


def wlq():
    import weight_only_quantized_rtn_b200 as m
    return m


def unpack_codes(codes_dev, K):
    c = codes_dev.cpu().numpy()
    out = np.empty((c.shape[0], K), np.uint8)
    out[:, 0::2] = c & 15
    out[:, 1::2] = c >> 4
    return out


def unswizzle_scales(scales_dev, rows, K):
    """The 512-byte atom layout back to [rows, K / 16]."""
    s = scales_dev.cpu().numpy()
    KA = ((K + 255) // 256) * 4
    out = np.empty((rows, K // 16), np.uint8)
    r = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    off = ((r // 128) * KA + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)
    out[:, :] = s[off]
    return out


def check_quantize(X, bits_input=None):
    """X: fp32 array, or (when bits_input is given) bf16 bit patterns."""
    m = wlq()
    if bits_input is not None:
        xd = dev_bf16(bits_input)
        co, so, go = oracle.nvfp4_quantize(bits_input)
    else:
        xd = dev_f32(X)
        co, so, go = oracle.nvfp4_quantize(X)
    rows, K = xd.shape
    c, s, g = m.nvfp4_quantize(xd)
    m.check_status()
    gg = g.cpu().numpy()
    assert gg[0].view(np.uint32) == np.float32(go).view(np.uint32), (gg[0], go)
    np.testing.assert_array_equal(unswizzle_scales(s, rows, K), so)
    cg = unpack_codes(c, K)
    bad = np.count_nonzero(cg != co)
    assert bad == 0, "%d codes differ" % bad
    # padding rows / blocks of the atom layout hold 0
    full = np.zeros(s.numel(), bool)
    KA = ((K + 255) // 256) * 4
    r = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    full[(((r // 128) * KA + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)).ravel()] = True
    assert not s.cpu().numpy()[~full].any()
    return c, s, g


@pytest.mark.parametrize("rows,K", [(1, 64), (7, 192), (130, 320), (256, 4096), (300, 1024)])
def test_quantize_fp32_bit_exact(rows, K):
    g = wi.rng(rows * 7 + K, 1)
    X = (g.standard_normal((rows, K)) * np.exp(g.standard_normal((rows, 1)))).astype(np.float32)
    check_quantize(X)


@pytest.mark.parametrize("rows,K", [(40, 512), (129, 256), (1560, 4096)])
def test_quantize_bf16_activations_bit_exact(rows, K):
    check_quantize(None, bits_input=wi.activations(rows + K, 2, rows, K))


def test_quantize_workload_weights_bit_exact():
    W = wi.weight(5, 1, 4096, 4096)
    check_quantize(W)


def test_quantize_edge_cases():
    K = 256
    g = wi.rng(3, 3)
    X = g.standard_normal((9, K)).astype(np.float32)
    X[0, :] = 0.0                                   # zero row
    X[1, 16:32] = 0.0                               # zero block
    X[2, 32:48] = 1e-30                             # block scale underflows to 0
    X[3, :16] = -0.0                                # negative zeros
    X[4, 0] = 2688.0 * 4                            # tensor amax; g = 4 exactly
    # E2M1 midpoints and E4M3 midpoints in units of the block scale (cf. the oracle pins)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.75, -5.0, 6.0, 0.5, 1.5, 3.0, 4.0])
    X[5, :16] = (mids * 4.0).astype(np.float32)     # d = s_b g = 1 * 4
    X[6, :16] = 0.0
    X[6, 3] = 4.0 * 6.0 * 1.0625                    # s_b tie between 1 and 1.125 -> 1
    X[7, :16] = 0.0
    X[7, 5] = -4.0 * 6.0 * 1.1875                   # s_b tie between 1.125 and 1.25 -> 1.25
    X[8, :16] = np.float32(4.0 * 6.0 * 2.0 ** -9 * 1.5)  # E4M3 subnormal tie -> 2 steps
    check_quantize(X)
    check_quantize(np.zeros((3, 64), np.float32))   # all-zero tensor: g = 0, every code 0


def _linear_case(M, N, K, r, bias, out_dtype, seed=0, rows=None):
    m = wlq()
    x_bits = wi.activations(seed + 1, 1, M, K)
    W = wi.weight(seed + 2, 2, N, K)
    b_bits = wi.bias(seed + 3, 3, N) if bias else None
    L1 = wi.normal_bf16(wi.rng(seed + 4, 4), (K, r), 0.05) if r else None
    L2 = wi.normal_bf16(wi.rng(seed + 5, 5), (r, N), 0.05) if r else None
    xq_o, xs_o, xg_o = oracle.nvfp4_quantize(x_bits)
    wq_o, ws_o, wg_o = oracle.nvfp4_quantize(W)
    x = dev_bf16(x_bits)
    wq, ws, wg = m.nvfp4_quantize(dev_f32(W))
    y = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
    m.w4a4_linear_into(y, x, wq, ws, wg, N, K, dev_bf16(b_bits) if bias else None,
                       dev_bf16(L1) if r else None, dev_bf16(L2) if r else None)
    m.check_status()
    if rows is None:
        rows = np.arange(M)
    y_ref = oracle.nvfp4_linear(xq_o[rows], xs_o[rows], xg_o, x_bits[rows], wq_o, ws_o, wg_o, b_bits, L1, L2)
    yg = y.float().cpu().numpy()[rows]
    assert not np.isnan(yg).any()
    if out_dtype == torch.bfloat16:
        # each value's own rounding taken out first: what is left must meet the fp32 bound
        rms = float(np.sqrt(np.mean(y_ref ** 2)))
        excess = np.abs(yg - y_ref) - 2.0 ** -8 * np.abs(y_ref)
        return max(float(excess.max()), 0.0) / rms
    return rel_err(yg, y_ref)


@pytest.mark.parametrize("M,N,K,r,bias", [
    (40, 320, 512, 0, True),
    (128, 128, 256, 0, False),
    (130, 200, 320, 32, True),      # ragged M, N and a K that is not a multiple of 256
    (256, 384, 1024, 16, True),
    (5, 128, 256, 64, False),
    (300, 640, 2048, 32, True),     # several tiles per CTA in both directions
])
def test_w4a4_linear_matches_oracle(M, N, K, r, bias):
    assert _linear_case(M, N, K, r, bias, torch.float32, seed=M + N) <= TOL_F32


@pytest.mark.parametrize("r", [0, 32])
def test_w4a4_linear_bf16_output(r):
    assert _linear_case(200, 256, 512, r, True, torch.bfloat16, seed=11) <= TOL_F32


def test_w4a4_linear_full_size_sampled_rows():
    """The SVDQuant-shaped projection (4096 x 4096, r = 32) at 4096 tokens: the
    rows of every 128-token tile checked against the oracle."""
    M = 4096
    rows = np.unique(np.concatenate([np.arange(0, M, 128), np.arange(127, M, 128),
                                     (np.arange(M // 128) * 128 + (np.arange(M // 128) * 37) % 128)]))
    assert _linear_case(M, 4096, 4096, 32, True, torch.float32, seed=21, rows=rows) <= TOL_F32


def test_nvfp4_linear_from_quantized_operands_equals_w4a4():
    """wlq_nvfp4_linear over codes from wlq_nvfp4_quantize is the same
    computation as the one-call W4A4 forward: bit-identical outputs."""
    m = wlq()
    M, N, K, r = 96, 256, 768, 16
    x_bits = wi.activations(31, 1, M, K)
    W = wi.weight(31, 2, N, K)
    L1 = dev_bf16(wi.normal_bf16(wi.rng(31, 4), (K, r), 0.05))
    L2 = dev_bf16(wi.normal_bf16(wi.rng(31, 5), (r, N), 0.05))
    x = dev_bf16(x_bits)
    wq, ws, wg = m.nvfp4_quantize(dev_f32(W))
    xq, xs, xg = m.nvfp4_quantize(x)
    y1 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    y2 = torch.empty_like(y1)
    m.nvfp4_linear_into(y1, xq, xs, xg, wq, ws, wg, N, K, x=x, L1=L1, L2=L2)
    m.w4a4_linear_into(y2, x, wq, ws, wg, N, K, L1=L1, L2=L2)
    m.check_status()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("M,N,K,r,out", [
    (1, 301, 128, 0, torch.float32),     # one token; odd N: rows of y are not 16-byte units (plain stores)
    (17, 300, 192, 16, torch.bfloat16),  # N * 2 bytes not a multiple of 16 (plain stores), K % 256 != 0
    (257, 136, 320, 32, torch.float32),  # a second 256-token tile holding one token
])
def test_w4a4_linear_ragged_shapes_and_plain_store_epilogue(M, N, K, r, out):
    assert _linear_case(M, N, K, r, True, out, seed=M + N + K) <= TOL_F32


def test_w4a4_linear_misaligned_output_takes_plain_stores():
    """y 4 bytes past a 16-byte boundary: the epilogue cannot use TMA stores
    and must write the same values with plain stores."""
    m = wlq()
    M, N, K = 64, 256, 256
    x_bits = wi.activations(41, 1, M, K)
    W = wi.weight(41, 2, N, K)
    x = dev_bf16(x_bits)
    wq, ws, wg = m.nvfp4_quantize(dev_f32(W))
    y_al = torch.empty((M, N), dtype=torch.float32, device="cuda")
    buf = torch.empty(M * N + 4, dtype=torch.float32, device="cuda")
    y_mis = buf[1:1 + M * N].view(M, N)
    m.w4a4_linear_into(y_al, x, wq, ws, wg, N, K)
    m.w4a4_linear_into(y_mis, x, wq, ws, wg, N, K)
    m.check_status()
    assert torch.equal(y_al, y_mis)


def test_w4a4_zero_weights_keep_the_low_rank_term_and_zero_x_gives_bias():
    """An all-zero weight tensor has tensor scale 0: the low-rank operand is then
    left unscaled, so y = (x L1) L2 + b.  An all-zero x gives y = b."""
    m = wlq()
    M, N, K, r = 48, 128, 256, 32
    x_bits = wi.activations(43, 1, M, K)
    b_bits = wi.bias(43, 3, N)
    L1 = wi.normal_bf16(wi.rng(43, 4), (K, r), 0.05)
    L2 = wi.normal_bf16(wi.rng(43, 5), (r, N), 0.05)
    W = np.zeros((N, K), np.float32)
    wq, ws, wg = m.nvfp4_quantize(dev_f32(W))
    assert float(wg[0]) == 0.0
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    m.w4a4_linear_into(y, dev_bf16(x_bits), wq, ws, wg, N, K, dev_bf16(b_bits), dev_bf16(L1), dev_bf16(L2))
    m.check_status()
    xq_o, xs_o, xg_o = oracle.nvfp4_quantize(x_bits)
    wq_o, ws_o, wg_o = oracle.nvfp4_quantize(W)
    y_ref = oracle.nvfp4_linear(xq_o, xs_o, xg_o, x_bits, wq_o, ws_o, wg_o, b_bits, L1, L2)
    assert rel_err(y.cpu().numpy(), y_ref) <= TOL_F32
    # x = 0: every code and the low-rank term vanish
    xz = np.zeros((M, K), np.uint16)
    W2 = wi.weight(43, 2, N, K)
    wq2, ws2, wg2 = m.nvfp4_quantize(dev_f32(W2))
    m.w4a4_linear_into(y, dev_bf16(xz), wq2, ws2, wg2, N, K, dev_bf16(b_bits), dev_bf16(L1), dev_bf16(L2))
    m.check_status()
    np.testing.assert_array_equal(y.cpu().numpy(), np.broadcast_to(oracle._bf16_value(b_bits), (M, N)))


def test_nvfp4_nonfinite_input_is_reported():
    m = wlq()
    X = np.ones((4, 64), np.float32)
    X[2, 5] = np.inf
    m.nvfp4_quantize(dev_f32(X))
    with pytest.raises(m.WlqError):
        m.check_status()
    m.check_status()  # the status word was cleared by the report


def test_w4a4_forward_is_bitwise_reproducible():
    m = wlq()
    M, N, K, r = 300, 384, 512, 32
    x = dev_bf16(wi.activations(47, 1, M, K))
    wq, ws, wg = m.nvfp4_quantize(dev_f32(wi.weight(47, 2, N, K)))
    L1 = dev_bf16(wi.normal_bf16(wi.rng(47, 4), (K, r), 0.05))
    L2 = dev_bf16(wi.normal_bf16(wi.rng(47, 5), (r, N), 0.05))
    ys = []
    for _ in range(3):
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        m.w4a4_linear_into(y, x, wq, ws, wg, N, K, L1=L1, L2=L2)
        ys.append(y)
    m.check_status()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])
