"""GPU weight-only quantized Linear against the oracle.

Bar ("Joy-face_change_optimized" files table: weight-only Linear; "Nunchaku
Lite" 16-bit low-rank correction): with identical codes,
max|y - y_ref| <= 1e-2 * rms(y_ref) in the fp32-output mode; the bf16-output
mode equals bf16(fp32-output y) bit for bit; results are bitwise
reproducible.  Small cases span several 128 x BN tiles with ragged tails in
N, K and M; the five workloads run at full size in the launch configuration
the benchmark uses and are checked on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import wlq_inputs as wi
from tests.gpu_helpers import TOL, assert_codes_equal, dev_bf16, dev_f32, linear_case, rel_err, sample_rows

pytestmark = pytest.mark.gpu

RECIPES = [(8, 0), (4, 64), (4, 16)]


def wlq():
    import weight_only_quantized_rtn_b200 as m
    return m


def small_case(seed, M, N, K, bits, group, bias=True, r=0, outliers=0.02):
    x = wi.activations(seed, 1, M, K)
    W = wi.weight(seed, 2, N, K, outlier_frac=outliers)
    b = wi.bias(seed, 3, N) if bias else None
    L1 = L2 = None
    if r:
        L1 = wi.normal_bf16(wi.rng(seed, 4), (K, r), 0.05)
        L2 = wi.normal_bf16(wi.rng(seed, 5), (r, N), 0.05)
    return x, W, b, L1, L2


@pytest.mark.parametrize("bits,group", RECIPES)
@pytest.mark.parametrize("M", [1, 16, 17, 40, 64, 100, 128, 200, 300, 520])
def test_parity_small_ragged(bits, group, M):
    N, K = 300, 448  # 3 n-tiles (last one ragged), 7 K blocks
    x, W, b, _, _ = small_case(100 + M, M, N, K, bits, group)
    err, _, _ = linear_case(x, W, bits, group, b)
    assert err <= TOL, err


@pytest.mark.parametrize("bits,group", RECIPES)
@pytest.mark.parametrize("N,K", [(1, 64), (129, 64), (64, 1088), (513, 2112)])
def test_parity_shapes(bits, group, N, K):
    M = 37
    x, W, b, _, _ = small_case(7 * N + K, M, N, K, bits, group, bias=(N % 2 == 1))
    err, _, _ = linear_case(x, W, bits, group, b)
    assert err <= TOL, err


@pytest.mark.parametrize("bits,group", RECIPES)
@pytest.mark.parametrize("M,N,K", [
    (1, 4096, 4096),    # direct-load kernel: one token
    (5, 1000, 576),     # ragged tokens and channels (not a multiple of 32)
    (9, 33, 2048),      # 9..16 tokens: two 8-token MMA columns; one ragged channel tile
    (16, 2080, 4096),   # 16 tokens, 17 tiles on 8-CTA clusters
    (16, 512, 16384),   # direct-load kernel: K split over an 8-CTA cluster
])
def test_parity_few_tokens(bits, group, M, N, K):
    x, W, b, _, _ = small_case(60 + M, M, N, K, bits, group)
    err, _, _ = linear_case(x, W, bits, group, b)
    assert err <= TOL, err


@pytest.mark.parametrize("bits,group", RECIPES)
def test_few_tokens_per_token_magnitudes(bits, group):
    """Direct-load kernel: each CTA rescales each token's x by its own power
    of two before the fp16 MMAs.  Tokens of size 1e-30 and 1e30, an all-zero
    token, tokens with one large entry among small ones, and ordinary tokens:
    each row within 1e-2 of its own rms (the zero row exactly 0).  At most 16
    tokens no workspace is needed."""
    m = wlq()
    M, N, K = 12, 384, 1536
    assert m.workspace_bytes(M, N, K, bits, group) == 0
    g = np.random.default_rng(31 + bits + group)
    x = g.standard_normal((M, K)).astype(np.float32)
    x[0] *= 1e-30
    x[1] *= 1e30
    x[2] = 0.0
    x[3] *= 1e-4
    x[3, 100] = 3e4
    x[4] = 1e-3
    x[4, 1500] = -2e5   # in the last K split of a cluster
    x[5, ::2] *= 1e-20  # every other input tiny
    W = wi.weight(5, 2, N, K)
    _, yg, y_ref = linear_case(wi.bf16_bits(x), W, bits, group)
    for i in range(M):
        rms = float(np.sqrt(np.mean(y_ref[i] ** 2)))
        if rms == 0.0:
            assert np.all(yg[i] == 0.0), i
        else:
            assert np.max(np.abs(yg[i] - y_ref[i])) <= TOL * rms, (i, np.max(np.abs(yg[i] - y_ref[i])) / rms)


@pytest.mark.parametrize("bits,group,M,N,K", [
    (8, 0, 3, 200, 200),      # one K split, three whole K blocks and 8 inputs
    (8, 0, 12, 700, 4040),    # 8-CTA clusters, the last split ends in a ragged block
    (4, 16, 16, 300, 1232),   # int4 groups of 16, ragged last block
])
def test_parity_few_tokens_ragged_k(bits, group, M, N, K):
    """Direct-load kernel with K not a multiple of 64: the inputs of the last
    K block beyond K must read as zero (their codes are 0)."""
    x, W, b, _, _ = small_case(80 + M, M, N, K, bits, group)
    err, _, _ = linear_case(x, W, bits, group, b)
    assert err <= TOL, err


@pytest.mark.parametrize("M,N,K", [(24, 512, 16384), (32, 512, 16384), (20, 1024, 12288)])
def test_ring_reuse_after_reads_complete(M, N, K):
    """Warp-MMA kernel with a large resident x and 4-8 CTA clusters: its weight
    ring slots are refilled as soon as all warps release them, so every read
    of a slot must have completed first.  These shapes once lost that race
    (a band of channels wrong in one CTA per run); five runs, all exact repeats
    and within tolerance."""
    m = wlq()
    x, W, b, _, _ = small_case(70 + M, M, N, K, 8, 0)
    codes, scales = m.quantize(dev_f32(W), 8, 0)
    packed = m.pack(codes, scales, 8, 0)
    co, so = oracle.quantize(W, 8, 0)
    ref = oracle.linear(x, co, so, 0, b, None, None)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    xd, bd = dev_bf16(x), dev_bf16(b)
    first = None
    for _ in range(5):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        m.linear_into(y, xd, packed, N, K, 8, 0, bd)
        m.check_status()
        yh = y.cpu().numpy()
        assert float(np.max(np.abs(yh - ref))) <= TOL * rms
        if first is None:
            first = yh
        assert np.array_equal(yh, first)


def test_parity_k_not_multiple_of_64():
    # int8 per channel only needs K % 8 == 0: the last K block is partial
    for K in (8, 72, 200):
        x, W, b, _, _ = small_case(K, 50, 140, K, 8, 0)
        err, _, _ = linear_case(x, W, 8, 0, b)
        assert err <= TOL, (K, err)


@pytest.mark.parametrize("bits,group", RECIPES)
@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("M", [16, 130])
def test_parity_low_rank(bits, group, r, M):
    x, W, b, L1, L2 = small_case(300 + r + M, M, 260, 512, bits, group, r=r)
    err, _, _ = linear_case(x, W, bits, group, b, L1, L2)
    assert err <= TOL, err


@pytest.mark.parametrize("bits,group", RECIPES)
@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("M", [16, 300, 600])
def test_parity_low_rank_zero_weight_rows(bits, group, r, M):
    """All-zero weight rows (scale 0, row factor 0) still carry their low-rank
    term: the branch shares the main accumulator, so such a row's operand is
    left unscaled and the epilogue scales it by 1."""
    x, W, b, L1, L2 = small_case(900 + r + M, M, 512, 512, bits, group, r=r)
    W[[0, 3, 130, 511]] = 0.0
    err, y, y_ref = linear_case(x, W, bits, group, b, L1, L2)
    assert err <= TOL, err
    assert np.abs(y_ref[:, 3]).max() > 0  # the low-rank term of a zero row is not zero


@pytest.mark.parametrize("bits,group", RECIPES)
@pytest.mark.parametrize("M,N,K,r,cap", [
    (600, 4096, 1024, 32, 0),  # low rank on CTA pairs (256-token tiles, the term in the pair's accumulator)
    (512, 1024, 512, 32, 0),   # low rank on split pairs: the term on K split 0 only
    (256, 1920, 1024, 64, 0),  # low rank, 256-token tiles on single CTAs with the partial in the ring
    (1024, 2048, 1024, 16, 20),# low rank on pairs, several tiles per pair
    (256, 4096, 1024, 0, 0),   # pairs over 128-token tiles, K split over the two pairs of a 4-CTA cluster
    (200, 4096, 512, 32, 0),   # the same with low rank and a ragged token tile

    (40, 1100, 320, 0, 4),     # 9 tiles on 4 CTAs: both accumulator buffers in use
    (16, 33000, 128, 0, 16),   # 258 tiles of 16 tokens on 16 CTAs
    (300, 700, 256, 0, 3),     # 128-token tiles, several per CTA
    (16, 1024, 2048, 0, 4),    # K split over clusters, each cluster several tiles
    (16, 4096, 1024, 0, 8),    # direct-load kernel on 8 CTAs: four tiles each
    (16, 4096, 16384, 0, 8),   # direct-load kernel: x needs 4-CTA clusters, sixteen tiles per cluster
    (24, 4096, 1024, 0, 8),    # warp-MMA kernel: K split over a cluster, several tiles per cluster
    (32, 1001, 512, 0, 3),     # warp-MMA kernel: ragged N (scalar stores), one cluster for all tiles
    (64, 2048, 1024, 0, 8),    # resident-x tensor-core kernel: K split over 4, several tiles per cluster
    (100, 1024, 512, 32, 4),   # low rank + K split, several tiles per cluster
    (600, 640, 640, 16, 5),    # low rank, single accumulator buffer, ring wrap-around
    (600, 4096, 448, 0, 0),    # CTA pairs (256 channels x 256 tokens per MMA), partial last slot
    (600, 4096, 1024, 0, 6),   # CTA pairs, three pairs for 48 tiles
    (256, 512, 1024, 0, 16),   # split pairs: K split over four pairs, one tile per 8-CTA cluster
    (512, 1024, 512, 0, 0),    # split pairs: two 256-token tiles per channel pair, K split over pairs
    (256, 1920, 1024, 0, 0),   # odd channel-tile count: single-CTA 256-token tiles, K split over 4, partial in the ring
    (512, 4096, 512, 0, 12),   # pairs in clusters of two pairs: 30 tiles in full rounds, 2 leftover tiles K-halved
    (1024, 2048, 1024, 0, 20), # the same with five clusters: 30 full, 2 leftover
])
def test_parity_several_tiles_per_cta(bits, group, M, N, K, r, cap):
    m = wlq()
    x, W, b, L1, L2 = small_case(M + N + K + r, M, N, K, bits, group, r=r)
    m.set_grid_limit(cap)
    try:
        err, _, _ = linear_case(x, W, bits, group, b, L1, L2)
    finally:
        m.set_grid_limit(0)
    assert err <= TOL, err


@pytest.mark.parametrize("bits,group", RECIPES)
@pytest.mark.parametrize("M,N,K", [
    (16, 384, 512),     # few-token kernel
    (300, 384, 512),    # K split over a cluster (partial in shared memory)
    (300, 16384, 512),  # unsplit 256-token tiles, CTA pairs: the bf16 fast epilogue
    (1560, 4096, 1024), # pairs with a tail round, ragged last token tile
    (600, 4096, 448),   # pairs, partial last ring slot
    (64, 4096, 1024),   # resident-x tensor-core kernel
    (100, 1000, 512),   # ragged N: scalar stores
])
def test_bf16_output_is_rounded_fp32_output(bits, group, M, N, K):
    """The bf16 output is the fp32 output rounded to nearest even, bit for
    bit, on every engine and epilogue variant (the int4 row factor of x
    included)."""
    m = wlq()
    x, W, b, _, _ = small_case(5 + M, M, N, K, bits, group)
    codes, scales = m.quantize(dev_f32(W), bits, group)
    packed = m.pack(codes, scales, bits, group)
    xd, bd = dev_bf16(x), dev_bf16(b)
    y32 = m.linear(xd, packed, N, K, bits, group, bd, out_dtype=torch.float32)
    y16 = m.linear(xd, packed, N, K, bits, group, bd, out_dtype=torch.bfloat16)
    m.check_status()
    assert not torch.isnan(y32).any()
    assert torch.equal(y16, y32.to(torch.bfloat16))


@pytest.mark.parametrize("bits,group", RECIPES)
def test_bitwise_reproducible(bits, group):
    m = wlq()
    for M in (16, 48, 1000):  # split-K and persistent paths
        x, W, b, L1, L2 = small_case(6, M, 1024, 1024, bits, group, r=32)
        codes, scales = m.quantize(dev_f32(W), bits, group)
        packed = m.pack(codes, scales, bits, group)
        args = (dev_bf16(x), packed, 1024, 1024, bits, group, dev_bf16(b), dev_bf16(L1), dev_bf16(L2))
        ws = m.new_workspace(M, 1024, 1024, bits, group, 32)
        ys = []
        for _ in range(3):
            # NaN never equals itself: an output left unwritten cannot pass
            y = torch.full((M, 1024), float("nan"), dtype=torch.float32, device="cuda")
            m.linear_into(y, *args, workspace=ws)
            ys.append(y)
        assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


def test_empty_and_errors():
    m = wlq()
    W = wi.weight(8, 1, 64, 128)
    codes, scales = m.quantize(dev_f32(W), 8, 0)
    packed = m.pack(codes, scales, 8, 0)
    x = torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda")
    assert m.linear(x, packed, 64, 128, 8, 0).shape == (0, 64)
    x = dev_bf16(wi.activations(8, 2, 16, 128))
    y = torch.empty((16, 64), dtype=torch.float32, device="cuda")
    need = m.workspace_bytes(16, 64, 128, 8, 0)
    if need:
        small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
        with pytest.raises(m.WlqError) as e:
            m.linear_into(y, x, packed, 64, 128, 8, 0, workspace=small)
        assert e.value.status == m.ERR_WORKSPACE
    # int4 beyond 16 tokens prepares x in a workspace: none given is an error
    c4, s4 = m.quantize(dev_f32(W), 4, 64)
    p4 = m.pack(c4, s4, 4, 64)
    x32 = dev_bf16(wi.activations(8, 4, 32, 128))
    y32 = torch.empty((32, 64), dtype=torch.float32, device="cuda")
    assert m.workspace_bytes(32, 64, 128, 4, 64) > 0
    with pytest.raises(m.WlqError) as e:
        m.linear_into(y32, x32, p4, 64, 128, 4, 64)
    assert e.value.status == m.ERR_WORKSPACE
    m.check_status()


# ------------------------------------------------------------ full workloads
def _check_full(x, W, bits, group, b, L1=None, L2=None):
    M = x.shape[0]
    rows = sample_rows(M, 12, seed=M)
    err, _, _ = linear_case(x, W, bits, group, b, L1, L2, rows=rows)
    assert err <= TOL, err
    return err


def test_full_tiny_w8():
    d = wi.tiny_w8()
    err, _, _ = linear_case(d["x"], d["W"], 8, 0, d["b"])
    assert err <= TOL, err


@pytest.mark.parametrize("M", [16, 256, 4096])
def test_full_attention_w8(M):
    d = wi.attn_w8(M)
    _check_full(d["x"], d["W"], 8, 0, d["b"])


@pytest.mark.parametrize("which", ["up", "down"])
@pytest.mark.parametrize("M", [16, 1560, 6240])
def test_full_mlp_w4_gs64(which, M):
    d = wi.mlp_w4(M, which)
    _check_full(d["x"], d["W"], 4, 64, d["b"])


def _bf16_close(y_bf16_rows: np.ndarray, ref: np.ndarray):
    """A bf16 output against the fp64 oracle: the parity bound plus the bf16
    rounding of each value (half a bf16 unit in the last place, at most
    2^-8 of the value)."""
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bad = np.abs(y_bf16_rows.astype(np.float64) - ref) > TOL * rms + 2.0 ** -8 * np.abs(ref)
    assert not bad.any(), "%d bf16 outputs outside the bound" % int(bad.sum())


def _oracle_chain(x_rows, up_q, up_b, down_q, down_b, group):
    """The oracle's chained pair on the same rows: up in fp64, handed on as
    bf16 (rounded to nearest even, as the product hands on its bf16 output),
    then down in fp64."""
    y_up = oracle.linear(x_rows, up_q[0], up_q[1], group, up_b)
    y_dn = oracle.linear(oracle._bf16_rne_bits(y_up), down_q[0], down_q[1], group, down_b)
    return y_up, y_dn


@pytest.mark.parametrize("M", [16, 1560, 6240])
def test_full_mlp_chained_up_then_down(M):
    """The MLP workload as configured: a GELU-free chained pair, down
    consuming up's bf16 output on the same stream, with both weights
    quantized by the fused quantize-pack pass (its codes and scales checked
    against the oracle too)."""
    m = wlq()
    up, dn = wi.mlp_w4(M, "up"), wi.mlp_w4(M, "down")
    N1, K1 = up["W"].shape
    N2, K2 = dn["W"].shape
    s_up, p_up = m.quantize_pack(dev_f32(up["W"]), 4, 64)
    s_dn, p_dn = m.quantize_pack(dev_f32(dn["W"]), 4, 64)
    q_up, q_dn = oracle.quantize(up["W"], 4, 64), oracle.quantize(dn["W"], 4, 64)
    assert_codes_equal(m.unpack(p_up, N1, K1, 4, 64), s_up, *q_up)
    assert_codes_equal(m.unpack(p_dn, N2, K2, 4, 64), s_dn, *q_dn)
    x = dev_bf16(up["x"])
    y_up = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
    y_dn = torch.full((M, N2), float("nan"), dtype=torch.float32, device="cuda")
    m.linear_into(y_up, x, p_up, N1, K1, 4, 64, dev_bf16(up["b"]),
                  workspace=m.new_workspace(M, N1, K1, 4, 64))
    m.linear_into(y_dn, y_up, p_dn, N2, K2, 4, 64, dev_bf16(dn["b"]),
                  workspace=m.new_workspace(M, N2, K2, 4, 64))
    m.check_status()
    rows = sample_rows(M, 12, seed=M)
    ref_up, ref_dn = _oracle_chain(up["x"][rows], q_up, up["b"], q_dn, dn["b"], 64)
    _bf16_close(y_up.float().cpu().numpy()[rows], ref_up)
    err = rel_err(y_dn.cpu().numpy()[rows], ref_dn)
    assert err <= TOL, err


def test_full_mixed_block_back_to_back():
    """The mixed-precision block as configured: q, k, v, o (int8 per channel)
    and up (int4 gs16) on x, then down (int4 gs16) on up's bf16 output -- six
    launches back to back on one stream, nothing synchronised between them."""
    m = wlq()
    M = 4096
    blk = wi.mixed_block(M)
    x_bits = blk["x"]
    x = dev_bf16(x_bits)
    dev_layers, outs = {}, {}
    for name, N, K, bits, group in wi.MIXED_LAYERS:
        L = blk["layers"][name]
        s, p = m.quantize_pack(dev_f32(L["W"]), bits, group)
        dev_layers[name] = (p, dev_bf16(L["b"]), m.new_workspace(M, N, K, bits, group))
        dt = torch.bfloat16 if name == "up" else torch.float32
        outs[name] = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    torch.cuda.synchronize()
    for name, N, K, bits, group in wi.MIXED_LAYERS:
        p, b, ws = dev_layers[name]
        inp = outs["up"] if name == "down" else x
        m.linear_into(outs[name], inp, p, N, K, bits, group, b, workspace=ws)
    m.check_status()
    rows = sample_rows(M, 12, seed=3)
    q = {name: oracle.quantize(blk["layers"][name]["W"], bits, group)
         for name, N, K, bits, group in wi.MIXED_LAYERS}
    for name in ("q", "k", "v", "o"):
        ref = oracle.linear(x_bits[rows], *q[name], 0, blk["layers"][name]["b"])
        err = rel_err(outs[name].cpu().numpy()[rows], ref)
        assert err <= TOL, (name, err)
    ref_up, ref_dn = _oracle_chain(x_bits[rows], q["up"], blk["layers"]["up"]["b"], q["down"],
                                   blk["layers"]["down"]["b"], 16)
    _bf16_close(outs["up"].float().cpu().numpy()[rows], ref_up)
    err = rel_err(outs["down"].cpu().numpy()[rows], ref_dn)
    assert err <= TOL, ("down", err)


@pytest.mark.parametrize("M", [256, 4096])
def test_full_svdq_low_rank(M):
    d = wi.svdq_w4_lr(M)
    _check_full(d["x"], d["W"], 4, 64, d["b"], d["L1"], d["L2"])
