"""Shared helpers for the GPU parity tests: move seeded numpy inputs to the
device, run the library through its C ABI, and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import wlq_inputs as wi

TOL = 1e-2  # max|y - y_ref| <= TOL * rms(y_ref), with identical codes


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def quantize_both(W: np.ndarray, bits: int, group: int):
    """GPU codes/scales and oracle codes/scales for the same weights."""
    import weight_only_quantized_rtn_b200 as wlq
    codes_g, scales_g = wlq.quantize(dev_f32(W), bits, group)
    codes_o, scales_o = oracle.quantize(W, bits, group)
    return codes_g, scales_g, codes_o, scales_o


def assert_codes_equal(codes_g, scales_g, codes_o, scales_o):
    cg = codes_g.cpu().numpy()
    sg = scales_g.cpu().numpy()
    bad = np.count_nonzero(cg != codes_o)
    assert bad == 0, "%d codes differ" % bad
    np.testing.assert_array_equal(sg.view(np.uint32), scales_o.view(np.uint32))


def rel_err(y: np.ndarray, y_ref: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(y_ref.astype(np.float64) ** 2)))
    return float(np.max(np.abs(y.astype(np.float64) - y_ref))) / max(rms, 1e-300)


def linear_case(x_bits, W, bits, group, b_bits=None, L1=None, L2=None, rows=None,
                out_dtype=torch.float32, check_codes=True):
    """Run quantize -> pack -> linear on the GPU and the oracle on `rows`.

    Returns (relative max error, y_gpu[rows], y_ref)."""
    import weight_only_quantized_rtn_b200 as wlq
    N, K = W.shape
    codes_g, scales_g, codes_o, scales_o = quantize_both(W, bits, group)
    if check_codes:
        assert_codes_equal(codes_g, scales_g, codes_o, scales_o)
    packed = wlq.pack(codes_g, scales_g, bits, group)
    x = dev_bf16(x_bits)
    b = dev_bf16(b_bits) if b_bits is not None else None
    l1 = dev_bf16(L1) if L1 is not None else None
    l2 = dev_bf16(L2) if L2 is not None else None
    # y starts as NaN, so an output the kernel never wrote cannot pass as a
    # stale copy of an earlier correct result
    M = x.shape[0]
    y = torch.full((M, N), float("nan"), dtype=out_dtype, device=x.device)
    ws = wlq.new_workspace(M, N, K, bits, group, 0 if l1 is None else l1.shape[1], device=x.device)
    wlq.linear_into(y, x, packed, N, K, bits, group, b, l1, l2, workspace=ws)
    wlq.check_status()
    if rows is None:
        rows = np.arange(x_bits.shape[0])
    y_ref = oracle.linear(x_bits[rows], codes_o, scales_o, group, b_bits, L1, L2)
    yg = y.float().cpu().numpy()[rows]
    return rel_err(yg, y_ref), yg, y_ref


def sample_rows(M: int, n: int = 12, seed: int = 0, block: int = 128) -> np.ndarray:
    """Rows checked at full size: every row up to 64 tokens; beyond that the
    first and last row of every `block`-token block (so each token tile of
    every plan, 64 to 256 tokens, has at least two checked rows, and each CTA
    of a CTA pair, which stages 128 of a 256-token tile, has its own), plus
    one row at an offset that moves by 37 from block to block (so the
    checked rows fall on every position inside a tile), plus `n` random rows."""
    if M <= 64:
        return np.arange(M)
    g = np.random.default_rng(seed)
    r = set(g.choice(M, min(n, M), replace=False).tolist())
    for i, b0 in enumerate(range(0, M, block)):
        end = min(M, b0 + block)
        r |= {b0, end - 1, min(end - 1, b0 + (37 * i) % block)}
    return np.array(sorted(r))
