"""wlq_linear_noalloc: the entry point for callers that cannot allocate
device memory (a host framework that owns a fixed memory pool, or a loop
where cudaMalloc / cudaFree would synchronise the device).

On two calls in a row (the built-in scratch keeps the previous call's
contents, including those of the previous parametrized shape) it must give
exactly the bytes wlq_linear gives with a caller workspace -- both run the
same plan and the same deterministic kernels -- and stay within the parity
tolerance of the oracle.  Shapes whose scratch does not fit in its 32 MiB are
refused.

Kept in its own file, collected last, so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import wlq_inputs as wi
from tests.gpu_helpers import TOL, dev_bf16, dev_f32, rel_err

pytestmark = pytest.mark.gpu

CASES = [
    # bits, group, M, N, K, r     (what the scratch holds)
    (4, 64, 24, 1024, 2048, 0),   # 17-32 tokens, warp-MMA kernel: fp16 copy of x + row scales
    (4, 64, 300, 640, 1024, 0),   # tensor-core kernel: fp16 copy of x + row scales
    (4, 16, 40, 384, 512, 32),    # fp16 x, low-rank T (hi/lo) and L2^T, K split over a cluster
    (8, 0, 200, 256, 320, 16),    # low rank with int8 weights: T and L2^T only
]


@pytest.mark.parametrize("bits,group,M,N,K,r", CASES)
def test_noalloc_matches_workspace_entry_point_twice(bits, group, M, N, K, r):
    import weight_only_quantized_rtn_b200 as wlq
    assert wlq.workspace_bytes(M, N, K, bits, group, r) > 0  # the case really uses the scratch
    x_bits = wi.activations(41, M, M, K)
    W = wi.weight(41, N, N, K, outlier_frac=0.02)
    b_bits = wi.bias(41, 3, N)
    L1_bits = wi.normal_bf16(wi.rng(41, 4), (K, r), 0.05) if r else None
    L2_bits = wi.normal_bf16(wi.rng(41, 5), (r, N), 0.05) if r else None
    x, b = dev_bf16(x_bits), dev_bf16(b_bits)
    L1 = dev_bf16(L1_bits) if r else None
    L2 = dev_bf16(L2_bits) if r else None
    codes, scales = wlq.quantize(dev_f32(W), bits, group)
    packed = wlq.pack(codes, scales, bits, group)
    ws = wlq.new_workspace(M, N, K, bits, group, r)
    y_ref = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    wlq.linear_into(y_ref, x, packed, N, K, bits, group, b, L1, L2, workspace=ws)
    wlq.check_status()
    co, so = oracle.quantize(W, bits, group)
    y_oracle = oracle.linear(x_bits, co, so, group, b_bits, L1_bits, L2_bits)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        wlq.linear_noalloc_into(y, x, packed, N, K, bits, group, b, L1, L2)
        wlq.check_status()
        assert torch.equal(y, y_ref)  # NaN never equals itself: every output was written
        err = rel_err(y.cpu().numpy(), y_oracle)
        assert err <= TOL, err


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import weight_only_quantized_rtn_b200 as wlq
    M, N, K = 4096, 4096, 4096  # int4 needs 2*M*K = 32 MiB for x16 alone, plus row scales
    assert wlq.workspace_bytes(M, N, K, 4, 64) > 32 << 20
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros(wlq.packed_bytes(N, K, 4, 64), dtype=torch.uint8, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wlq.WlqError) as e:
        wlq.linear_noalloc_into(y, x, packed, N, K, 4, 64)
    assert e.value.status == wlq.ERR_WORKSPACE
    assert "scratch" in str(e.value)
    wlq.check_status()
