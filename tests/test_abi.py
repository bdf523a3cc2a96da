"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/wlq.h declares, and its host-only logic (sizes, argument
checks that run before any device access) behaves as documented."""
import ctypes
import os
import re

import pytest

from tests.test_golden_shapes import load_golden

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wlq.h")


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_wlq_build", os.path.join(ROOT, "weight_only_quantized_rtn_b200", "_build.py"))
    _build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(_build)
    path = _build.build()
    L = ctypes.CDLL(path)
    L.wlq_packed_bytes.restype = ctypes.c_size_t
    L.wlq_packed_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
    L.wlq_linear_workspace.restype = ctypes.c_size_t
    L.wlq_linear_workspace.argtypes = [ctypes.c_int64] * 3 + [ctypes.c_int] * 3
    L.wlq_version.restype = ctypes.c_char_p
    L.wlq_last_error.restype = ctypes.c_char_p
    return L


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wlq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def test_version(lib):
    assert lib.wlq_version().decode().count(".") == 2


def test_packed_bytes(lib):
    # int8: 8192 B per 128x64 tile + 4 B per padded row
    assert lib.wlq_packed_bytes(4096, 4096, 8, 0) == 32 * 64 * 8192 + 4096 * 4
    assert lib.wlq_packed_bytes(4096, 4096, 4, 64) == 32 * 64 * (4096 + 256) + 4096 * 4
    assert lib.wlq_packed_bytes(4096, 4096, 4, 16) == 32 * 64 * (4096 + 1024) + 4096 * 4
    # ragged: N and K are padded to the tile
    assert lib.wlq_packed_bytes(130, 72, 8, 0) == 2 * 2 * 8192 + 256 * 4
    # unsupported recipes / shapes
    assert lib.wlq_packed_bytes(64, 64, 4, 0) == 0
    assert lib.wlq_packed_bytes(64, 60, 8, 0) == 0
    assert lib.wlq_packed_bytes(64, 72, 4, 64) == 0


def test_packed_bytes_match_the_pages_weight_totals(lib):
    """'Joy-face_change_optimized', quantization results table: 15.2 GiB
    (int8 per channel), 8.1 GiB (int4 gs64), 11.4 GiB (attention int8 + MLP
    int4 gs16).  The block Linears (80 = 40 blocks x 2 streams, 99% of the
    parameters) packed in this library's layout must come in just under each
    total, the rest being the remaining 1% of the model; fp32 group scales
    would overshoot the int4 figures, which is why group scales are packed as
    16-bit values."""
    g = load_golden()
    n_blocks = int(g["blocks"] * g["streams"])
    GiB = 2.0 ** 30
    attn = [(4096, 4096)] * 4
    mlp = [(16384, 4096), (4096, 16384)]

    def total(recipe_attn, recipe_mlp):
        b = sum(lib.wlq_packed_bytes(N, K, *recipe_attn) for N, K in attn)
        b += sum(lib.wlq_packed_bytes(N, K, *recipe_mlp) for N, K in mlp)
        return n_blocks * b / GiB

    cases = [
        (total((8, 0), (8, 0)), g["bytes_int8_per_channel_GiB"]),
        (total((4, 64), (4, 64)), g["bytes_int4_gs64_GiB"]),
        (total((8, 0), (4, 16)), g["bytes_attn_int8_mlp_int4_gs16_GiB"]),
    ]
    for ours, page in cases:
        assert page - 0.3 < ours < page, (ours, page)
    # with 4-byte group scales the int4 totals would exceed what the page prints
    fp32_scales_gs64 = n_blocks * sum(N * K // 2 + N * K // 64 * 4 for N, K in attn + mlp) / GiB
    assert fp32_scales_gs64 > g["bytes_int4_gs64_GiB"]


def test_workspace_sizes(lib):
    assert lib.wlq_linear_workspace(0, 4096, 4096, 8, 0, 0) == 0
    # int8 at large M needs no workspace
    assert lib.wlq_linear_workspace(4096, 4096, 4096, 8, 0, 0) == 0
    # small M splits K across a cluster; partial sums stay in shared memory
    assert lib.wlq_linear_workspace(16, 4096, 4096, 8, 0, 0) == 0
    # int4 at most 16 tokens: the few-token kernel reads the bf16 x itself
    assert lib.wlq_linear_workspace(16, 4096, 4096, 4, 64, 0) == 0
    assert lib.wlq_linear_workspace(16, 4096, 4096, 4, 16, 0) == 0
    assert lib.wlq_linear_workspace(17, 4096, 4096, 4, 64, 0) >= 17 * 4096 * 2
    # ... while its x rows fit in shared memory; beyond that the warp-MMA
    # kernel takes the shape and needs the fp16 copy of x again
    assert lib.wlq_linear_workspace(16, 4096, 40960, 4, 16, 0) == 0
    assert lib.wlq_linear_workspace(16, 4096, 65536, 4, 64, 0) >= 16 * 65536 * 2
    # int8 without low rank: none at any M and K
    for M, K in ((1, 131072), (16, 65536), (300, 4096)):
        assert lib.wlq_linear_workspace(M, 4096, K, 8, 0, 0) == 0
    # int4 stages an fp16 copy of x (+ row scales)
    assert lib.wlq_linear_workspace(4096, 4096, 4096, 4, 64, 0) >= 4096 * 4096 * 2 + 4096 * 4
    # low rank adds T (hi/lo) and the transposed L2
    assert (lib.wlq_linear_workspace(4096, 4096, 4096, 4, 64, 32)
            > lib.wlq_linear_workspace(4096, 4096, 4096, 4, 64, 0))
    assert lib.wlq_linear_workspace(16, 64, 64, 4, 64, 8) == 0  # bad rank


def test_argument_errors_before_any_device_access(lib):
    vp = ctypes.c_void_p
    lib.wlq_quantize.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, vp, vp, vp]
    lib.wlq_linear.argtypes = [vp, ctypes.c_int64, vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                               vp, vp, vp, ctypes.c_int, vp, ctypes.c_int, vp, ctypes.c_size_t, vp]
    assert lib.wlq_quantize(None, 4, 64, 5, 0, None, None, None) == 4          # bits
    assert lib.wlq_quantize(None, 4, 64, 4, 48, None, None, None) == 4         # group
    assert lib.wlq_quantize(None, 4, 60, 8, 0, None, None, None) == 2          # K % 8
    assert lib.wlq_quantize(None, 4, 64, 8, 0, None, None, None) == 1          # null
    assert lib.wlq_quantize(None, 0, 64, 8, 0, None, None, None) == 0          # N == 0: no-op
    assert lib.wlq_quantize(vp(16), 4, 64, 8, 0, vp(17), vp(16), None) == 3    # alignment
    assert b"16-byte" in lib.wlq_last_error()
    lib.wlq_quantize_pack.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, vp, vp, vp]
    assert lib.wlq_quantize_pack(None, 4, 64, 8, 64, None, None, None) == 4     # no packed layout for (8, 64)
    assert lib.wlq_quantize_pack(None, 4, 60, 8, 0, None, None, None) == 2      # K % 8
    assert lib.wlq_quantize_pack(None, 4, 40960, 8, 0, None, None, None) == 2   # row longer than the registers hold
    assert lib.wlq_quantize_pack(None, 4, 64, 8, 0, None, None, None) == 1      # null
    assert lib.wlq_quantize_pack(None, 0, 64, 8, 0, None, None, None) == 0      # N == 0: no-op
    assert lib.wlq_quantize_pack(vp(16), 4, 64, 8, 0, vp(16), vp(40), None) == 3  # packed misaligned
    i64, i32 = ctypes.c_int64, ctypes.c_int
    lib.wlq_quantize_ex.argtypes = [vp, i32, i64, i64, i32, i32, i32, vp, vp, vp]
    assert lib.wlq_quantize_ex(None, 0, 4, 64, 9, 0, 0, None, None, None) == 4    # bits 2..8
    assert lib.wlq_quantize_ex(None, 0, 4, 64, 1, 0, 0, None, None, None) == 4
    assert lib.wlq_quantize_ex(None, 2, 4, 64, 8, 0, 0, None, None, None) == 4    # input dtype
    assert lib.wlq_quantize_ex(None, 0, 4, 64, 8, 0, 3, None, None, None) == 4    # scale dtype
    assert lib.wlq_quantize_ex(None, 0, 4, 64, 8, 6, 0, None, None, None) == 2    # group % 4
    assert lib.wlq_quantize_ex(None, 1, 4, 64, 5, 16, 1, None, None, None) == 1   # null
    assert lib.wlq_quantize_ex(vp(16), 1, 4, 64, 5, 16, 1, vp(16), vp(17), None) == 3  # fp16 scales 2-byte aligned
    lib.wlq_quantize_fp8.argtypes = [vp, i32, i64, i64, i32, vp, vp, vp]
    assert lib.wlq_quantize_fp8(None, 0, 4, 64, 10, None, None, None) == 2        # group % 4
    assert lib.wlq_quantize_fp8(None, 0, 4, 60, 0, None, None, None) == 2         # K % 8
    assert lib.wlq_quantize_fp8(None, 0, 4, 64, 32, None, None, None) == 1        # null
    assert lib.wlq_quantize_fp8(None, 0, 0, 64, 32, None, None, None) == 0        # N == 0
    # M == 0 is a no-op
    assert lib.wlq_linear(None, 0, None, 64, 64, 8, 0, None, None, None, 0, None, 0, None, 0, None) == 0
    assert lib.wlq_linear(None, 4, None, 64, 64, 4, 0, None, None, None, 0, None, 0, None, 0, None) == 4
    assert lib.wlq_linear(None, 4, None, 64, 64, 8, 0, None, None, None, 8, None, 0, None, 0, None) == 2
    assert lib.wlq_linear(None, 4, None, 64, 64, 8, 0, None, None, None, 16, None, 0, None, 0, None) == 1
    assert lib.wlq_linear(None, 4, None, 64, 64, 8, 0, None, None, None, 0, None, 7, None, 0, None) == 1
    # misaligned x is rejected before any device access
    assert lib.wlq_linear(vp(18), 4, vp(32), 64, 64, 8, 0, None, None, None, 0, vp(64), 0, None, 0, None) == 3


def test_noalloc_argument_errors_match_the_workspace_entry_point(lib):
    """wlq_linear_noalloc makes wlq_linear's argument checks before it plans or
    sizes its scratch: a bad rank with a large M is a shape error, not a
    scratch-size or no-plan error, and every status comes before any device
    access (this machine has no GPU)."""
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.wlq_linear.argtypes = [vp, i64, vp, i64, i64, i32, i32, vp, vp, vp, i32, vp, i32, vp, ctypes.c_size_t, vp]
    lib.wlq_linear_noalloc.argtypes = [vp, i64, vp, i64, i64, i32, i32, vp, vp, vp, i32, vp, i32, vp]
    big = 1 << 20
    cases = [
        # x, M, packed, N, K, bits, group, bias, L1, L2, r, y, y_dtype -> status
        ((vp(16), big, vp(16), 4096, 4096, 4, 64, None, vp(16), vp(16), 8, vp(16), 0), 2),   # bad rank, large M
        ((vp(16), (1 << 30) + 1, vp(16), 64, 64, 8, 0, None, None, None, 0, vp(16), 0), 2),  # M > 2^30
        ((vp(16), -1, vp(16), 64, 64, 8, 0, None, None, None, 0, vp(16), 0), 1),             # M < 0
        ((vp(16), 4, vp(16), 64, 64, 4, 0, None, None, None, 0, vp(16), 0), 4),              # no packed layout
        ((vp(16), 4, vp(16), 64, 64, 8, 0, None, None, None, 16, vp(16), 0), 1),             # r > 0 without L1, L2
        ((vp(16), 4, vp(16), 64, 64, 8, 0, None, None, None, 0, vp(16), 5), 1),              # bad y dtype
        ((None, 4, vp(16), 64, 64, 8, 0, None, None, None, 0, vp(16), 0), 1),                # null x
        ((vp(18), 4, vp(16), 64, 64, 8, 0, None, None, None, 0, vp(16), 0), 3),              # misaligned x
        ((None, 0, None, 64, 64, 8, 0, None, None, None, 0, None, 0), 0),                    # M == 0: no-op
    ]
    for args, want in cases:
        assert lib.wlq_linear(*args, None, 0, None) == want, args
        assert lib.wlq_linear_noalloc(*args, None) == want, args


def test_nvfp4_sizes_and_argument_errors(lib):
    """NVFP4 scale storage: one 512-byte atom per 128 rows and 64 inputs, K
    padded to 256 and rows to 128; argument checks of the NVFP4 calls come
    before any device access."""
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.wlq_nvfp4_scales_bytes.restype = sz
    lib.wlq_nvfp4_scales_bytes.argtypes = [i64, i64]
    assert lib.wlq_nvfp4_scales_bytes(4096, 4096) == 32 * 64 * 512     # = 4096 * 4096 / 16 bytes
    assert lib.wlq_nvfp4_scales_bytes(130, 320) == 2 * 8 * 512          # rows -> 256, K -> 512
    assert lib.wlq_nvfp4_scales_bytes(4, 96) == 0                       # K % 64
    lib.wlq_nvfp4_quantize.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp]
    assert lib.wlq_nvfp4_quantize(vp(16), 2, 4, 64, vp(16), vp(16), vp(16), None) == 4    # input dtype
    assert lib.wlq_nvfp4_quantize(vp(16), 0, 4, 96, vp(16), vp(16), vp(16), None) == 2    # K % 64
    assert lib.wlq_nvfp4_quantize(None, 0, 4, 64, vp(16), vp(16), vp(16), None) == 1      # null
    assert lib.wlq_nvfp4_quantize(vp(16), 0, 4, 64, vp(24), vp(16), vp(16), None) == 3    # codes misaligned
    assert lib.wlq_nvfp4_quantize(vp(16), 0, 4, 64, vp(16), vp(16), vp(12), None) == 3    # gscale misaligned
    lib.wlq_nvfp4_linear_workspace.restype = sz
    lib.wlq_nvfp4_linear_workspace.argtypes = [i64, i64, i64, i32]
    assert lib.wlq_nvfp4_linear_workspace(256, 4096, 4096, 0) == 0
    # r = 32: T [M, 128] and L2 [N_pad, 128] in bf16, each 256-byte aligned
    assert lib.wlq_nvfp4_linear_workspace(200, 300, 512, 32) == 200 * 128 * 2 + 384 * 128 * 2
    assert lib.wlq_nvfp4_linear_workspace(200, 300, 512, 8) == 0        # bad rank
    lib.wlq_w4a4_workspace.restype = sz
    lib.wlq_w4a4_workspace.argtypes = [i64, i64, i64, i32]
    # codes M * K / 2, scale atoms, 256 bytes for the tensor scale, then the Linear's own
    assert lib.wlq_w4a4_workspace(256, 4096, 4096, 0) == 256 * 2048 + 2 * 64 * 512 + 256
    lib.wlq_nvfp4_linear.argtypes = [vp, vp, vp, vp, i64, vp, vp, vp, i64, i64, vp, vp, vp, i32, vp, i32, vp, sz, vp]
    ok = dict(xq=vp(16), xs=vp(16), xg=vp(16), x=vp(16), M=4, wq=vp(16), ws=vp(16), wg=vp(16), N=64, K=64,
              bias=None, L1=None, L2=None, r=0, y=vp(16), yd=0)
    cases = [
        (dict(K=96), 2), (dict(r=8), 2), (dict(r=16), 1), (dict(yd=3), 1), (dict(M=-1), 1),
        (dict(xq=None), 1), (dict(wg=None), 1), (dict(xs=vp(24)), 3), (dict(y=vp(18)), 3),
        (dict(M=0, xq=None), 0),
    ]
    for change, want in cases:
        a = dict(ok, **change)
        got = lib.wlq_nvfp4_linear(a["xq"], a["xs"], a["xg"], a["x"], a["M"], a["wq"], a["ws"], a["wg"], a["N"],
                                   a["K"], a["bias"], a["L1"], a["L2"], a["r"], a["y"], a["yd"], None, 0, None)
        assert got == want, (change, got)
    lib.wlq_w4a4_linear.argtypes = [vp, i64, vp, vp, vp, i64, i64, vp, vp, vp, i32, vp, i32, vp, sz, vp]
    assert lib.wlq_w4a4_linear(vp(16), 4, vp(16), vp(16), vp(16), 64, 64, None, None, None, 0, vp(16), 0,
                               None, 0, None) == 6                      # no workspace
    assert lib.wlq_w4a4_linear(None, 4, vp(16), vp(16), vp(16), 64, 64, None, None, None, 0, vp(16), 0,
                               vp(256), 1 << 20, None) == 1            # null x
    assert lib.wlq_w4a4_linear(vp(16), 4, vp(16), vp(16), vp(16), 64, 96, None, None, None, 0, vp(16), 0,
                               vp(256), 1 << 20, None) == 2            # K % 64
