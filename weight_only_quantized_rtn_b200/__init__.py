"""Python binding of the wlq C ABI (include/wlq.h): argument marshalling only.

Every step of the quantization and of the Linear runs in the CUDA library
``libwlq.so`` (sm_100a); this module only turns torch tensors into pointers,
sizes and the current stream.  PyTorch provides device memory and streams.
There is no fallback: if the library is missing or fails to load, importing
this package raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwlq.so")

OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_NONFINITE, ERR_WORKSPACE, ERR_TIMEOUT, ERR_CUDA = range(9)
OUT_BF16, OUT_F32 = 0, 1
STATUS_NAMES = {
    OK: "WLQ_OK", ERR_INVALID_ARG: "WLQ_ERR_INVALID_ARG", ERR_SHAPE: "WLQ_ERR_SHAPE",
    ERR_ALIGN: "WLQ_ERR_ALIGN", ERR_UNSUPPORTED: "WLQ_ERR_UNSUPPORTED",
    ERR_NONFINITE: "WLQ_ERR_NONFINITE", ERR_WORKSPACE: "WLQ_ERR_WORKSPACE",
    ERR_TIMEOUT: "WLQ_ERR_TIMEOUT", ERR_CUDA: "WLQ_ERR_CUDA",
}
EXPORTS = ("wlq_quantize", "wlq_quantize_pack", "wlq_quantize_ex", "wlq_quantize_fp8", "wlq_packed_bytes",
           "wlq_pack", "wlq_unpack", "wlq_linear_workspace", "wlq_linear", "wlq_linear_noalloc",
           "wlq_lowrank_workspace", "wlq_lowrank_split", "wlq_lowrank_residual", "wlq_nvfp4_scales_bytes",
           "wlq_nvfp4_quantize", "wlq_nvfp4_linear_workspace", "wlq_nvfp4_linear", "wlq_w4a4_workspace",
           "wlq_w4a4_linear", "wlq_get_status",
           "wlq_probe_wait_timeout", "wlq_set_grid_limit", "wlq_last_error", "wlq_version")

if not os.path.exists(LIB_PATH):
    raise ImportError("libwlq.so is not built; run `python weight_only_quantized_rtn_b200/_build.py`")

lib = ctypes.CDLL(LIB_PATH)
_i64, _i32, _vp, _sz, _u64 = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64
lib.wlq_quantize.argtypes = [_vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp]
lib.wlq_packed_bytes.argtypes = [_i64, _i64, _i32, _i32]
lib.wlq_packed_bytes.restype = _sz
lib.wlq_pack.argtypes = [_vp, _vp, _i64, _i64, _i32, _i32, _vp, _vp]
lib.wlq_unpack.argtypes = [_vp, _i64, _i64, _i32, _i32, _vp, _vp]
lib.wlq_quantize_pack.argtypes = [_vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp]
lib.wlq_quantize_ex.argtypes = [_vp, _i32, _i64, _i64, _i32, _i32, _i32, _vp, _vp, _vp]
lib.wlq_quantize_fp8.argtypes = [_vp, _i32, _i64, _i64, _i32, _vp, _vp, _vp]
lib.wlq_linear_workspace.argtypes = [_i64, _i64, _i64, _i32, _i32, _i32]
lib.wlq_linear_workspace.restype = _sz
lib.wlq_linear.argtypes = [_vp, _i64, _vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _sz, _vp]
lib.wlq_linear_noalloc.argtypes = [_vp, _i64, _vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _vp]
lib.wlq_lowrank_workspace.argtypes = [_i64, _i64, _i32, _i32]
lib.wlq_lowrank_workspace.restype = _sz
lib.wlq_lowrank_split.argtypes = [_vp, _i64, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.wlq_lowrank_residual.argtypes = [_vp, _vp, _vp, _i64, _i64, _i32, _vp, _vp]
lib.wlq_nvfp4_scales_bytes.argtypes = [_i64, _i64]
lib.wlq_nvfp4_scales_bytes.restype = _sz
lib.wlq_nvfp4_quantize.argtypes = [_vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp]
lib.wlq_nvfp4_linear_workspace.argtypes = [_i64, _i64, _i64, _i32]
lib.wlq_nvfp4_linear_workspace.restype = _sz
lib.wlq_nvfp4_linear.argtypes = [_vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _i32, _vp, _i32,
                                 _vp, _sz, _vp]
lib.wlq_w4a4_workspace.argtypes = [_i64, _i64, _i64, _i32]
lib.wlq_w4a4_workspace.restype = _sz
lib.wlq_w4a4_linear.argtypes = [_vp, _i64, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _sz, _vp]
lib.wlq_get_status.argtypes = [_vp]
lib.wlq_probe_wait_timeout.argtypes = [_u64, _vp]
lib.wlq_set_grid_limit.argtypes = [_i32]
lib.wlq_set_grid_limit.restype = None
lib.wlq_last_error.restype = ctypes.c_char_p
lib.wlq_version.restype = ctypes.c_char_p
for _f in ("wlq_quantize", "wlq_quantize_pack", "wlq_quantize_ex", "wlq_quantize_fp8", "wlq_pack", "wlq_unpack", "wlq_linear",
           "wlq_linear_noalloc", "wlq_lowrank_split", "wlq_lowrank_residual", "wlq_nvfp4_quantize", "wlq_nvfp4_linear",
           "wlq_w4a4_linear", "wlq_get_status", "wlq_probe_wait_timeout"):
    getattr(lib, _f).restype = ctypes.c_int


class WlqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), msg))
        self.status = status


def _check(rc: int):
    if rc != OK:
        raise WlqError(rc, lib.wlq_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def groups(K: int, group: int) -> int:
    return 1 if group == 0 else K // group


def quantize(W: torch.Tensor, bits: int, group: int, stream=None):
    """RTN symmetric quantization of fp32 W [N, K] -> (codes int8 [N,K], scales fp32 [N,G])."""
    assert W.dtype == torch.float32 and W.is_cuda and W.is_contiguous()
    N, K = W.shape
    codes = torch.empty((N, K), dtype=torch.int8, device=W.device)
    scales = torch.empty((N, groups(K, group)), dtype=torch.float32, device=W.device)
    _check(lib.wlq_quantize(_ptr(W), N, K, bits, group, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


SCALE_F32, SCALE_F16, SCALE_BF16 = 0, 1, 2
_SCALE_TORCH = {SCALE_F32: torch.float32, SCALE_F16: torch.float16, SCALE_BF16: torch.bfloat16}


def _in_dtype(W: torch.Tensor) -> int:
    if W.dtype == torch.float32:
        return 0
    if W.dtype == torch.bfloat16:
        return 1
    raise WlqError(ERR_UNSUPPORTED, "input must be fp32 or bf16")


def quantize_ex(W: torch.Tensor, bits: int, group: int, scale_dtype: int = SCALE_F32, stream=None):
    """RTN for 2..8 bits from fp32 or bf16 W [N, K] -> (codes int8 [N,K], scales [N,G] in scale_dtype)."""
    assert W.is_cuda and W.is_contiguous()
    N, K = W.shape
    codes = torch.empty((N, K), dtype=torch.int8, device=W.device)
    scales = torch.empty((N, groups(K, group)), dtype=_SCALE_TORCH[scale_dtype], device=W.device)
    _check(lib.wlq_quantize_ex(_ptr(W), _in_dtype(W), N, K, bits, group, scale_dtype, _ptr(codes), _ptr(scales),
                               _stream(stream)))
    return codes, scales


def quantize_fp8(W: torch.Tensor, group: int, stream=None):
    """fp8 e4m3 block quantization of fp32 or bf16 W [N, K] -> (codes uint8 [N,K], scales fp32 [N,G])."""
    assert W.is_cuda and W.is_contiguous()
    N, K = W.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N, groups(K, group)), dtype=torch.float32, device=W.device)
    _check(lib.wlq_quantize_fp8(_ptr(W), _in_dtype(W), N, K, group, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def packed_bytes(N: int, K: int, bits: int, group: int) -> int:
    return int(lib.wlq_packed_bytes(N, K, bits, group))


def pack(codes: torch.Tensor, scales: torch.Tensor, bits: int, group: int, stream=None) -> torch.Tensor:
    N, K = codes.shape
    nbytes = packed_bytes(N, K, bits, group)
    if nbytes == 0:
        raise WlqError(ERR_UNSUPPORTED, "no packed layout for bits=%d group=%d K=%d" % (bits, group, K))
    out = torch.empty(nbytes, dtype=torch.uint8, device=codes.device)
    _check(lib.wlq_pack(_ptr(codes), _ptr(scales), N, K, bits, group, _ptr(out), _stream(stream)))
    return out


def quantize_pack(W: torch.Tensor, bits: int, group: int, stream=None):
    """quantize then pack in one pass: fp32 W [N, K] -> (scales fp32 [N,G], packed uint8)."""
    assert W.dtype == torch.float32 and W.is_cuda and W.is_contiguous()
    N, K = W.shape
    nbytes = packed_bytes(N, K, bits, group)
    if nbytes == 0:
        raise WlqError(ERR_UNSUPPORTED, "no packed layout for bits=%d group=%d K=%d" % (bits, group, K))
    scales = torch.empty((N, groups(K, group)), dtype=torch.float32, device=W.device)
    out = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _check(lib.wlq_quantize_pack(_ptr(W), N, K, bits, group, _ptr(scales), _ptr(out), _stream(stream)))
    return scales, out


def unpack(packed: torch.Tensor, N: int, K: int, bits: int, group: int, stream=None) -> torch.Tensor:
    codes = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    _check(lib.wlq_unpack(_ptr(packed), N, K, bits, group, _ptr(codes), _stream(stream)))
    return codes


def workspace_bytes(M: int, N: int, K: int, bits: int, group: int, r: int = 0) -> int:
    return int(lib.wlq_linear_workspace(M, N, K, bits, group, r))


def new_workspace(M, N, K, bits, group, r=0, device="cuda"):
    """A zero-filled workspace of the size wlq_linear needs (None when it needs none)."""
    n = workspace_bytes(M, N, K, bits, group, r)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


def linear_into(y, x, packed, N, K, bits, group, bias=None, L1=None, L2=None, workspace=None, stream=None):
    """y = x deq(W)^T [+ (x L1) L2] [+ b] into a preallocated y (bf16 or fp32 [M, N])."""
    M = x.shape[0]
    r = 0 if L1 is None else L1.shape[1]
    out = OUT_F32 if y.dtype == torch.float32 else OUT_BF16
    ws_n = 0 if workspace is None else workspace.numel()
    _check(lib.wlq_linear(_ptr(x), M, _ptr(packed), N, K, bits, group, _ptr(bias), _ptr(L1), _ptr(L2), r,
                          _ptr(y), out, _ptr(workspace), ws_n, _stream(stream)))
    return y


def linear(x, packed, N, K, bits, group, bias=None, L1=None, L2=None, out_dtype=torch.bfloat16,
           workspace=None, stream=None):
    assert x.dtype == torch.bfloat16 and x.is_contiguous()
    M = x.shape[0]
    y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    r = 0 if L1 is None else L1.shape[1]
    if workspace is None:
        workspace = new_workspace(M, N, K, bits, group, r, device=x.device)
    return linear_into(y, x, packed, N, K, bits, group, bias, L1, L2, workspace, stream)


def linear_noalloc_into(y, x, packed, N, K, bits, group, bias=None, L1=None, L2=None, stream=None):
    """wlq_linear_noalloc: like linear_into, with the library's built-in scratch."""
    M = x.shape[0]
    r = 0 if L1 is None else L1.shape[1]
    out = OUT_F32 if y.dtype == torch.float32 else OUT_BF16
    _check(lib.wlq_linear_noalloc(_ptr(x), M, _ptr(packed), N, K, bits, group, _ptr(bias), _ptr(L1), _ptr(L2), r,
                                  _ptr(y), out, _stream(stream)))
    return y


def lowrank_split(W: torch.Tensor, r: int, omega: torch.Tensor, power_iters: int = 2, stream=None):
    """Top-r split of W's transpose for the low-rank branch: fp32 W [N, K] and a
    caller-drawn test matrix omega fp32 [N, l] -> (L1 bf16 [K, r], L2 bf16
    [r, N], sigma fp32 [r])."""
    assert W.dtype == torch.float32 and W.is_cuda and W.is_contiguous()
    N, K = W.shape
    l = omega.shape[1]
    L1 = torch.empty((K, r), dtype=torch.bfloat16, device=W.device)
    L2 = torch.empty((r, N), dtype=torch.bfloat16, device=W.device)
    sigma = torch.empty(r, dtype=torch.float32, device=W.device)
    n = int(lib.wlq_lowrank_workspace(N, K, r, l))
    if n == 0:
        raise WlqError(ERR_SHAPE, "no low-rank split for N=%d K=%d r=%d l=%d" % (N, K, r, l))
    ws = torch.empty(n, dtype=torch.uint8, device=W.device)
    _check(lib.wlq_lowrank_split(_ptr(W), N, K, r, l, power_iters, _ptr(omega), _ptr(L1), _ptr(L2), _ptr(sigma),
                                 _ptr(ws), n, _stream(stream)))
    return L1, L2, sigma


def lowrank_residual(W: torch.Tensor, L1: torch.Tensor, L2: torch.Tensor, stream=None) -> torch.Tensor:
    """R = fp32(W - (L1 L2)^T), the part left for quantization."""
    N, K = W.shape
    r = L1.shape[1]
    R = torch.empty_like(W)
    _check(lib.wlq_lowrank_residual(_ptr(W), _ptr(L1), _ptr(L2), N, K, r, _ptr(R), _stream(stream)))
    return R


def nvfp4_scales_bytes(rows: int, K: int) -> int:
    return int(lib.wlq_nvfp4_scales_bytes(rows, K))


def nvfp4_quantize(X: torch.Tensor, stream=None):
    """NVFP4 quantization of fp32 or bf16 X [rows, K] -> (codes uint8 [rows, K/2]
    (two E2M1 codes a byte, low nibble first), scales uint8 (E4M3, the MMA's
    512-byte atom layout), gscale fp32 [2] = (tensor scale, amax))."""
    assert X.is_cuda and X.is_contiguous()
    rows, K = X.shape
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=X.device)
    scales = torch.empty(max(nvfp4_scales_bytes(rows, K), 16), dtype=torch.uint8, device=X.device)
    gscale = torch.empty(2, dtype=torch.float32, device=X.device)
    _check(lib.wlq_nvfp4_quantize(_ptr(X), _in_dtype(X), rows, K, _ptr(codes), _ptr(scales), _ptr(gscale),
                                  _stream(stream)))
    return codes, scales, gscale


def nvfp4_linear_into(y, xq, xs, xg, wq, ws, wg, N, K, x=None, bias=None, L1=None, L2=None, workspace=None,
                      stream=None):
    """y = deq(xq) deq(wq)^T [+ (x L1) L2] [+ b] (NVFP4 operands from nvfp4_quantize)."""
    M = xq.shape[0]
    r = 0 if L1 is None else L1.shape[1]
    out = OUT_F32 if y.dtype == torch.float32 else OUT_BF16
    if workspace is None:
        n = int(lib.wlq_nvfp4_linear_workspace(M, N, K, r))
        workspace = torch.empty(n, dtype=torch.uint8, device=y.device) if n else None
    ws_n = 0 if workspace is None else workspace.numel()
    _check(lib.wlq_nvfp4_linear(_ptr(xq), _ptr(xs), _ptr(xg), _ptr(x), M, _ptr(wq), _ptr(ws), _ptr(wg), N, K,
                                _ptr(bias), _ptr(L1), _ptr(L2), r, _ptr(y), out, _ptr(workspace), ws_n,
                                _stream(stream)))
    return y


def w4a4_workspace(M: int, N: int, K: int, r: int = 0, device="cuda"):
    n = int(lib.wlq_w4a4_workspace(M, N, K, r))
    return torch.empty(n, dtype=torch.uint8, device=device) if n else None


def w4a4_linear_into(y, x, wq, ws, wg, N, K, bias=None, L1=None, L2=None, workspace=None, stream=None):
    """The W4A4 forward from bf16 x [M, K]: x quantized to NVFP4 in the
    workspace, then y = deq(xq) deq(wq)^T [+ (x L1) L2] [+ b]."""
    M = x.shape[0]
    r = 0 if L1 is None else L1.shape[1]
    out = OUT_F32 if y.dtype == torch.float32 else OUT_BF16
    if workspace is None:
        workspace = w4a4_workspace(M, N, K, r, device=x.device)
    ws_n = 0 if workspace is None else workspace.numel()
    _check(lib.wlq_w4a4_linear(_ptr(x), M, _ptr(wq), _ptr(ws), _ptr(wg), N, K, _ptr(bias), _ptr(L1), _ptr(L2), r,
                               _ptr(y), out, _ptr(workspace), ws_n, _stream(stream)))
    return y


def get_status(stream=None) -> int:
    """Synchronise and return (and clear) the device error status as a code."""
    return int(lib.wlq_get_status(_stream(stream)))


def check_status(stream=None):
    _check(get_status(stream))


def probe_wait_timeout(timeout_ns: int, stream=None):
    _check(lib.wlq_probe_wait_timeout(timeout_ns, _stream(stream)))


def set_grid_limit(max_ctas: int):
    """Cap the CTAs of every later wlq_linear launch (0: no cap)."""
    lib.wlq_set_grid_limit(int(max_ctas))


def version() -> str:
    return lib.wlq_version().decode()
