"""CPU oracle for the weight-only quantized Linear -- TEST INFRASTRUCTURE ONLY.

A plain fp64 C statement of RTN quantization and of the quantized Linear (see
``wlq_oracle.c`` for the arithmetic and the pages each step follows).  It is
independent of the CUDA library: the two share no code, and the oracle never
calls the library or the library the oracle.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import it.

Parity: every function here is pinned by tests that do not re-use it
(brute-force enumeration, closed-form bounds, invariants, special cases that
reduce to library routines).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wlq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

OK, ERR_ARG, ERR_NONFINITE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, strict IEEE: no contraction)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(path: str):
    """Load an oracle shared object and declare its entry points."""
    lib = ctypes.CDLL(path)
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.oracle_quantize.argtypes = [vp, i64, i64, i32, i32, vp, vp]
    lib.oracle_dequantize.argtypes = [vp, vp, i64, i64, i32, vp]
    lib.oracle_linear.argtypes = [vp, i64, i64, vp, vp, i64, i32, vp, vp, vp, i32, vp]
    lib.oracle_quantize_ex.argtypes = [vp, i32, i64, i64, i32, i32, i32, vp, vp]
    lib.oracle_quantize_fp8.argtypes = [vp, i32, i64, i64, i32, vp, vp]
    lib.oracle_lowrank_residual.argtypes = [vp, vp, vp, i64, i64, i32, vp]
    lib.oracle_nvfp4_quantize.argtypes = [vp, i32, i64, i64, vp, vp, vp]
    lib.oracle_nvfp4_dequantize.argtypes = [vp, vp, ctypes.c_float, i64, i64, vp]
    lib.oracle_nvfp4_linear.argtypes = [vp, vp, ctypes.c_float, vp, i64, i64, vp, vp, ctypes.c_float, i64,
                                        vp, vp, vp, i32, vp]
    for f in (lib.oracle_quantize, lib.oracle_dequantize, lib.oracle_linear, lib.oracle_quantize_ex,
              lib.oracle_quantize_fp8, lib.oracle_lowrank_residual, lib.oracle_nvfp4_quantize,
              lib.oracle_nvfp4_dequantize, lib.oracle_nvfp4_linear):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class OracleError(RuntimeError):
    pass


def _check(rc):
    if rc == ERR_NONFINITE:
        raise OracleError("non-finite weight")
    if rc != OK:
        raise OracleError("invalid argument (rc=%d)" % rc)


def groups_of(K: int, group: int) -> int:
    return 1 if group == 0 else K // group


def quantize(W: np.ndarray, bits: int, group: int):
    """RTN symmetric quantization: returns (codes int8 [N,K], scales fp32 [N,G])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.empty((N, K), np.int8)
    scales = np.empty((N, groups_of(K, group)), np.float32)
    _check(_load().oracle_quantize(_p(W), N, K, bits, group, _p(codes), _p(scales)))
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, group: int) -> np.ndarray:
    """deq[n,k] = q[n,k] * s[n, k/g], exact in fp64."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    N, K = codes.shape
    out = np.empty((N, K), np.float64)
    _check(_load().oracle_dequantize(_p(codes), _p(scales), N, K, group, _p(out)))
    return out


def linear(x_bits: np.ndarray, codes: np.ndarray, scales: np.ndarray, group: int,
           bias_bits=None, L1_bits=None, L2_bits=None) -> np.ndarray:
    """y = x deq(codes, scales)^T [+ (x L1) L2] [+ b] in fp64.

    x_bits, bias_bits, L1_bits, L2_bits are bf16 bit patterns (uint16):
    x [M,K], bias [N], L1 [K,r], L2 [r,N].
    """
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    M, K = x_bits.shape
    N = codes.shape[0]
    assert codes.shape[1] == K
    r = 0
    if L1_bits is not None:
        L1_bits = np.ascontiguousarray(L1_bits, dtype=np.uint16)
        L2_bits = np.ascontiguousarray(L2_bits, dtype=np.uint16)
        r = L1_bits.shape[1]
        assert L1_bits.shape == (K, r) and L2_bits.shape == (r, N)
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        assert bias_bits.shape == (N,)
    y = np.empty((M, N), np.float64)
    _check(_load().oracle_linear(_p(x_bits), M, K, _p(codes), _p(scales), N, group,
                                 _p(bias_bits), _p(L1_bits), _p(L2_bits), r, _p(y)))
    return y


SCALE_F32, SCALE_F16, SCALE_BF16 = 0, 1, 2


def quantize_ex(W: np.ndarray, bits: int, group: int, scale_dtype: int = SCALE_F32):
    """RTN for 2..8 bits with a 32- or 16-bit stored scale.

    W: fp32 array, or uint16 bf16 bit patterns.  Returns (codes int8 [N,K],
    scale values fp32 [N,G]: the stored scales, exactly)."""
    if W.dtype == np.uint16:
        W = np.ascontiguousarray(W)
        w_dtype = 1
    else:
        W = np.ascontiguousarray(W, dtype=np.float32)
        w_dtype = 0
    N, K = W.shape
    codes = np.empty((N, K), np.int8)
    scales = np.empty((N, groups_of(K, group)), np.float32)
    _check(_load().oracle_quantize_ex(_p(W), w_dtype, N, K, bits, group, scale_dtype, _p(codes), _p(scales)))
    return codes, scales


def quantize_fp8(W: np.ndarray, group: int):
    """fp8 e4m3 block quantization: returns (codes uint8 e4m3 bits [N,K], scales fp32 [N,G])."""
    if W.dtype == np.uint16:
        W = np.ascontiguousarray(W)
        w_dtype = 1
    else:
        W = np.ascontiguousarray(W, dtype=np.float32)
        w_dtype = 0
    N, K = W.shape
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N, groups_of(K, group)), np.float32)
    _check(_load().oracle_quantize_fp8(_p(W), w_dtype, N, K, group, _p(codes), _p(scales)))
    return codes, scales


def _bf16_rne_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns, round to nearest even in one step (via the
    exact fp64 value: scale to 8 significant bits and round half to even).
    Element by element, written with whole-array operations."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                           # |x| = m 2^e, m in [0.5, 1) (e = 0 for x = 0)
    lead = np.maximum(e - 1, -126)               # bf16 normals from 2^-126, subnormals below
    spacing = np.ldexp(1.0, lead - 7)            # bf16 spacing in that binade
    q = a / spacing                              # exact: spacing is a power of two
    f = np.floor(q)
    d = q - f
    r = np.where((d > 0.5) | ((d == 0.5) & (np.fmod(f, 2.0) == 1.0)), f + 1.0, f)
    f32 = (r * spacing).astype(np.float32)       # exact: at most 8 significant bits
    bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
    return bits | np.where(np.signbit(x), np.uint16(0x8000), np.uint16(0)).astype(np.uint16)


def _bf16_value(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def lowrank_split(W: np.ndarray, r: int):
    """Top-r SVD split before quantizing the residual ("Nunchaku Lite" article,
    why it matters / how it works: the hardest part of the weights goes to a
    16-bit low-rank branch, the rest is quantized).

    With W [N, K] and the Linear y = x W^T, the branch is y += (x L1) L2 with
    L1 [K, r], L2 [r, N], so L1 L2 approximates W^T:  W^T = U S V^T (fp64
    SVD), L1 = U_r S_r^(1/2), L2 = S_r^(1/2) V_r^T.  L1 and L2 are stored in
    bf16 (round to nearest even); the residual R = W - (bf16(L1) bf16(L2))^T
    is formed in fp64 and rounded to fp32 for quantization.

    Returns dict(L1 [K,r] fp64, L2 [r,N] fp64, L1_bits, L2_bits (bf16 bit
    patterns), R [N,K] fp32, sigma (all singular values, descending)).  The
    factors are unique only up to the sign of each component (their product
    is unique when the singular values are distinct)."""
    W = np.asarray(W, dtype=np.float64)
    U, S, Vt = np.linalg.svd(W.T, full_matrices=False)
    sq = np.sqrt(S[:r])
    L1 = U[:, :r] * sq[None, :]
    L2 = sq[:, None] * Vt[:r, :]
    L1b, L2b = _bf16_rne_bits(L1), _bf16_rne_bits(L2)
    R = (W - (_bf16_value(L1b) @ _bf16_value(L2b)).T).astype(np.float32)
    return dict(L1=L1, L2=L2, L1_bits=L1b, L2_bits=L2b, R=R, sigma=S)


def lowrank_residual(W: np.ndarray, L1_bits: np.ndarray, L2_bits: np.ndarray) -> np.ndarray:
    """R = fp32(W - (L1 L2)^T): the part of W the low-rank branch leaves for
    quantization ("Nunchaku Lite" article, why it matters), for given bf16
    factors (bit patterns L1 [K, r], L2 [r, N]).  The sum over the rank is
    taken in fp64 in increasing j, then rounded once to fp32 (``wlq_oracle.c``)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    L1_bits = np.ascontiguousarray(L1_bits, dtype=np.uint16)
    L2_bits = np.ascontiguousarray(L2_bits, dtype=np.uint16)
    N, K = W.shape
    r = L1_bits.shape[1]
    assert L1_bits.shape == (K, r) and L2_bits.shape == (r, N)
    R = np.empty((N, K), np.float32)
    _check(_load().oracle_lowrank_residual(_p(W), _p(L1_bits), _p(L2_bits), N, K, r, _p(R)))
    return R


def nvfp4_quantize(X: np.ndarray):
    """NVFP4 quantization of a [rows, K] tensor (the 4-bit format of the W4A4
    path on Blackwell: "Nunchaku Lite" article, hardware and precision
    support): E2M1 codes, one E4M3 scale per 16 inputs of a row, one fp32
    tensor scale g = fp32(amax / 2688).  X: fp32, or uint16 bf16 bit patterns.
    Returns (codes uint8 [rows, K] (E2M1 bits, sign in bit 3), scales uint8
    [rows, K/16] (E4M3 bits), g)."""
    if X.dtype == np.uint16:
        X = np.ascontiguousarray(X)
        x_dtype = 1
    else:
        X = np.ascontiguousarray(X, dtype=np.float32)
        x_dtype = 0
    rows, K = X.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 16 if K % 16 == 0 else 1), np.uint8)
    g = ctypes.c_float(0.0)
    _check(_load().oracle_nvfp4_quantize(_p(X), x_dtype, rows, K, _p(codes), _p(scales), ctypes.byref(g)))
    return codes, scales, float(g.value)


def nvfp4_dequantize(codes: np.ndarray, scales: np.ndarray, g: float) -> np.ndarray:
    """x^ = q s_b g (exact, fp64 [rows, K])."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    _check(_load().oracle_nvfp4_dequantize(_p(codes), _p(scales), g, rows, K, _p(out)))
    return out


def nvfp4_linear(xq, xs, xg, x_bits, wq, ws, wg, bias_bits=None, L1_bits=None, L2_bits=None) -> np.ndarray:
    """The W4A4 Linear in fp64: y = deq(xq) deq(wq)^T [+ (x L1) L2] [+ b].

    xq/xs/xg, wq/ws/wg: NVFP4 codes, block scales and tensor scale of the
    activations [M, K] and the weights [N, K]; x_bits: the 16-bit activations
    (bf16 bit patterns, used by the low-rank branch only); bias [N], L1 [K, r],
    L2 [r, N]: bf16 bit patterns."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    xs = np.ascontiguousarray(xs, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    ws = np.ascontiguousarray(ws, dtype=np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    assert wq.shape[1] == K
    r = 0
    if L1_bits is not None:
        L1_bits = np.ascontiguousarray(L1_bits, dtype=np.uint16)
        L2_bits = np.ascontiguousarray(L2_bits, dtype=np.uint16)
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        r = L1_bits.shape[1]
        assert L1_bits.shape == (K, r) and L2_bits.shape == (r, N) and x_bits.shape == (M, K)
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        assert bias_bits.shape == (N,)
    y = np.empty((M, N), np.float64)
    _check(_load().oracle_nvfp4_linear(_p(xq), _p(xs), xg, _p(x_bits) if r else None, M, K, _p(wq), _p(ws), wg,
                                       N, _p(bias_bits), _p(L1_bits), _p(L2_bits), r, _p(y)))
    return y
