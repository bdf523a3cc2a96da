"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no step of the quantization or of the Linear: it only draws
random tensors (numpy PCG64, ``default_rng``) and rounds fp32 draws to bf16 bit
patterns (round to nearest, ties to even), so that the oracle and the CUDA
library are fed byte-identical inputs.

Shapes follow the video DiT described on the "Joy-face_change_optimized"
model card (section "strip the text-stream weights", parameter table):
hidden size 4096, MLP size 16384, 4*4096^2 + 2*4096*16384 = 201 M Linear
parameters per block and stream.  Token counts follow 832x480 video with
16-pixel patches: 1560 tokens per latent frame, 6240 for four.
"""
from __future__ import annotations

import numpy as np

HIDDEN = 4096
MLP = 16384
RANK = 32


def rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(list(key))


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_f32(g: np.random.Generator, shape, std: float) -> np.ndarray:
    return (g.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def normal_bf16(g: np.random.Generator, shape, std: float) -> np.ndarray:
    return bf16_bits(normal_f32(g, shape, std))


def weight(seed: int, tag: int, N: int, K: int, std: float = 0.02,
           outlier_frac: float = 0.0, outlier_mult: float = 20.0) -> np.ndarray:
    """W fp32 [N, K] ~ N(0, std); optionally a seeded set of input columns
    (round(outlier_frac * K) of them) multiplied by outlier_mult."""
    g = rng(seed, tag)
    W = normal_f32(g, (N, K), std)
    n_out = int(round(outlier_frac * K))
    if n_out:
        cols = np.sort(g.permutation(K)[:n_out])
        W[:, cols] *= np.float32(outlier_mult)
    return W


def activations(seed: int, tag: int, M: int, K: int, std: float = 1.0) -> np.ndarray:
    """x bf16 bits [M, K] ~ N(0, std)."""
    return normal_bf16(rng(seed, tag, M), (M, K), std)


def bias(seed: int, tag: int, N: int, std: float = 0.01) -> np.ndarray:
    return normal_bf16(rng(seed, tag), (N,), std)


# ---------------------------------------------------------------------------
# The five workloads.  Each returns a dict of numpy arrays (bf16 as uint16 bit
# patterns, weights as fp32) plus the quantization recipe of every weight.
# ---------------------------------------------------------------------------

def tiny_w8(M: int = 64):
    """Tiny W8A16: x [64,256] N(0,1); W [512,256] N(0,0.02) int8 per channel;
    bias [512] N(0,0.01); seed 0."""
    return dict(x=activations(0, 1, M, 256), W=weight(0, 2, 512, 256),
                b=bias(0, 3, 512), bits=8, group=0)


def attn_w8(M: int, N: int = HIDDEN, K: int = HIDDEN):
    """DiT attention projection W8A16: W [4096,4096] N(0,0.02) with 1% of the
    input columns x20 (outlier channels), int8 per channel; x [M,4096];
    bias N(0,0.01); seed 1."""
    return dict(x=activations(1, 1, M, K),
                W=weight(1, 2, N, K, outlier_frac=0.01), b=bias(1, 3, N), bits=8, group=0)


def mlp_w4(M: int, which: str = "up"):
    """DiT MLP W4A16 RTN gs=64: up W [16384,4096], down W [4096,16384],
    N(0,0.02); x [M, K] N(0,1); seed 2.  When the pair runs chained, down
    consumes up's output instead of its own x."""
    if which == "up":
        N, K, tag = MLP, HIDDEN, 10
    else:
        N, K, tag = HIDDEN, MLP, 20
    return dict(x=activations(2, tag + 1, M, K), W=weight(2, tag + 2, N, K),
                b=bias(2, tag + 3, N), bits=4, group=64)


MIXED_LAYERS = (
    # name, N, K, bits, group
    ("q", HIDDEN, HIDDEN, 8, 0),
    ("k", HIDDEN, HIDDEN, 8, 0),
    ("v", HIDDEN, HIDDEN, 8, 0),
    ("o", HIDDEN, HIDDEN, 8, 0),
    ("up", MLP, HIDDEN, 4, 16),
    ("down", HIDDEN, MLP, 4, 16),
)


def mixed_block(M: int = 4096):
    """Mixed-precision DiT block: q/k/v/o int8 per channel, MLP up/down int4
    gs=16; x [4096,4096] N(0,1); seed 3."""
    layers = {}
    for i, (name, N, K, bits, group) in enumerate(MIXED_LAYERS):
        layers[name] = dict(W=weight(3, 10 * (i + 1), N, K), b=bias(3, 10 * (i + 1) + 1, N),
                            bits=bits, group=group)
    return dict(x=activations(3, 1, M, HIDDEN), layers=layers)


def svdq_w4_lr(M: int, N: int = HIDDEN, K: int = HIDDEN, r: int = RANK):
    """SVDQuant-style W4A16 + low-rank: L1 [K,r], L2 [r,N] ~ N(0,0.05) bf16
    (planted low-rank part), residual R [N,K] ~ N(0,0.02) quantized int4
    gs=64; x [M,K] N(0,1); seed 4."""
    return dict(x=activations(4, 1, M, K), W=weight(4, 2, N, K),
                L1=normal_bf16(rng(4, 3), (K, r), 0.05),
                L2=normal_bf16(rng(4, 4), (r, N), 0.05),
                b=bias(4, 5, N), bits=4, group=64)
