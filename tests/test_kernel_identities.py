"""Bit-level identities the CUDA kernels rely on, restated in numpy and
checked exhaustively on the host (no GPU).  They are implementation
arithmetic, not the method: no passage of the pages defines them; the GPU
parity tests check the kernels that use them against the oracle.

- int4 packing, byte-parallel nibble placement (fused quantize-pack): four
  two's-complement codes q in [-8, 7], one per byte of a word, become the
  offset-binary nibbles q + 8 at nibble positions 0, 4, 1, 5 by one xor and
  four shift-and-mask terms; the next four codes land at 2, 6, 3, 7.
- int8 codes to fp16 (few-token kernel): the byte permute that puts 0x64
  above an offset-binary byte q + 128 reads as the fp16 1024 + q + 128, and
  one fp16 subtraction of 1152 leaves q exactly.
- int8 codes to bf16 (tensor-core GEMM): a byte under 0x4B (as fp32, 2^23 +
  the byte), one packed fp32 subtraction of 2^23 + 128 and a permute of the
  two upper halves give bf16 q exactly.
- int4 codes to fp16 (every int4 engine): a nibble OR-ed into 0x6400 reads
  as 1024 + n (low nibble of a half) or 1024 + 16 n (high nibble); less 1032,
  or times 1/16 less 72, leaves n - 8 exactly; with the packed nibble order
  the four results of a word are the consecutive code pairs (0,1) .. (6,7).
- x to fp16 (few-token kernel): a bf16 row whose largest magnitude has
  exponent field E is scaled by 2^e, e = min(126, 141 - E) (e = 0 for a
  non-finite maximum): nothing overflows fp16, the largest lands in
  [2^14, 2^15) when E >= 15, and every scaled value of at least 2^-17 (so
  every value within 2^-32 of the largest) converts to fp16 exactly.
"""
import numpy as np


def _nibble_pos(t):
    # the packed int4 layout: code t of a group of eight at nibble (t odd: 4 + t/2, even: t/2)
    return 4 + (t >> 1) if t & 1 else t >> 1


def _place_byte_parallel(c_lo, c_hi):
    """Two words of four code bytes each -> one 32-bit word of eight nibbles."""
    def four(c):
        x = c ^ np.uint32(0x08080808)
        return ((x & np.uint32(0xF)) | ((x >> np.uint32(12)) & np.uint32(0xF0)) |
                ((x << np.uint32(8)) & np.uint32(0xF0000)) | ((x >> np.uint32(4)) & np.uint32(0xF00000)))
    return four(c_lo) | (four(c_hi) << np.uint32(8))


def _place_per_nibble(codes8):
    """Eight codes -> word, one nibble at a time."""
    w = 0
    for t, q in enumerate(codes8):
        w |= ((int(q) + 8) & 0xF) << (4 * _nibble_pos(t))
    return w


def _words(codes):
    """[n, 4] int8 codes -> [n] uint32 words, byte j = code j."""
    return np.ascontiguousarray(codes.astype(np.int8)).view(np.uint32).reshape(-1)


def test_int4_byte_parallel_nibble_placement_exhaustive_per_position():
    # every code value at every one of the eight positions, the others random
    g = np.random.default_rng(0)
    for t in range(8):
        codes = g.integers(-8, 8, (16, 8)).astype(np.int8)
        codes[:, t] = np.arange(-8, 8)
        got = _place_byte_parallel(_words(codes[:, :4]), _words(codes[:, 4:]))
        want = np.array([_place_per_nibble(c) for c in codes], dtype=np.uint32)
        np.testing.assert_array_equal(got, want)


def test_int4_byte_parallel_nibble_placement_random_words():
    g = np.random.default_rng(1)
    codes = g.integers(-8, 8, (20000, 8)).astype(np.int8)
    got = _place_byte_parallel(_words(codes[:, :4]), _words(codes[:, 4:]))
    want = np.array([_place_per_nibble(c) for c in codes], dtype=np.uint32)
    np.testing.assert_array_equal(got, want)


def _prmt(a, b, sel):
    """PTX prmt.b32 (default mode): byte i of the result is byte (sel >> 4i) & 7
    of the eight bytes {b, a} (a = bytes 0-3), sign-replicated when bit 3 of
    that selector nibble is set."""
    src = [(a >> (8 * k)) & 0xFF for k in range(4)] + [(b >> (8 * k)) & 0xFF for k in range(4)]
    out = 0
    for i in range(4):
        s = (sel >> (4 * i)) & 0xF
        v = src[s & 7]
        if s & 8:
            v = 0xFF if v & 0x80 else 0x00
        out |= v << (8 * i)
    return out


def _f16_pair(u32):
    return np.array([u32 & 0xFFFF, u32 >> 16], dtype=np.uint16).view(np.float16)


def test_int8_codes_to_fp16_by_byte_permute_and_one_subtraction():
    k1152 = np.float16(1152.0)
    assert np.array([0x6480], dtype=np.uint16).view(np.float16)[0] == k1152
    for q in range(-128, 128):
        u = (q + 128) & 0xFF                                   # offset-binary byte
        h = np.array([0x6400 | u], dtype=np.uint16).view(np.float16)[0]
        assert float(h) == 1024.0 + u
        d = h - k1152                                          # fp16 arithmetic
        assert d.dtype == np.float16 and float(d) == float(q)
    # the two selectors pick bytes (0, 1) and (2, 3) of a word, each under 0x64
    g = np.random.default_rng(2)
    for _ in range(2000):
        q4 = g.integers(-128, 128, 4)
        w = int(np.array((q4 + 128) & 0xFF, dtype=np.uint8).view(np.uint32)[0])
        lo = _f16_pair(_prmt(w, 0x64646464, 0x4140)) - k1152
        hi = _f16_pair(_prmt(w, 0x64646464, 0x4342)) - k1152
        np.testing.assert_array_equal(np.concatenate([lo, hi]).astype(np.float64), q4.astype(np.float64))


def _bf16_values(bits):
    return (np.asarray(bits, dtype=np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _row_exponent(E):
    return 0 if E >= 255 else min(126, 141 - E)


def test_x_rescale_to_fp16_exhaustive_over_bf16():
    pos = np.arange(1, 0x7F80, dtype=np.uint32)              # every positive finite bf16
    vals = _bf16_values(pos)
    fields = pos >> np.uint32(7)
    for E in range(0, 255):
        e = _row_exponent(E)
        mask = fields <= E                                   # values a row with that maximum can hold
        y = vals[mask] * 2.0 ** e
        assert y.max() < 2.0 ** 15                           # never beyond fp16's range
        if E >= 15:
            top = vals[fields == E] * 2.0 ** e
            assert top.min() >= 2.0 ** 14 and top.max() < 2.0 ** 15
        big = y >= 2.0 ** -17
        conv = y[big].astype(np.float16).astype(np.float64)
        np.testing.assert_array_equal(conv, y[big])           # exact from 2^-17 up
        # 2^-17 is at most 2^-32 of the largest when that largest is in [2^14, 2^15)
        if E >= 15:
            assert 2.0 ** -17 <= 2.0 ** -32 * (2.0 ** 15)
    # a non-finite maximum (field 255) leaves the row unscaled
    assert _row_exponent(255) == 0
    # the inverse factor 2^-e is a normal float for every e used
    es = {_row_exponent(E) for E in range(0, 256)}
    assert min(es) >= -126 and max(es) <= 126
    for e in es:
        inv = np.float32(2.0 ** -e)
        assert np.isfinite(inv) and inv >= np.finfo(np.float32).tiny and float(inv) * 2.0 ** e == 1.0


def _f32(u):
    return np.array([u], dtype=np.uint32).view(np.float32)[0]


def test_int8_codes_to_bf16_by_magic_float():
    magic = np.float32(2.0 ** 23 + 128)
    assert _f32(0x4B000080) == magic
    g = np.random.default_rng(3)
    words = [int(v) for v in g.integers(0, 2 ** 32, 3000, dtype=np.uint64)]
    words += [int(np.array([b, b ^ 0xFF, (b + 1) & 0xFF, (b * 7) & 0xFF], dtype=np.uint8).view(np.uint32)[0])
              for b in range(256)]
    for w in words:
        q = [((w >> (8 * k)) & 0xFF) - 128 for k in range(4)]       # offset-binary bytes
        for sel_lo, sel_hi, pair in ((0x7440, 0x7441, q[0:2]), (0x7442, 0x7443, q[2:4])):
            a = _f32(_prmt(w, 0x4B000000, sel_lo)) - magic           # fp32 arithmetic
            b = _f32(_prmt(w, 0x4B000000, sel_hi)) - magic
            lo = int(np.array([a], dtype=np.float32).view(np.uint32)[0])
            hi = int(np.array([b], dtype=np.float32).view(np.uint32)[0])
            out = _prmt(lo, hi, 0x7632)                              # the two upper halves
            bf = (np.array([out & 0xFFFF, out >> 16], dtype=np.uint32) << np.uint32(16)).view(np.float32)
            np.testing.assert_array_equal(bf.astype(np.float64), np.array(pair, dtype=np.float64))


def _f16x2(u32):
    return np.array([u32 & 0xFFFF, u32 >> 16], dtype=np.uint16).view(np.float16).astype(np.float64)


def _nibbles_to_pairs(w):
    """The int4 dequantise of one packed word, unit group scale: four fp16
    pairs, each rounded once as the fp16 subtract / fused multiply-add does."""
    def f16(x):
        return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)
    w8 = w >> 8
    p0 = f16(_f16x2((w & 0x000F000F) | 0x64006400) - 1032.0)
    p1 = f16(_f16x2((w & 0x00F000F0) | 0x64006400) * (1.0 / 16.0) - 72.0)
    p2 = f16(_f16x2((w8 & 0x000F000F) | 0x64006400) - 1032.0)
    p3 = f16(_f16x2((w8 & 0x00F000F0) | 0x64006400) * (1.0 / 16.0) - 72.0)
    return np.concatenate([p0, p1, p2, p3])


def test_int4_packed_word_dequantises_to_consecutive_code_pairs():
    g = np.random.default_rng(4)
    cases = [g.integers(-8, 8, 8) for _ in range(3000)]
    for t in range(8):                                   # every value at every position
        for q in range(-8, 8):
            c = g.integers(-8, 8, 8)
            c[t] = q
            cases.append(c)
    for codes in cases:
        w = _place_per_nibble(codes)
        np.testing.assert_array_equal(_nibbles_to_pairs(w), codes.astype(np.float64))
