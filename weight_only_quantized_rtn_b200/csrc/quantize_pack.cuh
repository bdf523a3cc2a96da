// quantize_pack.cuh -- RTN quantization written straight into the packed
// operand ("Joy-face_change_optimized" model card, files table and tools row:
// int8 with one scale per output channel, int4 grouped along K with gs 64 /
// 16; the "loader" step lays the codes out for the GEMM).
//
// The result is bit-identical to quantize (quantize.cuh) followed by pack
// (pack.cuh): same absmax, same scale, same exactly rounded codes, same
// offset-binary bytes and nibble order, same fp16 scale normalisation and row
// factors, same zero fill beyond N and K.  The int8 [N, K] code array is never
// written or read back: W is read once and the packed operand written once.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "quantize.cuh"
#include "pack.cuh"

namespace wlq {

// One CTA per padded output row (grid-stride over ceil(N/128)*128 rows).  The
// row's ceil(K/64)*64 inputs (zeros past K and for rows >= N) are held in
// registers: thread j takes runs of Q adjacent float4 at j + i*blockDim, so
// the lanes of a warp hold consecutive runs (Q = 2 for int8, 4 for int4: the
// faster of the two for each).
//  - int8: the row's absmax is reduced over the CTA (magnitude bit patterns,
//    as in quantize_rows_cta_kernel); a lane's eight codes leave as one
//    8-byte store of offset-binary bytes at its place in the row.
//  - int4: a lane holds quads of adjacent float4 (16 inputs, one 64-byte run
//    per slot), so a group of g inputs is g/16 adjacent lanes (one lane for
//    gs16); each group's absmax is reduced over its lanes; the row's
//    largest group scale (over the CTA) fixes the fp16 normalisation 2^e_n
//    and the row factor 2^-e_n; a lane's sixteen codes make two 32-bit words.
template <int FMT, int V>
__global__ void __launch_bounds__(1024) quantize_pack_rows_kernel(
    const float* __restrict__ W, int64_t N, int64_t K, int KT, int64_t rows, int qmax,
    float* __restrict__ scales, float* __restrict__ rowf, uint8_t* __restrict__ packed) {
    grid_dependency_sync();
    constexpr uint32_t TB = tile_bytes(FMT);
    constexpr int L = (FMT == FMT_W4G64) ? 16 : 4;  // int4: lanes per group (group / 4)
    constexpr int GS = 4 * L;                        // int4: group size
    constexpr int Q = (FMT == FMT_W8) ? 2 : 4;       // float4 per run of a lane
    __shared__ uint32_t part[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int K4 = static_cast<int>(K / 4);
    const int KP4 = KT * 16;  // float4s of the padded row
    const int64_t G = (FMT == FMT_W8) ? 1 : K / GS;
    bool bad = false;
    for (int64_t n = blockIdx.x; n < rows; n += gridDim.x) {
        const bool row_ok = n < N;
        const int i_row = static_cast<int>(n & 127);
        uint8_t* tiles = packed + static_cast<size_t>(n >> 7) * KT * TB;
        const float4* row = reinterpret_cast<const float4*>(W + (row_ok ? n : 0) * K);
        float4 v[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            // runs of Q float4 at run p = threadIdx.x + (i / Q) * blockDim: int8 pairs (8 inputs, one
            // 8-byte code store), int4 quads (16 inputs, two whole code words); measured best each
            const int idx = Q * (threadIdx.x + (i / Q) * blockDim.x) + (i % Q);
            v[i] = (row_ok && idx < K4) ? __ldcs(row + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if constexpr (FMT == FMT_W8) {
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                m = max(m, __float_as_uint(v[i].x) & 0x7FFFFFFFu);
                m = max(m, __float_as_uint(v[i].y) & 0x7FFFFFFFu);
                m = max(m, __float_as_uint(v[i].z) & 0x7FFFFFFFu);
                m = max(m, __float_as_uint(v[i].w) & 0x7FFFFFFFu);
            }
            for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
            if (lane == 0) part[warp] = m;
            __syncthreads();
            m = part[0];
            for (int w = 1; w < nwarps; ++w) m = max(m, part[w]);
            const bool row_bad = m >= 0x7F800000u;  // NaN or infinity in the row
            bad |= row_bad;
            const GroupScale g = group_scale(row_bad ? 0.0f : __uint_as_float(m), qmax);
            if (threadIdx.x == 0) {
                if (row_ok) scales[n] = g.s;
                rowf[n] = row_ok ? g.s : 0.0f;
            }
            const float h = 0.5f * g.s;
#pragma unroll
            for (int i = 0; i < V / 2; ++i) {
                const int p8 = threadIdx.x + i * blockDim.x;
                if (p8 >= KP4 / 2) continue;
                bool unused = false;
                const uint32_t ca = g.normal ? rtn4_f32(v[2 * i], g.s, g.inv, h) : pack_codes4(v[2 * i], g, qmax, unused);
                const uint32_t cb = g.normal ? rtn4_f32(v[2 * i + 1], g.s, g.inv, h)
                                             : pack_codes4(v[2 * i + 1], g, qmax, unused);
                const int k = 8 * p8;  // inputs k..k+7 of block k/64, run (k%64)/16, bytes k%16 (0 or 8)
                *reinterpret_cast<uint2*>(tiles + (k >> 6) * TB + ((k >> 4) & 3) * 2048 + 16 * i_row + (k & 15)) =
                    make_uint2(ca ^ 0x80808080u, cb ^ 0x80808080u);  // offset binary q + 128
            }
            __syncthreads();  // part[] is rewritten for the next row
        } else {
            // each lane holds V / 4 slots of 16 adjacent inputs; a group is L16 = GS / 16 adjacent lanes
            // (one lane for gs16).  Group absmax (0 for a group holding a NaN or infinity) reduced over
            // its lanes, and the row's largest group scale over the CTA (scales are non-negative
            // floats: their bit patterns order them)
            constexpr int V4 = V / 4;
            constexpr int L16 = GS / 16;
            uint32_t gm[V4];
#pragma unroll
            for (int i = 0; i < V4; ++i) {
                uint32_t m = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 a = v[4 * i + j];
                    m = max(m, max(max(__float_as_uint(a.x) & 0x7FFFFFFFu, __float_as_uint(a.y) & 0x7FFFFFFFu),
                                   max(__float_as_uint(a.z) & 0x7FFFFFFFu, __float_as_uint(a.w) & 0x7FFFFFFFu)));
                }
                for (int off = L16 >> 1; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
                const bool gbad = m >= 0x7F800000u;
                bad |= gbad;
                gm[i] = gbad ? 0u : m;
            }
            // The warp holds V4 * GPW groups (GPW = 32 / L16 per slot).  Lane j takes groups j, j + 32,
            // ...: the IEEE division and the reciprocal once per group rather than once per lane of
            // it; the results go back to each group's lanes by shuffle.
            constexpr int GPW = 32 / L16;
            constexpr int NGW = V4 * GPW;
            constexpr int PER_LANE = (NGW + 31) / 32;
            float sj[PER_LANE], ij[PER_LANE];
            uint32_t smax = 0;
#pragma unroll
            for (int t = 0; t < PER_LANE; ++t) {
                const int j = lane + 32 * t, ji = j / GPW, jg = j % GPW;
                uint32_t mj = 0;
#pragma unroll
                for (int i = 0; i < V4; ++i) {
                    const uint32_t mi = __shfl_sync(0xffffffffu, gm[i], jg * L16);
                    if (ji == i) mj = mi;
                }
                const GroupScale gs = group_scale(__uint_as_float(mj), qmax);
                sj[t] = gs.s;
                ij[t] = gs.inv;
                if (j < NGW) smax = max(smax, __float_as_uint(gs.s));
            }
            for (int off = 16; off > 0; off >>= 1) smax = max(smax, __shfl_xor_sync(0xffffffffu, smax, off));
            if (lane == 0) part[warp] = smax;
            __syncthreads();
            smax = part[0];
            for (int w = 1; w < nwarps; ++w) smax = max(smax, part[w]);
            const float S = __uint_as_float(smax);
            float rf = 0.0f;
            if (row_ok && S > 0.0f) {
                int ex;
                frexpf(S, &ex);             // S in [2^(ex-1), 2^ex)
                rf = ldexpf(1.0f, ex - 9);  // 2^-e_n with e_n = 9 - ex
            }
            if (threadIdx.x == 0) rowf[n] = rf;
            const int sh = (rf > 0.0f) ? -ilogbf(rf) : 0;  // s * 2^sh = s / rf exactly
            const int KP16 = KP4 / 4;
#pragma unroll
            for (int i = 0; i < V4; ++i) {
                const int p16 = threadIdx.x + i * blockDim.x;  // this lane's 16 inputs: k = 16 p16 ..
                const int k = 16 * p16;
                // this slot's group scale, from the lane that worked it out (group i * GPW + lane / L16:
                // the same lane slot t = i * GPW / 32 for every lane, since GPW divides 32)
                const int src_t = (i * GPW) / 32;
                const int src = (i * GPW) % 32 + lane / L16;
                GroupScale gs;
                gs.s = __shfl_sync(0xffffffffu, sj[src_t], src);
                gs.inv = __shfl_sync(0xffffffffu, ij[src_t], src);
                gs.normal = gs.s >= 1.17549435e-38f;
                uint32_t c[4];
                if (gs.normal) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) c[j] = rtn4_f32(v[4 * i + j], gs.s, gs.inv, 0.5f * gs.s);
                } else {  // rare: a subnormal (or zero) scale takes the fp64 path
                    bool unused = false;
                    gs.inv64 = (gs.s > 0.0f) ? 1.0 / static_cast<double>(gs.s) : 0.0;
#pragma unroll
                    for (int j = 0; j < 4; ++j) c[j] = pack_codes4(v[4 * i + j], gs, qmax, unused);
                }
                // sixteen nibbles (q + 8): the low nibble of each code byte with its top bit flipped is
                // q + 8 (|q| <= 7, no carry between bytes); in each word of eight, codes t = 0..3 go to
                // nibbles 0, 4, 1, 5 and t = 4..7 to nibbles 2, 6, 3, 7
                uint32_t wn[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t x = c[j] ^ 0x08080808u;
                    wn[j] = (x & 0xFu) | ((x >> 12) & 0xF0u) | ((x << 8) & 0xF0000u) | ((x >> 4) & 0xF00000u);
                }
                if (p16 >= KP16) continue;
                uint8_t* blk = tiles + (k >> 6) * TB;  // words (k%32)/8 and +1 of run (k%64)/32
                *reinterpret_cast<uint2*>(blk + ((k >> 5) & 1) * 2048 + 16 * i_row + 4 * ((k >> 3) & 3)) =
                    make_uint2(wn[0] | (wn[1] << 8), wn[2] | (wn[3] << 8));
                if ((p16 & (L16 - 1)) == 0) {  // first lane of the group: its scales
                    const int64_t gi = k / GS;
                    const bool real = row_ok && gi < G;
                    if (real) scales[n * G + gi] = gs.s;
                    const __half h16 = (real && rf != 0.0f) ? __float2half_rn(ldexpf(gs.s, sh)) : __float2half_rn(0.0f);
                    if constexpr (FMT == FMT_W4G64)
                        *reinterpret_cast<__half*>(blk + 4096 + 2 * i_row) = h16;
                    else  // group (k%64)/16: half ((k%64)/32), slot ((k%32)/16)
                        *reinterpret_cast<__half*>(blk + 4096 + 512 * ((k >> 5) & 1) + 4 * i_row + 2 * ((k >> 4) & 1)) = h16;
                }
            }
            __syncthreads();  // part[] is rewritten for the next row
        }
    }
    if (bad) raise_error(ERRBIT_NONFINITE);
}

}  // namespace wlq
