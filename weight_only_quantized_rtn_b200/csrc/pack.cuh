// pack.cuh -- lay RTN codes and scales out for the tcgen05 GEMM (the pages'
// "loader" step: "Joy-face_change_optimized" model card, files table).
//
// Packed operand = ceil(N/128) x ceil(K/64) tiles, tile (nt, kb) at byte
// offset (nt * KT + kb) * tile_bytes, followed by NT*128 fp32 row factors.
//
// int8 tile (8192 B): four 2048-byte chunks; chunk c holds, for each of the
//   128 rows i, the 16 codes k = 64 kb + 16 c + [0,16) at bytes [16 i, 16 i + 16),
//   stored offset-binary (q + 128).  Row factor = the channel scale s[n].
// int4 tile (4096 B of codes + scales): two 2048-byte chunks; chunk c holds,
//   for each row i, the 32 codes k = 64 kb + 32 c + [0,32) in 16 bytes: four
//   32-bit words of 8 codes each, nibble q + 8.  Inside a word the code for
//   k-offset t sits at nibble t/2 when t is even and 4 + t/2 when t is odd, so
//   one mask-and-or yields the fp16 pair (k, k+1) in the (low, high) halves.
//   Scales follow as fp16(s * 2^e_n): gs64 -> [row i] at 4096 + 2 i;
//   gs16 -> [half c][row i][2] at 4096 + 512 c + 4 i.  Row factor = 2^-e_n
//   with e_n chosen so the row's largest scale lands in [2^8, 2^9).
// Everything beyond N rows or K inputs is encoded as code 0 / scale 0.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include "ptx.cuh"

namespace wlq {

enum WFmt : int { FMT_W8 = 0, FMT_W4G64 = 1, FMT_W4G16 = 2 };

__host__ __device__ constexpr uint32_t tile_bytes(int fmt) {
    return fmt == FMT_W8 ? 8192u : (fmt == FMT_W4G64 ? 4096u + 256u : 4096u + 1024u);
}

__device__ __forceinline__ int int4_nibble_pos(int t) { return (t & 1) ? 4 + (t >> 1) : (t >> 1); }

// int4: one warp per padded row, the fp32 factor the epilogue multiplies by.
__global__ void pack_rowfactor_kernel(const float* __restrict__ scales, int64_t N, int64_t G,
                                      int fmt, int64_t N_pad, float* __restrict__ rowf) {
    grid_dependency_sync();
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t n = w0; n < N_pad; n += nw) {
        float f = 0.0f;
        if (n < N) {
            if (fmt == FMT_W8) {
                f = scales[n];
            } else {
                float S = 0.0f;
                for (int64_t g = lane; g < G; g += 32) S = fmaxf(S, scales[n * G + g]);
                for (int off = 16; off > 0; off >>= 1) S = fmaxf(S, __shfl_xor_sync(0xffffffffu, S, off));
                if (S > 0.0f) {
                    int ex;
                    frexpf(S, &ex);             // S in [2^(ex-1), 2^ex)
                    f = ldexpf(1.0f, ex - 9);   // 2^-e_n with e_n = 9 - ex
                }
            }
        }
        if (lane == 0) rowf[n] = f;
    }
}

// One CTA (128 threads) per tile.  Codes are read as 8-byte runs (8 inputs of
// one row; rows start 8-byte aligned because K % 8 == 0), so a warp reads
// four rows' 64 contiguous bytes each; each thread issues all eight of its
// loads before its first store.  For int8 the K-block-0 CTAs also write the
// row factors (the channel scales); int4 row factors come from
// pack_rowfactor_kernel, which runs first.
__global__ void __launch_bounds__(128) pack_tiles_kernel(
    const int8_t* __restrict__ codes, const float* __restrict__ scales, int64_t N, int64_t K,
    int64_t G, int fmt, int KT, float* __restrict__ rowf, uint8_t* __restrict__ packed) {
    grid_dependency_sync();
    const int64_t tile = blockIdx.x;
    const int64_t nt = tile / KT;
    const int kb = static_cast<int>(tile % KT);
    const int64_t k0 = static_cast<int64_t>(kb) * 64;
    uint8_t* blk = packed + tile * tile_bytes(fmt);
    uint2 v[8];
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int idx = threadIdx.x + 128 * it;
        const int i = idx >> 3, part = idx & 7;
        const int64_t n = nt * 128 + i, k = k0 + 8 * part;
        v[it] = (n < N && k < K) ? __ldg(reinterpret_cast<const uint2*>(codes + n * K + k)) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int idx = threadIdx.x + 128 * it;
        const int i = idx >> 3, part = idx & 7;
        if (fmt == FMT_W8) {
            // offset binary q + 128 of a two's-complement byte is q ^ 0x80
            const uint2 o = make_uint2(v[it].x ^ 0x80808080u, v[it].y ^ 0x80808080u);
            *reinterpret_cast<uint2*>(blk + (part >> 1) * 2048 + 16 * i + (part & 1) * 8) = o;
        } else {
            const uint32_t b[2] = {v[it].x, v[it].y};
            uint32_t w = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const uint32_t u = ((b[t >> 2] >> (8 * (t & 3))) + 8u) & 0xFu;  // (q + 8) mod 16
                w |= u << (4 * int4_nibble_pos(t));
            }
            *reinterpret_cast<uint32_t*>(blk + (part >> 2) * 2048 + 16 * i + 4 * (part & 3)) = w;
        }
    }
    const int i = threadIdx.x;
    const int64_t n = nt * 128 + i;
    const bool row_ok = n < N;
    if (fmt == FMT_W8) {
        if (kb == 0) rowf[n] = row_ok ? scales[n] : 0.0f;
        return;
    }
    const float rf = row_ok ? rowf[n] : 0.0f;
    const int sh = (rf > 0.0f) ? -ilogbf(rf) : 0;  // s * 2^sh = s / rf exactly
    auto scale16 = [&](int64_t g) -> __half {
        if (!row_ok || rf == 0.0f || g * (fmt == FMT_W4G64 ? 64 : 16) >= K) return __float2half_rn(0.0f);
        return __float2half_rn(ldexpf(scales[n * G + g], sh));
    };
    if (fmt == FMT_W4G64) {
        *reinterpret_cast<__half*>(blk + 4096 + 2 * i) = scale16(k0 / 64);
    } else {
        for (int c = 0; c < 2; ++c) {
            const __half2 p = __halves2half2(scale16(k0 / 16 + 2 * c), scale16(k0 / 16 + 2 * c + 1));
            *reinterpret_cast<__half2*>(blk + 4096 + 512 * c + 4 * i) = p;
        }
    }
}

// Inverse of the code layout: one CTA per tile.
__global__ void __launch_bounds__(128) unpack_tiles_kernel(const uint8_t* __restrict__ packed,
                                                           int64_t N, int64_t K, int fmt, int KT,
                                                           int8_t* __restrict__ codes) {
    grid_dependency_sync();
    const int64_t tile = blockIdx.x;
    const int64_t nt = tile / KT;
    const int kb = static_cast<int>(tile % KT);
    const int i = threadIdx.x;
    const int64_t n = nt * 128 + i;
    if (n >= N) return;
    const int64_t k0 = static_cast<int64_t>(kb) * 64;
    const uint8_t* blk = packed + tile * tile_bytes(fmt);
    if (fmt == FMT_W8) {
        for (int c = 0; c < 4; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(blk + c * 2048 + 16 * i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            for (int j = 0; j < 16; ++j) {
                const int64_t k = k0 + 16 * c + j;
                if (k < K) codes[n * K + k] = static_cast<int8_t>(static_cast<int>((w[j >> 2] >> (8 * (j & 3))) & 0xFFu) - 128);
            }
        }
        return;
    }
    for (int c = 0; c < 2; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(blk + c * 2048 + 16 * i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        for (int j = 0; j < 4; ++j)
            for (int t = 0; t < 8; ++t) {
                const int64_t k = k0 + 32 * c + 8 * j + t;
                if (k < K)
                    codes[n * K + k] = static_cast<int8_t>(static_cast<int>((w[j] >> (4 * int4_nibble_pos(t))) & 0xFu) - 8);
            }
    }
}

}  // namespace wlq
