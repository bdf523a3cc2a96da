// gemv.cuh -- the weight-only quantized Linear for at most 16 tokens with a
// small x ("Joy-face_change_optimized" model card, files table: weight-only
// Linear; "Nunchaku Lite", how it works: 4-bit weights, 16-bit activations).
//
//   y[m,n] = rowf[n] * xs[m] * sum_k xin[m,k] * w16[n,k]  +  b[n]
//
// Same packed operand, row factors and x (bf16, or the fp16 x16 of the int4
// formats) as the other engines.  Here streaming the packed weights from HBM
// is the whole cost, so nothing stands between the weight bytes and the MMAs:
//
//  - one CTA per 32 output channels, no cluster, no K split across CTAs;
//  - 16 warps: warp w takes rows 16 (w % 2)..+15 of the CTA's 32 and K slice
//    w / 2 of 8; each lane loads its codes straight from global memory into
//    registers (four K blocks in flight), dequantises them and runs m16n8k16
//    warp MMAs (fp32 accumulate) against x fragments read from shared memory;
//  - x ([M][K], zero-padded to 8 or 16 tokens and to whole K blocks) is copied
//    to shared memory once per CTA by bulk copies, while the first weight
//    loads are in flight;
//  - the 8 K slices of each row are summed in slice order (deterministic) in
//    shared memory, then scaled, biased and stored.
//
// The input renumbering inside a 64-wide K block is the one of the skinny
// kernel: lane (g, t) takes inputs 16t..16t+15 of its rows, the run of 16
// codes the packed tile holds contiguously, and reads x the same way.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "pack.cuh"
#include "gemm.cuh"
#include "skinny.cuh"

namespace wlq {

constexpr int GV_SLICES = 8;                      // K slices per CTA
constexpr int GV_WARPS = 2 * GV_SLICES;           // x 2 row groups of 16
constexpr int GV_THREADS = GV_WARPS * 32;
constexpr int GV_ROWS = 32;                       // output channels per CTA
constexpr int GV_U = 4;                           // K blocks of codes in flight per warp

__host__ __device__ constexpr uint32_t gv_x_pitch(int KT) { return static_cast<uint32_t>(KT) * 128u + 16u; }

template <int FMT, int NB>
__global__ void __launch_bounds__(GV_THREADS, 1) gemv_kernel(const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* xsm = smem_raw + (((raw + 127u) & ~127u) - raw);      // [NB*8][pitch]
    const uint32_t pitch = gv_x_pitch(a.KT);
    float* red = reinterpret_cast<float*>(xsm + NB * 8 * pitch);   // [slices][2][32][NB*4]
    __shared__ uint64_t xbar;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rg = warp & 1, slice = warp >> 1;
    const int nt = blockIdx.x >> 2;                        // 128-channel tile of the packed operand
    const int row0 = (blockIdx.x & 3) * GV_ROWS + rg * 16 + g;  // rows row0, row0 + 8 of that tile
    const int kb_lo = slice * a.KT / GV_SLICES, kb_hi = (slice + 1) * a.KT / GV_SLICES;
    const int Mv = min(a.M, NB * 8);

    // x: zero what the copies do not cover (token rows >= M, inputs >= K),
    // then one bulk copy per token row
    if (threadIdx.x == 0) {
        mbar_init(&xbar, 1);
        fence_barrier_init();
    }
    const uint32_t row_bytes = static_cast<uint32_t>(a.K) * 2u;
    for (uint32_t i = threadIdx.x; i < static_cast<uint32_t>(NB * 8) * (pitch / 16u); i += GV_THREADS) {
        const uint32_t m = i / (pitch / 16u), off = (i % (pitch / 16u)) * 16u;
        if (static_cast<int>(m) >= Mv || off >= row_bytes)
            *reinterpret_cast<uint4*>(xsm + m * pitch + off) = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&xbar, static_cast<uint32_t>(Mv) * row_bytes);
        for (int m = 0; m < Mv; ++m)
            bulk_load(xsm + m * pitch, reinterpret_cast<const uint8_t*>(a.xg) + static_cast<size_t>(m) * row_bytes,
                      row_bytes, &xbar);
    }

    float acc[NB][4];
#pragma unroll
    for (int j = 0; j < NB; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    const uint8_t* band = a.packed + static_cast<size_t>(nt) * a.KT * a.wtile_bytes;
    bool have_x = false, bad = false;
    for (int kb = kb_lo; kb < kb_hi; kb += GV_U) {
        SkCodes<FMT> cv[GV_U];
#pragma unroll
        for (int j = 0; j < GV_U; ++j)
            if (kb + j < kb_hi) cv[j] = sk_load_codes<FMT>(band + static_cast<size_t>(kb + j) * a.wtile_bytes, row0, t);
        if (!have_x) {
            // bounded: on a timeout the error bit is set and the (garbage) sums
            // still flow to the end, so every thread reaches the barriers below
            if (!mbar_wait(&xbar, 0, a.timeout_ns)) bad = true;
            have_x = true;
        }
#pragma unroll
        for (int j = 0; j < GV_U; ++j) {
            if (kb + j >= kb_hi) break;
            uint32_t p0[8], p1[8];
            sk_convert<FMT>(cv[j], p0, p1);
            const uint8_t* xk = xsm + (kb + j) * 128 + 32 * t;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const uint8_t* xr = xk + (nb * 8 + g) * pitch;
                const uint4 u0 = *reinterpret_cast<const uint4*>(xr);
                const uint4 u1 = *reinterpret_cast<const uint4*>(xr + 16);
                const uint32_t b[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    if constexpr (FMT == FMT_W8)
                        mma16816_bf16(acc[nb], p0[2 * k4], p1[2 * k4], p0[2 * k4 + 1], p1[2 * k4 + 1], b[2 * k4],
                                      b[2 * k4 + 1]);
                    else
                        mma16816_f16(acc[nb], p0[2 * k4], p1[2 * k4], p0[2 * k4 + 1], p1[2 * k4 + 1], b[2 * k4],
                                     b[2 * k4 + 1]);
                }
            }
        }
    }
    if (!have_x && !mbar_wait(&xbar, 0, a.timeout_ns)) bad = true;  // a slice with no K blocks
    if (bad && lane == 0) raise_error(ERRBIT_TIMEOUT);

    // sum the slices in order, scale, add the bias, store
    float* mine = red + ((slice * 2 + rg) * 32 + lane) * (NB * 4);
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) mine[nb * 4 + e] = acc[nb][e];
    __syncthreads();
    if (slice != 0) return;
    float sum[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) sum[nb][e] = 0.0f;
    for (int sl = 0; sl < GV_SLICES; ++sl) {
        const float* p = red + ((sl * 2 + rg) * 32 + lane) * (NB * 4);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int e = 0; e < 4; ++e) sum[nb][e] += p[nb * 4 + e];
    }
    const int n0 = nt * 128 + row0, n1 = n0 + 8;
    const float rf0 = n0 < a.N ? a.rowf[n0] : 0.0f, rf1 = n1 < a.N ? a.rowf[n1] : 0.0f;
    const float b0 = (a.bias && n0 < a.N) ? bf16_to_f32(a.bias[n0]) : 0.0f;
    const float b1 = (a.bias && n1 < a.N) ? bf16_to_f32(a.bias[n1]) : 0.0f;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int m = nb * 8 + 2 * t + (e & 1);
            const int n = (e < 2) ? n0 : n1;
            if (m >= a.M || n >= a.N) continue;
            float v = sum[nb][e] * ((e < 2) ? rf0 : rf1);
            if constexpr (FMT != FMT_W8) v *= a.xs[m];
            store_y(a, m, n, v + ((e < 2) ? b0 : b1));
        }
    }
}

}  // namespace wlq
