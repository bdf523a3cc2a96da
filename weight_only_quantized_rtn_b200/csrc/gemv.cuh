// gemv.cuh -- the weight-only quantized Linear for at most 16 tokens
// ("Joy-face_change_optimized" model card, files table: weight-only Linear;
// "Nunchaku Lite", how it works: 4-bit weights, 16-bit activations).
//
//   y[m,n] = rowf[n] * sum_k x[m,k] * w16[n,k]  +  b[n]
//
// Same packed operand and row factors as the other engines; x is the bf16
// input itself for every format (no preparation pass).  Here streaming the
// packed weights from HBM is the whole cost, so the kernel is built around
// that stream:
//
//  - a cluster of S CTAs takes one 128-channel tile of the packed operand, CTA
//    (cluster rank) q its K split q of kbps 64-wide blocks; clusters are
//    persistent over tiles;
//  - one producer thread (a warp of its own) streams the split's packed
//    blocks, four per ring slot
//    (one contiguous bulk copy of 17-32 KB: a bulk copy costs a fixed
//    ~0.2 us of the SM's copy engine, so small copies cannot keep up);
//  - all 16 compute warps work on the same landed block: int8, warp w takes
//    rows 32 (w % 4)..+31 and MMA K step w / 4 (16 inputs); int4, warp w takes
//    rows 16 (w % 8)..+15 and 32-input half w / 8.  Codes reach registers by
//    ldmatrix (8 rows x 16 bytes per matrix: conflict-free), are dequantised
//    in registers and feed m16n8k16 warp MMAs (fp32 accumulate) against x
//    fragments read from shared memory once per block;
//  - the CTA's x rows ([M][its K range]) are copied to shared memory once,
//    warp m row m, by 16-byte asynchronous copies; token rows >= M are never
//    read back into an output.  The warp then rewrites its row in place as
//    fp16 of x times 2^e_m, e_m chosen from the largest |x| of the token over
//    the CTA's K range so that it lands in [2^14, 2^15): bf16 values keep all
//    8 significand bits (only those below 2^-32 of the largest can round),
//    and the partials are multiplied back by 2^-e_m (exact) before they are
//    summed.  The MMAs are fp16: int8 codes become fp16 in two instructions a
//    pair (0x64 above the offset-binary byte is 1024 + c + 128, less 1152),
//    int4 codes times their group scale as in the other engines;
//  - the warps' partial sums are staged in shared memory and added in K-part
//    order; each thread then sends four adjacent rows of one token of the sum
//    to the CTA that owns them (rows [q' 128/S, (q'+1) 128/S) belong to CTA
//    q') with one 16-byte distributed-shared-memory store; one cluster
//    barrier later CTA q' adds the S partials of its rows in split order,
//    scales, biases and stores them.  The summation order is fixed: results
//    are reproducible.
//
// Inputs inside a 64-wide K block are renumbered for the MMA (the dot
// products are unchanged; x is read with the same renumbering):
//   int8: step s (inputs 16s..16s+15 of the block, packed chunk s): lane
//         (g, t) holds inputs 16s + 4t + {0, 1} as fragment columns 2t, 2t+1
//         and 16s + 4t + {2, 3} as columns 2t+8, 2t+9 -- the four bytes
//         ldmatrix hands lane (g, t) from a 16-byte row;
//   int4: half h (inputs 32h..32h+31, packed chunk h), sub-step j = 0, 1:
//         lane (g, t) holds inputs 32h + 8t + 4j + {0, 1} and + {2, 3} -- the
//         32-bit word t of the 16-byte row, eight nibbles.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "pack.cuh"
#include "gemm.cuh"

namespace wlq {

constexpr int GV_WARPS = 16;                      // compute warps
constexpr int GV_THREADS = (GV_WARPS + 1) * 32;   // + the producer warp
constexpr int GV_SLOT_KB = 4;                     // K blocks per ring slot (one bulk copy)
constexpr int GV_MAX_STAGES = 8;
constexpr int GV_MAX_SPLITS = 8;                  // portable cluster size

// partials summed per output row and CTA of the cluster: int8 four K steps,
// int4 two K halves
__host__ __device__ constexpr int gv_parts(int fmt) { return fmt == FMT_W8 ? 4 : 2; }
// bytes per token row of the CTA's x (its K range + a skew that keeps the
// fragment reads conflict-free: 32 bytes for int8, 64 for int4)
__host__ __device__ constexpr uint32_t gv_x_pitch(int kbps, int fmt) {
    return static_cast<uint32_t>(kbps) * 128u + (fmt == FMT_W8 ? 32u : 64u);
}
__host__ __device__ constexpr uint32_t gv_slot_bytes(int fmt) { return GV_SLOT_KB * tile_bytes(fmt); }
// dynamic shared memory: alignment + barriers + token scales + x rows +
// staging (parts x NB*8 tokens x 128 rows, fp32) + the cluster's partials of
// this CTA's rows (S x NB*8 x 128/S, fp32) + ring
__host__ __device__ constexpr size_t gv_smem_bytes(int fmt, int nb, int kbps, int stages) {
    return 128 + 256 + 64 + static_cast<size_t>(nb * 8) * gv_x_pitch(kbps, fmt) +
           static_cast<size_t>(gv_parts(fmt) + 1) * (nb * 8) * 128u * 4u + static_cast<size_t>(stages) * gv_slot_bytes(fmt);
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void st_dsmem_v4(uint32_t cluster_addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&d)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t (&d)[2]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                 : "=r"(d[0]), "=r"(d[1]) : "r"(addr) : "memory");
}

// two int8 codes (offset-binary bytes b0, b1 of w picked by sel) -> fp16x2
// of the signed codes: 0x64 above each byte is the fp16 1024 + byte, less 1152
__device__ __forceinline__ uint32_t bytes_to_f16x2(uint32_t w, uint32_t sel) {
    uint32_t v;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(v) : "r"(w), "r"(0x64646464u), "r"(sel));
    return h2u(__hsub2(u2h(v), u2h(0x64806480u)));
}

// one landed 64-input int8 block, this warp's rows and K step: ldmatrix of
// the codes, fp16 x fragments of NB token groups (xrow: this lane's place in
// x row g), 2 RB x NB warp MMAs
template <int NB>
__device__ __forceinline__ void gv_w8_block(const uint8_t* blk, uint32_t lm_off, const uint8_t* xrow, int g,
                                            uint32_t pitch, float (&acc)[2][NB][4], uint32_t& held) {
    uint32_t d[4];
    ldmatrix_x4(smem_u32(blk) + lm_off, d);
    held ^= d[0] ^ d[1] ^ d[2] ^ d[3];
    uint32_t b[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const uint2 u = *reinterpret_cast<const uint2*>(xrow + (nb * 8 + g) * pitch);
        b[nb][0] = u.x;
        b[nb][1] = u.y;
    }
#pragma unroll
    for (int bk = 0; bk < 2; ++bk) {
        const uint32_t lo0 = bytes_to_f16x2(d[2 * bk], 0x4140u);
        const uint32_t hi0 = bytes_to_f16x2(d[2 * bk], 0x4342u);
        const uint32_t lo1 = bytes_to_f16x2(d[2 * bk + 1], 0x4140u);
        const uint32_t hi1 = bytes_to_f16x2(d[2 * bk + 1], 0x4342u);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) mma16816_f16(acc[bk][nb], lo0, lo1, hi0, hi1, b[nb][0], b[nb][1]);
    }
}

template <int FMT, int NB>
__global__ void __launch_bounds__(GV_THREADS, 1) gemv_kernel(const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 127u) & ~127u) - raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(base);            // [GV_MAX_STAGES]
    uint64_t* empty = full + GV_MAX_STAGES;                          // [GV_MAX_STAGES]
    float* xinv_sm = reinterpret_cast<float*>(base + 192);          // [16] 2^-e_m
    uint8_t* xsm = base + 256 + 64;                                  // [NB*8][pitch]
    const uint32_t pitch = gv_x_pitch(a.kbps, FMT);
    constexpr int P = gv_parts(FMT);
    float* stage = reinterpret_cast<float*>(xsm + NB * 8 * pitch);  // [P][NB*8][128]
    float* red = stage + P * NB * 8 * 128;                           // [S][NB*8][128/S]
    uint8_t* ring = reinterpret_cast<uint8_t*>(red + NB * 8 * 128);  // [stages][slot]
    constexpr uint32_t SLOT = gv_slot_bytes(FMT);
    constexpr uint32_t TB = tile_bytes(FMT);
    const int stages = a.stages;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int S = a.S;
    const int q = (S > 1) ? static_cast<int>(cluster_ctarank()) : 0;
    const int cid = (S > 1) ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
    const int ncl = (S > 1) ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
    const int kb0 = q * a.kbps, kb1 = min(a.KT, kb0 + a.kbps);
    const int nkb = kb1 - kb0;
    const int nslots = (nkb + GV_SLOT_KB - 1) / GV_SLOT_KB;  // ring slots per tile
    const int Mv = min(a.M, NB * 8);
    const int rows_per = 128 / S;  // rows of each tile this CTA sums and stores

    if (threadIdx.x < GV_MAX_STAGES) {
        mbar_init(&full[threadIdx.x], 1);
        mbar_init(&empty[threadIdx.x], GV_WARPS);
    }
    if (threadIdx.x == 0) fence_barrier_init();
    __syncthreads();
    grid_dependency_sync();  // nothing above touches global memory

    if (warp < GV_WARPS) {
        // ---- x rows m < M over this CTA's K range; inputs beyond K (a ragged
        // last K block) are zeroed, as their codes are 0
        const uint32_t chunks = static_cast<uint32_t>(nkb) * 8u;  // 16-byte chunks per row
        const int kin = min(a.K, kb1 * 64) - kb0 * 64;            // real inputs of the range
        const uint8_t* xg = static_cast<const uint8_t*>(a.xg);
        // warp m takes token row m: copies it, finds its largest |x|
        // (bf16 magnitudes order as integers) and rewrites it in place as
        // fp16 of x * 2^e_m, e_m = 141 - E for the bf16 exponent field E
        // of that largest |x| (at most 126, so 2^-e_m is a normal float
        // too; a non-finite x keeps e_m = 0 and carries through)
        const int m = warp;
        if (m < Mv) {
            uint8_t* row = xsm + m * pitch;
            const uint8_t* src = xg + (static_cast<size_t>(m) * a.K + kb0 * 64) * 2;
            for (uint32_t c = lane; c < chunks; c += 32) {
                if (static_cast<int>(c) * 8 < kin) cp_async_16(smem_u32(row + c * 16u), src + c * 16u);
                else *reinterpret_cast<uint4*>(row + c * 16u) = make_uint4(0u, 0u, 0u, 0u);
            }
            cp_async_wait_all();
            __syncwarp();
            uint32_t mx = 0;
            for (uint32_t c = lane; c < chunks; c += 32) {
                const uint4 v = *reinterpret_cast<const uint4*>(row + c * 16u);
                mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                           __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
            }
            mx = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const int E = static_cast<int>(mx >> 7);
            const int e = (E >= 255) ? 0 : min(126, 141 - E);
            const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
            for (uint32_t c = lane; c < chunks; c += 32) {
                uint4* p = reinterpret_cast<uint4*>(row + c * 16u);
                const uint4 v = *p;
                uint4 h;
                h.x = h2u(__floats2half2_rn(__uint_as_float(v.x << 16) * sc, __uint_as_float(v.x & 0xFFFF0000u) * sc));
                h.y = h2u(__floats2half2_rn(__uint_as_float(v.y << 16) * sc, __uint_as_float(v.y & 0xFFFF0000u) * sc));
                h.z = h2u(__floats2half2_rn(__uint_as_float(v.z << 16) * sc, __uint_as_float(v.z & 0xFFFF0000u) * sc));
                h.w = h2u(__floats2half2_rn(__uint_as_float(v.w << 16) * sc, __uint_as_float(v.w & 0xFFFF0000u) * sc));
                *p = h;
            }
            if (lane == 0) xinv_sm[m] = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
        } else if (m < NB * 8 && lane == 0) {
            xinv_sm[m] = 1.0f;
        }
        named_sync(1, GV_WARPS * 32);  // x in shared memory for every compute warp
    }

    int it = 0;
    for (int tile = cid; tile < a.NT; tile += ncl) {
        // epilogue operands of this thread's output row, fetched early
        const int n_out = tile * 128 + q * rows_per + static_cast<int>(threadIdx.x) % rows_per;
        const float rf = (warp < GV_WARPS && n_out < a.N) ? a.rowf[n_out] : 0.0f;
        const float bias = (warp < GV_WARPS && a.bias && n_out < a.N) ? bf16_to_f32(a.bias[n_out]) : 0.0f;

        if (warp == GV_WARPS) {
            // ---- producer: this tile's blocks of the split, four per slot
            if (lane == 0) {
                const uint8_t* src = a.packed + (static_cast<size_t>(tile) * a.KT + kb0) * TB;
                for (int i = 0; i < nslots; ++i, ++it) {
                    const int st = it % stages;
                    // bounded: on a timeout the error bit is set and the copy is
                    // issued anyway (the data are then garbage, never a fault)
                    mbar_wait(&empty[st], ((it / stages) & 1) ^ 1, a.timeout_ns);
                    const uint32_t bytes = static_cast<uint32_t>(min(GV_SLOT_KB, nkb - i * GV_SLOT_KB)) * TB;
                    mbar_arrive_expect_tx(&full[st], bytes);
                    bulk_load(ring + st * SLOT, src + static_cast<size_t>(i) * SLOT, bytes, &full[st]);
                }
            }
            __syncwarp();
        } else {
            // int8: rows 32 rb + {0..31} (two 16-row MMA blocks), K step ks;
            // int4: rows 16 rb + {0..15}, K half ks
            const int rb = (FMT == FMT_W8) ? (warp & 3) : (warp & 7);
            const int ks = (FMT == FMT_W8) ? (warp >> 2) : (warp >> 3);
            constexpr int RB = (FMT == FMT_W8) ? 2 : 1;  // 16-row MMA blocks per warp
            float acc[RB][NB][4];
#pragma unroll
            for (int b = 0; b < RB; ++b)
#pragma unroll
                for (int j = 0; j < NB; ++j) acc[b][j][0] = acc[b][j][1] = acc[b][j][2] = acc[b][j][3] = 0.0f;
            // ldmatrix row address of this lane inside a block's tile
            uint32_t lm_off;
            if constexpr (FMT == FMT_W8) {
                // matrices: (block 0, rows 0-7), (block 0, rows 8-15), (block 1, ...), (block 1, ...)
                const int row = 32 * rb + 16 * (lane >> 4) + 8 * ((lane >> 3) & 1) + (lane & 7);
                lm_off = static_cast<uint32_t>(ks * 2048 + 16 * row);
            } else {
                const int row = 16 * rb + 8 * ((lane >> 3) & 1) + (lane & 7);  // lanes 16-31: ignored
                lm_off = static_cast<uint32_t>(ks * 2048 + 16 * row);
            }
            const int row_g = (FMT == FMT_W8) ? 32 * rb + g : 16 * rb + g;  // this lane's first row
            for (int i = 0; i < nslots; ++i, ++it) {
                const int st = it % stages;
                mbar_wait(&full[st], (it / stages) & 1, a.timeout_ns);  // bounded (error bit on timeout)
                const uint8_t* slot = ring + st * SLOT;
                const int nk = min(GV_SLOT_KB, nkb - i * GV_SLOT_KB);
                uint32_t held = 0;
                if constexpr (FMT == FMT_W8) {
                    // a full slot: its four blocks unrolled, so the four
                    // ldmatrix and x reads are in flight together
                    if (nk == GV_SLOT_KB) {
#pragma unroll
                        for (int j = 0; j < GV_SLOT_KB; ++j)
                            gv_w8_block<NB>(slot + j * TB, lm_off, xsm + (i * GV_SLOT_KB + j) * 128 + 32 * ks + 8 * t, g,
                                            pitch, acc, held);
                    } else {
                        for (int j = 0; j < nk; ++j)
                            gv_w8_block<NB>(slot + j * TB, lm_off, xsm + (i * GV_SLOT_KB + j) * 128 + 32 * ks + 8 * t, g,
                                            pitch, acc, held);
                    }
                } else {
                    for (int j = 0; j < nk; ++j) {
                        const uint8_t* blk = slot + j * TB;
                        const int kx = (i * GV_SLOT_KB + j) * 128;  // byte offset of the block in an x row
                        uint32_t d[2];
                        ldmatrix_x2(smem_u32(blk) + lm_off, d);
                        uint16_t h0, h1;
                        if constexpr (FMT == FMT_W4G64) {
                            h0 = *reinterpret_cast<const uint16_t*>(blk + 4096 + 2 * row_g);
                            h1 = *reinterpret_cast<const uint16_t*>(blk + 4096 + 2 * (row_g + 8));
                        } else {  // group of inputs 32 ks + 8t..+7: 2 ks + t / 2
                            h0 = *reinterpret_cast<const uint16_t*>(blk + 4096 + 512 * ks + 4 * row_g + 2 * (t >> 1));
                            h1 = *reinterpret_cast<const uint16_t*>(blk + 4096 + 512 * ks + 4 * (row_g + 8) + 2 * (t >> 1));
                        }
                        held ^= d[0] ^ d[1] ^ h0 ^ h1;
                        uint32_t f0[4], f1[4];
                        nibbles_to_f16x2(d[0], __half2half2(__ushort_as_half(h0)), f0);
                        nibbles_to_f16x2(d[1], __half2half2(__ushort_as_half(h1)), f1);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            const uint4 u = *reinterpret_cast<const uint4*>(xsm + (nb * 8 + g) * pitch + kx + 64 * ks + 16 * t);
                            mma16816_f16(acc[0][nb], f0[0], f1[0], f0[1], f1[1], u.x, u.y);
                            mma16816_f16(acc[0][nb], f0[2], f1[2], f0[3], f1[3], u.z, u.w);
                        }
                    }
                }
                // the slot's codes are in registers: hand it back to the producer
                loads_done_before_release(held);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }

            // stage this warp's partial: stage[ks][m][row], times 2^-e_m
            float xi[NB][2];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int e = 0; e < 2; ++e) xi[nb][e] = xinv_sm[nb * 8 + 2 * t + e];
#pragma unroll
            for (int bk = 0; bk < RB; ++bk)
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int e = 0; e < 2; ++e)
                            stage[(ks * NB * 8 + nb * 8 + 2 * t + e) * 128 + row_g + 16 * bk + 8 * h] =
                                acc[bk][nb][2 * h + e] * xi[nb][e];
            named_sync(2, GV_WARPS * 32);
            // sum the P parts of four adjacent rows of one token, in part order,
            // and send them to the owner of the rows: slot q of its buffer
            for (int i = static_cast<int>(threadIdx.x); i < Mv * 32; i += GV_WARPS * 32) {
                const int m = i >> 5, r4 = 4 * (i & 31);
                float4 v = *reinterpret_cast<const float4*>(stage + m * 128 + r4);
#pragma unroll
                for (int pp = 1; pp < P; ++pp) {
                    const float4 u = *reinterpret_cast<const float4*>(stage + (pp * NB * 8 + m) * 128 + r4);
                    v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
                }
                const int owner = r4 / rows_per;
                const uint32_t addr =
                    smem_u32(red) + static_cast<uint32_t>((q * NB * 8 + m) * rows_per + r4 % rows_per) * 4u;
                if (S > 1) st_dsmem_v4(mapa_shared(addr, static_cast<uint32_t>(owner)), v);
                else *reinterpret_cast<float4*>(smem_raw + (addr - raw)) = v;
            }
        }
        // every partial of this CTA's rows has landed in its buffer
        if (S > 1) cluster_sync_all();
        else __syncthreads();

        // sum the S partials of each of this CTA's rows in split order, scale,
        // bias, store.  Thread i takes row i % rows_per and tokens
        // i / rows_per + k (512 / rows_per).
        if (warp < GV_WARPS) {
            const int rl = static_cast<int>(threadIdx.x) % rows_per;
            for (int m = static_cast<int>(threadIdx.x) / rows_per; m < Mv; m += GV_WARPS * 32 / rows_per) {
                float v = red[m * rows_per + rl];
                for (int sp = 1; sp < S; ++sp) v += red[(sp * NB * 8 + m) * rows_per + rl];
                if (n_out < a.N) store_y(a, m, n_out, v * rf + bias);
            }
        }
        // the buffers are rewritten by the next tile: every CTA of the cluster
        // must have read them first
        if (tile + ncl < a.NT) {
            if (S > 1) cluster_sync_all();
            else __syncthreads();
        }
    }
    // nothing may land in shared memory after the CTA has exited (every copy
    // has landed unless a wait above timed out)
    if (warp == GV_WARPS && lane == 0)
        for (int i = max(0, it - stages); i < it; ++i) mbar_wait(&full[i % stages], (i / stages) & 1, DRAIN_TIMEOUT_NS);
}

}  // namespace wlq
