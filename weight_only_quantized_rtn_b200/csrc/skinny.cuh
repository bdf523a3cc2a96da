// skinny.cuh -- the weight-only quantized GEMM for few tokens (one token tile
// of at most 64), where streaming the packed weights from HBM is all of the
// work ("Joy-face_change_optimized" model card, files table: weight-only
// Linear; "Nunchaku Lite", how it works: 4-bit weights, 16-bit activations).
//
//   y[m,n] = rowf[n] * xs[m] * sum_k xin[m,k] * w16[n,k]  +  b[n]
//
// Same packed operand, same row factors, same x (bf16, or the fp16 x16 of the
// int4 formats) as the large-token kernel; only the engine differs.  Sixteen
// compute warps in two groups: warp w owns channels 16(w%8)..+15 of the CTA's
// 128, and group w/8 takes K block w/8 of every two-block ring slot.  A warp
// reads the codes of its staged weight tile straight into registers, hands
// the ring slot back at once, dequantises in registers and feeds warp-level
// MMAs (m16n8k16, fp32 accumulate); the two groups' sums are added (in a fixed
// order) at the end of the tile.  No MMA-issuing thread, no tensor memory and
// no hand-off between warps sits between the weight stream and the math.  (A
// tcgen05.mma issues no faster than about one per 46 cycles: at 16 tokens
// that is ~1400 FLOP/clk/SM, below the ~2000 of m16n8k16 warp MMAs; at 32
// tokens it would be ~2800, but here the weight stream, not the MMA rate,
// bounds the kernel.)
//
// Inputs inside a 64-wide K block are renumbered for the MMA: lane (g, t) of
// a warp (g = lane / 4, t = lane % 4) takes inputs 16t..16t+15 of its rows
// (one 16-byte run of codes in the packed tile), and MMA step s uses inputs
// 16t + 4s + {0,1} (fragment columns 2t, 2t+1) and 16t + 4s + {2,3} (columns
// 2t+8, 2t+9).  x is read with the same renumbering, so the dot products are
// unchanged.
//
// The CTA's x rows for its whole K range stay in shared memory (TMA, 128-byte
// swizzle, one 64-input slab per K block), loaded by a warp of their own at
// kernel start; the weight ring is refilled as soon as the sixteen warps hold
// a slot's codes.  A K split over the CTAs of a
// cluster is summed through distributed shared memory in split order, as in
// the large-token kernel.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "pack.cuh"
#include "gemm.cuh"

namespace wlq {

constexpr int SK_GROUPS = 2;                        // warp groups = K blocks per ring slot
constexpr int SK_WARPS = 8 * SK_GROUPS;             // compute warps, 16 channels each
constexpr int SK_THREADS = (SK_WARPS + 2) * 32;     // + weight producer warp + x loader warp
constexpr int SK_PITCH = 132;                       // floats per token row of the partial / staging buffer

struct SkSmem {
    uint8_t* x;       // kbps slabs of BN rows x 128 bytes (swizzled)
    uint8_t* w;       // stages x wstage_bytes
    float* red;       // [BN][SK_PITCH] fp32: split partial, or the output staging
    uint64_t* full;   // weight slot landed
    uint64_t* empty;  // weight slot read by all compute warps (SK_WARPS arrivals)
    uint64_t* xfull;  // x rows landed
    uint64_t* xch;    // local: group 1 parked its sums in red (8 arrivals)
    uint64_t* fin;    // local: group 0 finished the tile's values in red (8 arrivals)
    uint64_t* cpy;    // local: the staged tile was stored (16 arrivals)
    uint64_t* readw;  // local: every compute warp finished reading the cluster's partials
    uint64_t* ready;  // cluster: every CTA's partial is in its smem
    uint64_t* freed;  // cluster: every CTA finished reading this CTA's partial
    volatile int* abort_flag;
};

__device__ __forceinline__ void sk_issue_x(const GemmArgs& a, const CUtensorMap* tm_x, const SkSmem& s,
                                           const TileCoord& c) {
    mbar_arrive_expect_tx(s.xfull, static_cast<uint32_t>(c.kb1 - c.kb0) * a.xsub_bytes);
    for (int kb = c.kb0; kb < c.kb1; ++kb) tma_load_2d(s.x + (kb - c.kb0) * a.xsub_bytes, tm_x, s.xfull, kb * 64, 0);
}

// Weight producer (one thread): the ring of two-block slots.
__device__ void sk_producer(const GemmArgs& a, const SkSmem& s, const Sched& sc) {
    int it = 0;
    Ring r;
    bool ok = true;
    for (int g = sc.cid; g < a.tiles_nm && ok; g += sc.ncl) {
        const TileCoord c = tile_coord<false>(a, g, sc.rank);
        for (int kb = c.kb0; kb < c.kb1; kb += SK_GROUPS) {
            const int nkb = min(SK_GROUPS, c.kb1 - kb);
            const int st = r.slot;
            if (!wait_or_abort(&s.empty[st], r.phase ^ 1, a, s.abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&s.full[st], nkb * a.wtile_bytes);
            bulk_load(s.w + st * a.wstage_bytes, a.packed + (static_cast<size_t>(c.nt) * a.KT + kb) * a.wtile_bytes,
                      nkb * a.wtile_bytes, &s.full[st]);
            ++it;
            r.next(a.stages);
        }
    }
    if (!ok)
        for (int i = max(0, it - a.stages); i < it; ++i)
            mbar_wait(&s.full[i % a.stages], (i / a.stages) & 1, DRAIN_TIMEOUT_NS);
}

// x loader (one thread): this CTA's x rows for its K range, once (every tile
// of the CTA has the same tokens and, being one split, the same K range).
__device__ void sk_load_x(const GemmArgs& a, const CUtensorMap* tm_x, const SkSmem& s, const Sched& sc) {
    if (sc.cid >= a.tiles_nm) return;
    const TileCoord c = tile_coord<false>(a, sc.cid, sc.rank);
    mbar_arrive_expect_tx(s.xfull, static_cast<uint32_t>(c.kb1 - c.kb0) * a.xsub_bytes);
    for (int kb = c.kb0; kb < c.kb1; ++kb) tma_load_2d(s.x + (kb - c.kb0) * a.xsub_bytes, tm_x, s.xfull, kb * 64, 0);
    // nothing may land in shared memory after the CTA has exited
    mbar_wait(s.xfull, 0, DRAIN_TIMEOUT_NS);
}

// Codes of one 64-wide K block for rows g and g+8 of this warp's 16, as MMA
// A-fragment pairs: p[i] holds inputs 16t + 2i, 16t + 2i + 1 (low, high).
template <int FMT>
struct SkCodes {
    uint4 r0, r1;        // int8: 16 codes per row; int4: .x/.y hold 16 nibbles per row
    __half2 s0, s1;      // int4: fp16 scale of this lane's group, rows g and g+8
};

template <int FMT>
__device__ __forceinline__ SkCodes<FMT> sk_load_codes(const uint8_t* blk, int row0, int t) {
    SkCodes<FMT> v;
    if constexpr (FMT == FMT_W8) {
        v.r0 = *reinterpret_cast<const uint4*>(blk + t * 2048 + 16 * row0);
        v.r1 = *reinterpret_cast<const uint4*>(blk + t * 2048 + 16 * (row0 + 8));
    } else {
        const uint2 a0 = *reinterpret_cast<const uint2*>(blk + (t >> 1) * 2048 + 16 * row0 + 8 * (t & 1));
        const uint2 a1 = *reinterpret_cast<const uint2*>(blk + (t >> 1) * 2048 + 16 * (row0 + 8) + 8 * (t & 1));
        v.r0 = make_uint4(a0.x, a0.y, 0u, 0u);
        v.r1 = make_uint4(a1.x, a1.y, 0u, 0u);
        if constexpr (FMT == FMT_W4G64) {
            v.s0 = __half2half2(*reinterpret_cast<const __half*>(blk + 4096 + 2 * row0));
            v.s1 = __half2half2(*reinterpret_cast<const __half*>(blk + 4096 + 2 * (row0 + 8)));
        } else {
            v.s0 = __half2half2(*reinterpret_cast<const __half*>(blk + 4096 + 512 * (t >> 1) + 4 * row0 + 2 * (t & 1)));
            v.s1 = __half2half2(
                *reinterpret_cast<const __half*>(blk + 4096 + 512 * (t >> 1) + 4 * (row0 + 8) + 2 * (t & 1)));
        }
    }
    return v;
}

template <int FMT>
__device__ __forceinline__ void sk_convert(const SkCodes<FMT>& v, uint32_t (&p0)[8], uint32_t (&p1)[8]) {
    if constexpr (FMT == FMT_W8) {
        const uint32_t a[4] = {v.r0.x, v.r0.y, v.r0.z, v.r0.w};
        const uint32_t b[4] = {v.r1.x, v.r1.y, v.r1.z, v.r1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            p0[2 * i] = bytes_to_bf16x2(a[i], 0x7440u, 0x7441u);
            p0[2 * i + 1] = bytes_to_bf16x2(a[i], 0x7442u, 0x7443u);
            p1[2 * i] = bytes_to_bf16x2(b[i], 0x7440u, 0x7441u);
            p1[2 * i + 1] = bytes_to_bf16x2(b[i], 0x7442u, 0x7443u);
        }
    } else {
        uint32_t t0[4], t1[4];
        nibbles_to_f16x2(v.r0.x, v.s0, t0);
        nibbles_to_f16x2(v.r0.y, v.s0, t1);
#pragma unroll
        for (int i = 0; i < 4; ++i) p0[i] = t0[i], p0[4 + i] = t1[i];
        nibbles_to_f16x2(v.r1.x, v.s1, t0);
        nibbles_to_f16x2(v.r1.y, v.s1, t1);
#pragma unroll
        for (int i = 0; i < 4; ++i) p1[i] = t0[i], p1[4 + i] = t1[i];
    }
}

// Compute warps: the K loop, then the epilogue (or this CTA's part of the
// cluster reduction).  NB = token tile / 8.
template <int FMT, int NB>
__device__ void sk_compute(const GemmArgs& a, const SkSmem& s, const Sched& sc, int warp, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int grp = warp >> 3;                 // K block of each slot this warp takes
    const int row0 = (warp & 7) * 16 + g;      // rows row0 and row0 + 8 of the 128-channel tile
    const bool split = a.S > 1;
    const int share = a.BN / a.S;
    const bool first_thread = (warp == 0 && lane == 0);
    Ring r;
    int tc = 0;
    bool have_x = false;
    for (int gt = sc.cid; gt < a.tiles_nm; gt += sc.ncl, ++tc) {
        const TileCoord c = tile_coord<false>(a, gt, sc.rank);
        // epilogue operands, fetched before the K loop hides their latency
        const int n0 = c.nt * 128 + row0, n1 = n0 + 8;
        const float rf0 = n0 < a.N ? a.rowf[n0] : 0.0f, rf1 = n1 < a.N ? a.rowf[n1] : 0.0f;
        const float b0 = (!split && a.bias && n0 < a.N) ? bf16_to_f32(a.bias[n0]) : 0.0f;
        const float b1 = (!split && a.bias && n1 < a.N) ? bf16_to_f32(a.bias[n1]) : 0.0f;
        float xsv[NB][2];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const int m = nb * 8 + 2 * t;
            xsv[nb][0] = (FMT == FMT_W8) ? 1.0f : (m < a.M ? a.xs[m] : 0.0f);
            xsv[nb][1] = (FMT == FMT_W8) ? 1.0f : (m + 1 < a.M ? a.xs[m + 1] : 0.0f);
        }
        if (!have_x) {
            if (!warp_wait_or_abort(s.xfull, 0, a, s.abort_flag)) return;
            have_x = true;
        }
        float acc[NB][4];
#pragma unroll
        for (int j = 0; j < NB; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
        for (int kb = c.kb0; kb < c.kb1; kb += SK_GROUPS, r.next(a.stages)) {
            const int st = r.slot;
            const bool mine = kb + grp < c.kb1;
            if (!warp_wait_or_abort(&s.full[st], r.phase, a, s.abort_flag)) return;
            SkCodes<FMT> cv;
            uint32_t held = 0;
            if (mine) {
                cv = sk_load_codes<FMT>(s.w + st * a.wstage_bytes + grp * a.wtile_bytes, row0, t);
                held = cv.r0.x ^ cv.r0.y ^ cv.r0.z ^ cv.r0.w ^ cv.r1.x ^ cv.r1.y ^ cv.r1.z ^ cv.r1.w;
                if constexpr (FMT != FMT_W8) held ^= h2u(cv.s0) ^ h2u(cv.s1);
            }
            loads_done_before_release(held);
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.empty[st]);
            if (!mine) continue;
            uint32_t p0[8], p1[8];
            sk_convert<FMT>(cv, p0, p1);
            // x slab of this K block: token rows of 128 bytes, 16-byte chunk c of
            // row m stored at chunk c ^ (m % 8)
            const uint8_t* slab = s.x + (kb + grp - c.kb0) * a.xsub_bytes;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int m = nb * 8 + g;
                const uint8_t* xr = slab + m * 128;
                const uint4 u0 = *reinterpret_cast<const uint4*>(xr + (((2 * t) ^ (m & 7)) << 4));
                const uint4 u1 = *reinterpret_cast<const uint4*>(xr + (((2 * t + 1) ^ (m & 7)) << 4));
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

        // ---- epilogue: acc[nb] = D[rows row0, row0+8][tokens nb*8 + 2t, +1] of
        // this group's K blocks.  Group 1 parks its sums in the buffer, group 0
        // adds its own (group 0 + group 1, always in that order), scales and
        // leaves the tile's fp32 values there: the split partial, or the output
        // staging.  The buffer is free again once the previous tile's copy-out
        // (or every CTA's read of the previous partial) is done.
        // (all hand-offs are bounded mbarrier waits, so that an abort anywhere
        // cannot leave a warp blocked)
        const uint32_t par = tc & 1;
        if (grp == 1) {
            if (tc > 0) {
                const bool free_again = split ? warp_wait_or_abort(s.freed, par ^ 1, a, s.abort_flag, true)
                                              : warp_wait_or_abort(s.cpy, par ^ 1, a, s.abort_flag);
                if (!free_again) return;
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int m = nb * 8 + 2 * t;
                s.red[m * SK_PITCH + row0] = acc[nb][0];
                s.red[(m + 1) * SK_PITCH + row0] = acc[nb][1];
                s.red[m * SK_PITCH + row0 + 8] = acc[nb][2];
                s.red[(m + 1) * SK_PITCH + row0 + 8] = acc[nb][3];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(s.xch);
        } else {
            if (!warp_wait_or_abort(s.xch, par, a, s.abort_flag)) return;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int m = nb * 8 + 2 * t;
                float* e0 = s.red + m * SK_PITCH + row0;
                float* e1 = s.red + (m + 1) * SK_PITCH + row0;
                e0[0] = (acc[nb][0] + e0[0]) * rf0 * xsv[nb][0] + b0;
                e1[0] = (acc[nb][1] + e1[0]) * rf0 * xsv[nb][1] + b0;
                e0[8] = (acc[nb][2] + e0[8]) * rf1 * xsv[nb][0] + b1;
                e1[8] = (acc[nb][3] + e1[8]) * rf1 * xsv[nb][1] + b1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(s.fin);
        }
        if (!split) {
            // store the staged tile: each thread takes four adjacent channels of a token
            if (!warp_wait_or_abort(s.fin, par, a, s.abort_flag)) return;
            const int tid = warp * 32 + lane;
            for (int i = tid; i < a.BN * 32; i += SK_WARPS * 32) {
                const int m = i >> 5, nq = c.nt * 128 + 4 * (i & 31);
                if (m >= a.M || nq >= a.N) continue;
                const float4 v = *reinterpret_cast<const float4*>(s.red + m * SK_PITCH + 4 * (i & 31));
                const float o[4] = {v.x, v.y, v.z, v.w};
                if (a.vec_out) {
                    if (a.y_f32) {
                        *reinterpret_cast<float4*>(static_cast<float*>(a.y) + static_cast<size_t>(m) * a.N + nq) = v;
                    } else {
                        const __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]);
                        const __nv_bfloat162 hi = __floats2bfloat162_rn(o[2], o[3]);
                        uint2 v2;
                        v2.x = *reinterpret_cast<const uint32_t*>(&lo);
                        v2.y = *reinterpret_cast<const uint32_t*>(&hi);
                        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.y) + static_cast<size_t>(m) * a.N + nq) = v2;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (nq + q < a.N) store_y(a, m, nq + q, o[q]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(s.cpy);
            continue;
        }
        // publish this CTA's partial to the cluster, sum this CTA's share of the tokens
        if (first_thread && wait_or_abort(s.fin, par, a, s.abort_flag)) {
            // the fence orders the partial at cluster scope; the arrives need no
            // release of their own (a release.cluster arrive costs ~1000 cycles)
            fence_acq_rel_cluster();
            for (int q = 0; q < a.S; ++q) mbar_arrive_peer(mapa_shared(smem_u32(s.ready), q));
        }
        if (!warp_wait_or_abort(s.ready, par, a, s.abort_flag, true)) return;
        reduce_share(a, s.red, SK_PITCH, c, sc, 0, share, warp, SK_WARPS, lane, a.S);
        __syncwarp();
        if (lane == 0) mbar_arrive(s.readw);
        if (first_thread && wait_or_abort(s.readw, par, a, s.abort_flag)) {
            fence_acq_rel_cluster();
            for (int q = 0; q < a.S; ++q) mbar_arrive_peer(mapa_shared(smem_u32(s.freed), q));
        }
    }
    // no CTA of the cluster may still read this CTA's shared memory when it exits
    if (split && tc > 0) warp_wait_or_abort(s.freed, (tc - 1) & 1, a, s.abort_flag, true);
}

template <int FMT, int NB>
__global__ void __launch_bounds__(SK_THREADS, 1)
skinny_kernel(const __grid_constant__ CUtensorMap tm_x, const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    SkSmem s;
    s.x = base;
    s.w = s.x + static_cast<size_t>(a.kbps) * a.xsub_bytes;
    s.red = reinterpret_cast<float*>(s.w + static_cast<size_t>(a.stages) * a.wstage_bytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(s.red) + a.red_bytes);
    s.full = bars;
    s.empty = s.full + MAX_STAGES;
    s.xfull = s.empty + MAX_STAGES;
    s.xch = s.xfull + 1;
    s.fin = s.xch + 1;
    s.cpy = s.fin + 1;
    s.readw = s.cpy + 1;
    s.ready = s.readw + 1;
    s.freed = s.ready + 1;
    s.abort_flag = reinterpret_cast<volatile int*>(s.freed + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // one barrier per thread
    const int i = threadIdx.x;
    if (i < a.stages) mbar_init(&s.full[i], 1);
    else if (i >= 32 && i < 32 + a.stages) mbar_init(&s.empty[i - 32], SK_WARPS);
    else if (i == 64) mbar_init(s.xfull, 1);
    else if (i == 65) mbar_init(s.xch, SK_WARPS / 2);
    else if (i == 66) mbar_init(s.fin, SK_WARPS / 2);
    else if (i == 67) mbar_init(s.cpy, SK_WARPS);
    else if (i == 68) mbar_init(s.readw, SK_WARPS);
    else if (i == 69) mbar_init(s.ready, a.S_red);
    else if (i == 70) mbar_init(s.freed, a.S_red);
    else if (i == 71) *s.abort_flag = 0;
    if (warp == SK_WARPS + 1 && lane == 0) prefetch_tensormap(&tm_x);
    if (i < 72) {
        fence_barrier_init();
        fence_proxy_async();
    }
    __syncthreads();
    // every CTA of the cluster has initialised its barriers before any remote arrive
    if (a.S > 1) cluster_sync_all();
    grid_dependency_sync();  // nothing above touches global memory
    const Sched sc = sched();
    if (warp < SK_WARPS) sk_compute<FMT, NB>(a, s, sc, warp, lane);
    else if (warp == SK_WARPS && lane == 0) sk_producer(a, s, sc);
    else if (warp == SK_WARPS + 1 && lane == 0) sk_load_x(a, &tm_x, s, sc);
    __syncthreads();
}

}  // namespace wlq
