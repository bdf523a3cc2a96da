// prep.cuh -- per-call operand preparation for wlq_linear.
//
//  * x16: for int4 weights the GEMM runs on fp16 operands (a bf16 product of
//    q * s would round the dequantised weight to 8 bits).  Each row of x is
//    scaled by a power of two 2^f_m that puts its largest magnitude in
//    [2^8, 2^9) and converted to fp16; the scaling is exact, and bf16's 8-bit
//    significand fits fp16's 11 bits, so x16 * 2^-f_m == x except for values
//    below 2^-23 of the row maximum.  xs[m] = 2^-f_m is undone in the epilogue.
//  * low-rank branch ("Nunchaku Lite", why it matters: a 16-bit low-rank
//    correction), folded into the GEMM's own accumulator.  The GEMM's
//    epilogue multiplies its accumulator by rowf[n] xs[m], so the branch is
//    fed pre-divided by those factors: T' = (x L1)[m] / xs[m] (a power of
//    two: exact) and L2' = L2[n] / rowf[n] (exact for int4, whose row
//    factors are powers of two; one fp32 rounding for int8's channel scales).
//    Each is carried as a bf16 pair hi + lo (~2^-17 relative) and the GEMM
//    adds [T'h | T'l | T'h] [L2'h | L2'h | L2'l]^T = T'L2' - T'l L2'l over 3r
//    extra inputs (bf16 MMAs into the same fp32 accumulator).  A row whose
//    factor is 0 (an all-zero weight row) keeps L2 unscaled, and the epilogue
//    then scales that row by 1 instead.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"

namespace wlq {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// One warp per row.
__global__ void __launch_bounds__(256) prep_x16_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                       __half* __restrict__ x16, float* __restrict__ xs) {
    grid_dependency_sync();
    const int lane = threadIdx.x & 31;
    const int w0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    const int K8 = K / 8;
    for (int m = w0; m < M; m += nw) {
        const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K);
        float amax = 0.0f;
        for (int i = lane; i < K8; i += 32) {
            const uint4 v = __ldg(row + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            for (int j = 0; j < 4; ++j) {
                amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)));
                amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[j] >> 16)));
            }
        }
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        int f = 0;
        if (amax > 0.0f && isfinite(amax)) {
            int ex;
            frexpf(amax, &ex);  // amax in [2^(ex-1), 2^ex)
            f = 9 - ex;
        }
        if (lane == 0) xs[m] = ldexpf(1.0f, -f);
        uint4* out = reinterpret_cast<uint4*>(x16 + static_cast<size_t>(m) * K);
        for (int i = lane; i < K8; i += 32) {
            const uint4 v = __ldg(row + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
            for (int j = 0; j < 4; ++j) {
                const __half2 h = __floats2half2_rn(ldexpf(bf16_bits_to_f32(w[j] & 0xFFFFu), f),
                                                    ldexpf(bf16_bits_to_f32(w[j] >> 16), f));
                o[j] = *reinterpret_cast<const uint32_t*>(&h);
            }
            out[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// The same conversion with one CTA per row (grid-stride over rows) and the
// row held in registers: PER 16-byte chunks per thread, K <= 8 * PER * THREADS.
// Row maximum over bf16 magnitude bit patterns (NaN ignored, as fmaxf does;
// an infinity leaves the row unscaled), then the same ldexpf / round to
// nearest fp16 per element as prep_x16_kernel: the outputs are identical.
// MINB > 1 caps the registers (65536 / (threads * MINB) per thread) so that a
// CTA of this kernel can run beside a streaming CTA on the same SM.
template <int PER, int THREADS, int MINB>
__global__ void __launch_bounds__(THREADS, MINB) prep_x16_rows_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                     __half* __restrict__ x16, float* __restrict__ xs) {
    grid_dependency_sync();
    __shared__ uint32_t wmax[32];
    __shared__ int fsh;
    const int K8 = K / 8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K);
        uint4 v[PER];
        uint32_t amax = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int i = threadIdx.x + j * blockDim.x;
            v[j] = (i < K8) ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t lo = w[e] & 0x7FFFu, hi = (w[e] >> 16) & 0x7FFFu;
                amax = max(amax, lo > 0x7F80u ? 0u : lo);  // a NaN does not count
                amax = max(amax, hi > 0x7F80u ? 0u : hi);
            }
        }
        for (int off = 16; off > 0; off >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) wmax[warp] = amax;
        __syncthreads();
        if (warp == 0) {
            uint32_t a = (lane < static_cast<int>((blockDim.x + 31) >> 5)) ? wmax[lane] : 0u;
            for (int off = 16; off > 0; off >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, off));
            if (lane == 0) {
                const float fa = bf16_bits_to_f32(a);
                int f = 0;
                if (fa > 0.0f && isfinite(fa)) {
                    int ex;
                    frexpf(fa, &ex);  // fa in [2^(ex-1), 2^ex)
                    f = 9 - ex;
                }
                fsh = f;
                xs[m] = ldexpf(1.0f, -f);
            }
        }
        __syncthreads();
        const int f = fsh;
        uint4* out = reinterpret_cast<uint4*>(x16 + static_cast<size_t>(m) * K);
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int i = threadIdx.x + j * blockDim.x;
            if (i >= K8) break;
            const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __half2 h = __floats2half2_rn(ldexpf(bf16_bits_to_f32(w[e] & 0xFFFFu), f),
                                                    ldexpf(bf16_bits_to_f32(w[e] >> 16), f));
                o[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            out[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncthreads();  // wmax / fsh are rewritten for the next row
    }
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

constexpr int LR_ROWS = 64;          // rows of x per CTA (16 per warp, 4 warps)
constexpr int LR_KC = 64;            // K chunk per pipeline stage
constexpr int LR_STAGES = 3;         // cp.async pipeline depth
constexpr int LR_XP = LR_KC + 8;     // x tile row pitch in bf16 elements (144 bytes: ldmatrix conflict-free)
constexpr int LR_LP = 64 + 8;        // L1 tile row pitch in bf16 elements (r <= 64)
constexpr int LR_MAX_SPLITS = 8;     // CTAs of a cluster splitting K
constexpr uint32_t LR_STAGE_BYTES = (LR_ROWS * LR_XP + LR_KC * LR_LP) * 2u;
__host__ __device__ constexpr size_t lr_t_smem_bytes() {
    return 128 + static_cast<size_t>(LR_STAGES) * LR_STAGE_BYTES + static_cast<size_t>(LR_ROWS) * 64 * 4;
}

__device__ __forceinline__ void lr_cp16(uint32_t dst, const void* src, bool valid) {
    // 16-byte asynchronous copy; an invalid source reads as zeros (src-size 0)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t (&r)[2], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr));
}

// T' = (x L1) / xs -> Thl[m] = [T'h(0..r) | T'l(0..r) | T'h(0..r) | 0 ...] with
// width W = lr_kb * 64, r in {16, 32, 64}; xs == null means 1.  CTA (q, i) of a cluster of S along x takes rows
// 64 i..64 i + 63 over K split q (whole 64-wide chunks); its 4 warps each own
// 16 rows and run m16n8k16 bf16 MMAs (fp32 accumulate) on x and L1 chunks
// staged by a three-deep cp.async pipeline (L1 read K-major as stored and
// turned by ldmatrix.trans).  The S partials are then added in split order
// through distributed shared memory, CTA q taking rows 64/S q..+64/S, and
// written as the bf16 pair hi = bf16(T), lo = bf16(T - hi).
__global__ void __launch_bounds__(128) prep_lr_t_kernel(const uint16_t* __restrict__ x,
                                                        const uint16_t* __restrict__ L1, const float* __restrict__ xs,
                                                        int M, int K, int r, int W, int S, int kc_per,
                                                        uint16_t* __restrict__ thl) {
    extern __shared__ uint8_t lr_smem_raw[];
    uint8_t* base = lr_smem_raw + ((128u - (smem_u32(lr_smem_raw) & 127u)) & 127u);
    uint16_t* stage0 = reinterpret_cast<uint16_t*>(base);
    float* part = reinterpret_cast<float*>(base + LR_STAGES * LR_STAGE_BYTES);  // [64 rows][r]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = (S > 1) ? static_cast<int>(cluster_ctarank()) : 0;
    const int KC = (K + LR_KC - 1) / LR_KC;
    const int c0 = q * kc_per, c1 = min(KC, c0 + kc_per);
    const int nchunks = max(0, c1 - c0);
    const int ntile = r / 8;
    const int lchunks = r / 8;  // 16-byte pieces per L1 row
    grid_dependency_sync();
    // every CTA of a cluster shares blockIdx.y, so all take the same row tiles
    for (int m0 = blockIdx.y * LR_ROWS; m0 < M; m0 += gridDim.y * LR_ROWS) {

    auto issue = [&](int c, int st) {
        uint16_t* xt = stage0 + st * (LR_STAGE_BYTES / 2);
        uint16_t* lt = xt + LR_ROWS * LR_XP;
        const int k0 = (c0 + c) * LR_KC;
        for (int idx = tid; idx < LR_ROWS * (LR_KC / 8); idx += 128) {
            const int rr = idx >> 3, c8 = idx & 7;
            const int m = m0 + rr, k = k0 + c8 * 8;
            const bool ok = m < M && k < K;
            lr_cp16(smem_u32(xt + rr * LR_XP + c8 * 8), ok ? x + static_cast<size_t>(m) * K + k : x, ok);
        }
        for (int idx = tid; idx < LR_KC * lchunks; idx += 128) {
            const int kk = idx / lchunks, j8 = idx % lchunks;
            const int k = k0 + kk;
            const bool ok = k < K;
            lr_cp16(smem_u32(lt + kk * LR_LP + j8 * 8), ok ? L1 + static_cast<size_t>(k) * r + j8 * 8 : L1, ok);
        }
    };

    float acc[8][4];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
#pragma unroll
    for (int st = 0; st < LR_STAGES - 1; ++st) {
        if (st < nchunks) issue(st, st);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int c = 0; c < nchunks; ++c) {
        asm volatile("cp.async.wait_group %0;" ::"n"(LR_STAGES - 2) : "memory");
        __syncthreads();  // chunk c has landed for every thread; chunk c - 1's stage is free
        if (c + LR_STAGES - 1 < nchunks) issue(c + LR_STAGES - 1, (c + LR_STAGES - 1) % LR_STAGES);
        asm volatile("cp.async.commit_group;" ::: "memory");
        const uint16_t* xt = stage0 + (c % LR_STAGES) * (LR_STAGE_BYTES / 2);
        const uint16_t* lt = xt + LR_ROWS * LR_XP;
#pragma unroll
        for (int ks = 0; ks < LR_KC / 16; ++ks) {
            uint32_t a[4];
            const int arow = warp * 16 + (lane & 15);
            ldsm_x4(a, smem_u32(xt + arow * LR_XP + ks * 16 + (lane >> 4) * 8));
            // B fragment of n-tile t: rows k = 16 ks + {0..7} (lanes 0-7) and
            // + {8..15} (lanes 8-15) of the K-major L1 tile, columns 8 t..8 t + 7
            const int krow = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (t < ntile) {
                    uint32_t b[2];
                    ldsm_x2_trans(b, smem_u32(lt + krow * LR_LP + t * 8));
                    mma_bf16_16816(acc[t], a, b);
                }
            }
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // this CTA's partial: part[row][j]; c0,c1 -> (row g, cols 2q', 2q'+1), c2,c3 -> row g + 8
    {
        const int g = lane >> 2, qq = lane & 3;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            if (t < ntile) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = warp * 16 + g + 8 * h;
                    part[row * r + t * 8 + 2 * qq] = acc[t][2 * h];
                    part[row * r + t * 8 + 2 * qq + 1] = acc[t][2 * h + 1];
                }
            }
        }
    }
    if (S > 1) cluster_sync_all();
    else __syncthreads();
    // rows of this CTA's share, summed over the S partials in split order
    const int rows_per = LR_ROWS / S;
    for (int idx = tid; idx < rows_per * r; idx += 128) {
        const int row = q * rows_per + idx / r, j = idx % r;
        const uint32_t a0 = smem_u32(part + row * r + j);
        float T = (S > 1) ? ld_dsmem_f32(mapa_shared(a0, 0)) : part[row * r + j];
        for (int sp = 1; sp < S; ++sp) T += ld_dsmem_f32(mapa_shared(a0, static_cast<uint32_t>(sp)));
        const int m = m0 + row;
        if (m < M) {
            if (xs) T /= xs[m];  // a power of two: exact
            uint16_t* out = thl + static_cast<size_t>(m) * W;
            const __nv_bfloat16 hi = __float2bfloat16_rn(T);
            const __nv_bfloat16 lo = __float2bfloat16_rn(T - __bfloat162float(hi));
            out[j] = *reinterpret_cast<const uint16_t*>(&hi);
            out[r + j] = *reinterpret_cast<const uint16_t*>(&lo);
            out[2 * r + j] = *reinterpret_cast<const uint16_t*>(&hi);
            for (int jj = 3 * r + j; jj < W; jj += r) out[jj] = 0;
        }
    }
    // no CTA may exit, or overwrite its partial, while another still reads it
    if (S > 1) cluster_sync_all();
    else __syncthreads();
    }  // row tiles
}

// L1t[j][k] = L1[k][j] (bf16, [r, K]): the fused pass below reads four
// consecutive inputs of one rank component as one 8-byte load.
__global__ void prep_l1t_kernel(const uint16_t* __restrict__ L1, int K, int r, uint16_t* __restrict__ l1t) {
    grid_dependency_sync();
    const int64_t total = static_cast<int64_t>(K) * r;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int j = static_cast<int>(e / K), k = static_cast<int>(e % K);  // coalesced writes along k
        l1t[e] = L1[static_cast<size_t>(k) * r + j];
    }
}

// x -> x16, xs and T' = (x L1) / xs = (x L1) 2^f in one pass over x (int4
// weights with a low-rank term, K <= 4096).  A CTA holds 16 rows of x in
// shared memory (the whole K), so each row's maximum -- which x16's scale
// needs before any element is converted -- is known without a second read.
// T is formed from the bf16 rows on the tensor cores (m16n8k16, fp32
// accumulate; the 8 warps split K, their partials added in warp order; each
// warp fetches the L1 fragments of four steps before using any), with
// the inputs of an MMA renumbered so that lane (g, t) takes inputs 4t..4t+3
// of its 16: A from one 8-byte shared-memory load per row, B from one 8-byte
// load of L1t.  Same x16 / xs arithmetic as prep_x16_kernel; T' written as
// [T'h | T'l | T'h | 0 ...] like prep_lr_t_kernel.
constexpr int XLR_ROWS = 16;
constexpr int XLR_WARPS = 8;
__host__ __device__ constexpr size_t xlr_smem_bytes(int K, int r) {
    return 128 + static_cast<size_t>(XLR_ROWS) * (K + 8) * 2 + static_cast<size_t>(XLR_WARPS) * XLR_ROWS * r * 4 + 256;
}
template <int R>
__global__ void __launch_bounds__(XLR_WARPS * 32) prep_x16_lr_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ l1t,
                                                          int M, int K, int W, __half* __restrict__ x16,
                                                          float* __restrict__ xs, uint16_t* __restrict__ thl) {
    extern __shared__ uint8_t xlr_smem_raw[];
    uint8_t* base = xlr_smem_raw + ((128u - (smem_u32(xlr_smem_raw) & 127u)) & 127u);
    const int KP = K + 8;  // row pitch (bf16 elements)
    uint16_t* slab = reinterpret_cast<uint16_t*>(base);
    float* tpart = reinterpret_cast<float*>(base + static_cast<size_t>(XLR_ROWS) * KP * 2);  // [8][16][R]
    uint32_t* rmax = reinterpret_cast<uint32_t*>(tpart + XLR_WARPS * XLR_ROWS * R);      // [16]
    int* rf = reinterpret_cast<int*>(rmax + XLR_ROWS);                                    // [16]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int K8 = K / 8;
    grid_dependency_sync();
    constexpr int NT_ = XLR_WARPS * 32;
    for (int m0 = blockIdx.x * XLR_ROWS; m0 < M; m0 += gridDim.x * XLR_ROWS) {
        // the slab: rows m0..m0+15 (zeros past M), 16-byte asynchronous copies
        for (int i = tid; i < XLR_ROWS * K8; i += NT_) {
            const int rr = i / K8, c8 = i % K8;
            const int m = m0 + rr;
            const bool ok = m < M;
            lr_cp16(smem_u32(slab + rr * KP + c8 * 8), ok ? x + static_cast<size_t>(m) * K + c8 * 8 : x, ok);
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
        __syncthreads();
        // row maxima over bf16 magnitude bit patterns (NaN ignored, as fmaxf
        // does): 16 threads per row (half a warp), then a shuffle reduction
        {
            const int rr = tid >> 4, q = tid & 15;
            uint32_t a = 0;
            for (int c8 = q; c8 < K8; c8 += 16) {
                const uint4 v = *reinterpret_cast<const uint4*>(slab + rr * KP + c8 * 8);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t lo = w[e] & 0x7FFFu, hi = (w[e] >> 16) & 0x7FFFu;
                    a = max(a, lo > 0x7F80u ? 0u : lo);
                    a = max(a, hi > 0x7F80u ? 0u : hi);
                }
            }
            for (int off = 8; off > 0; off >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, off));
            if (q == 0) rmax[rr] = a;
        }
        // T over this warp's quarter of K (16-input steps)
        float acc[R / 8][4];
#pragma unroll
        for (int jt = 0; jt < R / 8; ++jt) acc[jt][0] = acc[jt][1] = acc[jt][2] = acc[jt][3] = 0.0f;
        const int ksteps = K / 16;
        constexpr int B4 = 4;  // steps whose L1 fragments are fetched together
        for (int st0 = warp; st0 < ksteps; st0 += XLR_WARPS * B4) {
            uint2 bf[B4][R / 8];
#pragma unroll
            for (int u = 0; u < B4; ++u) {
                const int st = st0 + u * XLR_WARPS;
                const int k0 = st * 16 + 4 * t;
#pragma unroll
                for (int jt = 0; jt < R / 8; ++jt)
                    bf[u][jt] = (st < ksteps) ? __ldg(reinterpret_cast<const uint2*>(l1t + static_cast<size_t>(jt * 8 + g) * K + k0))
                                              : make_uint2(0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < B4; ++u) {
                const int st = st0 + u * XLR_WARPS;
                if (st >= ksteps) break;
                const int k0 = st * 16 + 4 * t;
                const uint2 alo = *reinterpret_cast<const uint2*>(slab + g * KP + k0);
                const uint2 ahi = *reinterpret_cast<const uint2*>(slab + (g + 8) * KP + k0);
                const uint32_t a[4] = {alo.x, ahi.x, alo.y, ahi.y};
#pragma unroll
                for (int jt = 0; jt < R / 8; ++jt) {
                    const uint32_t bb[2] = {bf[u][jt].x, bf[u][jt].y};
                    mma_bf16_16816(acc[jt], a, bb);
                }
            }
        }
        // this warp's partial: rows g, g + 8; columns 8 jt + 2t, + 1
#pragma unroll
        for (int jt = 0; jt < R / 8; ++jt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                tpart[(warp * XLR_ROWS + g + 8 * h) * R + jt * 8 + 2 * t] = acc[jt][2 * h];
                tpart[(warp * XLR_ROWS + g + 8 * h) * R + jt * 8 + 2 * t + 1] = acc[jt][2 * h + 1];
            }
        __syncthreads();
        if (tid < XLR_ROWS) {
            const float fa = bf16_bits_to_f32(rmax[tid]);
            int f = 0;
            if (fa > 0.0f && isfinite(fa)) {
                int ex;
                frexpf(fa, &ex);  // fa in [2^(ex-1), 2^ex)
                f = 9 - ex;
            }
            rf[tid] = f;
            if (m0 + tid < M) xs[m0 + tid] = ldexpf(1.0f, -f);
        }
        __syncthreads();
        // T' = T 2^f (the warps' partials in warp order), as the bf16 pair
        for (int i = tid; i < XLR_ROWS * R; i += NT_) {
            const int rr = i / R, j = i % R;
            const int m = m0 + rr;
            if (m >= M) continue;
            float T = tpart[rr * R + j];
#pragma unroll
            for (int w = 1; w < XLR_WARPS; ++w) T += tpart[(w * XLR_ROWS + rr) * R + j];
            T = ldexpf(T, rf[rr]);  // a power of two: exact
            uint16_t* out = thl + static_cast<size_t>(m) * W;
            const __nv_bfloat16 hi = __float2bfloat16_rn(T);
            const __nv_bfloat16 lo = __float2bfloat16_rn(T - __bfloat162float(hi));
            out[j] = *reinterpret_cast<const uint16_t*>(&hi);
            out[R + j] = *reinterpret_cast<const uint16_t*>(&lo);
            out[2 * R + j] = *reinterpret_cast<const uint16_t*>(&hi);
            for (int jj = 3 * R + j; jj < W; jj += R) out[jj] = 0;
        }
        // x16 = fp16(x 2^f), row by row
        for (int i = tid; i < XLR_ROWS * K8; i += NT_) {
            const int rr = i / K8, c8 = i % K8;
            const int m = m0 + rr;
            if (m >= M) continue;
            const uint4 v = *reinterpret_cast<const uint4*>(slab + rr * KP + c8 * 8);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            const int f = rf[rr];
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __half2 h = __floats2half2_rn(ldexpf(bf16_bits_to_f32(w[e] & 0xFFFFu), f),
                                                    ldexpf(bf16_bits_to_f32(w[e] >> 16), f));
                o[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            reinterpret_cast<uint4*>(x16 + static_cast<size_t>(m) * K)[c8] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncthreads();  // the slab and partials are rewritten for the next rows
    }
}

// L2t[n] = [L2'h(0..r) | L2'h(0..r) | L2'l(0..r) | 0 ...] (width W) with
// L2' = L2[., n] / rowf[n] (L2 itself where rowf[n] == 0), zero for n >= N.
// One thread per (row n, 8 columns): the reads of L2 are coalesced across
// consecutive n, each thread writes one 16-byte piece.
__global__ void prep_lr_l2t_kernel(const uint16_t* __restrict__ L2, const float* __restrict__ rowf, int N,
                                   int N_pad, int r, int W, uint16_t* __restrict__ l2t) {
    grid_dependency_sync();
    const int64_t total = static_cast<int64_t>(N_pad) * (W / 8);
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int n = static_cast<int>(idx % N_pad), c8 = static_cast<int>(idx / N_pad);
        const float rf = (n < N) ? rowf[n] : 0.0f;

        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t h[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int c = c8 * 8 + 2 * e + u;
                uint16_t v = 0;
                if (n < N && c < 3 * r) {
                    const float l2 = bf16_bits_to_f32(L2[static_cast<size_t>(c % r) * N + n]);
                    const float l = (rf != 0.0f) ? l2 / rf : l2;
                    const __nv_bfloat16 hi = __float2bfloat16_rn(l);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(l - __bfloat162float(hi));
                    const __nv_bfloat16 out = (c < 2 * r) ? hi : lo;
                    v = *reinterpret_cast<const uint16_t*>(&out);
                }
                h[u] = v;
            }
            w[e] = h[0] | (h[1] << 16);
        }
        reinterpret_cast<uint4*>(l2t + static_cast<size_t>(n) * W)[c8] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace wlq
