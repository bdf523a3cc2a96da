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
        // 2^f as a float when it is one (f in [-126, 127], every row but those
        // spanning extreme ranges): the product is then exact whenever it can
        // round to a nonzero fp16 (a product below 2^-126 gives fp16 0 either
        // way), so it converts exactly as ldexpf's result does
        const bool fast = f >= -126 && f <= 127;
        const float p2 = __int_as_float((f + 127) << 23);
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int i = threadIdx.x + j * blockDim.x;
            if (i >= K8) break;
            const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = bf16_bits_to_f32(w[e] & 0xFFFFu), b = bf16_bits_to_f32(w[e] >> 16);
                const __half2 h = fast ? __floats2half2_rn(a * p2, b * p2) : __floats2half2_rn(ldexpf(a, f), ldexpf(b, f));
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
constexpr int LR_STAGES = 4;         // cp.async pipeline depth
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
                                                        int xs_scalar, uint16_t* __restrict__ thl) {
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
            if (xs && !xs_scalar) T /= xs[m];  // a power of two: exact
            if (xs && xs_scalar && xs[0] != 0.0f) T /= xs[0];  // one tensor scale (0: left unscaled)
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

// L2t[n] = [L2'h(0..r) | L2'h(0..r) | L2'l(0..r) | 0 ...] (width W) with
// L2' = L2[., n] / rowf[n] (rowf[0] for every n when rowf_scalar; L2 itself
// where that factor is 0 or rowf is null), zero for n >= N.
// A CTA builds 32 rows of L2t in shared memory: its reads of L2 are 64-byte
// row pieces (consecutive n), its writes one contiguous 32 * W * 2-byte block.
constexpr int L2T_ROWS = 32;
constexpr int L2T_MAX_W = 192;  // lr_kb <= 3
__global__ void __launch_bounds__(256) prep_lr_l2t_kernel(const uint16_t* __restrict__ L2, const float* __restrict__ rowf,
                                                          int rowf_scalar, int N, int N_pad, int r, int W,
                                                          uint16_t* __restrict__ l2t) {
    grid_dependency_sync();
    __shared__ __align__(16) uint16_t tile[L2T_ROWS][L2T_MAX_W + 8];
    const int tid = threadIdx.x;
    for (int n0 = blockIdx.x * L2T_ROWS; n0 < N_pad; n0 += gridDim.x * L2T_ROWS) {
        for (int e = tid; e < L2T_ROWS * r; e += 256) {
            const int j = e / L2T_ROWS, nn = e % L2T_ROWS, n = n0 + nn;
            uint16_t hb = 0, lb = 0;
            if (n < N) {
                const float rf = rowf ? rowf[rowf_scalar ? 0 : n] : 0.0f;
                const float l2 = bf16_bits_to_f32(L2[static_cast<size_t>(j) * N + n]);
                const float l = (rf != 0.0f) ? l2 / rf : l2;
                const __nv_bfloat16 hi = __float2bfloat16_rn(l);
                const __nv_bfloat16 lo = __float2bfloat16_rn(l - __bfloat162float(hi));
                hb = *reinterpret_cast<const uint16_t*>(&hi);
                lb = *reinterpret_cast<const uint16_t*>(&lo);
            }
            tile[nn][j] = hb;
            tile[nn][r + j] = hb;
            tile[nn][2 * r + j] = lb;
        }
        for (int e = tid; e < L2T_ROWS * (W - 3 * r); e += 256) {
            const int nn = e / (W - 3 * r), c = 3 * r + e % (W - 3 * r);
            tile[nn][c] = 0;
        }
        __syncthreads();
        const int w8 = W / 8;  // 16-byte pieces per row
        uint4* dst = reinterpret_cast<uint4*>(l2t + static_cast<size_t>(n0) * W);
        for (int e = tid; e < L2T_ROWS * w8; e += 256) {
            const int nn = e / w8, c8 = e % w8;
            dst[e] = *reinterpret_cast<const uint4*>(&tile[nn][c8 * 8]);
        }
        __syncthreads();
    }
}

}  // namespace wlq
