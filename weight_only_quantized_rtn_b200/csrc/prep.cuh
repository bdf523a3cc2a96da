// prep.cuh -- per-call operand preparation for wlq_linear.
//
//  * x16: for int4 weights the GEMM runs on fp16 operands (a bf16 product of
//    q * s would round the dequantised weight to 8 bits).  Each row of x is
//    scaled by a power of two 2^f_m that puts its largest magnitude in
//    [2^8, 2^9) and converted to fp16; the scaling is exact, and bf16's 8-bit
//    significand fits fp16's 11 bits, so x16 * 2^-f_m == x except for values
//    below 2^-23 of the row maximum.  xs[m] = 2^-f_m is undone in the epilogue.
//  * low-rank branch ("Nunchaku Lite", why it matters: a 16-bit low-rank
//    correction): T = x L1 in fp32 on the tensor cores, stored as a bf16
//    pair T = Th + Tl (hi, lo) so the second GEMM T L2 sees T to ~2^-17;
//    L2 is transposed into a K-major [N_pad, 2r] operand [L2^T | L2^T] so
//    that one extra MMA K-step computes Th L2 + Tl L2.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

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

constexpr int LR_ROWS = 64;       // rows of x per CTA (16 per warp, 4 warps)
constexpr int LR_KC = 64;         // K chunk
constexpr int LR_PITCH = LR_KC + 8;  // smem row pitch in bf16 elements (144 bytes)

// T = x L1 -> Thl[m] = [Th(0..r) | Tl(0..r) | 0 ... ] with width W = lr_kb * 64.
// r in {16, 32, 64}.  128 threads, one CTA per 64 rows.
__global__ void __launch_bounds__(128) prep_lr_t_kernel(const uint16_t* __restrict__ x,
                                                        const uint16_t* __restrict__ L1, int M, int K,
                                                        int r, int W, uint16_t* __restrict__ thl) {
    grid_dependency_sync();
    __shared__ __align__(16) uint16_t xt[LR_ROWS * LR_PITCH];
    __shared__ __align__(16) uint16_t lt[64 * LR_PITCH];  // [j][k]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * LR_ROWS;
    const int ntile = r / 8;
    float acc[8][4];
    for (int t = 0; t < 8; ++t)
        for (int e = 0; e < 4; ++e) acc[t][e] = 0.0f;
    for (int k0 = 0; k0 < K; k0 += LR_KC) {
        // x tile: 64 rows x 64 k, 8 elements per uint4
        for (int idx = tid; idx < LR_ROWS * (LR_KC / 8); idx += 128) {
            const int rr = idx / (LR_KC / 8), c8 = idx % (LR_KC / 8);
            const int m = m0 + rr, k = k0 + c8 * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m < M && k < K) v = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K + k));
            *reinterpret_cast<uint4*>(&xt[rr * LR_PITCH + c8 * 8]) = v;
        }
        // L1 chunk transposed: lt[j][kk] = L1[k0 + kk][j]
        for (int idx = tid; idx < LR_KC * r; idx += 128) {
            const int kk = idx / r, j = idx % r;
            const int k = k0 + kk;
            lt[j * LR_PITCH + kk] = (k < K) ? L1[static_cast<size_t>(k) * r + j] : static_cast<uint16_t>(0);
        }
        __syncthreads();
        for (int ks = 0; ks < LR_KC / 16; ++ks) {
            uint32_t a[4];
            const int arow = warp * 16 + (lane & 15);
            ldsm_x4(a, static_cast<uint32_t>(__cvta_generic_to_shared(&xt[arow * LR_PITCH + ks * 16 + (lane >> 4) * 8])));
            for (int t = 0; t < ntile; ++t) {
                uint32_t b[2];
                const int brow = t * 8 + (lane & 7);
                ldsm_x2(b, static_cast<uint32_t>(__cvta_generic_to_shared(&lt[brow * LR_PITCH + ks * 16 + ((lane >> 3) & 1) * 8])));
                mma_bf16_16816(acc[t], a, b);
            }
        }
        __syncthreads();
    }
    // scatter: c0,c1 -> (row g, cols 2q, 2q+1); c2,c3 -> (row g+8, same cols)
    const int g = lane >> 2, q = lane & 3;
    for (int half = 0; half < 2; ++half) {
        const int m = m0 + warp * 16 + g + 8 * half;
        if (m >= M) continue;
        uint16_t* out = thl + static_cast<size_t>(m) * W;
        for (int t = 0; t < ntile; ++t)
            for (int e = 0; e < 2; ++e) {
                const int j = t * 8 + 2 * q + e;
                const float T = acc[t][2 * half + e];
                const __nv_bfloat16 hi = __float2bfloat16_rn(T);
                const __nv_bfloat16 lo = __float2bfloat16_rn(T - __bfloat162float(hi));
                out[j] = *reinterpret_cast<const uint16_t*>(&hi);
                out[r + j] = *reinterpret_cast<const uint16_t*>(&lo);
            }
        for (int j = 2 * r + q; j < W; j += 4) out[j] = 0;
    }
}

// L2t[n][c] = L2[c mod r][n] for c < 2r, zero beyond 2r or N.
__global__ void prep_lr_l2t_kernel(const uint16_t* __restrict__ L2, int N, int N_pad, int r, int W,
                                   uint16_t* __restrict__ l2t) {
    grid_dependency_sync();
    const int64_t total = static_cast<int64_t>(N_pad) * W;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int n = static_cast<int>(idx / W), c = static_cast<int>(idx % W);
        uint16_t v = 0;
        if (n < N && c < 2 * r) v = L2[static_cast<size_t>(c % r) * N + n];
        l2t[idx] = v;
    }
}

}  // namespace wlq
