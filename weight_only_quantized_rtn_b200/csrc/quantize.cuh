// quantize.cuh -- RTN symmetric weight quantization on the GPU
// ("Joy-face_change_optimized" model card, files table and tools row: int8
// with one scale per output channel, int4 grouped along K with gs 64 / 16).
//
// Per group: a = max|W| (exact), s = a / qmax as an IEEE fp32 division, and
// q = the integer nearest to W / s with ties to even, clamped to +-qmax.  An
// estimate k of the quotient (within one of the answer) is corrected with the
// exact residual e = W - k*s, compared against s/2: the code therefore equals
// the rounding of the exact real quotient, whatever rounding the estimate
// had.  Normal scales take an fp32 path (rtn_byte_f32); subnormal ones an
// fp64 path (rtn_code), where k*s has at most 32 significant bits and one
// fp64 fma gives e exactly.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace wlq {

__device__ __forceinline__ int rtn_code(float w, float s, double inv_s, int qmax) {
    if (s == 0.0f) return 0;
    double k = rint(static_cast<double>(w) * inv_s);             // within 1 of the answer
    const double e = fma(-k, static_cast<double>(s), static_cast<double>(w));  // exact
    const double h = 0.5 * static_cast<double>(s);
    if (e > h) {
        k += 1.0;
    } else if (e < -h) {
        k -= 1.0;
    } else if (e == h || e == -h) {  // exact tie between k and k +- 1: keep the even one
        if (static_cast<int>(k) & 1) k += (e > 0.0) ? 1.0 : -1.0;
    }
    const double qm = static_cast<double>(qmax);
    k = fmin(fmax(k, -qm), qm);
    return static_cast<int>(k);
}

// The same exact rounding in fp32 for a normal scale (s >= 2^-126).  Adding
// 1.5 * 2^23 rounds any |t| < 2^22 to an integer, ties to even.  The residual
// e = w - k*s from one fp32 fma is exact wherever it decides anything: for
// |e| near s/2 its significand fits in 24 bits (|w| >= s/2 there, so w's last
// bit is at least half of s's).  Returns the code's two's-complement byte.
__device__ __forceinline__ uint32_t rtn_byte_f32(float w, float s, float inv, float qmax) {
    const float kMagic = 12582912.0f;  // 1.5 * 2^23
    float k = __fsub_rn(__fadd_rn(__fmul_rn(w, inv), kMagic), kMagic);
    const float e = __fmaf_rn(-k, s, w);
    const float h = 0.5f * s;
    if (e > h) {
        k += 1.0f;
    } else if (e < -h) {
        k -= 1.0f;
    } else if (e == h || e == -h) {  // exact tie: keep the even neighbour
        if (__float_as_uint(__fadd_rn(k, kMagic)) & 1u) k += (e > 0.0f) ? 1.0f : -1.0f;
    }
    k = fminf(fmaxf(k, -qmax), qmax);
    return __float_as_uint(__fadd_rn(k, kMagic)) & 0xFFu;  // low byte of 0x4B400000 + k
}

__device__ __forceinline__ float abs_finite_max(float a, float v, bool& bad) {
    bad |= !isfinite(v);
    return fmaxf(a, fabsf(v));
}

struct GroupScale {
    float s;       // fp32(absmax / qmax)
    float inv;     // fp32 1/s (normal s only)
    double inv64;  // fp64 1/s
    bool normal;   // s >= 2^-126: the fp32 path is exact
};

__device__ __forceinline__ GroupScale group_scale(float a, int qmax) {
    GroupScale g;
    g.s = __fdiv_rn(a, static_cast<float>(qmax));
    g.normal = g.s >= 1.17549435e-38f;
    g.inv = g.normal ? __frcp_rn(g.s) : 0.0f;
    g.inv64 = (!g.normal && g.s > 0.0f) ? 1.0 / static_cast<double>(g.s) : 0.0;  // subnormal path only
    return g;
}

__device__ __forceinline__ uint32_t pack_codes4(float4 v, const GroupScale& g, int qmax, bool& bad) {
    const float f[4] = {v.x, v.y, v.z, v.w};
    uint32_t out = 0;
    for (int i = 0; i < 4; ++i) {
        uint32_t byte = 0;
        if (!isfinite(f[i])) bad = true;
        else if (g.normal) byte = rtn_byte_f32(f[i], g.s, g.inv, static_cast<float>(qmax));
        else byte = static_cast<uint32_t>(rtn_code(f[i], g.s, g.inv64, qmax)) & 0xFFu;
        out |= byte << (8 * i);
    }
    return out;
}

// One warp per row, for rows longer than the per-CTA kernel holds: the group
// is the whole row (per output channel).  Pass 1 reads the row for its absmax,
// pass 2 reads it again (from L2: the row was just read) to round and store
// the codes; eight loads in flight per lane.
__global__ void __launch_bounds__(256) quantize_rows_kernel(
    const float* __restrict__ W, int64_t N, int64_t K, int qmax, int8_t* __restrict__ codes,
    float* __restrict__ scales) {
    grid_dependency_sync();
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t K4 = K / 4;
    for (int64_t n = w0; n < N; n += nw) {
        const float4* row = reinterpret_cast<const float4*>(W + n * K);
        float a = 0.0f;
        bool bad = false;
#pragma unroll 8
        for (int64_t i = lane; i < K4; i += 32) {
            const float4 v = __ldg(row + i);
            a = abs_finite_max(a, v.x, bad);
            a = abs_finite_max(a, v.y, bad);
            a = abs_finite_max(a, v.z, bad);
            a = abs_finite_max(a, v.w, bad);
        }
        for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        const GroupScale g = group_scale(a, qmax);
        if (lane == 0) scales[n] = g.s;
        uint32_t* out = reinterpret_cast<uint32_t*>(codes + n * K);
#pragma unroll 8
        for (int64_t i = lane; i < K4; i += 32) out[i] = pack_codes4(__ldcs(row + i), g, qmax, bad);
        if (bad) raise_error(ERRBIT_NONFINITE);
    }
}

// RTN of four weights of one group with a normal fp32 scale (s >= 2^-126),
// packed as two's-complement bytes, bit-identical to rtn_byte_f32.
//  - t = W * (1/s) (two roundings) is within 2^-15 of the exact quotient W/s
//    for |W/s| <= 128, so k = rint(t) is the answer unless t lies within
//    2^-12 of a half-integer.  Such rare weights (and exact ties) take the
//    exact path: residual e = W - k*s from one fma, compared with s/2.
//  - No clamp: s = RN(a/qmax) and |W| <= a give |W/s| < qmax + 1/2, so the
//    code never leaves [-qmax, qmax].
//  - k + 1.5*2^23 holds k in its low bits; byte permutes gather the four
//    low bytes.  h = s / 2, inv = 1 / s rounded.
__device__ __forceinline__ uint32_t rtn4_f32(float4 v, float s, float inv, float h) {
    const float kMagic = 12582912.0f;  // 1.5 * 2^23
    const float w[4] = {v.x, v.y, v.z, v.w};
    float km[4];
    bool near_half = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float t = __fmul_rn(w[i], inv);
        km[i] = __fadd_rn(t, kMagic);
        const float d = __fsub_rn(t, __fsub_rn(km[i], kMagic));
        near_half |= fabsf(d) > 0.499755859375f;  // 1/2 - 2^-12
    }
    if (near_half) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float k = __fsub_rn(km[i], kMagic);
            const float e = __fmaf_rn(-k, s, w[i]);
            k = (e > h) ? k + 1.0f : k;
            k = (e < -h) ? k - 1.0f : k;
            if (fabsf(e) == h) {  // exact tie between k and k + sign(e): keep the even one
                if (__float_as_uint(__fadd_rn(k, kMagic)) & 1u) k += (e > 0.0f) ? 1.0f : -1.0f;
            }
            km[i] = __fadd_rn(k, kMagic);
        }
    }
    uint32_t lo, hi, out;
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(lo) : "r"(__float_as_uint(km[0])), "r"(__float_as_uint(km[1])));
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(hi) : "r"(__float_as_uint(km[2])), "r"(__float_as_uint(km[3])));
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(out) : "r"(lo), "r"(hi));
    return out;
}

// One CTA per row (grid-stride over rows) for rows of up to 32768 inputs: the
// row is read once, straight into registers (V float4 per thread, all loads
// in flight together), its absmax is reduced over the CTA, and the codes are
// computed from the registers.  Every byte of W crosses HBM exactly once.
// The absmax is taken on the magnitude bit patterns: for non-negative IEEE
// values the unsigned order is the numeric order, and any NaN or infinity
// sorts above every finite value, so one compare at the end detects them.
template <int V>
__global__ void __launch_bounds__(1024) quantize_rows_cta_kernel(
    const float* __restrict__ W, int64_t N, int64_t K, int qmax, int8_t* __restrict__ codes,
    float* __restrict__ scales) {
    grid_dependency_sync();
    __shared__ uint32_t part[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int K4 = static_cast<int>(K / 4);
    bool bad = false;
    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        const float4* row = reinterpret_cast<const float4*>(W + n * K);
        float4 v[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int idx = threadIdx.x + i * blockDim.x;
            v[i] = idx < K4 ? __ldcs(row + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
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
        if (threadIdx.x == 0) scales[n] = g.s;
        uint32_t* out = reinterpret_cast<uint32_t*>(codes + n * K);
        if (g.normal) {
            const float h = 0.5f * g.s;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int idx = threadIdx.x + i * blockDim.x;
                if (idx < K4) out[idx] = rtn4_f32(v[i], g.s, g.inv, h);
            }
        } else {
            bool unused = false;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int idx = threadIdx.x + i * blockDim.x;
                if (idx < K4) out[idx] = pack_codes4(v[i], g, qmax, unused);
            }
        }
        __syncthreads();  // part[] is rewritten for the next row
    }
    if (bad) raise_error(ERRBIT_NONFINITE);
}

// Groups of L = group/4 threads (one float4 each); groups never straddle a
// warp because L divides 32 and every row holds a whole number of groups.
// Four float4 per thread are loaded before any is processed; absmax and RTN
// as in quantize_rows_cta_kernel.
__global__ void __launch_bounds__(256) quantize_groups_kernel(
    const float* __restrict__ W, int64_t total4, int lanes_per_group, int qmax,
    int8_t* __restrict__ codes, float* __restrict__ scales) {
    grid_dependency_sync();
    constexpr int U = 4;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const float4* W4 = reinterpret_cast<const float4*>(W);
    uint32_t* out = reinterpret_cast<uint32_t*>(codes);
    bool bad = false;
    for (int64_t base = warp0 * 32 * U; base < total4; base += nwarps * 32 * U) {
        float4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + u * 32 + lane;
            v[u] = i < total4 ? __ldcs(W4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + u * 32 + lane;
            uint32_t m = max(max(__float_as_uint(v[u].x) & 0x7FFFFFFFu, __float_as_uint(v[u].y) & 0x7FFFFFFFu),
                             max(__float_as_uint(v[u].z) & 0x7FFFFFFFu, __float_as_uint(v[u].w) & 0x7FFFFFFFu));
            for (int off = lanes_per_group >> 1; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
            if (i >= total4) continue;
            const bool gbad = m >= 0x7F800000u;  // NaN or infinity in the group
            bad |= gbad;
            const GroupScale gs = group_scale(gbad ? 0.0f : __uint_as_float(m), qmax);
            if ((lane & (lanes_per_group - 1)) == 0) scales[i / lanes_per_group] = gs.s;
            bool unused = false;
            out[i] = gs.normal ? rtn4_f32(v[u], gs.s, gs.inv, 0.5f * gs.s) : pack_codes4(v[u], gs, qmax, unused);
        }
    }
    if (bad) raise_error(ERRBIT_NONFINITE);
}

}  // namespace wlq
