// quantize.cuh -- RTN symmetric weight quantization on the GPU
// ("Joy-face_change_optimized" model card, files table and tools row: int8
// with one scale per output channel, int4 grouped along K with gs 64 / 16).
//
// Per group: a = max|W| (exact), s = a / qmax as an IEEE fp32 division, and
// q = the integer nearest to W / s with ties to even, clamped to +-qmax.  The
// quotient is estimated in fp64 and then corrected with the exact residual
// W - k*s (k*s has at most 32 significant bits, so one fp64 fma gives it
// exactly); the code therefore equals the exact real rounding, independent of
// how the estimate was rounded.
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

__device__ __forceinline__ float abs_finite_max(float a, float v, bool& bad) {
    bad |= !isfinite(v);
    return fmaxf(a, fabsf(v));
}

__device__ __forceinline__ uint32_t pack_codes4(float4 v, float s, double inv, int qmax, bool& bad) {
    const float f[4] = {v.x, v.y, v.z, v.w};
    uint32_t out = 0;
    for (int i = 0; i < 4; ++i) {
        int q = 0;
        if (isfinite(f[i])) q = rtn_code(f[i], s, inv, qmax);
        else bad = true;
        out |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * i);
    }
    return out;
}

// One CTA per row: the group is the whole row (per output channel).
template <int THREADS>
__global__ void __launch_bounds__(THREADS) quantize_rows_kernel(
    const float* __restrict__ W, int64_t N, int64_t K, int qmax, int8_t* __restrict__ codes,
    float* __restrict__ scales) {
    __shared__ float red[THREADS / 32];
    const int64_t K4 = K / 4;
    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        const float4* row = reinterpret_cast<const float4*>(W + n * K);
        float a = 0.0f;
        bool bad = false;
        for (int64_t i = threadIdx.x; i < K4; i += THREADS) {
            const float4 v = __ldg(row + i);
            a = abs_finite_max(a, v.x, bad);
            a = abs_finite_max(a, v.y, bad);
            a = abs_finite_max(a, v.z, bad);
            a = abs_finite_max(a, v.w, bad);
        }
        for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
        __syncthreads();
        a = red[0];
        for (int i = 1; i < THREADS / 32; ++i) a = fmaxf(a, red[i]);
        __syncthreads();
        const float s = __fdiv_rn(a, static_cast<float>(qmax));
        const double inv = (s > 0.0f) ? 1.0 / static_cast<double>(s) : 0.0;
        if (threadIdx.x == 0) scales[n] = s;
        uint32_t* out = reinterpret_cast<uint32_t*>(codes + n * K);
        for (int64_t i = threadIdx.x; i < K4; i += THREADS)
            out[i] = pack_codes4(row[i], s, inv, qmax, bad);
        if (bad) raise_error(ERRBIT_NONFINITE);
    }
}

// Groups of L = group/4 threads (one float4 each); groups never straddle a
// warp because L divides 32 and every row holds a whole number of groups.
__global__ void __launch_bounds__(256) quantize_groups_kernel(
    const float* __restrict__ W, int64_t total4, int lanes_per_group, int qmax,
    int8_t* __restrict__ codes, float* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const float4* W4 = reinterpret_cast<const float4*>(W);
    uint32_t* out = reinterpret_cast<uint32_t*>(codes);
    bool bad = false;
    for (int64_t base = warp0 * 32; base < total4; base += nwarps * 32) {
        const int64_t i = base + lane;
        const bool valid = i < total4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) v = __ldg(W4 + i);
        float a = 0.0f;
        bool b2 = false;
        a = abs_finite_max(a, v.x, b2);
        a = abs_finite_max(a, v.y, b2);
        a = abs_finite_max(a, v.z, b2);
        a = abs_finite_max(a, v.w, b2);
        for (int off = lanes_per_group >> 1; off > 0; off >>= 1)
            a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        if (valid) {
            const float s = __fdiv_rn(a, static_cast<float>(qmax));
            const double inv = (s > 0.0f) ? 1.0 / static_cast<double>(s) : 0.0;
            if ((lane & (lanes_per_group - 1)) == 0) scales[i / lanes_per_group] = s;
            out[i] = pack_codes4(v, s, inv, qmax, bad);
        }
    }
    if (bad) raise_error(ERRBIT_NONFINITE);
}

}  // namespace wlq
