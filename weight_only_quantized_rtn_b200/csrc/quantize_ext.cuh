// quantize_ext.cuh -- RTN for other widths, inputs and scale formats, and fp8
// block quantization ("Joy-face_change_optimized" model card: tools row, RTN
// per channel or per group; section 1, the KV-dtype setting: image K/V cached
// as int8 with one scale per token and head; section 2, a 5-bit MLP; section
// 1.1, DiT blocks quantized to fp8 on the GPU).
//
// quantize_ex_kernel: for each group (g inputs of a row), a = max|W| exactly,
// the stored scale s = the value of the scale format nearest to a / qmax
// (fp32: IEEE division; fp16 / bf16: the exactly rounded quotient, found in
// fp32 arithmetic by stored_scale), and
// q = clamp(RTN(W / s), +-qmax) computed exactly with that stored s (a 16-bit
// s may lie below a / qmax, so the clamp can act).  A group holding a NaN or
// an infinity, or whose 16-bit scale overflows, gets s = 0 and codes 0 and
// sets the non-finite error bit.
//
// quantize_fp8_kernel: s = fp32(a / 448); each weight becomes
// e4m3(RN(fp32(W / s))) saturated to +-448 (one rounding from the fp32
// quotient, cvt.rn.satfinite); an all-zero group has s = 0 and codes 0.
//
// One warp per group (grid-stride); a lane takes four adjacent inputs at a
// time (groups are multiples of 4 inputs).  Pass 1 reduces the absmax, pass 2
// re-reads the group (from L1 / L2) and writes the codes.  Groups of at most
// 128 inputs whose g / 4 divides 32 take quantize_ex_short_kernel instead.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "quantize.cuh"

namespace wlq {

enum ScaleFmt : int { SCALE_F32 = 0, SCALE_F16 = 1, SCALE_BF16 = 2 };

template <bool IN_BF16>
__device__ __forceinline__ float4 load4(const void* W, int64_t i4) {
    if constexpr (IN_BF16) {
        const uint2 u = reinterpret_cast<const uint2*>(W)[i4];
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    } else {
        return reinterpret_cast<const float4*>(W)[i4];
    }
}

__device__ __forceinline__ uint32_t absbits_max4(float4 v) {
    return max(max(__float_as_uint(v.x) & 0x7FFFFFFFu, __float_as_uint(v.y) & 0x7FFFFFFFu),
               max(__float_as_uint(v.z) & 0x7FFFFFFFu, __float_as_uint(v.w) & 0x7FFFFFFFu));
}

// The stored scale: the value of the scale format nearest to a / qmax
// (ties to even).  fp32: the IEEE division.  fp16 / bf16, from fp32
// arithmetic: q = RN32(a / qmax) rounds to the same 16-bit value as the exact
// quotient unless q itself is the midpoint of two 16-bit neighbours (fp32
// rounding cannot step over such a midpoint, which fp32 represents); there
// the sign of the exact residual a - q qmax picks the neighbour (a midpoint
// of two 16-bit values has at most 12 significant bits and qmax at most 7,
// so q qmax is exact, and so is the fma's result, a small difference of
// nearby values).  An exact
// quotient on the midpoint keeps the even neighbour.
template <int SF>
__device__ __forceinline__ float stored_scale(float a, int qmax) {
    const float qf = static_cast<float>(qmax);
    const float q = __fdiv_rn(a, qf);
    if constexpr (SF == SCALE_F32) {
        return q;
    } else {
        float lo, hi, rn;
        if constexpr (SF == SCALE_F16) {
            lo = __half2float(__float2half_rd(q));
            hi = __half2float(__float2half_ru(q));
            rn = __half2float(__float2half_rn(q));
        } else {
            lo = __bfloat162float(__float2bfloat16_rd(q));
            hi = __bfloat162float(__float2bfloat16_ru(q));
            rn = __bfloat162float(__float2bfloat16_rn(q));
        }
        if (lo != hi && __fsub_rn(q, lo) == __fsub_rn(hi, q)) {
            const float r = __fmaf_rn(-q, qf, a);
            if (r > 0.0f) return hi;
            if (r < 0.0f) return lo;
        }
        return rn;
    }
}

// rtn4_f32 with the codes clamped to [-qmax, qmax] before they are packed:
// a 16-bit scale may lie below a / qmax, so |W / s| may pass qmax + 1/2 (by at
// most a 2^-8 fraction: still below 128, where rtn4_f32's estimate holds, but
// the rounded code can be qmax + 1).
__device__ __forceinline__ uint32_t rtn4_f32_clamped(float4 v, float s, float inv, float h, float qmax) {
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
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float k = __fsub_rn(km[i], kMagic);
        if (near_half) {
            const float e = __fmaf_rn(-k, s, w[i]);
            k = (e > h) ? k + 1.0f : k;
            k = (e < -h) ? k - 1.0f : k;
            if (fabsf(e) == h) {  // exact tie between k and k + sign(e): keep the even one
                if (__float_as_uint(__fadd_rn(k, kMagic)) & 1u) k += (e > 0.0f) ? 1.0f : -1.0f;
            }
        }
        km[i] = __fadd_rn(fminf(fmaxf(k, -qmax), qmax), kMagic);
    }
    uint32_t lo, hi, out;
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(lo) : "r"(__float_as_uint(km[0])), "r"(__float_as_uint(km[1])));
    asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(hi) : "r"(__float_as_uint(km[2])), "r"(__float_as_uint(km[3])));
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(out) : "r"(lo), "r"(hi));
    return out;
}

template <bool IN_BF16, int SF>
__global__ void __launch_bounds__(256) quantize_ex_kernel(const void* __restrict__ W, int64_t groups, int g4,
                                                          int qmax, int8_t* __restrict__ codes,
                                                          void* __restrict__ scales) {
    grid_dependency_sync();
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    bool bad = false;
    for (int64_t gi = w0; gi < groups; gi += nw) {
        const int64_t base = gi * g4;  // first float4 of the group
        uint32_t m = 0;
        for (int j = lane; j < g4; j += 32) m = max(m, absbits_max4(load4<IN_BF16>(W, base + j)));
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        bool gbad = m >= 0x7F800000u;  // NaN or infinity in the group
        const float a = gbad ? 0.0f : __uint_as_float(m);
        float s = stored_scale<SF>(a, qmax);
        if (isinf(s)) {  // the 16-bit scale overflowed
            gbad = true;
            s = 0.0f;
        }
        bad |= gbad;
        if (lane == 0) {
            if constexpr (SF == SCALE_F32) static_cast<float*>(scales)[gi] = s;
            else if constexpr (SF == SCALE_F16) static_cast<__half*>(scales)[gi] = __float2half_rn(s);
            else static_cast<__nv_bfloat16*>(scales)[gi] = __float2bfloat16_rn(s);
        }
        GroupScale gs;
        gs.s = s;
        gs.normal = s >= 1.17549435e-38f;
        gs.inv = gs.normal ? __frcp_rn(s) : 0.0f;
        gs.inv64 = (!gs.normal && s > 0.0f) ? 1.0 / static_cast<double>(s) : 0.0;
        uint32_t* out = reinterpret_cast<uint32_t*>(codes);
        for (int j = lane; j < g4; j += 32) {
            const float4 v = load4<IN_BF16>(W, base + j);
            uint32_t c = 0;
            if (gs.normal) {
                const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    c |= rtn_byte_f32(w[e], gs.s, gs.inv, static_cast<float>(qmax)) << (8 * e);
            } else {
                bool unused = false;
                c = pack_codes4(v, gs, qmax, unused);  // s == 0 (and non-finite weights) give code 0
            }
            out[base + j] = c;
        }
    }
    if (bad) raise_error(ERRBIT_NONFINITE);
}

// Short groups (g / 4 divides 32: g <= 128), one pass: a warp takes 32 / L
// groups at once, L = g / 4 lanes each (one float4 per lane), and U such
// warp-rounds are loaded before any is quantized.  Same arithmetic as
// quantize_ex_kernel, from registers.
template <bool IN_BF16, int SF, int L>
__global__ void __launch_bounds__(256) quantize_ex_short_kernel(const void* __restrict__ W, int64_t groups,
                                                                int qmax, int8_t* __restrict__ codes,
                                                                void* __restrict__ scales) {
    grid_dependency_sync();
    constexpr int U = 4;
    constexpr int GPW = 32 / L;  // groups per warp-round
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t total4 = groups * L;
    uint32_t* out = reinterpret_cast<uint32_t*>(codes);
    bool bad = false;
    for (int64_t r0 = w0 * U; r0 * GPW < groups; r0 += nw * U) {
        float4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i4 = (r0 + u) * 32 + lane;  // float4 index: group (r0+u)*GPW + lane / L
            v[u] = i4 < total4 ? load4<IN_BF16>(W, i4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        uint32_t m[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            m[u] = absbits_max4(v[u]);
#pragma unroll
            for (int off = L >> 1; off > 0; off >>= 1) m[u] = max(m[u], __shfl_xor_sync(0xffffffffu, m[u], off));
        }
        // The warp holds NGW = U * GPW groups.  When they fit one per lane, lane
        // j works out the scale of group (j / GPW, j % GPW) -- the division, the
        // 16-bit rounding and the reciprocal once per group, not once per lane
        // of it -- and the results go back to each group's lanes by shuffle.
        constexpr int NGW = U * GPW;
        float su[U], iu[U];
        if constexpr (NGW <= 32) {
            const int ju = lane / GPW, jg = lane % GPW;
            uint32_t mj = 0;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t mu = __shfl_sync(0xffffffffu, m[u], jg * L);
                if (ju == u) mj = mu;
            }
            bool gbad = mj >= 0x7F800000u;  // NaN or infinity in the group
            float sj = stored_scale<SF>(gbad ? 0.0f : __uint_as_float(mj), qmax);
            if (isinf(sj)) {  // the 16-bit scale overflowed
                gbad = true;
                sj = 0.0f;
            }
            const float ij = (sj >= 1.17549435e-38f) ? __frcp_rn(sj) : 0.0f;
            const int64_t gj = (r0 + ju) * GPW + jg;
            if (lane < NGW && gj < groups) {
                bad |= gbad;
                if constexpr (SF == SCALE_F32) static_cast<float*>(scales)[gj] = sj;
                else if constexpr (SF == SCALE_F16) static_cast<__half*>(scales)[gj] = __float2half_rn(sj);
                else static_cast<__nv_bfloat16*>(scales)[gj] = __float2bfloat16_rn(sj);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                su[u] = __shfl_sync(0xffffffffu, sj, u * GPW + lane / L);
                iu[u] = __shfl_sync(0xffffffffu, ij, u * GPW + lane / L);
            }
        } else {
            // short groups (4 or 8 inputs): at most two lanes share a group
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t i4 = (r0 + u) * 32 + lane;
                bool gbad = m[u] >= 0x7F800000u;
                float sg = stored_scale<SF>(gbad ? 0.0f : __uint_as_float(m[u]), qmax);
                if (isinf(sg)) {
                    gbad = true;
                    sg = 0.0f;
                }
                su[u] = sg;
                iu[u] = (sg >= 1.17549435e-38f) ? __frcp_rn(sg) : 0.0f;
                if (i4 < total4) {
                    bad |= gbad;
                    if ((lane & (L - 1)) == 0) {
                        const int64_t gi = i4 / L;
                        if constexpr (SF == SCALE_F32) static_cast<float*>(scales)[gi] = sg;
                        else if constexpr (SF == SCALE_F16) static_cast<__half*>(scales)[gi] = __float2half_rn(sg);
                        else static_cast<__nv_bfloat16*>(scales)[gi] = __float2bfloat16_rn(sg);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i4 = (r0 + u) * 32 + lane;
            if (i4 >= total4) continue;
            const float sg = su[u];
            uint32_t c = 0;
            if (sg >= 1.17549435e-38f) {
                if constexpr (SF == SCALE_F32) c = rtn4_f32(v[u], sg, iu[u], 0.5f * sg);  // |W/s| < qmax + 1/2
                else c = rtn4_f32_clamped(v[u], sg, iu[u], 0.5f * sg, static_cast<float>(qmax));
            } else if (sg > 0.0f) {
                GroupScale gs;
                gs.s = sg;
                gs.normal = false;
                gs.inv = 0.0f;
                gs.inv64 = 1.0 / static_cast<double>(sg);
                bool unused = false;
                c = pack_codes4(v[u], gs, qmax, unused);
            }
            out[i4] = c;
        }
    }
    if (bad) raise_error(ERRBIT_NONFINITE);
}

// bf16 input, groups of G = E * LG inputs (LG a power of two, at most 32):
// a lane takes E = 8 or 16 adjacent inputs (one or two 16-byte loads) a
// round, so a warp covers 32 E inputs a round, with four loads a lane in
// flight; when the warp's groups fit one per lane, each scale is worked out
// once, by one lane.  The group's
// absmax is the maximum of the bf16 magnitude bits (two at a time, 16-bit
// lanes), reduced over its LG lanes; the stored scale and the exactly rounded
// codes are those of quantize_ex_short_kernel (same stored_scale, same
// rtn4_f32 / rtn4_f32_clamped), so the results are bit-identical.  Codes go
// out as one E-byte store per lane (codes E-byte aligned).
template <int SF, int LG, int E>
__global__ void __launch_bounds__(256) quantize_ex_bf16_kernel(const uint16_t* __restrict__ W, int64_t totalE,
                                                               int qmax, int8_t* __restrict__ codes,
                                                               void* __restrict__ scales) {
    grid_dependency_sync();
    constexpr int NQ = E / 8;          // 16-byte loads a lane per round
    constexpr int U = 4 / NQ;          // rounds in flight (four 16-byte loads a lane)
    constexpr int GPR = 32 / LG;       // groups per warp-round
    constexpr int NGW = U * GPR;       // groups the warp holds
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const uint4* W8 = reinterpret_cast<const uint4*>(W);
    bool bad = false;
    for (int64_t r0 = w0 * U; r0 * 32 < totalE; r0 += nw * U) {
        uint4 raw[U][NQ];
        uint32_t m[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t ie = (r0 + u) * 32 + lane;
#pragma unroll
            for (int q = 0; q < NQ; ++q)
                raw[u][q] = ie < totalE ? __ldcs(W8 + ie * NQ + q) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            uint32_t m2 = 0;
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const uint4 r = raw[u][q];
                m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(r.x & 0x7FFF7FFFu, r.y & 0x7FFF7FFFu),
                                           __vmaxu2(r.z & 0x7FFF7FFFu, r.w & 0x7FFF7FFFu)));
            }
            m[u] = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
            for (int off = LG >> 1; off > 0; off >>= 1) m[u] = max(m[u], __shfl_xor_sync(0xffffffffu, m[u], off));
        }
        float su[U], iu[U];
        bool bu[U];
        if constexpr (NGW <= 32) {
            // lane j works out the scale of group (j / GPR, j % GPR) once -- the 16-bit rounding and
            // the reciprocal per group, not per lane of it -- and the results go back by shuffle
            const int ju = lane / GPR, jg = lane % GPR;
            uint32_t mj = 0;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t mu = __shfl_sync(0xffffffffu, m[u], jg * LG);
                if (ju == u) mj = mu;
            }
            bool gbad = mj >= 0x7F80u;  // NaN or infinity in the group
            float sj = stored_scale<SF>(gbad ? 0.0f : __uint_as_float(mj << 16), qmax);
            if (isinf(sj)) {  // the 16-bit scale overflowed
                gbad = true;
                sj = 0.0f;
            }
            const float ij = (sj >= 1.17549435e-38f) ? __frcp_rn(sj) : 0.0f;
            const int gb = gbad ? 1 : 0;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                su[u] = __shfl_sync(0xffffffffu, sj, u * GPR + lane / LG);
                iu[u] = __shfl_sync(0xffffffffu, ij, u * GPR + lane / LG);
                bu[u] = __shfl_sync(0xffffffffu, gb, u * GPR + lane / LG) != 0;
            }
        } else {
            // one group per lane or two lanes a group: each lane its own
#pragma unroll
            for (int u = 0; u < U; ++u) {
                bool gbad = m[u] >= 0x7F80u;
                float sg = stored_scale<SF>(gbad ? 0.0f : __uint_as_float(m[u] << 16), qmax);
                if (isinf(sg)) {
                    gbad = true;
                    sg = 0.0f;
                }
                su[u] = sg;
                iu[u] = (sg >= 1.17549435e-38f) ? __frcp_rn(sg) : 0.0f;
                bu[u] = gbad;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t ie = (r0 + u) * 32 + lane;
            if (ie >= totalE) continue;
            const float sg = su[u];
            bad |= bu[u];
            if ((lane & (LG - 1)) == 0) {
                const int64_t gi = ie / LG;
                if constexpr (SF == SCALE_F32) static_cast<float*>(scales)[gi] = sg;
                else if constexpr (SF == SCALE_F16) static_cast<__half*>(scales)[gi] = __float2half_rn(sg);
                else static_cast<__nv_bfloat16*>(scales)[gi] = __float2bfloat16_rn(sg);
            }
            uint32_t c[2 * NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const uint4 r = raw[u][q];
                const float4 lo = make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xFFFF0000u),
                                              __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xFFFF0000u));
                const float4 hi = make_float4(__uint_as_float(r.z << 16), __uint_as_float(r.z & 0xFFFF0000u),
                                              __uint_as_float(r.w << 16), __uint_as_float(r.w & 0xFFFF0000u));
                c[2 * q] = c[2 * q + 1] = 0;
                if (sg >= 1.17549435e-38f) {
                    if constexpr (SF == SCALE_F32) {
                        c[2 * q] = rtn4_f32(lo, sg, iu[u], 0.5f * sg);
                        c[2 * q + 1] = rtn4_f32(hi, sg, iu[u], 0.5f * sg);
                    } else {
                        c[2 * q] = rtn4_f32_clamped(lo, sg, iu[u], 0.5f * sg, static_cast<float>(qmax));
                        c[2 * q + 1] = rtn4_f32_clamped(hi, sg, iu[u], 0.5f * sg, static_cast<float>(qmax));
                    }
                } else if (sg > 0.0f) {
                    GroupScale gs;
                    gs.s = sg;
                    gs.normal = false;
                    gs.inv = 0.0f;
                    gs.inv64 = 1.0 / static_cast<double>(sg);
                    bool unused = false;
                    c[2 * q] = pack_codes4(lo, gs, qmax, unused);
                    c[2 * q + 1] = pack_codes4(hi, gs, qmax, unused);
                }
            }
            if constexpr (NQ == 1) reinterpret_cast<uint2*>(codes)[ie] = make_uint2(c[0], c[1]);
            else reinterpret_cast<uint4*>(codes)[ie] = make_uint4(c[0], c[1], c[2], c[3]);
        }
    }
    if (bad) raise_error(ERRBIT_NONFINITE);
}

__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

template <bool IN_BF16>
__global__ void __launch_bounds__(256) quantize_fp8_kernel(const void* __restrict__ W, int64_t groups, int g4,
                                                           uint8_t* __restrict__ codes, float* __restrict__ scales) {
    grid_dependency_sync();
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    bool bad = false;
    for (int64_t gi = w0; gi < groups; gi += nw) {
        const int64_t base = gi * g4;
        uint32_t m = 0;
        for (int j = lane; j < g4; j += 32) m = max(m, absbits_max4(load4<IN_BF16>(W, base + j)));
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        const bool gbad = m >= 0x7F800000u;
        bad |= gbad;
        const float s = gbad ? 0.0f : __fdiv_rn(__uint_as_float(m), 448.0f);
        if (lane == 0) scales[gi] = s;
        uint32_t* out = reinterpret_cast<uint32_t*>(codes);
        for (int j = lane; j < g4; j += 32) {
            uint32_t c = 0;
            if (s != 0.0f) {
                const float4 v = load4<IN_BF16>(W, base + j);
                const uint32_t lo = cvt_e4m3x2(__fdiv_rn(v.x, s), __fdiv_rn(v.y, s));
                const uint32_t hi = cvt_e4m3x2(__fdiv_rn(v.z, s), __fdiv_rn(v.w, s));
                c = lo | (hi << 16);
            }
            out[base + j] = c;
        }
    }
    if (bad) raise_error(ERRBIT_NONFINITE);
}

}  // namespace wlq
