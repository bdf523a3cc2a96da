// nvfp4.cuh -- NVFP4 (4-bit E2M1 elements, one E4M3 scale per 16 inputs of a
// row, one fp32 scale per tensor): the number format of the W4A4 SVDQuant
// kernels on Blackwell ("Nunchaku Lite: loading and running 4-bit SVDQuant",
// section "hardware and precision support": the NVFP4 variant of svdq_w4a4
// runs on Blackwell, B200 included; section "why it matters": weights and
// activations in 4 bits, the hard part of the weights in a 16-bit low-rank
// branch).
//
// Quantization of a [rows, K] tensor X:
//   g   = fp32(amax(X) / 2688)                 2688 = 6 (largest E2M1) x 448 (largest E4M3)
//   s_b = E4M3 nearest a_b / (6 g)             a_b = max |x| over the 16 inputs of block b;
//                                              ties to even, saturated at 448; 0 when g = 0
//   q   = E2M1 nearest x / (s_b g)             ties to an even significand, saturated at 6;
//                                              0 when s_b = 0
// Every decision is exact.  a_b / (6 g) is formed in fp64 from the fp32
// operands: a quotient of a 24-bit by a 26-bit number is either an E4M3
// midpoint exactly or at least 2^-31 away from one (relative), far above
// fp64's rounding error.  The element decision compares |x| with the seven
// midpoints t (0.25, 0.75, ..., 5) times d = s_b g: each threshold's rounded
// product and exact fma error give the smallest fp32 value that passes it,
// so the decision is one exact fp32 comparison per threshold (in fp64 for
// tensors with amax below ~1e-26, where the error could underflow); no
// division is rounded.
//
// Layouts (what the block-scaled tensor-core MMA reads):
//   codes  : [rows, K / 2] bytes, input k in byte k / 2, low nibble for even k;
//            E2M1 code = sign << 3 | magnitude code (0, 0.5, 1, 1.5, 2, 3, 4, 6)
//   scales : 512-byte atoms, one per (128-row tile, 64 inputs of K); atom
//            (t, a) at ((t * KA) + a) * 512 with KA = ceil(K / 256) * 4, and in
//            it the scale of row 128 t + 32 i + j, block 4 a + c at byte
//            16 j + 4 i + c; rows are padded to a multiple of 256 and K to one
//            of 256, and rows and blocks past the tensor hold 0
//   gscale : [0] g, [1] amax(X) (the first pass's accumulator)
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "prep.cuh"
#include "ptx.cuh"

namespace wlq {

constexpr int NV_ATOM_BYTES = 512;

__host__ __device__ constexpr int64_t nv_atoms_per_row_tile(int64_t K) { return ((K + 255) / 256) * 4; }
// rows padded to 256 (two 128-row tiles): a 256-token GEMM tile always has both halves
__host__ __device__ constexpr size_t nv_scale_bytes(int64_t rows, int64_t K) {
    return static_cast<size_t>((rows + 255) / 256) * 2 * static_cast<size_t>(nv_atoms_per_row_tile(K)) * NV_ATOM_BYTES;
}
__device__ __forceinline__ size_t nv_scale_offset(int64_t row, int64_t blk, int64_t KA) {
    const int64_t atom = (row >> 7) * KA + (blk >> 2);
    return static_cast<size_t>(atom) * NV_ATOM_BYTES + static_cast<size_t>((row & 31) * 16 + ((row >> 5) & 3) * 4 + (blk & 3));
}

// E4M3 (no infinities; 0x7f is NaN) nearest to q >= 0, ties to an even
// mantissa, saturated at 448 (0x7e).  Spacing 2^(E-3) in [2^E, 2^(E+1)),
// 2^-9 below 2^-6: q / spacing is an exact scaling, rounded half to even by
// the conversion to an integer.  q is an fp64 normal here (a quotient of
// fp32 values), so its exponent field is E + 1023.
__device__ __forceinline__ uint32_t e4m3_from_f64(double q) {
    if (!(q > 0.0)) return 0u;
    if (q >= 448.0) return 0x7eu;
    int E = static_cast<int>((static_cast<unsigned long long>(__double_as_longlong(q)) >> 52) & 0x7ff) - 1023;
    if (E < -6) E = -6;
    const double sc = __longlong_as_double(static_cast<long long>(1023 + 3 - E) << 52);  // 2^(3-E)
    long long n = __double2ll_rn(q * sc);                                                   // in [0, 16]
    if (n >= 16) {
        n = 8;
        E += 1;
    }
    if (n < 8) return static_cast<uint32_t>(n);  // below 2^-6 (E = -6): subnormal, or zero
    return (static_cast<uint32_t>(E + 7) << 3) | static_cast<uint32_t>(n - 8);
}
__device__ __forceinline__ double e4m3_to_f64(uint32_t b) {
    const int e = (b >> 3) & 15, m = b & 7;
    return e == 0 ? ldexp(static_cast<double>(m), -9) : ldexp(static_cast<double>(8 + m), e - 10);
}
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    const int e = (b >> 3) & 15, m = b & 7;
    return e == 0 ? static_cast<float>(m) * 0x1p-9f : static_cast<float>(8 + m) * __int_as_float((e - 10 + 127) << 23);
}

// |x| of 16 inputs (fp32 or bf16) into v[], with the sign bits in *sign.
template <int DT>
__device__ __forceinline__ void nv_load16(const void* X, size_t off, float (&v)[16], uint32_t* sign) {
    if constexpr (DT == 0) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(X) + off);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 f = __ldg(p + i);
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(X) + off);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint4 u = __ldg(p + i);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
            }
        }
    }
    uint32_t s = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        s |= (__float_as_uint(v[i]) >> 31) << i;
        v[i] = fabsf(v[i]);
    }
    *sign = s;
}

// Pass 1: amax(X) into gscale[1] (zeroed beforehand), as the bits of a
// non-negative float (their integer order is the float order).  Non-finite
// inputs set ERRBIT_NONFINITE.
template <int DT>
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const void* __restrict__ X, int64_t nblocks,
                                                         float* __restrict__ gscale) {
    grid_dependency_sync();
    float m = 0.0f;
    bool bad = false;
    for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks;
         b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float v[16];
        uint32_t sg;
        nv_load16<DT>(X, static_cast<size_t>(b) * 16, v, &sg);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            bad |= !(v[i] <= 3.4028234663852886e38f);  // inf or NaN
            m = fmaxf(m, v[i]);
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) raise_error(ERRBIT_NONFINITE);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wm[8];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float mm = wm[0];
        for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) mm = fmaxf(mm, wm[i]);
        atomicMax(reinterpret_cast<unsigned int*>(gscale + 1), __float_as_uint(mm));
    }
}

// Pass 2: one thread per block of 16 inputs (consecutive threads take
// consecutive blocks of a row, 2^lg_tpr threads a row): block scale, then each code by a three-step
// search over the midpoints.  A midpoint between codes i and i + 1 rounds up
// when i is odd (the even neighbour is i + 1), so "passed" is |x| >= T_i for
// odd i and |x| > T_i for even i.
template <int DT>
__global__ void __launch_bounds__(256) nvfp4_quantize_kernel(const void* __restrict__ X, int64_t rows, int64_t K,
                                                             float* __restrict__ gscale, uint8_t* __restrict__ codes,
                                                             uint8_t* __restrict__ scales, int lg_tpr) {
    grid_dependency_sync();
    const float amax = __uint_as_float(*reinterpret_cast<const volatile unsigned int*>(gscale + 1));
    const float g = __fdiv_rn(amax, 2688.0f);
    const int kb_per_row = static_cast<int>(K / 16);
    const int64_t KA = nv_atoms_per_row_tile(K);
    if (blockIdx.x == 0 && threadIdx.x == 0) gscale[0] = g;
    // 2^lg_tpr threads per row (the CTA covers 256 >> lg_tpr rows a pass): no index division
    const int tpr = 1 << lg_tpr, rpc = 256 >> lg_tpr;
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * rpc + (threadIdx.x >> lg_tpr); row < rows;
         row += static_cast<int64_t>(gridDim.x) * rpc)
    for (int kb = threadIdx.x & (tpr - 1); kb < kb_per_row; kb += tpr) {
        const int64_t b = row * kb_per_row + kb;
        float v[16];
        uint32_t sg;
        nv_load16<DT>(X, static_cast<size_t>(b) * 16, v, &sg);
        float ab = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) ab = fmaxf(ab, v[i]);
        const uint32_t sb = (g > 0.0f) ? e4m3_from_f64(static_cast<double>(ab) / (6.0 * static_cast<double>(g))) : 0u;
        uint32_t lo = 0, hi = 0;
        if (sb != 0 && g >= 1e-30f) {
            // T_i = t_i s_b g is carried as p_i = fl(u_i g) plus its exact fma error e_i (u_i = t_i s_b
            // has at most 7 bits; the error is exact while u_i g stays far above the subnormals).  From
            // them, A_i = the smallest fp32 value that passes T_i: p_i itself when p_i already passes
            // (p_i >= T_i for odd i, > T_i for even i), else the next float up.  |x| is an fp32 value,
            // so |x| passes T_i exactly when |x| >= A_i: one comparison per threshold.
            const float sf = e4m3_to_f32(sb);
            float A[7];
            const float tau[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
#pragma unroll
            for (int t = 0; t < 7; ++t) {
                const float u = tau[t] * sf;
                const float pt = __fmul_rn(u, g);
                const float et = __fmaf_rn(u, g, -pt);  // T_t - p_t, exact
                const bool p_passes = (t & 1) ? (et <= 0.0f) : (et < 0.0f);
                A[t] = p_passes ? pt : __int_as_float(__float_as_int(pt) + 1);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float a = v[i];
                const bool p4 = a >= A[3];
                const bool p2 = a >= (p4 ? A[5] : A[1]);
                const bool p1 = a >= (p4 ? (p2 ? A[6] : A[4]) : (p2 ? A[2] : A[0]));
                const uint32_t c = (p4 ? 4u : 0u) + (p2 ? 2u : 0u) + (p1 ? 1u : 0u) + (((sg >> i) & 1u) << 3);
                if (i < 8) lo |= c << (4 * i);
                else hi |= c << (4 * (i - 8));
            }
        } else if (sb != 0) {
            // tensors whose amax is below ~1e-26: the same decisions in fp64
            const double d = e4m3_to_f64(sb) * static_cast<double>(g);  // exact
            const double T0 = 0.25 * d, T1 = 0.75 * d, T2 = 1.25 * d, T3 = 1.75 * d, T4 = 2.5 * d, T5 = 3.5 * d,
                         T6 = 5.0 * d;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const double a = static_cast<double>(v[i]);
                const bool p4 = a >= T3;
                const bool p2 = a >= (p4 ? T5 : T1);
                const bool p1 = a > (p4 ? (p2 ? T6 : T4) : (p2 ? T2 : T0));
                const uint32_t c = (p4 ? 4u : 0u) + (p2 ? 2u : 0u) + (p1 ? 1u : 0u) + (((sg >> i) & 1u) << 3);
                if (i < 8) lo |= c << (4 * i);
                else hi |= c << (4 * (i - 8));
            }
        }
        *reinterpret_cast<uint2*>(codes + static_cast<size_t>(row) * (K / 2) + kb * 8) = make_uint2(lo, hi);
        scales[nv_scale_offset(row, kb, KA)] = static_cast<uint8_t>(sb);
    }
}


// ---------------------------------------------------------------------------
// W4A4 GEMM: y = (xq^ wq^T) g_x g_w + (x L1) L2 + b on the block-scaled
// tensor cores (tcgen05.mma kind::mxf4nvf4, E2M1 operands, one UE4M3 scale
// per 16 inputs, fp32 accumulation in tensor memory).
//
// Tile: 128 output channels (the MMA's M: weight rows, operand A) x 256
// tokens (its N: activation rows, operand B).  A stage holds 256 inputs of K:
// the 128 x 128-byte weight code tile and the 256 x 128-byte token code tile
// (TMA, 128-byte swizzle), the weights' four 512-byte scale atoms and the
// tokens' eight (two 128-row halves; bulk copies).  The MMA thread moves the
// atoms into tensor memory (tcgen05.cp 32x128b.warpx4: lane 32 i + j gets
// atom bytes 16 j .. 16 j + 15 for every i, i.e. rows j, j + 32, j + 64,
// j + 96 of the atom in four columns; the token atoms of one 64-input block
// take eight columns, rows 0-127 then 128-255) and issues four K = 64 MMAs.
// The low-rank term shares the accumulator: its operands are pre-divided by
// the tensor scales (T / g_x and L2 / g_w, each as a bf16 hi + lo pair, the
// [T_h | T_l | T_h] x [L2_h | L2_h | L2_l] split the W4A16 path uses) and
// pass through the same ring as ceil(3r / 64) bf16 stages ahead of each
// tile's FP4 stages (a 128 x 64 bf16 tile is 16 KB like the weight codes, a
// 256 x 64 one 32 KB like the token codes), so y = acc g_x g_w + b.  A tensor
// scale of 0 (an all-zero operand) is taken as 1 on both sides.
// Persistent CTAs walk the tiles (channel tile fastest); warp 0 loads, warp 1
// issues MMAs, warps 2-5 drain the accumulator.  One 256-column accumulator
// and 48 scale columns per stage fill the 512 TMEM columns, so a tile's
// epilogue and the next tile's MMAs do not overlap.
constexpr int NV_TM = 128;  // channels per tile
constexpr int NV_TN = 256;  // tokens per tile
constexpr uint32_t NV_A_BYTES = 128u * 128u;
constexpr uint32_t NV_B_BYTES = 256u * 128u;
constexpr uint32_t NV_SFA_BYTES = 4u * NV_ATOM_BYTES;
constexpr uint32_t NV_SFB_BYTES = 8u * NV_ATOM_BYTES;
constexpr uint32_t NV_STAGE_BYTES = NV_A_BYTES + NV_B_BYTES + NV_SFA_BYTES + NV_SFB_BYTES;  // 54 KB
constexpr uint32_t NV_LR_STAGE_BYTES = NV_A_BYTES + NV_B_BYTES;  // one bf16 low-rank block
constexpr int NV_MAX_STAGES = 4;
constexpr int NV_THREADS = 192;
constexpr uint32_t NV_TMEM_COLS = 512;
constexpr uint32_t NV_SF_COL0 = 256;  // stage s: weight scales at 256 + 48 s, token scales 16 columns after
constexpr uint32_t NV_SF_COLS = 48;

constexpr uint32_t NV_EPI_STAGE = 2048;  // per epilogue warp: 16 tokens x 32 channels of y (two bf16 halves or one fp32)

__host__ __device__ constexpr size_t nv_smem_bytes(int stages) {
    return 1024 + static_cast<size_t>(stages) * NV_STAGE_BYTES + 256 + 4 * NV_EPI_STAGE;
}

struct NvArgs {
    const uint8_t* wsf;  // weight scale atoms
    const uint8_t* xsf;  // activation scale atoms
    const float* wg;     // [0]: weight tensor scale
    const float* xg;     // [0]: activation tensor scale
    const uint16_t* bias;
    void* y;
    int M, N, K;
    int NT, MT, KS;  // channel tiles (128), token tiles (256), 256-input stages
    int KA;          // scale atoms per 128-row tile
    int tiles, stages, lr_kb, y_f32;
    int tma_store;  // y written by TMA stores from a per-warp staging tile (y 16-byte aligned, rows 16-byte multiples)
    uint64_t timeout_ns;
};

// y[box] <- shared staging (bulk async group of this thread).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// D[tmem] (+)= A[smem] B[smem]^T with one UE4M3 scale per 16 inputs of each
// operand row (scales in tensor memory at sfa / sfb).
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}
// 32 rows x 16 bytes of shared memory into four columns of every lane quarter.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// Shared-memory descriptor of 32 contiguous 16-byte rows, no swizzle: 8-row
// groups 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_rows16(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(128 >> 4) << 32;  // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;         // descriptor version
    return d;                                     // layout type 0: no swizzle
}
// Instruction descriptor, block-scaled kinds: E2M1 A and B (format 1), K-major,
// N / 8 at bit 17, UE4M3 scales (bit 23 clear), M / 16 at bit 24, dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(uint32_t m, uint32_t n) {
    return (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

__device__ __forceinline__ bool nv_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > timeout_ns) {
            raise_error(ERRBIT_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

template <bool LR>
__global__ void __launch_bounds__(NV_THREADS, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_l2, const __grid_constant__ CUtensorMap tm_t,
                      const __grid_constant__ CUtensorMap tm_y, const NvArgs a) {
    extern __shared__ uint8_t nv_smem_raw[];
    uint8_t* base = nv_smem_raw + ((1024u - (smem_u32(nv_smem_raw) & 1023u)) & 1023u);
    uint8_t* stage0 = base;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + static_cast<size_t>(a.stages) * NV_STAGE_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = full + NV_MAX_STAGES;
    uint64_t* accfull = empty + NV_MAX_STAGES;
    uint64_t* accempty = accfull + 1;
    uint64_t* drain = accempty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    uint8_t* epi_stage = reinterpret_cast<uint8_t*>(bars) + 256;  // 4 x NV_EPI_STAGE, 256-byte aligned

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < a.stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(accfull, 1);
        mbar_init(accempty, 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
        if (a.tma_store) prefetch_tensormap(&tm_y);
        if (LR) {
            prefetch_tensormap(&tm_l2);
            prefetch_tensormap(&tm_t);
        }
    }
    if (warp == 1) tmem_alloc(tmem_slot, NV_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dependency_sync();
    const int per_tile = a.KS + (LR ? a.lr_kb : 0);  // ring stages per tile

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- loads
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < a.tiles && ok; tile += gridDim.x) {
                const int nt = tile % a.NT, mt = tile / a.NT;
                for (int s = 0; s < per_tile; ++s, ++it) {
                    const uint32_t st = it % a.stages, ph = (it / a.stages) & 1;
                    if (!nv_wait(&empty[st], ph ^ 1, a.timeout_ns, abort_flag)) { ok = false; break; }
                    uint8_t* sb = stage0 + static_cast<size_t>(st) * NV_STAGE_BYTES;
                    const int ks = s - (LR ? a.lr_kb : 0);
                    if (ks < 0) {  // low-rank block j: L2'' rows of this channel tile, T'' rows of this token tile
                        const int j = s;
                        mbar_arrive_expect_tx(&full[st], NV_LR_STAGE_BYTES);
                        tma_load_2d(sb, &tm_l2, &full[st], j * 64, nt * NV_TM);
                        tma_load_2d(sb + NV_A_BYTES, &tm_t, &full[st], j * 64, mt * NV_TN);
                    } else {
                        mbar_arrive_expect_tx(&full[st], NV_STAGE_BYTES);
                        tma_load_2d(sb, &tm_w, &full[st], ks * 128, nt * NV_TM);
                        tma_load_2d(sb + NV_A_BYTES, &tm_x, &full[st], ks * 128, mt * NV_TN);
                        uint8_t* sf = sb + NV_A_BYTES + NV_B_BYTES;
                        bulk_load(sf, a.wsf + (static_cast<size_t>(nt) * a.KA + ks * 4) * NV_ATOM_BYTES, NV_SFA_BYTES,
                                  &full[st]);
                        // the two 128-row halves of the token tile (scale rows are padded to 256)
                        bulk_load(sf + NV_SFA_BYTES, a.xsf + (static_cast<size_t>(2 * mt) * a.KA + ks * 4) * NV_ATOM_BYTES,
                                  NV_SFA_BYTES, &full[st]);
                        bulk_load(sf + 2 * NV_SFA_BYTES,
                                  a.xsf + (static_cast<size_t>(2 * mt + 1) * a.KA + ks * 4) * NV_ATOM_BYTES, NV_SFA_BYTES,
                                  &full[st]);
                    }
                }
            }
            // copies still in flight land before the CTA leaves (bounded)
            const uint32_t n = it < static_cast<uint32_t>(a.stages) ? it : static_cast<uint32_t>(a.stages);
            for (uint32_t i = it - n; i < it; ++i) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&full[i % a.stages], (i / a.stages) & 1) && globaltimer_ns() - t0 < a.timeout_ns) {
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ----------------------------------------------------------- MMAs
            const uint32_t idesc = idesc_nvf4(NV_TM, NV_TN);
            const uint32_t idesc_lr = idesc_f16(1, NV_TM, NV_TN);
            uint32_t it = 0, tc = 0;
            for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++tc) {
                if (!nv_wait(accempty, (tc & 1) ^ 1, a.timeout_ns, abort_flag)) break;
                tc_fence_after();
                bool ok = true;
                for (int s = 0; s < per_tile; ++s, ++it) {
                    const uint32_t st = it % a.stages, ph = (it / a.stages) & 1;
                    if (!nv_wait(&full[st], ph, a.timeout_ns, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint8_t* sb = stage0 + static_cast<size_t>(st) * NV_STAGE_BYTES;
                    const uint64_t da = smem_desc_sw128(smem_u32(sb)), db = smem_desc_sw128(smem_u32(sb + NV_A_BYTES));
                    if (LR && s < a.lr_kb) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ss(tmem, da + 2 * kk, db + 2 * kk, idesc_lr, (s > 0 || kk > 0) ? 1u : 0u);
                    } else {
                        const bool first = s == 0;  // no low-rank block before it
                        const uint32_t sfa = tmem + NV_SF_COL0 + NV_SF_COLS * st, sfb = sfa + 16;
                        const uint32_t sa = smem_u32(sb + NV_A_BYTES + NV_B_BYTES);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            tmem_cp_32x128b_x4(sfa + 4 * i, smem_desc_rows16(sa + i * NV_ATOM_BYTES));
                            tmem_cp_32x128b_x4(sfb + 8 * i, smem_desc_rows16(sa + NV_SFA_BYTES + i * NV_ATOM_BYTES));
                            tmem_cp_32x128b_x4(sfb + 8 * i + 4, smem_desc_rows16(sa + 2 * NV_SFA_BYTES + i * NV_ATOM_BYTES));
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_nvf4(tmem, da + 2 * k, db + 2 * k, idesc, sfa + 4 * k, sfb + 8 * k,
                                     (first && k == 0) ? 0u : 1u);
                    }
                    mma_commit(&empty[st]);
                }
                if (!ok) break;
                mma_commit(accfull);
            }
            // every MMA issued has completed before tensor memory is freed
            mma_commit(drain);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may read
        const float gx = __ldg(a.xg), gw = __ldg(a.wg);
        const float ex = (gx != 0.0f) ? gx : 1.0f, ew = (gw != 0.0f) ? gw : 1.0f;
        uint32_t tc = 0, chunk = 0;  // chunk: staging halves alternate across tiles too
        for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++tc) {
            const int nt = tile % a.NT, mt = tile / a.NT;
            // every lane polls (each acquires for itself); lane 0 decides to give up
            bool ready = false;
            uint64_t t0 = 0;
            for (uint32_t spin = 0;; ++spin) {
                ready = mbar_try_wait(accfull, tc & 1);
                if (__all_sync(0xffffffffu, ready)) break;
                int give_up = 0;
                if (lane == 0 && (spin & 255) == 255) {
                    if (t0 == 0) t0 = globaltimer_ns();
                    if (*abort_flag) {
                        give_up = 1;
                    } else if (globaltimer_ns() - t0 > a.timeout_ns) {
                        raise_error(ERRBIT_TIMEOUT);
                        *abort_flag = 1;
                        give_up = 1;
                    }
                }
                if (__shfl_sync(0xffffffffu, give_up, 0)) break;
            }
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after();
            const int n = nt * NV_TM + q * 32 + lane;
            const float bv = (a.bias && n < a.N) ? bf16_bits_to_f32(a.bias[n]) : 0.0f;
            const uint32_t acc = tmem + (static_cast<uint32_t>(q * 32) << 16);
            const int m_end = min(NV_TN, a.M - mt * NV_TN);
            uint8_t* stg = epi_stage + static_cast<size_t>(warp - 2) * NV_EPI_STAGE;
            for (int c0 = 0; c0 < m_end; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(acc + c0, v);
                tmem_wait_ld();
                if (a.tma_store) {
                    // 16 tokens x this warp's 32 channels into the staging tile (token-major, like y),
                    // then one TMA store; out-of-range rows and channels are clipped by the store
                    uint8_t* buf = a.y_f32 ? stg : stg + (chunk++ & 1) * 1024;
                    if (lane == 0) {
                        if (a.y_f32) bulk_wait_read<0>();
                        else bulk_wait_read<1>();  // the other half may still be read
                    }
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float o = (__uint_as_float(v[j]) * ex) * ew + bv;
                        if (a.y_f32) reinterpret_cast<float*>(buf)[j * 32 + lane] = o;
                        else reinterpret_cast<__nv_bfloat16*>(buf)[j * 32 + lane] = __float2bfloat16_rn(o);
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0 && nt * NV_TM + q * 32 < a.N) tma_store_2d(&tm_y, buf, nt * NV_TM + q * 32, mt * NV_TN + c0);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = mt * NV_TN + c0 + j;
                        const float o = (__uint_as_float(v[j]) * ex) * ew + bv;
                        if (c0 + j < m_end && n < a.N) {
                            const size_t off = static_cast<size_t>(m) * a.N + n;
                            if (a.y_f32) static_cast<float*>(a.y)[off] = o;
                            else static_cast<__nv_bfloat16*>(a.y)[off] = __float2bfloat16_rn(o);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accempty);
        }
        // the staging tiles stay valid until their stores have read them
        if (a.tma_store && lane == 0) bulk_wait_read<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, NV_TMEM_COLS);
    }
}

}  // namespace wlq
