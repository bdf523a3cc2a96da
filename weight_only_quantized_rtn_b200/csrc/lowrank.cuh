// lowrank.cuh -- the split W ~ (L1 L2)^T + R that feeds the low-rank branch
// ("Nunchaku Lite: loading and running 4-bit SVDQuant", section "why it
// matters": the hardest part of the weights is carried by a 16-bit low-rank
// correction and only the rest is quantized).  L1 L2 is the best rank-r part
// of A = W^T [K, N] (its top-r singular triplets, split evenly: L1 = U_r
// S_r^(1/2), L2 = S_r^(1/2) V_r^T), reached by randomized subspace iteration
// with l = r + p columns:
//
//   Y = A Omega                 (Omega [N, l]: a test matrix the caller draws)
//   q times:  Z = W Q; P = orth(Z); Y = A P        (Q = orth(Y) before each)
//   Q = orth(Y);  C = W Q [N, l];  H = C^T C = U~ Lambda U~^T (Jacobi, fp64)
//   L1 = Q U~_r Lambda_r^(1/4) [K, r],   L2^T = C U~_r Lambda_r^(-1/4) [N, r]
//
// (H = B B^T for B = Q^T A = C^T, so Lambda holds the squared singular
// values of B, and B's right singular vectors are C U~ Lambda^(-1/2).)
// orth() is CholeskyQR2: G = Y^T Y in fp64, G = R^T R, Y <- Y R^-1, twice.
//
// Kernels: a deterministic fp32 "tall times skinny" GEMM (every product the
// method needs: W X, W^T X, and Y B with a small B), fp64 Gram partials over
// row chunks, and one single-CTA fp64 kernel that sums the partials in chunk
// order and runs Cholesky + triangular inverse, or a parallel-order Jacobi
// eigensolver.  The residual kernel forms R = W - (L1 L2)^T in fp64, the
// products added in j order with no fused multiply-add, and rounds once to
// fp32, so a plain fp64 statement of the same sum reproduces it bit for bit.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace wlq {

constexpr int LRS_MAX_L = 64;      // columns of the sketch (l)
constexpr int LRS_ROWS = 64;       // output rows per CTA of the skinny GEMM
constexpr int LRS_KC = 32;         // inner chunk
constexpr int LRS_THREADS = 256;

// part[split][R, c] = op(A)[R, inner-range of split] * B[inner-range, c], fp32.
// op(A): TRANS == false: A is [R, inner] row-major;
//        TRANS == true : A is [inner, R] row-major, read transposed.
// B is [inner, c] row-major, c in {16, 32, 64}.  A CTA takes 64 rows and one
// inner range (blockIdx.y); thread (tr, tc) accumulates rows 4 tr..+3 and
// columns 4 tc..+3; the next chunk is loaded into registers while the
// current one is used.
template <bool TRANS>
__global__ void __launch_bounds__(LRS_THREADS) lr_skinny_gemm(const float* __restrict__ A, const float* __restrict__ B,
                                                              int R, int inner, int c, int kper,
                                                              float* __restrict__ part) {
    grid_dependency_sync();
    __shared__ __align__(16) float As[2][LRS_KC][LRS_ROWS + 4];  // [k][row]
    __shared__ __align__(16) float Bs[2][LRS_KC][LRS_MAX_L];     // [k][col]
    const int r0 = blockIdx.x * LRS_ROWS;
    const int kb = blockIdx.y * kper, ke = min(inner, kb + kper);
    const int tid = threadIdx.x;
    const int cg = c / 4;
    const bool active = tid < 16 * cg;
    const int tr = tid / cg, tc = tid % cg;
    constexpr int AV = LRS_KC * LRS_ROWS / LRS_THREADS;  // A values per thread per chunk (8)
    float ra[AV], rb[AV];
    auto load = [&](int k0) {
#pragma unroll
        for (int u = 0; u < AV; ++u) {
            const int idx = tid + u * LRS_THREADS;
            int kk, rr;
            if (TRANS) { rr = idx % LRS_ROWS; kk = idx / LRS_ROWS; }
            else { kk = idx % LRS_KC; rr = idx / LRS_KC; }
            const int row = r0 + rr, k = k0 + kk;
            ra[u] = (row < R && k < ke) ? (TRANS ? A[static_cast<size_t>(k) * R + row] : A[static_cast<size_t>(row) * inner + k]) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < AV; ++u) {
            const int idx = tid + u * LRS_THREADS;
            const int kk = idx / c, j = idx % c;
            const int k = k0 + kk;
            rb[u] = (idx < LRS_KC * c && k < ke) ? B[static_cast<size_t>(k) * c + j] : 0.0f;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int u = 0; u < AV; ++u) {
            const int idx = tid + u * LRS_THREADS;
            int kk, rr;
            if (TRANS) { rr = idx % LRS_ROWS; kk = idx / LRS_ROWS; }
            else { kk = idx % LRS_KC; rr = idx / LRS_KC; }
            As[buf][kk][rr] = ra[u];
        }
#pragma unroll
        for (int u = 0; u < AV; ++u) {
            const int idx = tid + u * LRS_THREADS;
            if (idx < LRS_KC * c) Bs[buf][idx / c][idx % c] = rb[u];
        }
    };
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    int buf = 0;
    if (kb < ke) {
        load(kb);
        store(0);
    }
    __syncthreads();
    for (int k0 = kb; k0 < ke; k0 += LRS_KC) {
        const bool more = k0 + LRS_KC < ke;
        if (more) load(k0 + LRS_KC);
        if (active) {
#pragma unroll 8
            for (int kk = 0; kk < LRS_KC; ++kk) {
                const float4 a = *reinterpret_cast<const float4*>(&As[buf][kk][4 * tr]);
                const float4 b = *reinterpret_cast<const float4*>(&Bs[buf][kk][4 * tc]);
                const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
        }
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    if (!active) return;
    float* out = part + static_cast<size_t>(blockIdx.y) * R * c;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = r0 + 4 * tr + i;
        if (row < R)
            *reinterpret_cast<float4*>(out + static_cast<size_t>(row) * c + 4 * tc) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
}

// out = sum over the S splits of part (in split order), as fp32 [R, c],
// bf16 [R, c] and / or bf16 transposed [c, R] (each optional).
__global__ void lr_sum_splits(const float* __restrict__ part, int S, int R, int c, float* __restrict__ out,
                              uint16_t* __restrict__ out_bf16, uint16_t* __restrict__ out_bf16_t) {
    grid_dependency_sync();
    const int64_t total = static_cast<int64_t>(R) * c;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float v = part[e];
        for (int sp = 1; sp < S; ++sp) v += part[static_cast<size_t>(sp) * total + e];
        const int row = static_cast<int>(e / c), j = static_cast<int>(e % c);
        if (out) out[e] = v;
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        if (out_bf16) out_bf16[e] = *reinterpret_cast<const uint16_t*>(&h);
        if (out_bf16_t) out_bf16_t[static_cast<size_t>(j) * R + row] = *reinterpret_cast<const uint16_t*>(&h);
    }
}

// Gram partials: part[b][i][j] = sum over rows of chunk b of Y[row][i] Y[row][j]
// (fp64, rows in order inside the chunk).  One CTA per chunk of rows_per rows;
// thread t owns the entries t, t + 256, ... of the l x l matrix.
template <int L>
__global__ void __launch_bounds__(256) lr_gram_partial(const float* __restrict__ Y, int R, int rows_per,
                                                       double* __restrict__ part) {
    grid_dependency_sync();
    constexpr int l = L;
    __shared__ float rows[32][L];
    const int b = blockIdx.x;
    const int rs = b * rows_per, re = min(R, rs + rows_per);
    constexpr int ll = L * L;
    constexpr int OWN = (ll + 255) / 256;
    double acc[OWN];
#pragma unroll
    for (int i = 0; i < OWN; ++i) acc[i] = 0.0;
    for (int r0 = rs; r0 < re; r0 += 32) {
        const int nr = min(32, re - r0);
        for (int idx = threadIdx.x; idx < nr * l; idx += 256) rows[idx / l][idx % l] = Y[static_cast<size_t>(r0 + idx / l) * l + idx % l];
        __syncthreads();
        for (int rr = 0; rr < nr; ++rr) {
#pragma unroll
            for (int o = 0; o < OWN; ++o) {
                const int e = threadIdx.x + 256 * o;
                if (e < ll) acc[o] += static_cast<double>(rows[rr][e / l]) * static_cast<double>(rows[rr][e % l]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int o = 0; o < OWN; ++o) {
        const int e = threadIdx.x + 256 * o;
        if (e < ll) part[static_cast<size_t>(b) * ll + e] = acc[o];
    }
}

// Single-CTA fp64 kernels on l x l matrices held in shared memory.
// mode 0: G = sum of nparts partials; Cholesky G = R^T R (upper R); out =
//         R^-1 (fp32, row-major [l][l]), so that Y R^-1 has orthonormal
//         columns.  A pivot at or below 1e-12 of G's largest diagonal entry
//         (a column the fp32 sketch does not resolve: W of lower rank than
//         l) drops that column (its row of R and column of R^-1 are zero)
//         and sets *status = 1.
// mode 1: H = sum of partials; Jacobi eigen-decomposition H = V diag(w) V^T
//         (parallel round-robin order, sweeps until the off-diagonal mass
//         is below 1e-20 of the total -- a norm ratio of 1e-10, far below the
//         fp32 the results are stored in -- or 40 sweeps); then for the r largest
//         eigenvalues w_k (descending): out1 [l][r] = V_k w_k^(1/4),
//         out2 [l][r] = V_k w_k^(-1/4) (fp32), sigma[k] = sqrt(w_k).
__global__ void __launch_bounds__(256) lr_small_kernel(const double* __restrict__ part, int nparts, int l, int r,
                                                       int mode, float* __restrict__ out1, float* __restrict__ out2,
                                                       float* __restrict__ sigma, int* __restrict__ status) {
    grid_dependency_sync();
    extern __shared__ double sm[];
    double* Am = sm;                    // [l][l]
    double* Vm = sm + l * l;            // [l][l]
    __shared__ double cs[LRS_MAX_L / 2][2];
    __shared__ int pairs[LRS_MAX_L];
    __shared__ int order[LRS_MAX_L];
    __shared__ double wsum[2];
    const int tid = threadIdx.x;
    const int ll = l * l;
    for (int e = tid; e < ll; e += 256) {
        // chunk order, eight partials loaded at a time
        double s = 0.0;
        int b = 0;
        for (; b + 8 <= nparts; b += 8) {
            double p[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) p[u] = part[static_cast<size_t>(b + u) * ll + e];
#pragma unroll
            for (int u = 0; u < 8; ++u) s += p[u];
        }
        for (; b < nparts; ++b) s += part[static_cast<size_t>(b) * ll + e];
        Am[e] = s;
    }
    __syncthreads();
    if (mode == 0) {
        // Cholesky, column by column (R upper: Am's upper triangle becomes R)
        __shared__ int bad;
        __shared__ double tol;
        if (tid == 0) {
            bad = 0;
            double mx = 0.0;
            for (int i = 0; i < l; ++i) mx = fmax(mx, Am[i * l + i]);
            tol = 1e-12 * mx;
        }
        __syncthreads();
        for (int k = 0; k < l; ++k) {
            if (tid == 0) {
                const double d = Am[k * l + k];
                if (!(d > tol)) { bad = 1; Am[k * l + k] = 0.0; }
                else Am[k * l + k] = sqrt(d);
            }
            __syncthreads();
            const double rkk = Am[k * l + k];
            for (int j = k + 1 + tid; j < l; j += 256) Am[k * l + j] = (rkk > 0.0) ? Am[k * l + j] / rkk : 0.0;
            __syncthreads();
            for (int e = tid; e < (l - k - 1) * (l - k - 1); e += 256) {
                const int i = k + 1 + e / (l - k - 1), j = k + 1 + e % (l - k - 1);
                if (j >= i) Am[i * l + j] -= Am[k * l + i] * Am[k * l + j];
            }
            __syncthreads();
        }
        // R^-1 (upper triangular) by back substitution, one column per thread
        for (int j = tid; j < l; j += 256) {
            for (int i = l - 1; i >= 0; --i) {
                double v = (i == j) ? 1.0 : 0.0;
                for (int k = i + 1; k <= j; ++k) v -= Am[i * l + k] * Vm[k * l + j];
                const double rii = Am[i * l + i];
                Vm[i * l + j] = (i <= j && rii > 0.0) ? v / rii : 0.0;
            }
        }
        __syncthreads();
        for (int e = tid; e < ll; e += 256) out1[e] = static_cast<float>(Vm[e]);
        if (tid == 0 && status) *status = bad;
        return;
    }
    // ---- Jacobi eigen-decomposition, round-robin pairing (l even)
    for (int e = tid; e < ll; e += 256) Vm[e] = (e / l == e % l) ? 1.0 : 0.0;
    if (tid < l) order[tid] = tid;
    __syncthreads();
    for (int sweep = 0; sweep < 40; ++sweep) {
        if (tid < 2) wsum[tid] = 0.0;
        __syncthreads();
        double off = 0.0, tot = 0.0;
        for (int e = tid; e < ll; e += 256) {
            const double v = Am[e] * Am[e];
            tot += v;
            if (e / l != e % l) off += v;
        }
        for (int o = 16; o > 0; o >>= 1) {
            off += __shfl_xor_sync(0xffffffffu, off, o);
            tot += __shfl_xor_sync(0xffffffffu, tot, o);
        }
        if ((tid & 31) == 0) {
            atomicAdd(&wsum[0], off);
            atomicAdd(&wsum[1], tot);
        }
        __syncthreads();
        if (wsum[0] <= 1e-20 * wsum[1]) break;  // off-diagonal norm <= 1e-10 of the whole: far below fp32
        for (int step = 0; step < l - 1; ++step) {
            // pairs of this step: (order[i], order[l-1-i]), i < l/2
            if (tid < l / 2) {
                const int p = order[tid], q = order[l - 1 - tid];
                const int a = min(p, q), b = max(p, q);
                pairs[2 * tid] = a;
                pairs[2 * tid + 1] = b;
                const double apq = Am[a * l + b], app = Am[a * l + a], aqq = Am[b * l + b];
                double c = 1.0, s = 0.0;
                if (apq != 0.0) {
                    const double tau = (aqq - app) / (2.0 * apq);
                    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    s = t * c;
                }
                cs[tid][0] = c;
                cs[tid][1] = s;
            }
            __syncthreads();
            // A <- A J (columns a, b of every row), V <- V J
            for (int e = tid; e < (l / 2) * l; e += 256) {
                const int pi = e / l, i = e % l;
                const int a = pairs[2 * pi], b = pairs[2 * pi + 1];
                const double c = cs[pi][0], s = cs[pi][1];
                const double xa = Am[i * l + a], xb = Am[i * l + b];
                Am[i * l + a] = c * xa - s * xb;
                Am[i * l + b] = s * xa + c * xb;
                const double va = Vm[i * l + a], vb = Vm[i * l + b];
                Vm[i * l + a] = c * va - s * vb;
                Vm[i * l + b] = s * va + c * vb;
            }
            __syncthreads();
            // A <- J^T A (rows a, b of every column)
            for (int e = tid; e < (l / 2) * l; e += 256) {
                const int pi = e / l, j = e % l;
                const int a = pairs[2 * pi], b = pairs[2 * pi + 1];
                const double c = cs[pi][0], s = cs[pi][1];
                const double xa = Am[a * l + j], xb = Am[b * l + j];
                Am[a * l + j] = c * xa - s * xb;
                Am[b * l + j] = s * xa + c * xb;
            }
            __syncthreads();
            // rotate the tournament: position 0 fixed, the others move by one
            if (tid == 0) {
                const int last = order[l - 1];
                for (int i = l - 1; i > 1; --i) order[i] = order[i - 1];
                order[1] = last;
            }
            __syncthreads();
        }
    }
    // r largest eigenvalues, descending (ties by index), one thread
    if (tid == 0) {
        for (int i = 0; i < l; ++i) pairs[i] = i;
        for (int i = 0; i < r; ++i) {
            int best = i;
            for (int j = i + 1; j < l; ++j)
                if (Am[pairs[j] * l + pairs[j]] > Am[pairs[best] * l + pairs[best]]) best = j;
            const int t = pairs[i];
            pairs[i] = pairs[best];
            pairs[best] = t;
        }
    }
    __syncthreads();
    for (int e = tid; e < l * r; e += 256) {
        const int i = e / r, k = e % r;
        const int col = pairs[k];
        const double w = fmax(Am[col * l + col], 0.0);
        const double q4 = sqrt(sqrt(w));
        out1[e] = static_cast<float>(Vm[i * l + col] * q4);
        out2[e] = static_cast<float>(q4 > 0.0 ? Vm[i * l + col] / q4 : 0.0);
    }
    if (tid < r && sigma) sigma[tid] = static_cast<float>(sqrt(fmax(Am[pairs[tid] * l + pairs[tid]], 0.0)));
}

// R[n][k] = fp32( W[n][k] - sum_j L1[k][j] L2[j][n] ), the sum over j = 0..r-1
// in fp64, in order, each product and addition rounded separately (no fused
// multiply-add), then one rounding to fp32.  A 32 x 32 tile of (n, k) per
// 256-thread CTA; the tile's L1 rows and L2 columns are staged in fp64.
__global__ void __launch_bounds__(256) lr_residual_kernel(const float* __restrict__ W, const uint16_t* __restrict__ L1,
                                                          const uint16_t* __restrict__ L2, int N, int K, int r,
                                                          float* __restrict__ R) {
    grid_dependency_sync();
    __shared__ double l1s[32][65];  // [k][j]
    __shared__ double l2s[64][33];  // [j][n]
    const int n0 = blockIdx.y * 32, k0 = blockIdx.x * 32;
    for (int idx = threadIdx.x; idx < 32 * r; idx += 256) {
        const int kk = idx / r, j = idx % r, k = k0 + kk;
        l1s[kk][j] = (k < K) ? static_cast<double>(__uint_as_float(static_cast<uint32_t>(L1[static_cast<size_t>(k) * r + j]) << 16)) : 0.0;
    }
    for (int idx = threadIdx.x; idx < r * 32; idx += 256) {
        const int j = idx / 32, nn = idx % 32, n = n0 + nn;
        l2s[j][nn] = (n < N) ? static_cast<double>(__uint_as_float(static_cast<uint32_t>(L2[static_cast<size_t>(j) * N + n]) << 16)) : 0.0;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * 32; e += 256) {
        const int nn = e / 32, kk = e % 32;  // consecutive threads: consecutive k (coalesced rows of W)
        const int n = n0 + nn, k = k0 + kk;
        if (n >= N || k >= K) continue;
        double p = 0.0;
        for (int j = 0; j < r; ++j) p = __dadd_rn(p, __dmul_rn(l1s[kk][j], l2s[j][nn]));
        const size_t o = static_cast<size_t>(n) * K + k;
        R[o] = __double2float_rn(__dsub_rn(static_cast<double>(W[o]), p));
    }
}

}  // namespace wlq
