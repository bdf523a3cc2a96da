/*
 * wlq.h -- weight-only quantized Linear for NVIDIA B200 (sm_100a).
 *
 * What the library computes (web pages, cited by title and section):
 *  - "Joy-face_change_optimized" model card (README), section "what this
 *    branch does", files table: a weight-only Linear whose weights are int8
 *    with one scale per output channel, or int4 grouped along the input
 *    dimension, plus a loader for the exported codes; tools row: RTN int8,
 *    RTN int4 with group size 64, and attention-int8 / MLP-int4 with group
 *    size 16.
 *  - "Nunchaku Lite: loading and running 4-bit SVDQuant" (news article),
 *    section "why it matters": the hard part of the weights is carried by a
 *    16-bit low-rank correction; section "how it works": the W4A16 kernels
 *    keep activations in 16 bits.
 *  - The same model card, section 1 (the KV-dtype setting: cached K/V in int8
 *    with one scale per token and head), section 1.1 (DiT blocks quantized to
 *    fp8 on the GPU) and section 2 (a 5-bit MLP): the wider quantizers
 *    wlq_quantize_ex and wlq_quantize_fp8.
 *
 * Conventions shared by every call:
 *  - W is [N, K] row-major (N outputs, K inputs); x is [M, K] and y is [M, N],
 *    both row-major.  qmax = 2^(bits-1) - 1.
 *  - Every pointer is a DEVICE pointer owned by the caller, on the current
 *    CUDA device, unless stated otherwise.  The library allocates no device
 *    memory and keeps no state other than one error word per device.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Compute calls are asynchronous on it: argument errors are
 *    returned before anything is enqueued; faults detected on the device
 *    (non-finite weights, a bounded wait that ran out) are recorded in the
 *    device error word and returned by wlq_get_status().
 *  - Every kernel is launched with programmatic dependent launch: it may be
 *    scheduled while the previous kernel on the stream is finishing, but it
 *    touches no global memory before that kernel has completed and its writes
 *    are visible, so stream order holds as for a plain launch.
 *  - Supported recipes (bits, group): (8, 0) = int8 per output channel;
 *    (4, 64) and (4, 16) = int4 grouped along K.  wlq_quantize also accepts
 *    (8, g) and (4, 0) for g in {16, 32, 64, 128}.
 *  - Requirements: K % 8 == 0, K % group == 0, pointers 16-byte aligned.
 *  - Only sm_100 devices are supported (WLQ_ERR_UNSUPPORTED otherwise).
 */
#ifndef WLQ_H_
#define WLQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WLQ_OK = 0,
    WLQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad dtype     */
    WLQ_ERR_SHAPE = 2,       /* K % 8, K % group, r out of range           */
    WLQ_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned           */
    WLQ_ERR_UNSUPPORTED = 4, /* recipe or device architecture not handled  */
    WLQ_ERR_NONFINITE = 5,   /* a weight was NaN or +-Inf (device-detected) */
    WLQ_ERR_WORKSPACE = 6,   /* workspace missing or smaller than required */
    WLQ_ERR_TIMEOUT = 7,     /* a bounded device wait ran out              */
    WLQ_ERR_CUDA = 8         /* a CUDA runtime / driver call failed        */
} wlq_status;

typedef enum { WLQ_OUT_BF16 = 0, WLQ_OUT_F32 = 1 } wlq_out_dtype;
typedef enum { WLQ_IN_F32 = 0, WLQ_IN_BF16 = 1 } wlq_in_dtype;
typedef enum { WLQ_SCALE_F32 = 0, WLQ_SCALE_F16 = 1, WLQ_SCALE_BF16 = 2 } wlq_scale_dtype;

/*
 * RTN symmetric quantization ("Joy-face_change_optimized", files table and
 * tools row).  For each group (a whole row when group == 0, else `group`
 * contiguous inputs of a row, starting at k = 0):
 *   a = max |W|,  s = fp32(a / qmax)  (IEEE division, round to nearest even),
 *   q = clamp(round_half_even(W / s), -qmax, qmax) computed exactly,
 *   s == 0 (all-zero group) gives q = 0.
 * W      : fp32 [N, K]
 * codes  : int8 [N, K] (values in [-qmax, qmax])
 * scales : fp32 [N, K / g] with g = K when group == 0
 * A non-finite weight sets WLQ_ERR_NONFINITE in the device error word (its
 * code is written as 0); the call itself still returns WLQ_OK.
 * N == 0 is a no-op.
 */
wlq_status wlq_quantize(const float* W, int64_t N, int64_t K, int bits, int group,
                        int8_t* codes, float* scales, void* stream);

/*
 * Bytes of the packed operand produced by wlq_pack (0 for an unsupported
 * recipe or a bad shape).  Host-only, no device access.  No passage of the
 * pages defines it: a sizing helper for the layout below, which is this
 * library's own (the pages name the loader step, not its layout).
 * Layout: ceil(N/128) * ceil(K/64) tiles of 128 outputs x 64 inputs, each
 * holding the codes (int8: 8192 B; int4: 4096 B) followed, for int4, by the
 * tile's group scales in fp16 (gs64: 256 B; gs16: 1024 B), then one fp32
 * factor per padded output row (int8: the channel scale; int4: the power of
 * two that undoes the row's fp16 scale normalisation).
 */
size_t wlq_packed_bytes(int64_t N, int64_t K, int bits, int group);

/*
 * Lay codes and scales out for the GEMM (the pages' "loader" step).  Codes
 * are stored offset-binary (q + 2^(bits-1)); int4 group scales are stored as
 * fp16(s * 2^e_n) with one power of two e_n per output row, chosen so the
 * row's largest scale lands in [2^8, 2^9).  Rows and inputs beyond N and K
 * are zero-filled.
 * codes: int8 [N, K]; scales: fp32 [N, K / g]; packed: wlq_packed_bytes().
 */
wlq_status wlq_pack(const int8_t* codes, const float* scales, int64_t N, int64_t K,
                    int bits, int group, void* packed, void* stream);

/*
 * wlq_quantize followed by wlq_pack in one pass over W (the same two steps
 * of the pages: RTN quantization, then the loader's layout), without the
 * int8 [N, K] codes: W is read once and the packed operand written once.
 * The packed bytes and the scales are bit-identical to those of
 * wlq_pack(wlq_quantize(W)) for the same recipe.
 * W      : fp32 [N, K], 16-byte aligned, K <= 32768 (else WLQ_ERR_SHAPE)
 * scales : fp32 [N, K / g] (as wlq_quantize), 4-byte aligned
 * packed : wlq_packed_bytes(N, K, bits, group) bytes, 16-byte aligned
 * Recipes (8, 0), (4, 64), (4, 16).  A non-finite weight sets
 * WLQ_ERR_NONFINITE in the device error word, as wlq_quantize does.
 */
wlq_status wlq_quantize_pack(const float* W, int64_t N, int64_t K, int bits, int group,
                             float* scales, void* packed, void* stream);

/*
 * RTN symmetric quantization for any width of 2..8 bits, from fp32 or bf16,
 * with fp32, fp16 or bf16 stored scales ("Joy-face_change_optimized" model
 * card: tools row, RTN per channel or per group; section 1, the KV-dtype
 * setting: image K/V cached as int8 with one scale per token and head -- a
 * [tokens*heads, head_dim] input with group = head_dim; section 2: a 5-bit
 * MLP).  qmax = 2^(bits-1) - 1.  Per group (the row when group == 0):
 *   a = max |W|;  s = the value of the scale format nearest to a / qmax;
 *   q = clamp(round_half_even(W / s), -qmax, qmax) exactly, with that s.
 * W      : [N, K] fp32 or bf16 (w_dtype), 16-byte aligned
 * codes  : int8 [N, K], 4-byte aligned
 * scales : [N, K / g] in scale_dtype, aligned to its type
 * group  : 0 or a multiple of 4 dividing K; K % 8 == 0.
 * bits = 8, group and fp32 scales as in wlq_quantize give the same result.
 * A NaN or infinity in a group, or a 16-bit scale that overflows, sets
 * WLQ_ERR_NONFINITE in the device error word; that group gets s = 0, codes 0.
 */
wlq_status wlq_quantize_ex(const void* W, int w_dtype, int64_t N, int64_t K, int bits, int group,
                           int scale_dtype, int8_t* codes, void* scales, void* stream);

/*
 * fp8 block quantization ("Joy-face_change_optimized" model card, section
 * 1.1: DiT blocks quantized to fp8 on the GPU for small cards).  Format e4m3
 * (no infinity, largest finite 448).  Per group of g inputs of a row (the row
 * when group == 0): s = fp32(max|W| / 448); code = e4m3 nearest to
 * fp32(W / s), ties to an even significand, saturated to +-448; s = 0 gives
 * codes 0.
 * W: [N, K] fp32 or bf16, 16-byte aligned; codes: uint8 [N, K] e4m3 bit
 * patterns; scales: fp32 [N, K / g].  Non-finite weights as wlq_quantize_ex.
 */
wlq_status wlq_quantize_fp8(const void* W, int w_dtype, int64_t N, int64_t K, int group,
                            uint8_t* codes, float* scales, void* stream);

/*
 * NVFP4 quantization: the 4-bit format of the W4A4 SVDQuant kernels on
 * Blackwell ("Nunchaku Lite: loading and running 4-bit SVDQuant", section
 * "hardware and precision support": the NVFP4 variant of svdq_w4a4 runs on
 * Blackwell GPUs, B200 included; section "why it matters": weights AND
 * activations in 4 bits).  The pages name the format without defining it;
 * it is read as NVIDIA's NVFP4:
 *   g   = fp32(amax(X) / 2688)                 (one scale per tensor)
 *   s_b = E4M3 nearest a_b / (6 g)             (a_b = max |x| of 16 inputs of
 *                                               a row; ties to even, <= 448)
 *   q   = E2M1 nearest x / (s_b g)             (values 0, .5, 1, 1.5, 2, 3, 4, 6
 *                                               with sign; ties to even; <= 6)
 * with every rounding decision exact (see nvfp4.cuh).  An all-zero block
 * (or one whose scale rounds to 0) gets codes 0.
 * X      : [rows, K] fp32 or bf16 (x_dtype), 16-byte aligned; K % 64 == 0
 * codes  : uint8 [rows, K / 2]: input k in byte k / 2, low nibble for even k;
 *          a code is sign << 3 | magnitude index; 16-byte aligned
 * scales : wlq_nvfp4_scales_bytes(rows, K) bytes, E4M3 bits in the tensor
 *          cores' 512-byte atom layout: atom (t, a) = 128 rows from 128 t,
 *          inputs 64 a .. 64 a + 63, at ((t * KA) + a) * 512 with
 *          KA = ceil(K / 256) * 4; the scale of row 128 t + 32 i + j, block
 *          4 a + c (16 inputs each) at byte 16 j + 4 i + c of its atom; padding
 *          rows and blocks hold 0; 16-byte aligned
 * gscale : fp32 [2], 8-byte aligned: [0] = g, [1] = amax(X)
 * Non-finite inputs set the device error word (WLQ_ERR_NONFINITE).
 */
size_t wlq_nvfp4_scales_bytes(int64_t rows, int64_t K);
wlq_status wlq_nvfp4_quantize(const void* X, int x_dtype, int64_t rows, int64_t K, void* codes,
                              void* scales, float* gscale, void* stream);

/*
 * Inverse of the code part of wlq_pack: packed -> codes int8 [N, K].  No
 * passage of the pages defines it: a layout helper that lets a caller (and
 * the tests) read the packed codes back.
 */
wlq_status wlq_unpack(const void* packed, int64_t N, int64_t K, int bits, int group,
                      int8_t* codes, void* stream);

/*
 * Workspace bytes wlq_linear needs for this shape (host-only; 0 when it
 * needs none: without the low-rank branch, int8 weights at any M, and int4
 * weights at M <= 16 where the few-token kernel, which reads x itself, holds
 * its x rows in shared memory -- K up to about 40,000 at 9..16 tokens and
 * 88,000 at 1..8).  No passage of the
 * pages defines it: a sizing helper for the caller-owned scratch.  The contents need
 * no initialisation.  A workspace must not be shared by calls that may run
 * concurrently.
 */
size_t wlq_linear_workspace(int64_t M, int64_t N, int64_t K, int bits, int group, int r);

/*
 * Weight-only quantized Linear ("Joy-face_change_optimized", files table;
 * "Nunchaku Lite", why it matters / how it works):
 *   y[m,n] = sum_k x[m,k] q[n,k] s[n, k/g]  +  sum_j (x L1)[m,j] L2[j,n]  +  b[n]
 * accumulated in fp32 on the tensor cores.
 * x      : bf16 [M, K]
 * packed : output of wlq_pack for (N, K, bits, group)
 * bias   : bf16 [N] or NULL
 * L1, L2 : bf16 [K, r] (16-byte aligned) and [r, N], or NULL with r == 0;
 *          r in {0, 16, 32, 64}
 * y      : [M, N] in y_dtype (WLQ_OUT_BF16 or WLQ_OUT_F32)
 * workspace / ws_bytes : at least wlq_linear_workspace(M, N, K, bits, group, r)
 *                        bytes (may be NULL when that is 0)
 * M == 0 or N == 0 is a no-op.  Results are bitwise reproducible run to run.
 */
wlq_status wlq_linear(const void* x, int64_t M, const void* packed, int64_t N, int64_t K,
                      int bits, int group, const void* bias, const void* L1, const void* L2,
                      int r, void* y, int y_dtype, void* workspace, size_t ws_bytes,
                      void* stream);

/*
 * wlq_linear without a workspace argument, for callers that cannot allocate
 * device memory: for example code running inside a host framework that owns
 * a fixed device-memory pool and does not let libraries call cudaMalloc, or a
 * latency-critical loop where cudaMalloc / cudaFree would synchronise the
 * device.  (The pages have no counterpart to this entry point; it is a
 * deployment convenience.)
 *
 * The scratch it needs lives in one built-in device array of 32 MiB, which
 * every GPU that loads the library holds until the process exits.  Shapes
 * whose scratch (wlq_linear_workspace) exceeds 32 MiB are rejected with
 * WLQ_ERR_WORKSPACE; int4 weights need about 2*M*K bytes, so e.g. K = 4096
 * allows up to roughly 4000 tokens.  This call allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Its first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call shares the one array and leaves its
 * contents behind; nothing in it has to start at zero, because each call
 * writes every byte it later reads.  Calls that may overlap on the GPU (other
 * streams, other host threads) race on the array and must be serialised by
 * the caller.  Arguments and results are otherwise those of wlq_linear.
 */
wlq_status wlq_linear_noalloc(const void* x, int64_t M, const void* packed, int64_t N, int64_t K,
                              int bits, int group, const void* bias, const void* L1, const void* L2,
                              int r, void* y, int y_dtype, void* stream);

/*
 * Workspace bytes wlq_lowrank_split needs (host-only; 0 for an unsupported
 * shape).  No passage of the pages defines it: a sizing helper.
 */
size_t wlq_lowrank_workspace(int64_t N, int64_t K, int r, int l);

/*
 * Low-rank split of a weight before it is quantized ("Nunchaku Lite", section
 * "why it matters": the hardest part of the weights is carried by a 16-bit
 * low-rank correction and only the rest is quantized).  The best rank-r part
 * of W^T [K, N] (its top r singular triplets), split evenly:
 *   W^T ~ U_r S_r V_r^T,   L1 = U_r S_r^(1/2) [K, r],   L2 = S_r^(1/2) V_r^T [r, N]
 * found by randomized subspace iteration with l sketch columns and
 * power_iters passes of W W^T (each followed by a re-orthonormalisation),
 * then an fp64 eigen-solve of the l x l projected problem.  Like any SVD,
 * each component's sign is arbitrary; the product L1 L2 is not.  The error
 * against the exact split shrinks with the gap between the r-th and the
 * (l+1)-th singular values, like (s_(l+1) / s_r)^(2 power_iters + 1).
 * W      : fp32 [N, K], 16-byte aligned
 * omega  : fp32 [N, l], a test matrix drawn by the caller (e.g. independent
 *          standard normals), 16-byte aligned
 * L1, L2 : bf16 [K, r] and [r, N] (round to nearest even), 16-byte aligned
 * sigma  : fp32 [r] estimated singular values, descending, or NULL
 * workspace / ws_bytes : at least wlq_lowrank_workspace(N, K, r, l) bytes
 * r in {16, 32, 64}; l in {32, 64}, l >= r; 0 <= power_iters <= 8; N, K >= l.
 * Asynchronous on `stream`; deterministic run to run.
 */
wlq_status wlq_lowrank_split(const float* W, int64_t N, int64_t K, int r, int l, int power_iters,
                             const float* omega, void* L1, void* L2, float* sigma, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * The part of W the low-rank branch leaves for quantization (same passage):
 *   R[n][k] = fp32( W[n][k] - sum_{j<r} L1[k][j] L2[j][n] )
 * the sum taken in fp64 over j in increasing order (products and additions
 * rounded one by one, no fused multiply-add), then one rounding to fp32.
 * Quantize R with wlq_quantize / wlq_quantize_pack and give (L1, L2) to
 * wlq_linear.  W, R: fp32 [N, K] (4-byte aligned; R must not overlap W);
 * L1: bf16 [K, r]; L2: bf16 [r, N]; r in {16, 32, 64}.
 */
wlq_status wlq_lowrank_residual(const float* W, const void* L1, const void* L2, int64_t N, int64_t K, int r,
                                float* R, void* stream);

/*
 * Synchronise `stream`, then read and clear this device's error word:
 * WLQ_OK, WLQ_ERR_NONFINITE or WLQ_ERR_TIMEOUT (or WLQ_ERR_CUDA).
 * The error path follows "Nunchaku Lite", section "hardware and precision
 * support": the quantizer checks the GPU's compute capability when it loads
 * and raises a clear error on a mismatch.  Here every call returns
 * WLQ_ERR_UNSUPPORTED on a device other than sm_100, and errors found on the
 * device are kept until this call reads them.
 */
wlq_status wlq_get_status(void* stream);

/*
 * Exercise the bounded device wait on its own: one CTA waits, through the
 * same helper the GEMM uses, on a barrier that nothing ever arrives at, for
 * at most `timeout_ns` nanoseconds (capped at 10 s), then records
 * WLQ_ERR_TIMEOUT in the device error word and exits.  No other work is
 * touched; the device stays usable.  For failure-path tests.
 */
wlq_status wlq_probe_wait_timeout(uint64_t timeout_ns, void* stream);

/*
 * Cap the number of CTAs (thread blocks) every later wlq_linear launch uses
 * on any device; 0 removes the cap.  Host-only, process-wide, not thread
 * safe against concurrent launches.  For tests that need several output
 * tiles per CTA, and for tuning; results do not depend on it.
 */
void wlq_set_grid_limit(int max_ctas);

/*
 * Human-readable text of the last error returned on this host thread (the
 * clear error of "Nunchaku Lite", section "hardware and precision support").
 */
const char* wlq_last_error(void);

/* Library version, e.g. "0.1.0". */
const char* wlq_version(void);

/*
 * The W4A4 Linear of the NVFP4 SVDQuant path ("Nunchaku Lite", section "how
 * it works": svdq_w4a4 = 4-bit weights and activations plus the SVDQuant
 * low-rank correction, used for the attention and MLP projections):
 *   y[m, n] = g_x g_w sum_k qx[m,k] sx[m,k/16] qw[n,k] sw[n,k/16]
 *             + sum_j (sum_k x[m,k] L1[k,j]) L2[j,n] + b[n]
 * on the block-scaled tensor cores (E2M1 x E2M1 products scaled by UE4M3
 * block scales, fp32 accumulation); the low-rank term from the 16-bit x
 * through a bf16 hi/lo split (relative error ~2^-16) into a second fp32
 * accumulator.
 * xq, xs, xg : the activations [M, K] as wlq_nvfp4_quantize writes them
 *              (xg: its gscale, read on the device)
 * x          : bf16 [M, K] (only read when r > 0; may be NULL otherwise)
 * wq, ws, wg : the weights [N, K] from wlq_nvfp4_quantize
 * bias [N], L1 [K, r], L2 [r, N]: bf16 (bias may be NULL; r in {0,16,32,64})
 * y          : [M, N] in y_dtype
 * workspace  : wlq_nvfp4_linear_workspace(M, N, K, r) bytes (0 when r == 0),
 *              16-byte aligned
 * K % 64 == 0; codes, scales, x, L1 and the workspace 16-byte aligned.
 */
size_t wlq_nvfp4_linear_workspace(int64_t M, int64_t N, int64_t K, int r);
wlq_status wlq_nvfp4_linear(const void* xq, const void* xs, const float* xg, const void* x, int64_t M,
                            const void* wq, const void* ws, const float* wg, int64_t N, int64_t K,
                            const void* bias, const void* L1, const void* L2, int r, void* y,
                            int y_dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * The W4A4 forward from bf16 activations: x [M, K] is quantized to NVFP4 in
 * the workspace (wlq_nvfp4_quantize), then wlq_nvfp4_linear runs.  Same
 * arguments as wlq_nvfp4_linear otherwise; workspace: wlq_w4a4_workspace()
 * bytes (never 0 for M, N > 0), 16-byte aligned.
 */
size_t wlq_w4a4_workspace(int64_t M, int64_t N, int64_t K, int r);
wlq_status wlq_w4a4_linear(const void* x, int64_t M, const void* wq, const void* ws, const float* wg,
                           int64_t N, int64_t K, const void* bias, const void* L1, const void* L2, int r,
                           void* y, int y_dtype, void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WLQ_H_ */
