// wlq_api.cu -- the C ABI (include/wlq.h): argument checks, launch plans,
// TMA descriptors and kernel launches.  Single translation unit: every kernel
// header is included here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <utility>
#include <mutex>
#include <unordered_map>

#include "../../include/wlq.h"
#include "gemm.cuh"
#include "skinny.cuh"
#include "gemv.cuh"
#include "quantize_pack.cuh"
#include "quantize_ext.cuh"
#include "pack.cuh"
#include "prep.cuh"
#include "lowrank.cuh"
#include "ptx.cuh"
#include "quantize.cuh"
#include "nvfp4.cuh"

namespace {

thread_local char g_msg[512] = "no error";

wlq_status fail(wlq_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

wlq_status cuda_fail(cudaError_t e, const char* what) {
    return fail(WLQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int fmt_of(int bits, int group) {
    if (bits == 8 && group == 0) return wlq::FMT_W8;
    if (bits == 4 && group == 64) return wlq::FMT_W4G64;
    if (bits == 4 && group == 16) return wlq::FMT_W4G16;
    return -1;
}

// ----------------------------------------------------------------- device
struct DeviceInfo {
    int checked = 0;  // 0 unknown, 1 supported, -1 not
    int sms = 0;
    bool smem_set[64] = {};
    // resident clusters per (format, cluster size, dynamic smem), queried once
    std::unordered_map<uint64_t, int> max_clusters;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

wlq_status current_device(int* dev_out, DeviceInfo** info_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(WLQ_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (d.checked == 0) {
        int major = 0, minor = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        d.checked = (major == 10 && minor == 0) ? 1 : -1;
        d.sms = sms;
    }
    if (d.checked < 0) return fail(WLQ_ERR_UNSUPPORTED, "this library is built for sm_100 (B200) only");
    *dev_out = dev;
    *info_out = &d;
    return WLQ_OK;
}

// ------------------------------------------------------------- TMA encode
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D tensor of 16-bit elements [rows, cols] (cols contiguous), tiles of
// box_rows x 64 with a 128-byte swizzle; out-of-range elements read as zero.
wlq_status make_map_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(WLQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(WLQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return WLQ_OK;
}

// ------------------------------------------------------------------ plan
constexpr uint64_t kDefaultTimeoutNs = 2ull * 1000 * 1000 * 1000;
constexpr size_t kSmemLimit = 232448;  // 227 KB opt-in per block on sm_100
constexpr size_t kXresMaxBytes = 128 * 1024;  // largest resident x block (tokens x K range, bf16)

struct Plan {
    int fmt = -1;
    int M = 0, N = 0, K = 0, r = 0;
    int NT = 0, KT = 0, MT = 0, S = 1, kbps = 0, BN = 0, tiles_nm = 0, grid = 0;
    int stages = 0, ks = 1, lr_kb = 0, acc_bufs = 1;
    bool pair = false;  // two CTAs per MMA (cta_group::2)
    bool xres = false;  // x resident in shared memory; weight ring released by the dequant warps
    bool skinny = false;  // one token tile of <= 64 tokens: the warp-MMA streaming kernel
    bool gemv = false;    // <= 16 tokens, x small enough for shared memory: the direct-load kernel
    bool red_alias = false;  // split partial in the ring's memory (one tile per cluster)
    int astages = 0;    // resident x: TMEM A-stage ring depth
    uint32_t tmem_cols = 0, acc_col0 = 0, lr_col0 = 0, a_col0 = 0, wtile = 0, wstage = 0, xsub = 0, xstage = 0, red = 0, stage = 0;
    size_t smem = 0;
    size_t off_x16 = 0, off_xs = 0, off_thl = 0, off_l2t = 0, ws = 0;
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int token_tile(int64_t M, int r) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

int g_grid_limit = 0;  // 0: no cap on the GEMM's CTAs (see wlq_set_grid_limit)

// Returned by a launcher when the plan's cluster shape cannot get one tile per
// cluster on this device; the caller plans again without split pairs.
constexpr wlq_status kRetryPlan = static_cast<wlq_status>(-100);

// Launch plan: token tile BN, K split S (a power of two up to 8, the CTAs of
// one cluster), TMEM columns, shared-memory ring depth, workspace layout.
// variant 0: CTA pairs may split K (over up to four pairs of a cluster);
// variant 1: no split pairs, but 256-token tiles may split K (partial in the
// ring); variant 2: splits use 128-token tiles (partial beside the ring).
// Variant 0 needs one tile per cluster; the launcher reports kRetryPlan when
// the device cannot hold that many clusters.
bool make_plan(Plan& p, int64_t M, int64_t N, int64_t K, int fmt, int r, int sms, int variant = 0) {
    p.fmt = fmt;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.r = r;
    p.NT = static_cast<int>(cdiv(N, 128));
    p.KT = static_cast<int>(cdiv(K, 64));
    p.lr_kb = r ? static_cast<int>(cdiv(3 * r, 64)) : 0;  // [T'h|T'l|T'h] x [L2'h|L2'h|L2'l]
    p.BN = token_tile(M, r);
    p.MT = static_cast<int>(cdiv(M, p.BN));
    // Few 256-token tiles: CTA pairs, with the K range split over up to four
    // pairs of one cluster when plain pairs would leave most SMs idle.  Each
    // cluster then holds exactly one tile (its partial reuses the ring).
    const int cap = (g_grid_limit > 0) ? std::min(g_grid_limit, sms) : sms;
    int S = 1;
    bool pair_split = false;
    if (variant == 0 && p.BN == 256 && p.NT % 2 == 0) {
        const int64_t tp = static_cast<int64_t>(p.NT / 2) * p.MT;  // pair tiles
        if (tp * 2 * 2 <= cap) {
            while (S * 2 <= 4 && tp * 2 * (S * 2) <= cap && p.KT >= S * 2 * 4) S *= 2;
            pair_split = S > 1;
        }
    }
    // Split K when the output tiles cannot cover half of the SMs.  128-token
    // split tiles keep their fp32 partial beside the ring; 256-token ones
    // (variants 0-1, no low-rank term) keep it in the ring's memory.
    if (!pair_split && p.NT * p.MT * 2 <= sms) {
        if (p.BN > 128 && variant == 2) {
            p.BN = 128;
            p.MT = static_cast<int>(cdiv(M, p.BN));
        }
        // each CTA of a split cluster sums BN / S tokens of the tile, four at a
        // time (vector loads from distributed shared memory): keep BN / S >= 4
        while (S * 2 <= wlq::MAX_SPLITS && p.NT * p.MT * S * 2 <= sms && S * 8 <= p.BN && p.KT >= S * 4) S *= 2;
    }
    // every split must own at least one K block
    for (;;) {
        p.kbps = static_cast<int>(cdiv(p.KT, S));
        if (S == 1 || static_cast<int64_t>(S - 1) * p.kbps < p.KT) break;
        S /= 2;
    }
    p.S = S;
    if (S > 1 && p.BN % S != 0) return false;  // every CTA of a split cluster sums whole tokens
    // CTA pairs for large token tiles: two 128-channel tiles share each MMA
    if (pair_split && S == 1) pair_split = false;  // the K range was too short to split
    p.pair = (p.BN == 256 && p.NT % 2 == 0) && (S == 1 || pair_split);
    p.red_alias = S > 1 && p.BN == 256;  // split 256-token tiles: pairs or single CTAs
    p.tiles_nm = p.pair ? (p.NT / 2) * p.MT : p.NT * p.MT;
    // TMEM: accumulator(s) first, from column 0, so each starts at a multiple
    // of its own width (main accumulators at ab*BN, low-rank ones after them);
    // then a ks * 32-column A stage per ring slot.  The accumulators are
    // double-buffered when that still leaves room for four 32-column blocks.
    const uint32_t acc_cols = static_cast<uint32_t>(p.BN);  // the low-rank term shares the accumulator
    if (acc_cols + 2 * wlq::A_STAGE_COLS > 512) return false;
    p.acc_bufs = (2 * acc_cols + 4 * wlq::A_STAGE_COLS <= 512) ? 2 : 1;
    const uint32_t acc_total = p.acc_bufs * acc_cols;
    const uint32_t a_col0 = (acc_total + wlq::A_STAGE_COLS - 1) / wlq::A_STAGE_COLS * wlq::A_STAGE_COLS;
    // shared memory: ring slots + low-rank tiles + split partial + barriers
    p.wtile = wlq::tile_bytes(fmt);
    p.xsub = static_cast<uint32_t>(p.pair ? p.BN / 2 : p.BN) * 128u;  // a pair's CTA stages half the tokens
    // token-major fp32 partial (256-token split tiles: in the ring's memory)
    p.red = (S > 1 && !p.red_alias) ? static_cast<uint32_t>(p.BN) * 128u * 4u : 0u;
    const size_t lr_bytes = r ? static_cast<size_t>(p.lr_kb) * (wlq::LR_TILE_A_BYTES + p.xsub) : 0;
    p.stage = (S == 1) ? wlq::NUM_EPI_WARPS * wlq::EPI_STAGE_BYTES : 0u;  // epilogue transpose buffers
    const size_t fixed = 1024 /* alignment */ + 1024 /* barriers */ + lr_bytes + p.red + p.stage;
    // Resident x (one token tile, small K range): the CTA's x rows stay in
    // shared memory for the whole K range, the weight ring is released as soon
    // as the dequant warps hold the codes, and the TMEM A stages form a ring of
    // their own, so weight loads never wait for the MMA.
    const size_t xres_bytes = static_cast<size_t>(p.kbps) * p.BN * 128u;
    p.ks = 0;
    // At most 16 tokens, no low rank: the direct-load kernel.  A cluster of
    // S CTAs splits each 128-channel tile's K range; S grows while the tiles
    // times S fit on the SMs (and every split keeps two K blocks), then while
    // the CTA's x rows and a two-slot weight ring do not fit in shared memory.
    // The ring takes what shared memory is left, up to eight slots.
    if (r == 0 && M <= 16) {
        const int nb = (M <= 8) ? 1 : 2;
        const size_t lim = kSmemLimit - 1024;
        int gs = 1;
        while (gs * 2 <= wlq::GV_MAX_SPLITS && static_cast<int64_t>(p.NT) * gs * 2 <= cap && p.KT >= gs * 2 * 2)
            gs *= 2;
        auto kbps_of = [&](int s_) { return static_cast<int>(cdiv(p.KT, s_)); };
        while (wlq::gv_smem_bytes(fmt, nb, kbps_of(gs), 2) > lim && gs * 2 <= wlq::GV_MAX_SPLITS && p.KT >= gs * 2)
            gs *= 2;
        // every split owns at least one K block
        while (gs > 1 && static_cast<int64_t>(gs - 1) * kbps_of(gs) >= p.KT) gs /= 2;
        const size_t fixed = wlq::gv_smem_bytes(fmt, nb, kbps_of(gs), 0);
        const int st = (fixed < lim) ? static_cast<int>(std::min<size_t>(wlq::GV_MAX_STAGES,
                                                                          (lim - fixed) / wlq::gv_slot_bytes(fmt)))
                                     : 0;
        if (st >= 2) {
            p.gemv = true;
            p.S = gs;
            p.kbps = kbps_of(gs);
            p.stages = st;
            p.smem = wlq::gv_smem_bytes(fmt, nb, p.kbps, st);
            p.tiles_nm = p.NT;
            p.grid = static_cast<int>(std::min<int64_t>(p.NT, std::max(1, cap / gs))) * gs;  // persistent over tiles
            p.ws = 0;  // the kernel reads the bf16 x itself, every format
            return true;
        }
    }
    // Few tokens (at most 32): the skinny kernel (x resident, warp MMAs, no
    // tensor memory).  At 64 tokens the resident-x tensor-core kernel is faster.
    p.skinny = !p.pair && r == 0 && p.MT == 1 && p.BN <= 32 && xres_bytes <= kXresMaxBytes;
    if (p.skinny) {
        p.red = static_cast<uint32_t>(p.BN) * wlq::SK_PITCH * 4u;  // split partial or output staging
        p.stage = 0;
        const size_t sk_fixed = 1024 /* alignment */ + 1024 /* barriers */ + xres_bytes + p.red;
        {
            const int ks = wlq::SK_GROUPS;  // one K block per warp group in every slot
            const uint32_t wstage = (static_cast<uint32_t>(ks) * p.wtile + 1023u) & ~1023u;
            const int stages = std::min(wlq::MAX_STAGES, static_cast<int>((kSmemLimit - sk_fixed) / wstage));
            if (sk_fixed + 2 * static_cast<size_t>(wstage) <= kSmemLimit && stages >= 2) {
                p.ks = ks;
                p.stages = stages;
                p.wstage = wstage;
                p.xstage = 0;
                p.smem = sk_fixed + stages * static_cast<size_t>(wstage);
            }
        }
        if (p.ks == 0) {
            p.skinny = false;
            p.red = (S > 1) ? static_cast<uint32_t>(p.BN) * 128u * 4u : 0u;
            p.stage = (S == 1) ? wlq::NUM_EPI_WARPS * wlq::EPI_STAGE_BYTES : 0u;
        } else {
            p.kbps = (S > 1) ? p.kbps : p.KT;
            p.tmem_cols = 0;
            size_t off = 0;
            if (fmt != wlq::FMT_W8) {
                p.off_x16 = off; off = align256(off + static_cast<size_t>(M) * K * 2);
                p.off_xs = off;  off = align256(off + static_cast<size_t>(M) * 4);
            }
            p.ws = off;
            return true;
        }
    }
    p.xres = !p.pair && r == 0 && p.MT == 1 && p.BN <= 64 && xres_bytes <= kXresMaxBytes;
    if (p.xres) {
        for (int ks : {4, 2, 1}) {
            const uint32_t wstage = (static_cast<uint32_t>(ks) * p.wtile + 1023u) & ~1023u;
            const int astages = static_cast<int>((512 - a_col0) / (static_cast<uint32_t>(ks) * wlq::A_STAGE_COLS));
            if (fixed + xres_bytes + 2 * wstage > kSmemLimit) continue;
            const int stages = std::min(wlq::MAX_STAGES, static_cast<int>((kSmemLimit - fixed - xres_bytes) / wstage));
            const int ast = std::min(wlq::MAX_STAGES, astages);
            if (stages >= 2 && (ast >= 3 || (ks == 1 && ast >= 2))) {
                p.ks = ks;
                p.stages = stages;
                p.astages = ast;
                p.wstage = wstage;
                p.xstage = 0;
                p.smem = fixed + xres_bytes + stages * static_cast<size_t>(wstage);
                break;
            }
        }
        if (p.ks == 0) p.xres = false;
    }
    // K blocks per ring slot: the largest of 4, 2, 1 that still leaves three
    // slots in both TMEM and shared memory (one handshake per slot)
    for (int ks : {4, 2, 1}) {
        if (p.ks) break;
        const uint32_t wstage = (static_cast<uint32_t>(ks) * p.wtile + 1023u) & ~1023u;
        const uint32_t xstage = static_cast<uint32_t>(ks) * p.xsub;
        const size_t per_stage = xstage + wstage;
        if (fixed + 2 * per_stage > kSmemLimit) continue;
        const int tmem_slots = static_cast<int>((512 - a_col0) / (static_cast<uint32_t>(ks) * wlq::A_STAGE_COLS));
        const int smem_slots = static_cast<int>((kSmemLimit - fixed) / per_stage);
        const int stages = std::min({wlq::MAX_STAGES, tmem_slots, smem_slots});
        if (stages >= 3 || (ks == 1 && stages >= 2)) {
            p.ks = ks;
            p.stages = stages;
            p.wstage = wstage;
            p.xstage = xstage;
            p.smem = fixed + stages * per_stage;
            break;
        }
    }
    if (p.ks == 0) return false;
    if (p.red_alias && p.stages * static_cast<size_t>(p.xstage + p.wstage) < static_cast<size_t>(p.BN) * 128u * 4u)
        return variant < 2 ? make_plan(p, M, N, K, fmt, r, sms, variant + 1) : false;
    p.acc_col0 = 0;
    p.lr_col0 = 0;
    p.a_col0 = a_col0;
    const uint32_t need = a_col0 + static_cast<uint32_t>((p.xres ? p.astages : p.stages) * p.ks) * wlq::A_STAGE_COLS;
    p.tmem_cols = 32;
    while (p.tmem_cols < need) p.tmem_cols <<= 1;
    // workspace
    size_t off = 0;
    if (fmt != wlq::FMT_W8) {
        p.off_x16 = off; off = align256(off + static_cast<size_t>(M) * K * 2);
        p.off_xs = off;  off = align256(off + static_cast<size_t>(M) * 4);
    }
    if (r) {
        p.off_thl = off; off = align256(off + static_cast<size_t>(M) * p.lr_kb * 64 * 2);
        p.off_l2t = off; off = align256(off + static_cast<size_t>(p.NT) * 128 * p.lr_kb * 64 * 2);
    }
    p.ws = off;
    return true;
}

wlq_status check_shape(int64_t N, int64_t K, int bits, int group) {
    if (N < 0 || K <= 0) return fail(WLQ_ERR_INVALID_ARG, "N must be >= 0 and K > 0");
    if (N > (int64_t(1) << 30) || K > (int64_t(1) << 30)) return fail(WLQ_ERR_SHAPE, "N or K too large");
    if (K % 8) return fail(WLQ_ERR_SHAPE, "K %% 8 != 0 (K = %lld)", static_cast<long long>(K));
    if (group && K % group) return fail(WLQ_ERR_SHAPE, "K %% group != 0");
    (void)bits;
    return WLQ_OK;
}


// Adds programmatic dependent launch to a configuration (keeping its cluster
// attribute, if any): see launch_k.
void add_pdl(cudaLaunchConfig_t& cfg, cudaLaunchAttribute (&all)[2]) {
    int na = 0;
    if (cfg.numAttrs > 0) all[na++] = cfg.attrs[0];
    all[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    all[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    cfg.attrs = all;
    cfg.numAttrs = static_cast<unsigned>(na);
}

template <int FMT, bool PAIR, bool XRES>
wlq_status launch_gemm(Plan& p, const CUtensorMap& tx, const CUtensorMap& tt, const CUtensorMap& tl,
                       wlq::GemmArgs& a, DeviceInfo* d, cudaStream_t st) {
    auto kern = wlq::gemm_kernel<FMT, PAIR, XRES>;
    const int kid = FMT * 4 + (PAIR ? 2 : 0) + (XRES ? 1 : 0);
    if (!d->smem_set[kid]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemLimit));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        d->smem_set[kid] = true;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(wlq::GEMM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    const int cta_cap = (g_grid_limit > 0) ? std::min(g_grid_limit, d->sms) : d->sms;
    // clusters of `csize` CTAs that the device can hold at once (cached)
    auto resident_clusters = [&](int csize) {
        const uint64_t key = (static_cast<uint64_t>(kid) << 48) | (static_cast<uint64_t>(csize) << 32) | p.smem;
        int active = 0;
        {
            std::lock_guard<std::mutex> lk(g_dev_mu);
            auto it = d->max_clusters.find(key);
            if (it != d->max_clusters.end()) active = it->second;
        }
        if (active == 0) {
            cudaLaunchAttribute at;
            at.id = cudaLaunchAttributeClusterDimension;
            at.val.clusterDim.x = static_cast<unsigned>(csize);
            at.val.clusterDim.y = 1;
            at.val.clusterDim.z = 1;
            cudaLaunchConfig_t c2 = cfg;
            c2.attrs = &at;
            c2.numAttrs = 1;
            c2.gridDim = dim3(static_cast<unsigned>((cta_cap / csize) * csize), 1, 1);
            if (cudaOccupancyMaxActiveClusters(&active, kern, &c2) != cudaSuccess || active <= 0) {
                cudaGetLastError();
                active = d->sms / csize;
            }
            std::lock_guard<std::mutex> lk(g_dev_mu);
            d->max_clusters[key] = active;
        }
        return std::min(active, cta_cap / csize);
    };
    int csize = PAIR ? 2 * p.S : p.S;  // CTAs per cluster
    // Pairs over whole K: when the tiles do not fill the last round of pairs,
    // run clusters of two pairs and split each leftover tile's K range over
    // one cluster's two pairs (a half-length last round).
    a.tail = 0;
    if (PAIR && p.S == 1 && p.stages * static_cast<size_t>(p.xstage + p.wstage) >= static_cast<size_t>(p.BN) * 512u) {
        const int c4 = resident_clusters(4);
        const int P = 2 * c4;
        const int rem = (P > 0) ? p.tiles_nm % P : 0;
        if (c4 > 0 && p.tiles_nm > P && rem > 0 && rem <= c4) {
            csize = 4;
            a.tail = 1;
            a.tiles_full = p.tiles_nm - rem;
            a.red_alias = 1;
            a.S_red = 2;
        }
    }
    int clusters = std::max(1, std::min(a.tail ? resident_clusters(4) : p.tiles_nm, cta_cap / csize));
    if (csize > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        // persistent clusters: no more than can be resident at once
        clusters = std::min(clusters, resident_clusters(csize));
    }
    // a partial kept in the ring needs one tile per cluster
    if (p.red_alias && clusters < p.tiles_nm) return kRetryPlan;
    cfg.gridDim = dim3(static_cast<unsigned>(clusters * csize), 1, 1);
    p.grid = clusters * csize;
    cudaLaunchAttribute all_attrs[2];
    add_pdl(cfg, all_attrs);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tx, tt, tl, a);
    if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
    return WLQ_OK;
}

template <int FMT, int NB>
wlq_status launch_skinny(Plan& p, const CUtensorMap& tx, wlq::GemmArgs& a, DeviceInfo* d, cudaStream_t st) {
    auto kern = wlq::skinny_kernel<FMT, NB>;
    const int kid = 12 + FMT * 3 + (NB == 2 ? 0 : NB == 4 ? 1 : 2);  // 12..20 (gemm: 0..11, gemv: 21..26)
    if (!d->smem_set[kid]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemLimit));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        d->smem_set[kid] = true;
    }
    const int csize = p.S;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(wlq::SK_THREADS, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    const int cta_cap = (g_grid_limit > 0) ? std::min(g_grid_limit, d->sms) : d->sms;
    int clusters = std::max(1, std::min(p.tiles_nm, cta_cap / csize));
    if (csize > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const uint64_t key = (static_cast<uint64_t>(kid) << 48) | (static_cast<uint64_t>(csize) << 32) | p.smem;
        int active = 0;
        {
            std::lock_guard<std::mutex> lk(g_dev_mu);
            auto it = d->max_clusters.find(key);
            if (it != d->max_clusters.end()) active = it->second;
        }
        if (active == 0) {
            cfg.gridDim = dim3(static_cast<unsigned>(clusters * csize), 1, 1);
            if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess || active <= 0) {
                cudaGetLastError();
                active = d->sms / csize;
            }
            std::lock_guard<std::mutex> lk(g_dev_mu);
            d->max_clusters[key] = active;
        }
        clusters = std::min(clusters, active);
    }
    cfg.gridDim = dim3(static_cast<unsigned>(clusters * csize), 1, 1);
    p.grid = clusters * csize;
    cudaLaunchAttribute all_attrs[2];
    add_pdl(cfg, all_attrs);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tx, a);
    if (e != cudaSuccess) return cuda_fail(e, "skinny launch");
    return WLQ_OK;
}

template <int FMT, int NB>
wlq_status launch_gemv(Plan& p, wlq::GemmArgs& a, DeviceInfo* d, cudaStream_t st) {
    auto kern = wlq::gemv_kernel<FMT, NB>;
    const int kid = 21 + FMT * 2 + (NB == 1 ? 0 : 1);  // 21..26
    if (!d->smem_set[kid]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemLimit - 1024));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        d->smem_set[kid] = true;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(wlq::GV_THREADS, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    const int csize = p.S;
    int clusters = p.grid / csize;
    if (csize > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        // clusters are persistent over tiles: launch no more than fit at once
        const uint64_t key = (static_cast<uint64_t>(kid) << 48) | (static_cast<uint64_t>(csize) << 32) | p.smem;
        int active = 0;
        {
            std::lock_guard<std::mutex> lk(g_dev_mu);
            auto it = d->max_clusters.find(key);
            if (it != d->max_clusters.end()) active = it->second;
        }
        if (active == 0) {
            cfg.gridDim = dim3(static_cast<unsigned>(clusters * csize), 1, 1);
            if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess || active <= 0) {
                cudaGetLastError();
                active = d->sms / csize;
            }
            std::lock_guard<std::mutex> lk(g_dev_mu);
            d->max_clusters[key] = active;
        }
        clusters = std::max(1, std::min(clusters, active));
    }
    cfg.gridDim = dim3(static_cast<unsigned>(clusters * csize), 1, 1);
    p.grid = clusters * csize;
    cudaLaunchAttribute all_attrs[2];
    add_pdl(cfg, all_attrs);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return cuda_fail(e, "gemv launch");
    return WLQ_OK;
}

template <int FMT>
wlq_status launch_gemv_nb(Plan& p, wlq::GemmArgs& a, DeviceInfo* d, cudaStream_t st) {
    if (p.M <= 8) return launch_gemv<FMT, 1>(p, a, d, st);
    return launch_gemv<FMT, 2>(p, a, d, st);
}

template <int FMT>
wlq_status launch_skinny_nb(Plan& p, const CUtensorMap& tx, wlq::GemmArgs& a, DeviceInfo* d, cudaStream_t st) {
    if (p.BN == 16) return launch_skinny<FMT, 2>(p, tx, a, d, st);
    if (p.BN == 32) return launch_skinny<FMT, 4>(p, tx, a, d, st);
    return launch_skinny<FMT, 8>(p, tx, a, d, st);
}

// Every launch allows programmatic dependent launch: the kernel may start
// while the previous grid on the stream finishes; each kernel's first action
// is griddepcontrol.wait (ptx.cuh, grid_dependency_sync), which blocks until
// that grid has completed and its memory is visible.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

int grid_for(int64_t work, int per_block, int sms) {
    const int64_t b = cdiv(std::max<int64_t>(work, 1), per_block);
    return static_cast<int>(std::min<int64_t>(b, int64_t(sms) * 32));
}

// x -> x16 (int4 operands): one CTA per row with the row in registers when
// it fits (K <= 32768), else one warp per row.
wlq_status launch_prep_x16(const uint16_t* x, int M, int K, __half* x16, float* xs, DeviceInfo* d, cudaStream_t s) {
    const int K8 = K / 8;
    if (M <= 16 && K8 <= 8 * 256) {
        // few rows: one 256-thread CTA per row
        const int per = (K8 <= 256) ? 1 : (K8 <= 512) ? 2 : (K8 <= 1024) ? 4 : 8;
        const int threads = static_cast<int>(std::max<int64_t>(32, (cdiv(K8, per) + 31) / 32 * 32));
        if (per == 1) launch_k(wlq::prep_x16_rows_kernel<1, 256, 4>, M, threads, 0, s, x, M, K, x16, xs);
        else if (per == 2) launch_k(wlq::prep_x16_rows_kernel<2, 256, 4>, M, threads, 0, s, x, M, K, x16, xs);
        else if (per == 4) launch_k(wlq::prep_x16_rows_kernel<4, 256, 4>, M, threads, 0, s, x, M, K, x16, xs);
        else launch_k(wlq::prep_x16_rows_kernel<8, 256, 4>, M, threads, 0, s, x, M, K, x16, xs);
    } else if (K8 <= 16 * 128) {
        // many rows: 128-thread CTAs, up to 16 chunks of the row per thread, so
        // that the 16 CTAs an SM holds keep about 128 KB of x in flight
        const int per = (K8 <= 128) ? 1 : (K8 <= 256) ? 2 : (K8 <= 512) ? 4 : (K8 <= 1024) ? 8 : 16;
        const int threads = static_cast<int>(std::max<int64_t>(32, (cdiv(K8, per) + 31) / 32 * 32));
        const int grid = static_cast<int>(std::min<int64_t>(M, static_cast<int64_t>(d->sms) * 16));
        if (per == 1) launch_k(wlq::prep_x16_rows_kernel<1, 128, 1>, grid, threads, 0, s, x, M, K, x16, xs);
        else if (per == 2) launch_k(wlq::prep_x16_rows_kernel<2, 128, 1>, grid, threads, 0, s, x, M, K, x16, xs);
        else if (per == 4) launch_k(wlq::prep_x16_rows_kernel<4, 128, 1>, grid, threads, 0, s, x, M, K, x16, xs);
        else if (per == 8) launch_k(wlq::prep_x16_rows_kernel<8, 128, 1>, grid, threads, 0, s, x, M, K, x16, xs);
        else launch_k(wlq::prep_x16_rows_kernel<16, 128, 1>, grid, threads, 0, s, x, M, K, x16, xs);
    } else {
        launch_k(wlq::prep_x16_kernel, grid_for(static_cast<int64_t>(M) * 32, 256, d->sms), 256, 0, s, x, M, K, x16, xs);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? WLQ_OK : cuda_fail(e, "prep_x16 launch");
}

// x16, xs and T' in one pass (int4 + low rank, K <= 4096): 16 rows per CTA.
// T = x L1 as [Th | Tl]: 64-row tiles, K split over a cluster of S CTAs
// (S doubles while the CTAs fit twice on the SMs and every split keeps two
// 64-wide chunks).
wlq_status launch_prep_lr_t(const uint16_t* x, const uint16_t* L1, const float* xs, int xs_scalar, int M, int K, int r,
                            int W, uint16_t* thl, DeviceInfo* d, cudaStream_t s) {
    auto kern = wlq::prep_lr_t_kernel;
    const size_t smem = wlq::lr_t_smem_bytes();
    if (!d->smem_set[27]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        d->smem_set[27] = true;
    }
    const int64_t tiles = cdiv(M, wlq::LR_ROWS);
    const int KC = static_cast<int>(cdiv(K, wlq::LR_KC));
    int S = 1;
    while (S * 2 <= wlq::LR_MAX_SPLITS && tiles * S * 2 <= 2 * d->sms && KC >= S * 2 * 2) S *= 2;
    int kc_per = static_cast<int>(cdiv(KC, S));
    while (S > 1 && (S - 1) * kc_per >= KC) {  // every split owns at least one chunk
        S /= 2;
        kc_per = static_cast<int>(cdiv(KC, S));
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(static_cast<unsigned>(S), static_cast<unsigned>(std::min<int64_t>(tiles, 65535)), 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    if (S > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(S);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cudaLaunchAttribute all_attrs[2];
    add_pdl(cfg, all_attrs);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, x, L1, xs, M, K, r, W, S, kc_per, xs_scalar, thl);
    return e == cudaSuccess ? WLQ_OK : cuda_fail(e, "prep_lr_t launch");
}

wlq_status launch_linear(Plan& p, int fmt, int64_t M, int64_t N, int64_t K, int r, const void* xin, float* xs,
                         uint16_t* thl, uint16_t* l2t, int W, const void* packed, const void* bias, void* y,
                         int y_dtype, DeviceInfo* d, cudaStream_t s) {
    wlq_status st;
    const int64_t NT = p.NT, KT = p.KT;
    // --- descriptors
    CUtensorMap tx, tt, tl;
    std::memset(&tt, 0, sizeof tt);
    std::memset(&tl, 0, sizeof tl);
    std::memset(&tx, 0, sizeof tx);
    if (!p.gemv && (st = make_map_2d(&tx, xin, M, K, p.pair ? p.BN / 2 : p.BN)) != WLQ_OK) return st;
    if (r) {
        if ((st = make_map_2d(&tt, thl, M, W, p.pair ? p.BN / 2 : p.BN)) != WLQ_OK) return st;
        if ((st = make_map_2d(&tl, l2t, NT * 128, W, 128)) != WLQ_OK) return st;
    }
    wlq::GemmArgs a;
    std::memset(&a, 0, sizeof a);
    a.packed = static_cast<const uint8_t*>(packed);
    a.rowf = reinterpret_cast<const float*>(a.packed + NT * KT * wlq::tile_bytes(fmt));
    a.xs = xs;
    a.bias = static_cast<const uint16_t*>(bias);
    a.y = y;
    a.M = p.M; a.N = p.N; a.K = p.K;
    a.NT = p.NT; a.KT = p.KT; a.MT = p.MT; a.S = p.S; a.kbps = p.kbps; a.BN = p.BN;
    a.stages = p.stages; a.astages = p.astages; a.ks = p.ks; a.lr = r ? 1 : 0; a.lr_kb = p.lr_kb; a.acc_bufs = p.acc_bufs;
    a.y_f32 = (y_dtype == WLQ_OUT_F32) ? 1 : 0;
    a.tiles_nm = p.tiles_nm;
    a.tmem_cols = p.tmem_cols; a.acc_col0 = p.acc_col0; a.lr_col0 = p.lr_col0; a.a_col0 = p.a_col0;
    a.wtile_bytes = p.wtile; a.wstage_bytes = p.wstage; a.xsub_bytes = p.xsub; a.xstage_bytes = p.xstage; a.red_bytes = p.red;
    a.stage_bytes = p.stage;
    a.red_alias = p.red_alias ? 1 : 0;
    a.S_red = p.S;
    // vector stores of y: unsplit tiles store 16-byte runs (4 fp32 / 8 bf16
    // channels), the split reduction 4 adjacent channels (16 / 8 bytes)
    {
        const uintptr_t ya = reinterpret_cast<uintptr_t>(y);
        const bool f32 = y_dtype == WLQ_OUT_F32;
        if (p.S == 1) a.vec_out = ((ya & 15u) == 0 && N % (f32 ? 4 : 8) == 0) ? 1 : 0;
        else a.vec_out = ((ya & (f32 ? 15u : 7u)) == 0 && N % 4 == 0) ? 1 : 0;
    }
    a.timeout_ns = kDefaultTimeoutNs;
    a.xg = xin;
    if (p.gemv) {
        if (fmt == wlq::FMT_W8) return launch_gemv_nb<wlq::FMT_W8>(p, a, d, s);
        if (fmt == wlq::FMT_W4G64) return launch_gemv_nb<wlq::FMT_W4G64>(p, a, d, s);
        return launch_gemv_nb<wlq::FMT_W4G16>(p, a, d, s);
    }
    if (p.skinny) {
        if (fmt == wlq::FMT_W8) return launch_skinny_nb<wlq::FMT_W8>(p, tx, a, d, s);
        if (fmt == wlq::FMT_W4G64) return launch_skinny_nb<wlq::FMT_W4G64>(p, tx, a, d, s);
        return launch_skinny_nb<wlq::FMT_W4G16>(p, tx, a, d, s);
    }
    switch (fmt * 3 + (p.pair ? 1 : 0) + (p.xres ? 2 : 0)) {
        case 0: return launch_gemm<wlq::FMT_W8, false, false>(p, tx, tt, tl, a, d, s);
        case 1: return launch_gemm<wlq::FMT_W8, true, false>(p, tx, tt, tl, a, d, s);
        case 2: return launch_gemm<wlq::FMT_W8, false, true>(p, tx, tt, tl, a, d, s);
        case 3: return launch_gemm<wlq::FMT_W4G64, false, false>(p, tx, tt, tl, a, d, s);
        case 4: return launch_gemm<wlq::FMT_W4G64, true, false>(p, tx, tt, tl, a, d, s);
        case 5: return launch_gemm<wlq::FMT_W4G64, false, true>(p, tx, tt, tl, a, d, s);
        case 6: return launch_gemm<wlq::FMT_W4G16, false, false>(p, tx, tt, tl, a, d, s);
        case 7: return launch_gemm<wlq::FMT_W4G16, true, false>(p, tx, tt, tl, a, d, s);
        default: return launch_gemm<wlq::FMT_W4G16, false, true>(p, tx, tt, tl, a, d, s);
    }
}

}  // namespace

extern "C" {

const char* wlq_version(void) { return "0.1.0"; }

const char* wlq_last_error(void) { return g_msg; }

wlq_status wlq_quantize(const float* W, int64_t N, int64_t K, int bits, int group, int8_t* codes,
                        float* scales, void* stream) {
    if (bits != 8 && bits != 4) return fail(WLQ_ERR_UNSUPPORTED, "bits must be 8 or 4");
    if (!(group == 0 || group == 16 || group == 32 || group == 64 || group == 128))
        return fail(WLQ_ERR_UNSUPPORTED, "group must be 0, 16, 32, 64 or 128");
    wlq_status st = check_shape(N, K, bits, group);
    if (st != WLQ_OK) return st;
    if (N == 0) return WLQ_OK;
    if (!W || !codes || !scales) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(W) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return fail(WLQ_ERR_ALIGN, "W and codes must be 16-byte aligned, scales 4-byte aligned");
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int qmax = (1 << (bits - 1)) - 1;
    if (group == 0 && K <= 8 * 4 * 1024) {
        // one CTA per row, the row held in registers (8 float4 per thread)
        const int64_t per_thread = 8 * 4;
        const int threads = static_cast<int>(std::min<int64_t>(1024, std::max<int64_t>(32, (cdiv(K, per_thread) + 31) / 32 * 32)));
        const int grid = static_cast<int>(std::min<int64_t>(N, static_cast<int64_t>(d->sms) * (2048 / threads)));
        launch_k(wlq::quantize_rows_cta_kernel<8>, grid, threads, 0, s, W, N, K, qmax, codes, scales);
    } else if (group == 0) {
        launch_k(wlq::quantize_rows_kernel, grid_for(N * 32, 256, d->sms), 256, 0, s, W, N, K, qmax, codes, scales);
    } else {
        const int64_t total4 = N * K / 4;
        launch_k(wlq::quantize_groups_kernel, grid_for(cdiv(total4, 4), 256, d->sms), 256, 0, s, W, total4, group / 4, qmax,
                                                                                   codes, scales);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    return WLQ_OK;
}

wlq_status wlq_quantize_pack(const float* W, int64_t N, int64_t K, int bits, int group, float* scales,
                             void* packed, void* stream) {
    const int fmt = fmt_of(bits, group);
    if (fmt < 0) return fail(WLQ_ERR_UNSUPPORTED, "quantize_pack supports (8,0), (4,64) and (4,16)");
    wlq_status st = check_shape(N, K, bits, group);
    if (st != WLQ_OK) return st;
    if (N == 0) return WLQ_OK;
    if (K > 8 * 4 * 1024) return fail(WLQ_ERR_SHAPE, "quantize_pack holds a row in registers: K <= 32768");
    if (!W || !scales || !packed) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(W) || !aligned16(packed) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return fail(WLQ_ERR_ALIGN, "W and packed must be 16-byte aligned, scales 4-byte aligned");
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t NT = cdiv(N, 128), KT = cdiv(K, 64);
    uint8_t* base = static_cast<uint8_t*>(packed);
    float* rowf = reinterpret_cast<float*>(base + NT * KT * wlq::tile_bytes(fmt));
    const int qmax = (1 << (bits - 1)) - 1;
    // one CTA per padded row, the row in registers: 8 float4 per thread
    const int64_t kp4 = KT * 16;
    const int threads = static_cast<int>(std::min<int64_t>(1024, std::max<int64_t>(32, (cdiv(kp4, 8) + 31) / 32 * 32)));
    const int64_t rows = NT * 128;
    const int grid = static_cast<int>(std::min<int64_t>(rows, static_cast<int64_t>(d->sms) * (2048 / threads)));
    if (fmt == wlq::FMT_W8)
        launch_k(wlq::quantize_pack_rows_kernel<wlq::FMT_W8, 8>, grid, threads, 0, s, W, N, K, static_cast<int>(KT), rows,
                                                                               qmax, scales, rowf, base);
    else if (fmt == wlq::FMT_W4G64)
        launch_k(wlq::quantize_pack_rows_kernel<wlq::FMT_W4G64, 8>, grid, threads, 0, s, W, N, K, static_cast<int>(KT), rows,
                                                                                  qmax, scales, rowf, base);
    else
        launch_k(wlq::quantize_pack_rows_kernel<wlq::FMT_W4G16, 8>, grid, threads, 0, s, W, N, K, static_cast<int>(KT), rows,
                                                                                  qmax, scales, rowf, base);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "quantize_pack launch");
    return WLQ_OK;
}

wlq_status wlq_quantize_ex(const void* W, int w_dtype, int64_t N, int64_t K, int bits, int group, int scale_dtype,
                           int8_t* codes, void* scales, void* stream) {
    if (bits < 2 || bits > 8) return fail(WLQ_ERR_UNSUPPORTED, "bits must be 2..8");
    if (w_dtype != WLQ_IN_F32 && w_dtype != WLQ_IN_BF16) return fail(WLQ_ERR_UNSUPPORTED, "input must be fp32 or bf16");
    if (scale_dtype < WLQ_SCALE_F32 || scale_dtype > WLQ_SCALE_BF16)
        return fail(WLQ_ERR_UNSUPPORTED, "scales must be fp32, fp16 or bf16");
    if (group < 0 || (group && group % 4)) return fail(WLQ_ERR_SHAPE, "group must be 0 or a positive multiple of 4");
    wlq_status st = check_shape(N, K, bits, group);
    if (st != WLQ_OK) return st;
    if (N == 0) return WLQ_OK;
    if (!W || !codes || !scales) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(W) || (reinterpret_cast<uintptr_t>(codes) & 3u) ||
        (reinterpret_cast<uintptr_t>(scales) & (scale_dtype == WLQ_SCALE_F32 ? 3u : 1u)))
        return fail(WLQ_ERR_ALIGN, "W must be 16-byte aligned, codes 4-byte, scales aligned to their type");
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t g = group ? group : K;
    const int64_t groups = N * (K / g);
    const int g4 = static_cast<int>(g / 4);
    const int qmax = (1 << (bits - 1)) - 1;
    const bool bf = (w_dtype == WLQ_IN_BF16);
    // bf16 with power-of-two groups of 8..512: E = 16 inputs a lane (codes 16-byte aligned, groups of
    // at least 16), else 8; four 16-byte loads a lane in flight, persistent
    const bool pow2 = g >= 8 && (g & (g - 1)) == 0;
    const int E = (pow2 && g >= 16 && g <= 512 && (reinterpret_cast<uintptr_t>(codes) & 15u) == 0) ? 16
                  : (pow2 && g <= 256 && (reinterpret_cast<uintptr_t>(codes) & 7u) == 0)          ? 8
                                                                                                  : 0;
    if (bf && E) {
        const int LG = static_cast<int>(g / E);
        const int64_t totalE = N * K / E;
        const int64_t rounds = cdiv(totalE, 32);
        const int U = 4 / (E / 8);
        const int grid = static_cast<int>(std::min<int64_t>(cdiv(cdiv(rounds, U), 8), static_cast<int64_t>(d->sms) * 8));
        const uint16_t* Wb = static_cast<const uint16_t*>(W);
#define WLQ_QB(F, L, EE) launch_k(wlq::quantize_ex_bf16_kernel<F, L, EE>, grid, 256, 0, s, Wb, totalE, qmax, codes, scales)
#define WLQ_QBL(F, EE)                 \
    switch (LG) {                      \
        case 1: WLQ_QB(F, 1, EE); break;   \
        case 2: WLQ_QB(F, 2, EE); break;   \
        case 4: WLQ_QB(F, 4, EE); break;   \
        case 8: WLQ_QB(F, 8, EE); break;   \
        case 16: WLQ_QB(F, 16, EE); break; \
        default: WLQ_QB(F, 32, EE); break; \
    }
        if (E == 16) {
            if (scale_dtype == WLQ_SCALE_F32) { WLQ_QBL(wlq::SCALE_F32, 16) }
            else if (scale_dtype == WLQ_SCALE_F16) { WLQ_QBL(wlq::SCALE_F16, 16) }
            else { WLQ_QBL(wlq::SCALE_BF16, 16) }
        } else {
            if (scale_dtype == WLQ_SCALE_F32) { WLQ_QBL(wlq::SCALE_F32, 8) }
            else if (scale_dtype == WLQ_SCALE_F16) { WLQ_QBL(wlq::SCALE_F16, 8) }
            else { WLQ_QBL(wlq::SCALE_BF16, 8) }
        }
#undef WLQ_QBL
#undef WLQ_QB
    } else if (g4 <= 32 && 32 % g4 == 0) {
        // short groups: one pass from registers, 32 / g4 groups per warp, four rounds in flight
        // persistent: the CTAs that fit at once (8 per SM) loop over the rounds
        const int64_t rounds = cdiv(groups * g4, 32);
        const int grid = static_cast<int>(std::min<int64_t>(cdiv(cdiv(rounds, 4), 8), static_cast<int64_t>(d->sms) * 8));
#define WLQ_QS(B, F, L) launch_k(wlq::quantize_ex_short_kernel<B, F, L>, grid, 256, 0, s, W, groups, qmax, codes, scales)
#define WLQ_QSL(B, F)                                                    \
    switch (g4) {                                                        \
        case 1: WLQ_QS(B, F, 1); break;                                  \
        case 2: WLQ_QS(B, F, 2); break;                                  \
        case 4: WLQ_QS(B, F, 4); break;                                  \
        case 8: WLQ_QS(B, F, 8); break;                                  \
        case 16: WLQ_QS(B, F, 16); break;                                \
        default: WLQ_QS(B, F, 32); break;                                \
    }
        if (scale_dtype == WLQ_SCALE_F32) { if (bf) { WLQ_QSL(true, wlq::SCALE_F32) } else { WLQ_QSL(false, wlq::SCALE_F32) } }
        else if (scale_dtype == WLQ_SCALE_F16) { if (bf) { WLQ_QSL(true, wlq::SCALE_F16) } else { WLQ_QSL(false, wlq::SCALE_F16) } }
        else { if (bf) { WLQ_QSL(true, wlq::SCALE_BF16) } else { WLQ_QSL(false, wlq::SCALE_BF16) } }
#undef WLQ_QSL
#undef WLQ_QS
    } else {
        const int grid = static_cast<int>(std::min<int64_t>(cdiv(groups, 8), static_cast<int64_t>(d->sms) * 8));
#define WLQ_QX(B, F) launch_k(wlq::quantize_ex_kernel<B, F>, grid, 256, 0, s, W, groups, g4, qmax, codes, scales)
        if (scale_dtype == WLQ_SCALE_F32) { if (bf) WLQ_QX(true, wlq::SCALE_F32); else WLQ_QX(false, wlq::SCALE_F32); }
        else if (scale_dtype == WLQ_SCALE_F16) { if (bf) WLQ_QX(true, wlq::SCALE_F16); else WLQ_QX(false, wlq::SCALE_F16); }
        else { if (bf) WLQ_QX(true, wlq::SCALE_BF16); else WLQ_QX(false, wlq::SCALE_BF16); }
#undef WLQ_QX
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "quantize_ex launch");
    return WLQ_OK;
}

wlq_status wlq_quantize_fp8(const void* W, int w_dtype, int64_t N, int64_t K, int group, uint8_t* codes,
                            float* scales, void* stream) {
    if (w_dtype != WLQ_IN_F32 && w_dtype != WLQ_IN_BF16) return fail(WLQ_ERR_UNSUPPORTED, "input must be fp32 or bf16");
    if (group < 0 || (group && group % 4)) return fail(WLQ_ERR_SHAPE, "group must be 0 or a positive multiple of 4");
    wlq_status st = check_shape(N, K, 8, group);
    if (st != WLQ_OK) return st;
    if (N == 0) return WLQ_OK;
    if (!W || !codes || !scales) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(W) || (reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return fail(WLQ_ERR_ALIGN, "W must be 16-byte aligned, codes and scales 4-byte aligned");
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t g = group ? group : K;
    const int64_t groups = N * (K / g);
    const int g4 = static_cast<int>(g / 4);
    const int grid = static_cast<int>(std::min<int64_t>(cdiv(groups, 8), static_cast<int64_t>(d->sms) * 8));
    if (w_dtype == WLQ_IN_BF16) launch_k(wlq::quantize_fp8_kernel<true>, grid, 256, 0, s, W, groups, g4, codes, scales);
    else launch_k(wlq::quantize_fp8_kernel<false>, grid, 256, 0, s, W, groups, g4, codes, scales);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "quantize_fp8 launch");
    return WLQ_OK;
}

size_t wlq_nvfp4_scales_bytes(int64_t rows, int64_t K) {
    if (rows < 0 || K <= 0 || K % 64) return 0;
    return wlq::nv_scale_bytes(rows, K);
}

wlq_status wlq_nvfp4_quantize(const void* X, int x_dtype, int64_t rows, int64_t K, void* codes, void* scales,
                              float* gscale, void* stream) {
    if (x_dtype != WLQ_IN_F32 && x_dtype != WLQ_IN_BF16) return fail(WLQ_ERR_UNSUPPORTED, "input must be fp32 or bf16");
    if (rows < 0 || K <= 0 || K % 64) return fail(WLQ_ERR_SHAPE, "NVFP4 needs rows >= 0 and K a positive multiple of 64");
    if (!X || !codes || !scales || !gscale) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(X) || !aligned16(codes) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(gscale) & 7u))
        return fail(WLQ_ERR_ALIGN, "X, codes and scales must be 16-byte aligned, gscale 8-byte aligned");
    int dev;
    DeviceInfo* d;
    wlq_status st;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(gscale, 0, 2 * sizeof(float), s);
    if (e == cudaSuccess && (rows % 256 || K % 256)) e = cudaMemsetAsync(scales, 0, wlq::nv_scale_bytes(rows, K), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    const int64_t nblocks = rows * (K / 16);
    const int grid = static_cast<int>(std::min<int64_t>(std::max<int64_t>(cdiv(nblocks, 256), 1), int64_t(d->sms) * 8));
    int lg_tpr = 0;  // threads per row of the quantize pass: the 16-input blocks of a row, up to 256
    while ((1 << lg_tpr) < 256 && (int64_t(1) << lg_tpr) < K / 16) ++lg_tpr;
    const int qgrid = static_cast<int>(std::min<int64_t>(std::max<int64_t>(cdiv(rows, 256 >> lg_tpr), 1), int64_t(d->sms) * 8));
    if (x_dtype == WLQ_IN_BF16) {
        launch_k(wlq::nvfp4_amax_kernel<1>, grid, 256, 0, s, X, nblocks, gscale);
        launch_k(wlq::nvfp4_quantize_kernel<1>, qgrid, 256, 0, s, X, rows, K, gscale, static_cast<uint8_t*>(codes),
                 static_cast<uint8_t*>(scales), lg_tpr);
    } else {
        launch_k(wlq::nvfp4_amax_kernel<0>, grid, 256, 0, s, X, nblocks, gscale);
        launch_k(wlq::nvfp4_quantize_kernel<0>, qgrid, 256, 0, s, X, rows, K, gscale, static_cast<uint8_t*>(codes),
                 static_cast<uint8_t*>(scales), lg_tpr);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "nvfp4 quantize launch");
    return WLQ_OK;
}

size_t wlq_packed_bytes(int64_t N, int64_t K, int bits, int group) {
    const int fmt = fmt_of(bits, group);
    if (fmt < 0 || N < 0 || K <= 0 || K % 8 || (group && K % group)) return 0;
    const int64_t NT = cdiv(N, 128), KT = cdiv(K, 64);
    return static_cast<size_t>(NT * KT) * wlq::tile_bytes(fmt) + static_cast<size_t>(NT) * 128 * 4;
}

wlq_status wlq_pack(const int8_t* codes, const float* scales, int64_t N, int64_t K, int bits, int group,
                    void* packed, void* stream) {
    const int fmt = fmt_of(bits, group);
    if (fmt < 0) return fail(WLQ_ERR_UNSUPPORTED, "pack supports (8,0), (4,64) and (4,16)");
    wlq_status st = check_shape(N, K, bits, group);
    if (st != WLQ_OK) return st;
    if (N == 0) return WLQ_OK;
    if (!codes || !scales || !packed) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(packed) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return fail(WLQ_ERR_ALIGN, "packed and codes must be 16-byte aligned, scales 4-byte aligned");
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t NT = cdiv(N, 128), KT = cdiv(K, 64);
    const int64_t G = group ? K / group : 1;
    uint8_t* base = static_cast<uint8_t*>(packed);
    float* rowf = reinterpret_cast<float*>(base + NT * KT * wlq::tile_bytes(fmt));
    if (fmt != wlq::FMT_W8)  // int8 row factors are written by the tile kernel itself
        launch_k(wlq::pack_rowfactor_kernel, grid_for(NT * 128 * 32, 256, d->sms), 256, 0, s, scales, N, G, fmt, NT * 128, rowf);
    launch_k(wlq::pack_tiles_kernel, static_cast<unsigned>(NT * KT), 128, 0, s, codes, scales, N, K, G, fmt,
                                                                          static_cast<int>(KT), rowf, base);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pack launch");
    return WLQ_OK;
}

wlq_status wlq_unpack(const void* packed, int64_t N, int64_t K, int bits, int group, int8_t* codes,
                      void* stream) {
    const int fmt = fmt_of(bits, group);
    if (fmt < 0) return fail(WLQ_ERR_UNSUPPORTED, "unpack supports (8,0), (4,64) and (4,16)");
    wlq_status st = check_shape(N, K, bits, group);
    if (st != WLQ_OK) return st;
    if (N == 0) return WLQ_OK;
    if (!codes || !packed) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(packed)) return fail(WLQ_ERR_ALIGN, "packed must be 16-byte aligned");
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    const int64_t NT = cdiv(N, 128), KT = cdiv(K, 64);
    launch_k(wlq::unpack_tiles_kernel, static_cast<unsigned>(NT * KT), 128, 0, static_cast<cudaStream_t>(stream), 
        static_cast<const uint8_t*>(packed), N, K, fmt, static_cast<int>(KT), codes);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "unpack launch");
    return WLQ_OK;
}

size_t wlq_linear_workspace(int64_t M, int64_t N, int64_t K, int bits, int group, int r) {
    const int fmt = fmt_of(bits, group);
    if (fmt < 0 || M < 0 || N < 0 || K <= 0 || !(r == 0 || r == 16 || r == 32 || r == 64)) return 0;
    if (M == 0 || N == 0) return 0;
    int sms = 148;
    int dev;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
    } else {
        cudaGetLastError();
    }
    Plan p;
    if (!make_plan(p, M, N, K, fmt, r, sms)) return 0;
    return p.ws;
}

}  // extern "C"

namespace {

// Argument checks of the Linear entry points, all made before any device
// access or planning.  *noop is set when the call has nothing to do (M == 0
// or N == 0 after valid arguments).
wlq_status check_linear_args(const void* x, int64_t M, const void* packed, int64_t N, int64_t K, int bits,
                             int group, const void* bias, const void* L1, const void* L2, int r, const void* y,
                             int y_dtype, bool* noop) {
    *noop = false;
    if (fmt_of(bits, group) < 0) return fail(WLQ_ERR_UNSUPPORTED, "linear supports (8,0), (4,64) and (4,16)");
    wlq_status st = check_shape(N, K, bits, group);
    if (st != WLQ_OK) return st;
    if (M < 0) return fail(WLQ_ERR_INVALID_ARG, "M < 0");
    if (M > (int64_t(1) << 30)) return fail(WLQ_ERR_SHAPE, "M too large");
    if (!(r == 0 || r == 16 || r == 32 || r == 64)) return fail(WLQ_ERR_SHAPE, "r must be 0, 16, 32 or 64");
    if (r && (!L1 || !L2)) return fail(WLQ_ERR_INVALID_ARG, "r > 0 needs L1 and L2");
    if (y_dtype != WLQ_OUT_BF16 && y_dtype != WLQ_OUT_F32) return fail(WLQ_ERR_INVALID_ARG, "bad y_dtype");
    if (M == 0 || N == 0) {
        *noop = true;
        return WLQ_OK;
    }
    if (!x || !packed || !y) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x) || !aligned16(packed)) return fail(WLQ_ERR_ALIGN, "x and packed must be 16-byte aligned");
    if ((bias && (reinterpret_cast<uintptr_t>(bias) & 1u)) || (L1 && !aligned16(L1)) ||
        (L2 && (reinterpret_cast<uintptr_t>(L2) & 1u)) || (reinterpret_cast<uintptr_t>(y) & 3u))
        return fail(WLQ_ERR_ALIGN, "L1 must be 16-byte aligned, bias/L2 2-byte aligned, y 4-byte aligned");
    return WLQ_OK;
}

}  // namespace

extern "C" {

wlq_status wlq_linear(const void* x, int64_t M, const void* packed, int64_t N, int64_t K, int bits, int group,
                      const void* bias, const void* L1, const void* L2, int r, void* y, int y_dtype,
                      void* workspace, size_t ws_bytes, void* stream) {
    bool noop = false;
    wlq_status st = check_linear_args(x, M, packed, N, K, bits, group, bias, L1, L2, r, y, y_dtype, &noop);
    if (st != WLQ_OK || noop) return st;
    const int fmt = fmt_of(bits, group);
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    Plan p;
    if (!make_plan(p, M, N, K, fmt, r, d->sms)) return fail(WLQ_ERR_UNSUPPORTED, "no launch plan for this shape");
    if (p.ws > 0 && (!workspace || ws_bytes < p.ws))
        return fail(WLQ_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", p.ws, ws_bytes);
    if (workspace && !aligned16(workspace)) return fail(WLQ_ERR_ALIGN, "workspace must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int64_t NT = p.NT;

    // --- operand preparation
    const void* xin = x;
    float* xs = nullptr;
    if (fmt != wlq::FMT_W8 && !p.gemv) {
        __half* x16 = reinterpret_cast<__half*>(ws + p.off_x16);
        xs = reinterpret_cast<float*>(ws + p.off_xs);
        if ((st = launch_prep_x16(static_cast<const uint16_t*>(x), p.M, p.K, x16, xs, d, s)) != WLQ_OK) return st;
        xin = x16;
    }
    uint16_t* thl = nullptr;
    uint16_t* l2t = nullptr;
    const int W = p.lr_kb * 64;
    if (r) {
        thl = reinterpret_cast<uint16_t*>(ws + p.off_thl);
        l2t = reinterpret_cast<uint16_t*>(ws + p.off_l2t);
        // the branch is folded into the GEMM's accumulator: T' = T / xs (int4) and
        // L2' = L2 / rowf, rowf read from the packed operand
        if ((st = launch_prep_lr_t(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(L1), xs, 0, p.M, p.K,
                                   r, W, thl, d, s)) != WLQ_OK)
            return st;
        const float* rowf = reinterpret_cast<const float*>(static_cast<const uint8_t*>(packed) +
                                                           static_cast<size_t>(NT) * p.KT * wlq::tile_bytes(fmt));
        launch_k(wlq::prep_lr_l2t_kernel, static_cast<int>(NT * 128 / wlq::L2T_ROWS), 256, 0, s,
                 static_cast<const uint16_t*>(L2), rowf, 0, p.N, static_cast<int>(NT * 128), r, W, l2t);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prep launch");

    // plans that keep a split partial in the ring need one tile per cluster:
    // if the device cannot hold that many clusters, take the next variant
    for (int attempt = 0; attempt < 3; ++attempt) {
        if (attempt > 0 && !make_plan(p, M, N, K, fmt, r, d->sms, attempt))
            return fail(WLQ_ERR_UNSUPPORTED, "no launch plan for this shape");
        st = launch_linear(p, fmt, M, N, K, r, xin, xs, thl, l2t, W, packed, bias, y, y_dtype, d, s);
        if (st != kRetryPlan) return st;
    }
    return fail(WLQ_ERR_UNSUPPORTED, "no launch plan for this shape");
}


}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of wlq_linear.  Its scratch lives in this file-scope
// device array (held by every GPU that loads the library, until exit).  In
// host code the array's name only stands in for it; the device address is
// fetched once per device with cudaGetSymbolAddress, with that device current.
namespace {
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
}  // namespace
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

namespace {
void* g_static_scratch_ptr[kMaxDevices] = {};
std::mutex g_static_mu;

wlq_status static_scratch(int dev, cudaStream_t stream, void** out) {
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_scratch_ptr[dev]) {
        // The address lookup is not a stream operation and may load the
        // module; inside a stream capture it would fail or invalidate the
        // capture, so the first call on a device must come before any capture.
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaError_t ce = cudaStreamIsCapturing(stream, &cs);
        if (ce != cudaSuccess) return cuda_fail(ce, "cudaStreamIsCapturing");
        if (cs != cudaStreamCaptureStatusNone)
            return fail(WLQ_ERR_INVALID_ARG,
                        "the first wlq_linear_noalloc call on a device looks up its built-in scratch and must "
                        "come before any stream capture");
        void* ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
        g_static_scratch_ptr[dev] = ptr;
    }
    *out = g_static_scratch_ptr[dev];
    return WLQ_OK;
}
}  // namespace

extern "C" {

wlq_status wlq_linear_noalloc(const void* x, int64_t M, const void* packed, int64_t N, int64_t K, int bits,
                              int group, const void* bias, const void* L1, const void* L2, int r, void* y,
                              int y_dtype, void* stream) {
    // The same argument checks as wlq_linear, before any planning or device
    // access, so an invalid call gets the same status from both entry points.
    bool noop = false;
    wlq_status st = check_linear_args(x, M, packed, N, K, bits, group, bias, L1, L2, r, y, y_dtype, &noop);
    if (st != WLQ_OK || noop) return st;
    const int fmt = fmt_of(bits, group);
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    Plan p;
    if (!make_plan(p, M, N, K, fmt, r, d->sms)) return fail(WLQ_ERR_UNSUPPORTED, "no launch plan for this shape");
    if (p.ws > kStaticScratchBytes)
        return fail(WLQ_ERR_WORKSPACE,
                    "this shape needs %zu bytes of scratch but the built-in scratch holds %zu; "
                    "call wlq_linear with a caller-owned workspace instead",
                    p.ws, kStaticScratchBytes);
    void* scratch = nullptr;
    if ((st = static_scratch(dev, static_cast<cudaStream_t>(stream), &scratch)) != WLQ_OK) return st;
    // Nothing in the scratch has to start at zero: every region is fully
    // written by the call's preparation kernels before the GEMM reads it.
    return wlq_linear(x, M, packed, N, K, bits, group, bias, L1, L2, r, y, y_dtype, scratch, kStaticScratchBytes,
                      stream);
}

}  // extern "C"

namespace {

// Workspace of the low-rank split: two [K, l] and two [N, l] fp32 panels,
// the fp64 Gram partials (one per chunk of LR_GRAM_ROWS rows), the small
// l x l / l x r matrices.
constexpr int LR_GRAM_ROWS = 64;
struct LrLayout {
    size_t y0, y1, z0, z1, parts, rinv, b1, b2, gpart, total;
};
constexpr int LR_MAX_GSPLIT = 8;  // inner-dimension splits of the skinny GEMM
LrLayout lr_layout(int64_t N, int64_t K, int l, int r) {
    LrLayout o;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off = align256(off + bytes); return at; };
    o.y0 = take(static_cast<size_t>(K) * l * 4);
    o.y1 = take(static_cast<size_t>(K) * l * 4);
    o.z0 = take(static_cast<size_t>(N) * l * 4);
    o.z1 = take(static_cast<size_t>(N) * l * 4);
    const int64_t parts = cdiv(std::max(N, K), LR_GRAM_ROWS);
    o.parts = take(static_cast<size_t>(parts) * l * l * 8);
    o.rinv = take(static_cast<size_t>(l) * l * 4);
    o.b1 = take(static_cast<size_t>(l) * r * 4);
    o.b2 = take(static_cast<size_t>(l) * r * 4);
    o.gpart = take(static_cast<size_t>(LR_MAX_GSPLIT) * std::max(N, K) * l * 4);
    o.total = off;
    return o;
}

bool lr_shape_ok(int64_t N, int64_t K, int r, int l, int q) {
    return (r == 16 || r == 32 || r == 64) && (l == 32 || l == 64) && l >= r && q >= 0 && q <= 8 && N >= l &&
           K >= l && N <= (int64_t(1) << 24) && K <= (int64_t(1) << 24);
}

// out = op(A) B through the skinny GEMM: the inner range split S ways (S <= 8,
// each at least 256 long) until the CTAs cover the SMs twice, the splits'
// partials (in `gpart`) added in order by a second pass.
template <bool TRANS>
void lr_gemm(const float* A, const float* B, int R, int inner, int c, float* out, uint16_t* out_bf16,
             uint16_t* out_bf16_t, float* gpart, int sms, cudaStream_t s) {
    const int tiles = static_cast<int>(cdiv(R, wlq::LRS_ROWS));
    int S = 1;
    while (S * 2 <= LR_MAX_GSPLIT && tiles * S < 2 * sms && inner / (S * 2) >= 256) S *= 2;
    const int kper = static_cast<int>(cdiv(cdiv(inner, S), wlq::LRS_KC) * wlq::LRS_KC);
    launch_k(wlq::lr_skinny_gemm<TRANS>, dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(S), 1),
             wlq::LRS_THREADS, 0, s, A, B, R, inner, c, kper, gpart);
    launch_k(wlq::lr_sum_splits, grid_for(static_cast<int64_t>(R) * c, 256, sms), 256, 0, s,
             static_cast<const float*>(gpart), S, R, c, out, out_bf16, out_bf16_t);
}

wlq_status lr_small(const double* parts, int nparts, int l, int r, int mode, float* o1, float* o2, float* sigma,
                    DeviceInfo* d, cudaStream_t s) {
    const size_t smem = static_cast<size_t>(2) * l * l * 8;
    if (!d->smem_set[40]) {
        cudaError_t e = cudaFuncSetAttribute(wlq::lr_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(2 * wlq::LRS_MAX_L * wlq::LRS_MAX_L * 8));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        d->smem_set[40] = true;
    }
    launch_k(wlq::lr_small_kernel, 1, 256, smem, s, parts, nparts, l, r, mode, o1, o2, sigma, static_cast<int*>(nullptr));
    return WLQ_OK;
}

void lr_gram(const float* Y, int R, int l, double* parts, cudaStream_t s) {
    const int nparts = static_cast<int>(cdiv(R, LR_GRAM_ROWS));
    if (l == 32) launch_k(wlq::lr_gram_partial<32>, nparts, 256, 0, s, Y, R, LR_GRAM_ROWS, parts);
    else launch_k(wlq::lr_gram_partial<64>, nparts, 256, 0, s, Y, R, LR_GRAM_ROWS, parts);
}

// Y <- orth(Y) by CholeskyQR2 (Y [R, l] in `cur`, `tmp` the same size); the
// orthonormal result ends in `cur`.
wlq_status lr_orth(float* cur, float* tmp, int R, int l, const LrLayout& L, uint8_t* ws, DeviceInfo* d,
                   cudaStream_t s) {
    double* parts = reinterpret_cast<double*>(ws + L.parts);
    float* rinv = reinterpret_cast<float*>(ws + L.rinv);
    const int nparts = static_cast<int>(cdiv(R, LR_GRAM_ROWS));
    wlq_status st;
    for (int pass = 0; pass < 2; ++pass) {
        lr_gram(cur, R, l, parts, s);
        if ((st = lr_small(parts, nparts, l, 0, 0, rinv, nullptr, nullptr, d, s)) != WLQ_OK) return st;
        lr_gemm<false>(cur, rinv, R, l, l, tmp, nullptr, nullptr, reinterpret_cast<float*>(ws + L.gpart), d->sms, s);
        std::swap(cur, tmp);
    }
    // two swaps: the result is back in the caller's `cur`
    return WLQ_OK;
}

}  // namespace

extern "C" {

size_t wlq_lowrank_workspace(int64_t N, int64_t K, int r, int l) {
    if (!lr_shape_ok(N, K, r, l, 0)) return 0;
    return lr_layout(N, K, l, r).total;
}

wlq_status wlq_lowrank_split(const float* W, int64_t N, int64_t K, int r, int l, int power_iters, const float* omega,
                             void* L1, void* L2, float* sigma, void* workspace, size_t ws_bytes, void* stream) {
    if (!lr_shape_ok(N, K, r, l, power_iters))
        return fail(WLQ_ERR_SHAPE, "low-rank split needs r in {16,32,64}, l in {32,64} with l >= r, "
                                   "0 <= power_iters <= 8 and N, K >= l");
    if (!W || !omega || !L1 || !L2 || !workspace) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(W) || !aligned16(omega) || !aligned16(L1) || !aligned16(L2) || !aligned16(workspace) ||
        (sigma && (reinterpret_cast<uintptr_t>(sigma) & 3u)))
        return fail(WLQ_ERR_ALIGN, "W, omega, L1, L2 and workspace must be 16-byte aligned");
    const LrLayout L = lr_layout(N, K, l, r);
    if (ws_bytes < L.total) return fail(WLQ_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", L.total, ws_bytes);
    int dev;
    DeviceInfo* d;
    wlq_status st = current_device(&dev, &d);
    if (st != WLQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* y0 = reinterpret_cast<float*>(ws + L.y0);
    float* y1 = reinterpret_cast<float*>(ws + L.y1);
    float* z0 = reinterpret_cast<float*>(ws + L.z0);
    float* z1 = reinterpret_cast<float*>(ws + L.z1);
    float* gpart = reinterpret_cast<float*>(ws + L.gpart);
    const int n = static_cast<int>(N), k = static_cast<int>(K);
    // Y = W^T Omega, orthonormalised
    lr_gemm<true>(W, omega, k, n, l, y0, nullptr, nullptr, gpart, d->sms, s);
    if ((st = lr_orth(y0, y1, k, l, L, ws, d, s)) != WLQ_OK) return st;
    for (int it = 0; it < power_iters; ++it) {
        lr_gemm<false>(W, y0, n, k, l, z0, nullptr, nullptr, gpart, d->sms, s);   // Z = W Q
        if ((st = lr_orth(z0, z1, n, l, L, ws, d, s)) != WLQ_OK) return st;
        lr_gemm<true>(W, z0, k, n, l, y0, nullptr, nullptr, gpart, d->sms, s);    // Y = W^T P
        if ((st = lr_orth(y0, y1, k, l, L, ws, d, s)) != WLQ_OK) return st;
    }
    // C = W Q; H = C^T C = U~ Lambda U~^T
    lr_gemm<false>(W, y0, n, k, l, z0, nullptr, nullptr, gpart, d->sms, s);
    double* parts = reinterpret_cast<double*>(ws + L.parts);
    const int nparts = static_cast<int>(cdiv(N, LR_GRAM_ROWS));
    lr_gram(z0, n, l, parts, s);
    float* b1 = reinterpret_cast<float*>(ws + L.b1);
    float* b2 = reinterpret_cast<float*>(ws + L.b2);
    if ((st = lr_small(parts, nparts, l, r, 1, b1, b2, sigma, d, s)) != WLQ_OK) return st;
    // L1 = Q U~_r Lambda_r^(1/4) [K, r]; L2 = (C U~_r Lambda_r^(-1/4))^T [r, N]
    lr_gemm<false>(y0, b1, k, l, r, nullptr, static_cast<uint16_t*>(L1), nullptr, gpart, d->sms, s);
    lr_gemm<false>(z0, b2, n, l, r, nullptr, nullptr, static_cast<uint16_t*>(L2), gpart, d->sms, s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "low-rank split launch");
    return WLQ_OK;
}

wlq_status wlq_lowrank_residual(const float* W, const void* L1, const void* L2, int64_t N, int64_t K, int r, float* R,
                                void* stream) {
    if (N < 0 || K <= 0 || !(r == 16 || r == 32 || r == 64) || N > (int64_t(1) << 30) || K > (int64_t(1) << 30))
        return fail(WLQ_ERR_SHAPE, "residual needs r in {16,32,64}, N >= 0, K > 0");
    if (N == 0) return WLQ_OK;
    if (!W || !L1 || !L2 || !R) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if ((reinterpret_cast<uintptr_t>(W) & 3u) || (reinterpret_cast<uintptr_t>(R) & 3u) ||
        (reinterpret_cast<uintptr_t>(L1) & 1u) || (reinterpret_cast<uintptr_t>(L2) & 1u))
        return fail(WLQ_ERR_ALIGN, "W and R must be 4-byte aligned, L1 and L2 2-byte aligned");
    int dev;
    DeviceInfo* d;
    wlq_status st = current_device(&dev, &d);
    if (st != WLQ_OK) return st;
    const dim3 grid(static_cast<unsigned>(cdiv(K, 32)), static_cast<unsigned>(cdiv(N, 32)), 1);
    if (grid.y > 65535) return fail(WLQ_ERR_SHAPE, "N too large for the residual kernel");
    launch_k(wlq::lr_residual_kernel, grid, 256, 0, static_cast<cudaStream_t>(stream), W,
             static_cast<const uint16_t*>(L1), static_cast<const uint16_t*>(L2), static_cast<int>(N),
             static_cast<int>(K), r, R);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "residual launch");
    return WLQ_OK;
}

void wlq_set_grid_limit(int max_ctas) { g_grid_limit = max_ctas > 0 ? max_ctas : 0; }

wlq_status wlq_get_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned word = 0;
    if ((e = cudaMemcpyFromSymbol(&word, wlq::g_error_word, sizeof word)) != cudaSuccess)
        return cuda_fail(e, "read error word");
    if (word) {
        const unsigned zero = 0;
        if ((e = cudaMemcpyToSymbol(wlq::g_error_word, &zero, sizeof zero)) != cudaSuccess)
            return cuda_fail(e, "clear error word");
    }
    if (word & wlq::ERRBIT_TIMEOUT) return fail(WLQ_ERR_TIMEOUT, "a bounded device wait ran out");
    if (word & wlq::ERRBIT_NONFINITE) return fail(WLQ_ERR_NONFINITE, "non-finite weight");
    if (word & wlq::ERRBIT_LAUNCH) return fail(WLQ_ERR_CUDA, "a kernel was launched with a shape it cannot run");
    return WLQ_OK;
}

wlq_status wlq_probe_wait_timeout(uint64_t timeout_ns, void* stream) {
    int dev;
    DeviceInfo* d;
    wlq_status st = current_device(&dev, &d);
    if (st != WLQ_OK) return st;
    const uint64_t cap = 10ull * 1000 * 1000 * 1000;
    launch_k(wlq::wait_probe_kernel, 1, 32, 0, static_cast<cudaStream_t>(stream), std::min(timeout_ns, cap));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "probe launch");
    return WLQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// NVFP4 W4A4 Linear (block-scaled tensor-core GEMM plus the low-rank branch)
namespace {

// 2-D tensor of bytes [rows, cols] (cols contiguous), box_rows x 128-byte
// boxes with a 128-byte swizzle; out-of-range bytes read as zero.
wlq_status make_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(WLQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {128, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(WLQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return WLQ_OK;
}

struct NvPlan {
    int NT = 0, MT = 0, KS = 0, KA = 0, tiles = 0, stages = 0, lr_kb = 0, W = 0;
    size_t smem = 0, off_thl = 0, off_l2t = 0, ws = 0;
};

constexpr size_t kMaxDynSmem = 232448;  // 227 KB per CTA

bool nv_plan(NvPlan& p, int64_t M, int64_t N, int64_t K, int r) {
    p.NT = static_cast<int>(cdiv(N, wlq::NV_TM));
    p.MT = static_cast<int>(cdiv(M, wlq::NV_TN));
    p.KS = static_cast<int>(cdiv(K, 256));
    p.KA = p.KS * 4;
    p.tiles = p.NT * p.MT;
    p.lr_kb = r ? static_cast<int>(cdiv(3 * r, 64)) : 0;
    p.W = 64 * p.lr_kb;
    p.stages = 0;
    for (int st = wlq::NV_MAX_STAGES; st >= 2; --st)
        if (wlq::nv_smem_bytes(st) <= kMaxDynSmem) {
            p.stages = st;
            break;
        }
    if (!p.stages) return false;
    p.smem = wlq::nv_smem_bytes(p.stages);
    size_t off = 0;
    if (r) {
        p.off_thl = off;
        off = align256(off + static_cast<size_t>(M) * p.W * 2);
        p.off_l2t = off;
        off = align256(off + static_cast<size_t>(p.NT) * 128 * p.W * 2);
    }
    p.ws = off;
    return true;
}

wlq_status check_nvfp4_linear(const void* xq, const void* xs, const float* xg, const void* x, int64_t M, const void* wq,
                              const void* ws, const float* wg, int64_t N, int64_t K, const void* bias, const void* L1,
                              const void* L2, int r, const void* y, int y_dtype, bool* noop) {
    *noop = false;
    if (M < 0 || N < 0) return fail(WLQ_ERR_INVALID_ARG, "M and N must be >= 0");
    if (K <= 0 || K % 64) return fail(WLQ_ERR_SHAPE, "NVFP4 needs K a positive multiple of 64");
    if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return fail(WLQ_ERR_SHAPE, "M or N too large");
    if (!(r == 0 || r == 16 || r == 32 || r == 64)) return fail(WLQ_ERR_SHAPE, "r must be 0, 16, 32 or 64");
    if (r && (!L1 || !L2 || !x)) return fail(WLQ_ERR_INVALID_ARG, "r > 0 needs x, L1 and L2");
    if (y_dtype != WLQ_OUT_BF16 && y_dtype != WLQ_OUT_F32) return fail(WLQ_ERR_INVALID_ARG, "bad y_dtype");
    if (M == 0 || N == 0) {
        *noop = true;
        return WLQ_OK;
    }
    if (!xq || !xs || !xg || !wq || !ws || !wg || !y) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(xq) || !aligned16(xs) || !aligned16(wq) || !aligned16(ws) || (x && !aligned16(x)) ||
        (L1 && !aligned16(L1)) || (L2 && (reinterpret_cast<uintptr_t>(L2) & 1u)) ||
        (bias && (reinterpret_cast<uintptr_t>(bias) & 1u)) || (reinterpret_cast<uintptr_t>(y) & 3u) ||
        (reinterpret_cast<uintptr_t>(xg) & 3u) || (reinterpret_cast<uintptr_t>(wg) & 3u))
        return fail(WLQ_ERR_ALIGN, "codes, scales, x and L1 must be 16-byte aligned, bias/L2 2-byte, y/xg/wg 4-byte");
    return WLQ_OK;
}

template <bool LR>
wlq_status launch_nvfp4_gemm(const NvPlan& p, const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& tl,
                             const CUtensorMap& tt, const CUtensorMap& ty, const wlq::NvArgs& a, DeviceInfo* d,
                             cudaStream_t s) {
    auto kern = wlq::nvfp4_gemm_kernel<LR>;
    const int kid = LR ? 51 : 50;
    if (!d->smem_set[kid]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kMaxDynSmem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        d->smem_set[kid] = true;
    }
    const int grid = std::min(p.tiles, d->sms);
    cudaError_t e = launch_k(kern, grid, wlq::NV_THREADS, p.smem, s, tw, tx, tl, tt, ty, a);
    return e == cudaSuccess ? WLQ_OK : cuda_fail(e, "nvfp4 gemm launch");
}

wlq_status nvfp4_linear_impl(const void* xq, const void* xs, const float* xg, const void* x, int64_t M, const void* wq,
                             const void* wsf, const float* wg, int64_t N, int64_t K, const void* bias, const void* L1,
                             const void* L2, int r, void* y, int y_dtype, uint8_t* ws, size_t ws_bytes, DeviceInfo* d,
                             cudaStream_t s) {
    NvPlan p;
    if (!nv_plan(p, M, N, K, r)) return fail(WLQ_ERR_UNSUPPORTED, "no NVFP4 launch plan for this shape");
    if (p.ws > 0 && (!ws || ws_bytes < p.ws)) return fail(WLQ_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", p.ws, ws_bytes);
    if (ws && !aligned16(ws)) return fail(WLQ_ERR_ALIGN, "workspace must be 16-byte aligned");
    wlq_status st;
    uint16_t* thl = nullptr;
    uint16_t* l2t = nullptr;
    if (r) {
        thl = reinterpret_cast<uint16_t*>(ws + p.off_thl);
        l2t = reinterpret_cast<uint16_t*>(ws + p.off_l2t);
        // T / g_x and L2 / g_w, each split into bf16 [h | l | h] and [h | h | l]: the
        // branch then adds into the FP4 accumulator, which the epilogue scales by g_x g_w
        if ((st = launch_prep_lr_t(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(L1), xg, 1,
                                   static_cast<int>(M), static_cast<int>(K), r, p.W, thl, d, s)) != WLQ_OK)
            return st;
        launch_k(wlq::prep_lr_l2t_kernel, p.NT * 128 / wlq::L2T_ROWS, 256, 0, s, static_cast<const uint16_t*>(L2), wg, 1,
                 static_cast<int>(N), p.NT * 128, r, p.W, l2t);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "low-rank prep launch");
    }
    CUtensorMap tw, tx, tl, tt;
    std::memset(&tl, 0, sizeof tl);
    std::memset(&tt, 0, sizeof tt);
    if ((st = make_map_u8(&tw, wq, N, K / 2, wlq::NV_TM)) != WLQ_OK) return st;
    if ((st = make_map_u8(&tx, xq, M, K / 2, wlq::NV_TN)) != WLQ_OK) return st;
    if (r) {
        if ((st = make_map_2d(&tl, l2t, static_cast<uint64_t>(p.NT) * 128, p.W, wlq::NV_TM)) != WLQ_OK) return st;
        if ((st = make_map_2d(&tt, thl, M, p.W, wlq::NV_TN)) != WLQ_OK) return st;
    }
    wlq::NvArgs a;
    std::memset(&a, 0, sizeof a);
    a.wsf = static_cast<const uint8_t*>(wsf);
    a.xsf = static_cast<const uint8_t*>(xs);
    a.wg = wg;
    a.xg = xg;
    a.bias = static_cast<const uint16_t*>(bias);
    a.y = y;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.NT = p.NT;
    a.MT = p.MT;
    a.KS = p.KS;
    a.KA = p.KA;
    a.tiles = p.tiles;
    a.stages = p.stages;
    a.lr_kb = p.lr_kb;
    a.y_f32 = (y_dtype == WLQ_OUT_F32) ? 1 : 0;
    // y through TMA stores when its rows are whole 16-byte units (else plain stores)
    CUtensorMap ty;
    std::memset(&ty, 0, sizeof ty);
    const size_t esize = a.y_f32 ? 4 : 2;
    if (aligned16(y) && (static_cast<size_t>(N) * esize) % 16 == 0) {
        EncodeTiledFn fn = encode_fn();
        if (!fn) return fail(WLQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * esize};
        const cuuint32_t box[2] = {32, 16};
        const cuuint32_t estr[2] = {1, 1};
        CUresult cr = fn(&ty, a.y_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, y, dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS) return fail(WLQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(cr));
        a.tma_store = 1;
    }
    a.timeout_ns = kDefaultTimeoutNs;
    return r ? launch_nvfp4_gemm<true>(p, tw, tx, tl, tt, ty, a, d, s)
             : launch_nvfp4_gemm<false>(p, tw, tx, tl, tt, ty, a, d, s);
}

struct W4a4Layout {
    size_t off_xq = 0, off_xs = 0, off_xg = 0, off_lin = 0, total = 0;
};
W4a4Layout w4a4_layout(int64_t M, int64_t K, size_t lin) {
    W4a4Layout L;
    size_t off = 0;
    L.off_xq = off;
    off = align256(off + static_cast<size_t>(M) * (K / 2));
    L.off_xs = off;
    off = align256(off + wlq::nv_scale_bytes(M, K));
    L.off_xg = off;
    off = align256(off + 16);
    L.off_lin = off;
    L.total = off + lin;
    return L;
}

}  // namespace

extern "C" {

size_t wlq_nvfp4_linear_workspace(int64_t M, int64_t N, int64_t K, int r) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 64 || !(r == 0 || r == 16 || r == 32 || r == 64)) return 0;
    NvPlan p;
    if (!nv_plan(p, M, N, K, r)) return 0;
    return p.ws;
}

wlq_status wlq_nvfp4_linear(const void* xq, const void* xs, const float* xg, const void* x, int64_t M, const void* wq,
                            const void* ws, const float* wg, int64_t N, int64_t K, const void* bias, const void* L1,
                            const void* L2, int r, void* y, int y_dtype, void* workspace, size_t ws_bytes,
                            void* stream) {
    bool noop = false;
    wlq_status st = check_nvfp4_linear(xq, xs, xg, x, M, wq, ws, wg, N, K, bias, L1, L2, r, y, y_dtype, &noop);
    if (st != WLQ_OK || noop) return st;
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    return nvfp4_linear_impl(xq, xs, xg, x, M, wq, ws, wg, N, K, bias, L1, L2, r, y, y_dtype,
                             static_cast<uint8_t*>(workspace), ws_bytes, d, static_cast<cudaStream_t>(stream));
}

size_t wlq_w4a4_workspace(int64_t M, int64_t N, int64_t K, int r) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 64 || !(r == 0 || r == 16 || r == 32 || r == 64)) return 0;
    NvPlan p;
    if (!nv_plan(p, M, N, K, r)) return 0;
    return w4a4_layout(M, K, p.ws).total;
}

wlq_status wlq_w4a4_linear(const void* x, int64_t M, const void* wq, const void* ws, const float* wg, int64_t N,
                           int64_t K, const void* bias, const void* L1, const void* L2, int r, void* y, int y_dtype,
                           void* workspace, size_t ws_bytes, void* stream) {
    if (M > 0 && N > 0 && !x) return fail(WLQ_ERR_INVALID_ARG, "null pointer");
    if (M > 0 && N > 0 && !workspace) return fail(WLQ_ERR_WORKSPACE, "the W4A4 Linear needs a workspace");
    uint8_t* w = static_cast<uint8_t*>(workspace);
    bool noop = false;
    // the activations' codes and scales are checked as if they were already in the workspace
    const W4a4Layout L = w4a4_layout(std::max<int64_t>(M, 0), K > 0 ? K : 64, 0);
    const void* xq = w ? w + L.off_xq : nullptr;
    const void* xs = w ? w + L.off_xs : nullptr;
    const float* xg = w ? reinterpret_cast<const float*>(w + L.off_xg) : nullptr;
    wlq_status st = check_nvfp4_linear(xq, xs, xg, x, M, wq, ws, wg, N, K, bias, L1, L2, r, y, y_dtype, &noop);
    if (st != WLQ_OK || noop) return st;
    if (!aligned16(x) || !aligned16(workspace)) return fail(WLQ_ERR_ALIGN, "x and workspace must be 16-byte aligned");
    int dev;
    DeviceInfo* d;
    if ((st = current_device(&dev, &d)) != WLQ_OK) return st;
    NvPlan p;
    if (!nv_plan(p, M, N, K, r)) return fail(WLQ_ERR_UNSUPPORTED, "no NVFP4 launch plan for this shape");
    const W4a4Layout LL = w4a4_layout(M, K, p.ws);
    if (ws_bytes < LL.total) return fail(WLQ_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", LL.total, ws_bytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = wlq_nvfp4_quantize(x, WLQ_IN_BF16, M, K, w + LL.off_xq, w + LL.off_xs,
                                 reinterpret_cast<float*>(w + LL.off_xg), stream)) != WLQ_OK)
        return st;
    return nvfp4_linear_impl(w + LL.off_xq, w + LL.off_xs, reinterpret_cast<const float*>(w + LL.off_xg), x, M, wq, ws,
                             wg, N, K, bias, L1, L2, r, y, y_dtype, w + LL.off_lin, ws_bytes - LL.off_lin, d, s);
}

}  // extern "C"
