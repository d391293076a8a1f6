// wq_api.cu -- the C ABI of libwq.so (declared in include/wq.h).
//
// Host side only: argument checks, the choice of kernel family, launch configuration and
// status reporting. Every step of the computation runs in the kernels included below.
// One translation unit so that the device error word is a single symbol.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "wq.h"

#include "common.cuh"
#include "pack.cuh"
#include "smallm.cuh"
#include "gemm_tc.cuh"

namespace {

thread_local char g_last_error[512] = "";

wq_status fail(wq_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

wq_status cuda_fail(cudaError_t e, const char *what) {
    return fail(WQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
    int checked = 0;   // 0 unknown, 1 supported, -1 unsupported
    int sm_count = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// Current device must be sm_100 (B200). Fills the SM count.
wq_status current_device(int *dev_out, const DeviceInfo **info) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(WQ_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo &d = g_dev[dev];
    if (d.checked == 0) {
        int major = 0, minor = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetAttribute");
        d.checked = (major == 10 && minor == 0) ? 1 : -1;
        d.sm_count = sms;
    }
    if (d.checked < 0)
        return fail(WQ_ERR_UNSUPPORTED_DEVICE, "device %d is not compute capability 10.0 (sm_100a)", dev);
    *dev_out = dev;
    *info = &d;
    return WQ_OK;
}

std::atomic<uint64_t> g_launches{0};

// One-time per-device set-up (kernel attributes) that concurrent host threads may race to:
// the first caller runs f() under a mutex, later callers see the flag and skip it. A failed
// set-up is retried by the next call.
std::mutex g_setup_mutex;
template <class F>
cudaError_t setup_once(std::atomic<int> (&done)[kMaxDevices], int dev, F &&f) {
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    const cudaError_t e = f();
    if (e == cudaSuccess) done[dev].store(1, std::memory_order_release);
    return e;
}

// Called right after every kernel launch: counts it and reports a launch error.
wq_status check_launch(const char *what) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? WQ_OK : cuda_fail(e, what);
}

// ------------------------------------------------------------------ quantize + pack
template <int BITS>
wq_status launch_pack(const void *W, int64_t n_groups, uint8_t *packed, float *scales, int sm_count,
                      cudaStream_t st) {
    const int64_t per_block = (int64_t)wq::kPackGroupsPerWarp * (wq::kPackThreads / 32);
    const int64_t want = (n_groups + per_block - 1) / per_block;
    const int grid = (int)std::min<int64_t>(want, (int64_t)sm_count * 16);
    wq::quantize_pack_kernel<BITS><<<grid, wq::kPackThreads, 0, st>>>(
        static_cast<const uint16_t *>(W), n_groups, packed, scales);
    return check_launch("quantize_pack_kernel");
}

// The jobs of one width, packed by quantize_pack_many_kernel in launches of up to
// kPackMaxSegs tensors (in the order given; empty jobs are skipped).
template <int BITS>
wq_status launch_pack_many(const wq_pack_job *jobs, int n_jobs, int sm_count, cudaStream_t st) {
    constexpr int64_t GW = wq::kPackGroupsPerWarp;
    const int64_t per_block = GW * (wq::kPackThreads / 32);
    wq::PackSegments segs;
    int i = 0;
    while (i < n_jobs) {
        segs.n = 0;
        segs.vbegin[0] = 0;
        for (; i < n_jobs && segs.n < wq::kPackMaxSegs; ++i) {
            const wq_pack_job &j = jobs[i];
            if (j.bits != BITS || j.N == 0 || j.K == 0) continue;
            const int k = segs.n++;
            const int64_t n_groups = j.N * (j.K / 128);
            segs.n_groups[k] = n_groups;
            segs.W[k] = static_cast<const uint16_t *>(j.W);
            segs.packed[k] = j.packed;
            segs.scales[k] = j.scales;
            segs.vbegin[k + 1] = segs.vbegin[k] + (n_groups + GW - 1) / GW * GW;
        }
        if (segs.n == 0) break;
        const int64_t want = (segs.vbegin[segs.n] + per_block - 1) / per_block;
        const int grid = (int)std::min<int64_t>(want, (int64_t)sm_count * 16);
        wq::quantize_pack_many_kernel<BITS><<<grid, wq::kPackThreads, 0, st>>>(segs);
        const wq_status s = check_launch("quantize_pack_many_kernel");
        if (s != WQ_OK) return s;
    }
    return WQ_OK;
}

// ------------------------------------------------------------------ small-M path
constexpr uint32_t kSmemMax = 227 * 1024;        // dynamic shared memory per CTA on sm_100

uint32_t align_u32(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Stage and shared-memory layout of smallm_kernel for `rows` weight rows per stage and a
// CTA range of `gcta` groups (`even`: every CTA of the launch has exactly gcta groups).
// Chunk width gc: the largest candidate that keeps a ring of at least three stages (two at
// one group per chunk); with an even split the candidates are the divisors of gcta, so no
// chunk is short. gc * bits <= 64 keeps a weight box row within 256 32-bit words.
template <int TOK>
bool small_layout(int bits, int rows, int gcta, bool even, bool scale_tma, int sbox, wq::SmallMArgs &a,
                  uint32_t *total) {
    using T = wq::SmTok<TOK>;
    const uint32_t tree = 4u * T::kNR * 32u * 4u;
    const uint32_t part = align_u32((uint32_t)TOK * T::kPStride * 4u, 128);
    const uint32_t bars = (2u * wq::kSmMaxStages + 4u) * 8u + 16u;
    const uint32_t sres = scale_tma ? align_u32((uint32_t)rows * (uint32_t)sbox * 4u, 128) : 0u;
    if (tree + part + bars + sres >= kSmemMax) return false;
    const uint32_t budget = kSmemMax - tree - part - bars - sres;
    for (int gc = std::min(gcta, 64 / bits); gc >= 1; --gc) {
        if (even ? (gcta % gc != 0) : ((gc & (gc - 1)) != 0 || gc > 8)) continue;
        const uint32_t w_bytes = align_u32((uint32_t)rows * (uint32_t)gc * 16u * (uint32_t)bits, 128);
        const uint32_t x_bytes = align_u32((uint32_t)TOK * (uint32_t)gc * 256u, 128);
        const uint32_t s_bytes = scale_tma ? 0u : align_u32((uint32_t)gc * (uint32_t)rows * 4u, 128);
        const uint32_t stage = w_bytes + x_bytes + s_bytes;
        const uint32_t stages = std::min<uint32_t>(wq::kSmMaxStages, budget / stage);
        if (stages < 3 && !(gc == 1 && stages >= 2)) continue;
        a.gc = gc;
        a.stages = (int)stages;
        a.srows = rows;
        a.stage_bytes = stage;
        a.off_x = w_bytes;
        a.off_s = w_bytes + x_bytes;
        a.scale_tma = scale_tma ? 1 : 0;
        a.sbox = sbox;
        a.off_sres = stages * stage;
        a.off_tree = a.off_sres + sres;
        a.off_part = a.off_tree + tree;
        a.off_bar = a.off_part + part;
        *total = a.off_bar + bars;
        return true;
    }
    return false;
}

// Clusters of S CTAs that fit at once (one CTA per SM, the most shared memory), cached.
template <int BITS, int TOK>
int small_max_clusters(int dev, int S, int sm_count) {
    // computed once per device and cluster size; two threads racing here compute the same value
    static std::atomic<int> cache[kMaxDevices][3] = {};
    const int si = S == 1 ? 0 : (S == 2 ? 1 : 2);
    const int cached = cache[dev][si].load(std::memory_order_relaxed);
    if (cached != 0) return cached;
    int n = sm_count / S;
    if (S > 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(S * (sm_count / S)));
        cfg.blockDim = dim3(wq::kSmThreads);
        cfg.dynamicSmemBytes = kSmemMax;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int q = 0;
        if (cudaOccupancyMaxActiveClusters(&q, (void *)wq::smallm_kernel<BITS, TOK>, &cfg) != cudaSuccess) q = 0;
        cudaGetLastError();
        n = std::min(n, q);
    }
    const int v = n > 0 ? n : -1;
    cache[dev][si].store(v, std::memory_order_relaxed);
    return v;
}

wq_status get_encoder();
wq_status make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);
wq_status make_map_3d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, const uint64_t (&dims)[3],
                      const uint64_t (&strides)[2], const uint32_t (&box)[3]);

template <int BITS, int TOK>
wq_status launch_smallm_tok(wq::SmallMArgs a, const uint8_t *packed, int dev, int sm_count, cudaStream_t st) {
    using T = wq::SmTok<TOK>;
    static std::atomic<int> attr_done[kMaxDevices] = {};
    cudaError_t e = setup_once(attr_done, dev, [] {
        return cudaFuncSetAttribute(wq::smallm_kernel<BITS, TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kSmemMax);
    });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(smallm)");
    const int64_t U = (a.N + 15) / 16;
    const int G = (int)(a.K / 128);
    // cluster size S (K split) and cluster count C: the fewest items on the busiest CTA,
    // items = (16-row units per cluster) x (groups per CTA); ties go to the smaller S
    int bestS = 1, bestC = 1;
    int64_t best = -1;
    for (int S = 1; S <= 4; S *= 2) {
        if (S > G) break;
        const int mc = small_max_clusters<BITS, TOK>(dev, S, sm_count);
        if (mc <= 0) continue;
        const int C = (int)std::min<int64_t>(mc, U);
        const int64_t cost = ((U + C - 1) / C) * ((G + S - 1) / S);
        if (best < 0 || cost < best) { best = cost; bestS = S; bestC = C; }
    }
    a.S = bestS;
    a.n_clusters = bestC;
    const int rows = (int)std::min<int64_t>(T::kRP, (U + bestC - 1) / bestC) * 16;
    const int gcta = (G + bestS - 1) / bestS;
    const bool even = (G % bestS) == 0;
    // resident steps by TMA: rows of G fp32 must be 16-byte multiples; the box covers the
    // CTA's groups from the 4-aligned group below its first one
    const int sbox = (gcta + 3 + 3) / 4 * 4;
    bool scale_tma = (G % 4 == 0) && sbox <= 256 && (uint64_t)rows * sbox * 4 <= 48 * 1024;
    uint32_t smem = 0;
    if (!small_layout<TOK>(BITS, rows, gcta, even, scale_tma, sbox, a, &smem)) {
        scale_tma = false;
        if (!small_layout<TOK>(BITS, rows, gcta, even, false, sbox, a, &smem))
            return fail(WQ_ERR_INVALID_ARG, "no shared-memory layout for the small-M kernel");
    }
    // TMA maps: packed as [N][K*b/32] 32-bit words (boxes of gc groups x 64/32/16 rows) and,
    // for short chunks, as {16b bytes, G, N} one group at a time; x as {128 k, G, M};
    // steps as [N][G] fp32
    const uint64_t G64 = (uint64_t)G, kGB = 16u * BITS, row_bytes = (uint64_t)a.K * BITS / 8;
    CUtensorMap pm64, pm32, pm16, pm_tail, xm_full, xm_tail, sm_map;
    wq_status s;
    const uint64_t pdims[3] = {kGB, G64, (uint64_t)a.N};
    const uint64_t pstr[2] = {kGB, row_bytes};
    const uint64_t xdims[3] = {128, G64, (uint64_t)a.M};
    const uint64_t xstr[2] = {256, (uint64_t)a.K * 2};
    const uint32_t pbox_t[3] = {(uint32_t)kGB, 1, 16};
    const uint32_t xbox_f[3] = {128, (uint32_t)a.gc, (uint32_t)TOK}, xbox_t[3] = {128, 1, (uint32_t)TOK};
    const uint32_t wbox = (uint32_t)a.gc * 4u * BITS;
    if ((s = make_map_2d(&pm64, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, row_bytes / 4, (uint64_t)a.N, row_bytes, wbox, 64,
                         CU_TENSOR_MAP_SWIZZLE_NONE)) != WQ_OK ||
        (s = make_map_2d(&pm32, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, row_bytes / 4, (uint64_t)a.N, row_bytes, wbox, 32,
                         CU_TENSOR_MAP_SWIZZLE_NONE)) != WQ_OK ||
        (s = make_map_2d(&pm16, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, row_bytes / 4, (uint64_t)a.N, row_bytes, wbox, 16,
                         CU_TENSOR_MAP_SWIZZLE_NONE)) != WQ_OK ||
        (s = make_map_3d(&pm_tail, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, pdims, pstr, pbox_t)) != WQ_OK ||
        (s = make_map_3d(&xm_full, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, xdims, xstr, xbox_f)) != WQ_OK ||
        (s = make_map_3d(&xm_tail, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, xdims, xstr, xbox_t)) != WQ_OK)
        return s;
    if (scale_tma) {
        if ((s = make_map_2d(&sm_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.scales, G64, (uint64_t)a.N, G64 * 4,
                             (uint32_t)sbox, 16, CU_TENSOR_MAP_SWIZZLE_NONE)) != WQ_OK)
            return s;
    } else {
        sm_map = pm16;   // not read by the kernel
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(bestC * bestS));
    cfg.blockDim = dim3(wq::kSmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)bestS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = bestS > 1 ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, wq::smallm_kernel<BITS, TOK>, pm64, pm32, pm16, pm_tail, xm_full, xm_tail, sm_map, a);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(smallm_kernel)");
    return check_launch("smallm_kernel");
}

// Up to 16 tokens per launch; more tokens take several launches.
template <int BITS>
wq_status launch_smallm(const wq::SmallMArgs &base, const uint8_t *packed, int dev, int sm_count, cudaStream_t st) {
    for (int64_t m0 = 0; m0 < base.M; m0 += wq::kSmMaxTok) {
        wq::SmallMArgs a = base;
        a.M = std::min<int64_t>(wq::kSmMaxTok, base.M - m0);
        a.x = base.x + m0 * base.K;
        a.y = base.y + m0 * base.N;
        if (base.t) a.t = base.t + m0 * wq::kTStrideSm;
        wq_status s;
        if (a.M <= 8) s = launch_smallm_tok<BITS, 8>(a, packed, dev, sm_count, st);
        else s = launch_smallm_tok<BITS, 16>(a, packed, dev, sm_count, st);
        if (s != WQ_OK) return s;
    }
    return WQ_OK;
}


// ------------------------------------------------------------------ tensor-core path
constexpr int64_t kSmallMThreshold = 32;

struct TcArgs {
    const void *x;
    int64_t M, K;
    const uint8_t *packed;
    const float *scales;
    int bits;
    int64_t N;
    const void *L1, *L2;
    int rank;
    const void *bias;
    void *y;
    void *workspace;
};

size_t tc_workspace_bytes(int64_t M, int64_t /*N*/, int64_t /*K*/, int rank) {
    return rank > 0 ? ((size_t)M * wq::kTStride * 2 + 255) / 256 * 256 : 0;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

wq_status get_encoder() {
    std::call_once(g_encode_once, [] {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorName(g_encode_err));
    return WQ_OK;
}

wq_status make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    wq_status s = get_encoder();
    if (s != WQ_OK) return s;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return WQ_OK;
}

wq_status make_map_3d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, const uint64_t (&dims)[3],
                      const uint64_t (&strides)[2], const uint32_t (&box)[3]) {
    wq_status s = get_encoder();
    if (s != WQ_OK) return s;
    const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    const cuuint64_t st[2] = {strides[0], strides[1]};
    const cuuint32_t b[3] = {box[0], box[1], box[2]};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, dt, 3, const_cast<void *>(base), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled (3d) failed (%d)", (int)r);
    return WQ_OK;
}

template <int BITS>
wq_status launch_tc(const TcArgs &a, const CUtensorMap &xm, const CUtensorMap &pm, const CUtensorMap &tm,
                    const CUtensorMap &lm, int l_tma, int sm_count, cudaStream_t st) {
    using L = wq::TcLayout<BITS>;
    static std::atomic<int> attr_done[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const cudaError_t e = setup_once(attr_done, dev, [] {
        return cudaFuncSetAttribute(wq::tc_linear_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)L::kAlloc);
    });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tc_linear_kernel)");
    wq::TcParams p{};
    p.scales = a.scales;
    p.L2 = static_cast<const uint16_t *>(a.L2);
    p.bias = static_cast<const uint16_t *>(a.bias);
    p.y = static_cast<uint16_t *>(a.y);
    p.M = a.M; p.N = a.N; p.K = a.K; p.rank = a.rank;
    p.tiles_m = (int)((a.M + wq::kTcBT - 1) / wq::kTcBT);
    p.tiles_n = (int)((a.N + wq::kTcBW - 1) / wq::kTcBW);
    p.l_tma = l_tma;
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = std::min(tiles, sm_count);
    wq::tc_linear_kernel<BITS><<<grid, wq::kTcThreads, L::kAlloc, st>>>(xm, pm, tm, lm, p);
    return check_launch("tc_linear_kernel");
}

template <int R>
wq_status launch_prepass(const TcArgs &a, uint16_t *t, int sm_count, cudaStream_t st) {
    const int64_t mtiles = (a.M + 63) / 64;
    const int64_t nkb = a.K / 64;
    // The prepass is latency-bound (each CTA walks its K share one 64-k block at a time), so
    // K is split (clusters of up to 16 CTAs, a non-portable size) until about eight CTAs per
    // SM are in flight.
    static std::atomic<int> attr_done[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t e = setup_once(attr_done, dev, [] {
        return cudaFuncSetAttribute(wq::lowrank_prepass_kernel<R>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(lowrank_prepass_kernel)");
    const int kmax = 16;
    int ks = 1;
    while (ks < kmax && ks * 2 <= nkb && mtiles * ks < 8 * (int64_t)sm_count) ks *= 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)mtiles, (unsigned)ks, 1);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)ks;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, wq::lowrank_prepass_kernel<R>, static_cast<const uint16_t *>(a.x),
                                       static_cast<const uint16_t *>(a.L1), t, a.M, a.K);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(lowrank_prepass_kernel)");
    return check_launch("lowrank_prepass_kernel");
}

wq_status tc_linear(const TcArgs &a, int sm_count, cudaStream_t st) {
    wq_status s = get_encoder();
    if (s != WQ_OK) return s;
    if (a.M > (int64_t)INT32_MAX || a.N > (int64_t)INT32_MAX || a.K > (int64_t)INT32_MAX)
        return fail(WQ_ERR_INVALID_ARG, "dimension above 2^31 on the tensor-core path");
    CUtensorMap xm, pm, tm, lm;
    int l_tma = 0;
    if ((s = make_map_2d(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)a.K, (uint64_t)a.M,
                         (uint64_t)a.K * 2, wq::kTcBK, wq::kTcBT, CU_TENSOR_MAP_SWIZZLE_128B)) != WQ_OK)
        return s;
    const uint64_t row_bytes = (uint64_t)a.K * a.bits / 8;
    if ((s = make_map_2d(&pm, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.packed, row_bytes, (uint64_t)a.N, row_bytes,
                         16u * a.bits, wq::kTcBW, CU_TENSOR_MAP_SWIZZLE_NONE)) != WQ_OK)
        return s;
    tm = xm;
    if (a.rank > 0) {
        uint16_t *t = static_cast<uint16_t *>(a.workspace);
        switch (a.rank) {
            case 16: s = launch_prepass<16>(a, t, sm_count, st); break;
            case 32: s = launch_prepass<32>(a, t, sm_count, st); break;
            case 48: s = launch_prepass<48>(a, t, sm_count, st); break;
            default: s = launch_prepass<64>(a, t, sm_count, st); break;
        }
        if (s != WQ_OK) return s;
        if ((s = make_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, t, (uint64_t)wq::kTStride, (uint64_t)a.M,
                             (uint64_t)wq::kTStride * 2, wq::kTcBK, wq::kTcBT, CU_TENSOR_MAP_SWIZZLE_128B)) != WQ_OK)
            return s;
        // L2 (rank x N) by TMA when its rows are 16-byte multiples: a [rank][128] tile per weight tile
        if (a.N % 8 == 0) {
            if ((s = make_map_2d(&lm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L2, (uint64_t)a.N, (uint64_t)a.rank,
                                 (uint64_t)a.N * 2, wq::kTcBW, (uint32_t)a.rank, CU_TENSOR_MAP_SWIZZLE_NONE)) != WQ_OK)
                return s;
            l_tma = 1;
        }
    }
    if (!l_tma) lm = xm;   // not read by the kernel
    switch (a.bits) {
        case 3: return launch_tc<3>(a, xm, pm, tm, lm, l_tma, sm_count, st);
        case 4: return launch_tc<4>(a, xm, pm, tm, lm, l_tma, sm_count, st);
        case 5: return launch_tc<5>(a, xm, pm, tm, lm, l_tma, sm_count, st);
        case 6: return launch_tc<6>(a, xm, pm, tm, lm, l_tma, sm_count, st);
        default: return launch_tc<7>(a, xm, pm, tm, lm, l_tma, sm_count, st);
    }
}

size_t smallm_workspace(int64_t M, int rank) { return tc_workspace_bytes(M, 0, 0, rank); }

// ------------------------------------------------------------------ static scratch
// Scratch for wq_linear_no_workspace: a file-scope device array. In host code its name is
// only a stand-in, so the kernels get the address cudaGetSymbolAddress reports, looked up
// once per device with that device current.
static __device__ __align__(256) unsigned char g_static_scratch[WQ_STATIC_SCRATCH_BYTES];
void *g_static_scratch_ptr[kMaxDevices] = {};
std::mutex g_static_scratch_mutex;

wq_status static_scratch(int dev, void **out) {
    std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
    if (!g_static_scratch_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
        g_static_scratch_ptr[dev] = p;
    }
    *out = g_static_scratch_ptr[dev];
    return WQ_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int wq_version(void) { return 100; }

size_t wq_packed_bytes(int64_t N, int64_t K, int bits, int group) {
    if (N < 0 || K < 0 || bits < 3 || bits > 7 || group != 128 || K % group != 0) return 0;
    return (size_t)N * (size_t)K * (size_t)bits / 8;
}

int64_t wq_scales_count(int64_t N, int64_t K, int group) {
    if (N < 0 || K < 0 || group <= 0 || K % group != 0) return -1;
    return N * (K / group);
}

const char *wq_status_string(wq_status s) {
    switch (s) {
        case WQ_OK: return "ok";
        case WQ_ERR_INVALID_ARG: return "invalid argument";
        case WQ_ERR_UNSUPPORTED_BITS: return "unsupported bit width (3..7)";
        case WQ_ERR_UNSUPPORTED_GROUP: return "unsupported group size (128)";
        case WQ_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
        case WQ_ERR_CUDA: return "CUDA error";
        case WQ_ERR_TIMEOUT: return "device-side wait timed out";
        case WQ_ERR_WORKSPACE: return "workspace missing or too small";
        case WQ_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
    }
    return "unknown status";
}

const char *wq_last_error(void) { return g_last_error; }

uint64_t wq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

wq_status wq_quantize_pack(const void *W, int64_t N, int64_t K, int bits, int group, uint8_t *packed,
                           float *scales, wq_stream_t stream) {
    g_last_error[0] = 0;
    if (bits < 3 || bits > 7) return fail(WQ_ERR_UNSUPPORTED_BITS, "bits=%d", bits);
    if (group != 128) return fail(WQ_ERR_UNSUPPORTED_GROUP, "group=%d", group);
    if (N < 0 || K < 0) return fail(WQ_ERR_INVALID_ARG, "negative size N=%lld K=%lld", (long long)N, (long long)K);
    if (K % 128 != 0) return fail(WQ_ERR_INVALID_ARG, "K=%lld is not a multiple of 128", (long long)K);
    if (N == 0 || K == 0) return WQ_OK;
    if (!W || !packed || !scales) return fail(WQ_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(W) || !aligned16(packed) || !aligned16(scales))
        return fail(WQ_ERR_MISALIGNED, "W/packed/scales must be 16-byte aligned");
    int dev;
    const DeviceInfo *info;
    wq_status s = current_device(&dev, &info);
    if (s != WQ_OK) return s;
    const int64_t n_groups = N * (K / 128);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (bits) {
        case 3: return launch_pack<3>(W, n_groups, packed, scales, info->sm_count, st);
        case 4: return launch_pack<4>(W, n_groups, packed, scales, info->sm_count, st);
        case 5: return launch_pack<5>(W, n_groups, packed, scales, info->sm_count, st);
        case 6: return launch_pack<6>(W, n_groups, packed, scales, info->sm_count, st);
        default: return launch_pack<7>(W, n_groups, packed, scales, info->sm_count, st);
    }
}

wq_status wq_quantize_pack_many(const wq_pack_job *jobs, int n_jobs, int group, wq_stream_t stream) {
    g_last_error[0] = 0;
    if (group != 128) return fail(WQ_ERR_UNSUPPORTED_GROUP, "group=%d", group);
    if (n_jobs < 0) return fail(WQ_ERR_INVALID_ARG, "n_jobs=%d", n_jobs);
    if (n_jobs == 0) return WQ_OK;
    if (!jobs) return fail(WQ_ERR_INVALID_ARG, "NULL job array");
    bool any = false;
    for (int i = 0; i < n_jobs; ++i) {
        const wq_pack_job &j = jobs[i];
        if (j.bits < 3 || j.bits > 7) return fail(WQ_ERR_UNSUPPORTED_BITS, "job %d: bits=%d", i, j.bits);
        if (j.N < 0 || j.K < 0)
            return fail(WQ_ERR_INVALID_ARG, "job %d: negative size N=%lld K=%lld", i, (long long)j.N, (long long)j.K);
        if (j.K % 128 != 0) return fail(WQ_ERR_INVALID_ARG, "job %d: K=%lld is not a multiple of 128", i, (long long)j.K);
        if (j.N == 0 || j.K == 0) continue;
        if (!j.W || !j.packed || !j.scales) return fail(WQ_ERR_INVALID_ARG, "job %d: NULL tensor pointer", i);
        if (!aligned16(j.W) || !aligned16(j.packed) || !aligned16(j.scales))
            return fail(WQ_ERR_MISALIGNED, "job %d: W/packed/scales must be 16-byte aligned", i);
        any = true;
    }
    if (!any) return WQ_OK;
    int dev;
    const DeviceInfo *info;
    wq_status s = current_device(&dev, &info);
    if (s != WQ_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((s = launch_pack_many<3>(jobs, n_jobs, info->sm_count, st)) != WQ_OK) return s;
    if ((s = launch_pack_many<4>(jobs, n_jobs, info->sm_count, st)) != WQ_OK) return s;
    if ((s = launch_pack_many<5>(jobs, n_jobs, info->sm_count, st)) != WQ_OK) return s;
    if ((s = launch_pack_many<6>(jobs, n_jobs, info->sm_count, st)) != WQ_OK) return s;
    return launch_pack_many<7>(jobs, n_jobs, info->sm_count, st);
}

size_t wq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int rank) {
    if (M < 0 || N < 0 || K < 0 || bits < 3 || bits > 7 || rank < 0) return 0;
    return std::max(smallm_workspace(M, rank), tc_workspace_bytes(M, N, K, rank));
}

wq_status wq_linear_ex(const void *x, int64_t M, int64_t K, const uint8_t *packed, const float *scales, int bits,
                       int group, int64_t N, const void *L1, const void *L2, int rank, const void *bias, void *y,
                       void *workspace, size_t workspace_bytes, wq_path path, wq_stream_t stream) {
    g_last_error[0] = 0;
    if (bits < 3 || bits > 7) return fail(WQ_ERR_UNSUPPORTED_BITS, "bits=%d", bits);
    if (group != 128) return fail(WQ_ERR_UNSUPPORTED_GROUP, "group=%d", group);
    if (M < 0 || N < 0 || K < 0) return fail(WQ_ERR_INVALID_ARG, "negative size");
    if (K % 128 != 0) return fail(WQ_ERR_INVALID_ARG, "K=%lld is not a multiple of 128", (long long)K);
    if (rank < 0 || rank > 64 || rank % 16 != 0)
        return fail(WQ_ERR_INVALID_ARG, "rank=%d must be 0..64 and a multiple of 16", rank);
    if (rank > 0 && (!L1 || !L2)) return fail(WQ_ERR_INVALID_ARG, "rank > 0 needs L1 and L2");
    if (rank == 0 && (L1 || L2)) return fail(WQ_ERR_INVALID_ARG, "L1/L2 given with rank 0");
    if (path != WQ_PATH_AUTO && path != WQ_PATH_SMALL_M && path != WQ_PATH_TENSOR)
        return fail(WQ_ERR_INVALID_ARG, "unknown path %d", (int)path);
    if (M == 0 || N == 0) return WQ_OK;
    if (K == 0) return fail(WQ_ERR_INVALID_ARG, "K must be positive when M, N > 0");
    if (!x || !packed || !scales || !y) return fail(WQ_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y) ||
        (L1 && !aligned16(L1)) || (L2 && !aligned16(L2)) || (bias && !aligned16(bias)) ||
        (workspace && !aligned16(workspace)))
        return fail(WQ_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
    const size_t need = wq_linear_workspace_bytes(M, N, K, bits, rank);
    if (need > 0 && (!workspace || workspace_bytes < need))
        return fail(WQ_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : (size_t)0);
    int dev;
    const DeviceInfo *info;
    wq_status s = current_device(&dev, &info);
    if (s != WQ_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    const bool small = (path == WQ_PATH_SMALL_M) || (path == WQ_PATH_AUTO && M <= kSmallMThreshold);
    if (!small) {
        TcArgs ta{x, M, K, packed, scales, bits, N, L1, L2, rank, bias, y, workspace};
        return tc_linear(ta, info->sm_count, st);
    }

    wq::SmallMArgs a{};
    a.x = static_cast<const uint16_t *>(x);
    a.scales = scales;
    a.bias = static_cast<const uint16_t *>(bias);
    a.L2 = static_cast<const uint16_t *>(L2);
    a.y = static_cast<uint16_t *>(y);
    a.M = M; a.N = N; a.K = K; a.rank = rank;
    if (M > (int64_t)INT32_MAX || N > (int64_t)INT32_MAX || K > (int64_t)INT32_MAX)
        return fail(WQ_ERR_INVALID_ARG, "dimension above 2^31 on the small-M path");
    if (rank > 0) {
        // t = x L1 as [t_hi | t_lo] bf16 pairs, the same prepass as the tensor-core path
        TcArgs ta{x, M, K, packed, scales, bits, N, L1, L2, rank, bias, y, workspace};
        uint16_t *t = static_cast<uint16_t *>(workspace);
        switch (rank) {
            case 16: s = launch_prepass<16>(ta, t, info->sm_count, st); break;
            case 32: s = launch_prepass<32>(ta, t, info->sm_count, st); break;
            case 48: s = launch_prepass<48>(ta, t, info->sm_count, st); break;
            default: s = launch_prepass<64>(ta, t, info->sm_count, st); break;
        }
        if (s != WQ_OK) return s;
        a.t = t;
    }
    switch (bits) {
        case 3: return launch_smallm<3>(a, packed, dev, info->sm_count, st);
        case 4: return launch_smallm<4>(a, packed, dev, info->sm_count, st);
        case 5: return launch_smallm<5>(a, packed, dev, info->sm_count, st);
        case 6: return launch_smallm<6>(a, packed, dev, info->sm_count, st);
        default: return launch_smallm<7>(a, packed, dev, info->sm_count, st);
    }
}

wq_status wq_linear(const void *x, int64_t M, int64_t K, const uint8_t *packed, const float *scales, int bits,
                    int group, int64_t N, const void *L1, const void *L2, int rank, const void *bias, void *y,
                    void *workspace, size_t workspace_bytes, wq_stream_t stream) {
    return wq_linear_ex(x, M, K, packed, scales, bits, group, N, L1, L2, rank, bias, y, workspace,
                        workspace_bytes, WQ_PATH_AUTO, stream);
}

wq_status wq_linear_no_workspace(const void *x, int64_t M, int64_t K, const uint8_t *packed, const float *scales,
                                 int bits, int group, int64_t N, const void *L1, const void *L2, int rank,
                                 const void *bias, void *y, wq_stream_t stream) {
    g_last_error[0] = 0;
    const size_t need = wq_linear_workspace_bytes(M, N, K, bits, rank);
    if (need > WQ_STATIC_SCRATCH_BYTES)
        return fail(WQ_ERR_WORKSPACE, "scratch of %zu bytes needed, the static buffer holds %zu", need,
                    (size_t)WQ_STATIC_SCRATCH_BYTES);
    void *scratch = nullptr;
    size_t scratch_bytes = 0;
    if (need > 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
        if (dev < 0 || dev >= kMaxDevices) return fail(WQ_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
        wq_status s = static_scratch(dev, &scratch);
        if (s != WQ_OK) return s;
        scratch_bytes = WQ_STATIC_SCRATCH_BYTES;
    }
    return wq_linear_ex(x, M, K, packed, scales, bits, group, N, L1, L2, rank, bias, y, scratch, scratch_bytes,
                        WQ_PATH_AUTO, stream);
}

wq_status wq_device_status(wq_stream_t stream, int clear) {
    g_last_error[0] = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0;
    e = cudaMemcpyFromSymbolAsync(&v, wq::g_dev_status, sizeof v, 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    if (clear) {
        const int zero = 0;
        e = cudaMemcpyToSymbolAsync(wq::g_dev_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
    }
    if (v != 0) return fail((wq_status)v, "device recorded: %s", wq_status_string((wq_status)v));
    return WQ_OK;
}

wq_status wq_selftest_bounded_wait(uint32_t timeout_us, wq_stream_t stream) {
    g_last_error[0] = 0;
    if (timeout_us < 1 || timeout_us > 1000000) return fail(WQ_ERR_INVALID_ARG, "timeout_us=%u", timeout_us);
    int dev;
    const DeviceInfo *info;
    wq_status s = current_device(&dev, &info);
    if (s != WQ_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    wq::bounded_wait_selftest_kernel<<<1, 32, 0, st>>>((uint64_t)timeout_us * 1000ull);
    if ((s = check_launch("bounded_wait_selftest_kernel")) != WQ_OK) return s;
    return wq_device_status(stream, 1);
}

}  // extern "C"
