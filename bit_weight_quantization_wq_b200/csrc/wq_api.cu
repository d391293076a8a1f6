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
#include "error.cuh"
#include "dequant.cuh"
#include "smallm.cuh"
#include "gemm_tc.cuh"
#include "pd_search.h"

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

// ------------------------------------------------------------------ error table
// The jobs' outputs are zeroed, then quant_error_many_kernel runs over up to kErrMaxSegs
// tensors per launch.
wq_status launch_error_many(const wq_error_job *jobs, int n_jobs, int sm_count, cudaStream_t st) {
    wq::ErrSegments segs;
    int i = 0;
    while (i < n_jobs) {
        segs.n = 0;
        segs.vbegin[0] = 0;
        for (; i < n_jobs && segs.n < wq::kErrMaxSegs; ++i) {
            const wq_error_job &j = jobs[i];
            const int k = segs.n++;
            const int64_t n_groups = j.N * (j.K / 128);
            segs.n_groups[k] = n_groups;
            segs.W[k] = static_cast<const uint16_t *>(j.W);
            segs.out[k] = j.out;
            segs.vbegin[k + 1] = segs.vbegin[k] + (n_groups + 7) / 8 * 8;
        }
        wq::zero_error_outputs_kernel<<<1, wq::kErrMaxSegs * wq::kErrOut, 0, st>>>(segs);
        wq_status s = check_launch("zero_error_outputs_kernel");
        if (s != WQ_OK) return s;
        const int64_t per_block = 8 * (wq::kErrThreads / 32);
        const int64_t want = (segs.vbegin[segs.n] + per_block - 1) / per_block;
        if (want > 0) {
            const int grid = (int)std::min<int64_t>(want, (int64_t)sm_count * 12);
            wq::quant_error_many_kernel<<<grid, wq::kErrThreads, 0, st>>>(segs);
            if ((s = check_launch("quant_error_many_kernel")) != WQ_OK) return s;
        }
    }
    return WQ_OK;
}

// ------------------------------------------------------------------ small-M path
constexpr uint32_t kSmemMax = 227 * 1024;        // dynamic shared memory per CTA on sm_100

uint64_t align_u64(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

wq_status make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);

// Clusters of S CTAs that fit at once (one CTA per SM, the most shared memory), cached.
template <int BITS, int TOK>
int small_max_clusters(int dev, int S, int sm_count) {
    // computed once per device and cluster size; two threads racing here compute the same value
    static std::atomic<int> cache[kMaxDevices][4] = {};
    const int si = S == 1 ? 0 : (S == 2 ? 1 : (S == 4 ? 2 : 3));
    const int cached = cache[dev][si].load(std::memory_order_relaxed);
    if (cached != 0) return cached;
    int n = sm_count / S;
    if (S > 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(S * (sm_count / S)));
        cfg.blockDim = dim3(wq::SmCfg<TOK>::kThreads);
        cfg.dynamicSmemBytes = kSmemMax;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int q = 0;
        if (cudaOccupancyMaxActiveClusters(&q, (void *)wq::smallm_kernel<BITS, TOK, 1>, &cfg) != cudaSuccess) q = 0;
        cudaGetLastError();
        n = std::min(n, q);
    }
    const int v = n > 0 ? n : -1;
    cache[dev][si].store(v, std::memory_order_relaxed);
    return v;
}

// Work split and shared-memory layout of smallm_kernel for a cluster size S: C clusters own
// ~U/C units each, a CTA ~G/S groups. Inside the CTA, blocks of RB units go to the W warps
// (GW warps per block, each a share of the groups, when there are fewer blocks than warps);
// each warp streams its items through D ring slots. Returns the busiest warp's item count
// (scaled, with a small preference for deeper rings), or -1 when nothing fits.
//
// Layout: x [M][x_stride] | 256 zero bytes at 64 mod 128 | st [gc][rows_pad] | L2 [rank][rows_max] |
// mbarriers [W][D], staging mbarrier, abort word | rings [W][D][slot] | part [GW][TOK][rows_max].
template <int BITS, int TOK>
int64_t small_plan(int64_t U, int G, int S, int C, int M, wq::SmallMArgs &a, uint32_t *smem_total) {
    constexpr int W = wq::SmCfg<TOK>::kWarps;
    const int64_t uc = (U + C - 1) / C;
    const int gc = (G + S - 1) / S;
    // sizes in 64 bits: a layout is kept only when its total fits in shared memory
    const uint64_t x_stride = (uint64_t)gc * 256u + 64u;
    const uint64_t x_bytes = align_u64((uint64_t)M * x_stride, 128);
    const uint64_t off_zero = x_bytes + 64u;
    const uint64_t off_st = x_bytes + 384u;
    int64_t best = -1;
    // L2 columns of the cluster's rows are staged when its rows are 16-byte multiples and the
    // layout still fits; otherwise the finish reads them from global memory
    for (int l2_try = 1; l2_try >= 0 && best < 0; --l2_try) {
        const bool l2_staged = l2_try == 1 && a.rank > 0 && a.N % 8 == 0;
        if (l2_try == 1 && !l2_staged) continue;
        const uint64_t l2_bytes = l2_staged ? align_u64((uint64_t)a.rank * (uint64_t)(uc * 16) * 2u, 128) : 0u;
        for (int rb = wq::sm_max_rb<TOK>(); rb >= 1; --rb) {
            const int64_t nb = (uc + rb - 1) / rb;
            const int gw = nb >= W ? 1 : (int)(W / nb);
            // items (one group of one block) on the busiest warp; an item costs about one unit's
            // work on top of its units' (the x fragment, the correction MMAs, the wait and copy)
            const int64_t items = nb >= W ? ((nb + W - 1) / W) * gc : (gc + gw - 1) / gw;
            const int64_t rows_pad = uc * 16 + 16 * (rb - 1);
            const uint64_t st_bytes = align_u64((uint64_t)rows_pad * (uint64_t)gc * 4u, 128);
            const uint64_t off_l2 = off_st + st_bytes;
            const uint64_t off_bar = off_l2 + l2_bytes;
            const uint64_t part = align_u64((uint64_t)gw * TOK * (uint64_t)(uc * 16) * 4u, 128);
            const uint64_t slot = (uint64_t)rb * 16u * 16u * BITS;
            for (int d = wq::kSmMaxD; d >= 2; --d) {
                const uint64_t off_ring = off_bar + align_u64((uint64_t)W * d * 8u + 16u, 128);   // + staging bar, abort
                const uint64_t total = off_ring + (uint64_t)W * d * slot + part;
                if (total > kSmemMax) continue;
                // the least work on the busiest warp first; then a deeper ring
                const int64_t cost = items * (1 + rb) * 8 + (d >= 4 ? 0 : 4 - d);
                if (best < 0 || cost < best) {
                    best = cost;
                    a.RB = rb;
                    a.GW = gw;
                    a.D = d;
                    a.rows_max = (int)(uc * 16);
                    a.rows_pad = (int)rows_pad;
                    a.gmax = gc;
                    a.x_stride = (uint32_t)x_stride;
                    a.slot_bytes = (uint32_t)slot;
                    a.off_zero = (uint32_t)off_zero;
                    a.off_st = (uint32_t)off_st;
                    a.off_l2 = (uint32_t)off_l2;
                    a.off_bar = (uint32_t)off_bar;
                    a.off_ring = (uint32_t)off_ring;
                    a.off_part = (uint32_t)(off_ring + (uint64_t)W * d * slot);
                    a.l2_staged = l2_staged ? 1 : 0;
                    *smem_total = (uint32_t)total;
                }
                break;
            }
        }
    }
    return best;
}

template <int BITS, int TOK, int RB>
cudaError_t smallm_launch_rb(const cudaLaunchConfig_t &cfg, const CUtensorMap &pm, const wq::SmallMArgs &a) {
    return cudaLaunchKernelEx(&cfg, wq::smallm_kernel<BITS, TOK, RB>, pm, a);
}

// *no_layout is set (and nothing launched) when no cluster size has a shared-memory layout
// for this many tokens.
template <int BITS, int TOK>
wq_status launch_smallm_tok(wq::SmallMArgs a, const CUtensorMap &pm, int dev, int sm_count, cudaStream_t st,
                            bool *no_layout) {
    *no_layout = false;
    static std::atomic<int> attr_done[kMaxDevices] = {};
    cudaError_t e = setup_once(attr_done, dev, [] {
        cudaError_t r = cudaSuccess;
        const void *fs[4] = {(const void *)wq::smallm_kernel<BITS, TOK, 1>, (const void *)wq::smallm_kernel<BITS, TOK, 2>,
                             (const void *)wq::smallm_kernel<BITS, TOK, 3>,
                             (const void *)wq::smallm_kernel<BITS, TOK, wq::sm_max_rb<TOK>()>};
        for (const void *f : fs)
            if (r == cudaSuccess) r = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax);
        return r;
    });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(smallm)");
    const int64_t U = (a.N + 15) / 16;
    const int G = (int)(a.K / 128);
    // cluster size S (K split) and cluster count C: the fewest items on the busiest warp;
    // ties go to the smaller S
    int64_t best = -1;
    wq::SmallMArgs chosen = a;
    uint32_t smem = 0;
    for (int S = 1; S <= 8; S *= 2) {
        if (S > G) break;
        const int mc = small_max_clusters<BITS, TOK>(dev, S, sm_count);
        if (mc <= 0) continue;
        const int C = (int)std::min<int64_t>(mc, U);
        wq::SmallMArgs t = a;
        uint32_t total = 0;
        const int64_t cost = small_plan<BITS, TOK>(U, G, S, C, (int)a.M, t, &total);
        if (cost < 0) continue;
        if (best < 0 || cost < best) {
            best = cost;
            t.S = S;
            t.n_clusters = C;
            chosen = t;
            smem = total;
        }
    }
    if (best < 0) {
        *no_layout = true;
        return fail(WQ_ERR_INVALID_ARG, "no shared-memory layout for the small-M kernel");
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(chosen.n_clusters * chosen.S));
    cfg.blockDim = dim3(wq::SmCfg<TOK>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n_attr = 0;
    if (chosen.S > 1) {
        attr[n_attr].id = cudaLaunchAttributeClusterDimension;
        attr[n_attr].val.clusterDim.x = (unsigned)chosen.S;
        attr[n_attr].val.clusterDim.y = 1;
        attr[n_attr].val.clusterDim.z = 1;
        ++n_attr;
    }
    if (chosen.rank > 0) {
        // t comes from the prepass launched just before: the kernel streams the weight while
        // the prepass runs and waits for it (griddepcontrol.wait) only before reading t
        attr[n_attr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n_attr].val.programmaticStreamSerializationAllowed = 1;
        ++n_attr;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n_attr;
    switch (chosen.RB) {
        case 1: e = smallm_launch_rb<BITS, TOK, 1>(cfg, pm, chosen); break;
        case 2: e = smallm_launch_rb<BITS, TOK, 2>(cfg, pm, chosen); break;
        case 3: e = smallm_launch_rb<BITS, TOK, 3>(cfg, pm, chosen); break;
        default: e = smallm_launch_rb<BITS, TOK, wq::sm_max_rb<TOK>()>(cfg, pm, chosen); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(smallm_kernel)");
    return check_launch("smallm_kernel");
}

// Up to 16 tokens per launch; more tokens take several launches. A shape whose staged x
// and partial sums do not fit in shared memory for 16 tokens is run in launches of 8, 4, 2
// or 1 tokens (each streams the weight once more). The packed codes are read by TMA as
// [N][K*b/8] bytes, one unit (16 rows x 16*b bytes of one group) per copy.
template <int BITS>
wq_status launch_smallm(const wq::SmallMArgs &base, const uint8_t *packed, int dev, int sm_count, cudaStream_t st) {
    CUtensorMap pm;
    const uint64_t row_bytes = (uint64_t)base.K * BITS / 8;
    wq_status s = make_map_2d(&pm, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, row_bytes, (uint64_t)base.N, row_bytes,
                              16u * BITS, 16u, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (s != WQ_OK) return s;
    int64_t chunk = wq::kSmMaxTok;
    for (int64_t m0 = 0; m0 < base.M;) {
        wq::SmallMArgs a = base;
        a.M = std::min<int64_t>(chunk, base.M - m0);
        a.x = base.x + m0 * base.K;
        a.y = base.y + m0 * base.N;
        if (base.t) a.t = base.t + m0 * wq::kTStrideSm;
        bool no_layout = false;
        if (a.M <= 8) s = launch_smallm_tok<BITS, 8>(a, pm, dev, sm_count, st, &no_layout);
        else s = launch_smallm_tok<BITS, 16>(a, pm, dev, sm_count, st, &no_layout);
        if (no_layout && a.M > 1) {
            chunk = (a.M + 1) / 2;                     // nothing was launched: retry with fewer tokens
            g_last_error[0] = 0;
            continue;
        }
        if (s != WQ_OK) return s;
        m0 += a.M;
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

template <int BITS, int TT>
wq_status launch_tc(const TcArgs &a, const CUtensorMap &xm, const CUtensorMap &tm, const CUtensorMap &lm,
                    const CUtensorMap &pm, int l_tma, int sm_count, cudaStream_t st) {
    using L = wq::TcLayout<TT>;
    static std::atomic<int> attr_done[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const cudaError_t e = setup_once(attr_done, dev, [] {
        // The warpgroups re-split their registers with setmaxnreg, a split that adds up to
        // exactly 128 registers per thread at launch: a kernel built with any other count
        // would wait forever in setmaxnreg.inc, so it is never launched.
        cudaFuncAttributes fa;
        cudaError_t r = cudaFuncGetAttributes(&fa, wq::tc_linear_kernel<BITS, TT>);
        if (r != cudaSuccess) return r;
        if (fa.numRegs != wq::kTcRegsLaunch || fa.maxThreadsPerBlock < wq::kTcThreads) return cudaErrorInvalidKernelImage;
        return cudaFuncSetAttribute(wq::tc_linear_kernel<BITS, TT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)L::kAlloc);
    });
    if (e != cudaSuccess) return cuda_fail(e, "tc_linear_kernel set-up (register count / shared memory)");
    wq::TcParams p{};
    p.packed = a.packed;
    p.scales = a.scales;
    p.L2 = static_cast<const uint16_t *>(a.L2);
    p.bias = static_cast<const uint16_t *>(a.bias);
    p.y = static_cast<uint16_t *>(a.y);
    p.M = a.M; p.N = a.N; p.K = a.K; p.rank = a.rank;
    p.row_bytes = a.K * BITS / 8;
    p.tiles_m = (int)((a.M + TT - 1) / TT);
    p.tiles_n = (int)((a.N + wq::kTcBW - 1) / wq::kTcBW);
    p.l_tma = l_tma;
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = std::min(tiles, sm_count);
    wq::tc_linear_kernel<BITS, TT><<<grid, wq::kTcThreads, L::kAlloc, st>>>(xm, tm, lm, pm, p);
    return check_launch("tc_linear_kernel");
}

template <int BITS>
wq_status launch_tc_tt(const TcArgs &a, int tt, const CUtensorMap &xm, const CUtensorMap &tm, const CUtensorMap &lm,
                       const CUtensorMap &pm, int l_tma, int sm_count, cudaStream_t st) {
    if (tt == 256) return launch_tc<BITS, 256>(a, xm, tm, lm, pm, l_tma, sm_count, st);
    if (tt == 240) return launch_tc<BITS, 240>(a, xm, tm, lm, pm, l_tma, sm_count, st);
    return launch_tc<BITS, 128>(a, xm, tm, lm, pm, l_tma, sm_count, st);
}

template <int R>
wq_status launch_prepass(const TcArgs &a, uint16_t *t, int sm_count, cudaStream_t st) {
    using PL = wq::PreLayout<R>;
    const int64_t mtiles = (a.M + 63) / 64;
    const int64_t nkb = a.K / 64;
    // K is split over a cluster of up to 16 CTAs (a non-portable size) while the doubled split
    // still leaves at most two CTAs per SM (longer CTAs amortize the ring's start and the
    // cluster reduction)
    int ks = 1;
    while (ks < wq::kPreMaxKS && ks * 2 <= nkb && mtiles * ks * 2 <= 2 * (int64_t)sm_count) ks *= 2;
    static std::atomic<int> attr_done[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t e = setup_once(attr_done, dev, [] {
        cudaError_t r = cudaFuncSetAttribute(wq::lowrank_prepass_kernel<R>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (r != cudaSuccess) return r;
        return cudaFuncSetAttribute(wq::lowrank_prepass_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)PL::kAlloc);
    });
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(lowrank_prepass_kernel)");
    // x as 64-token x 64-k tiles (128-byte swizzle), L1 as 64-k x R tiles
    CUtensorMap xm, lm;
    wq_status s = make_map_2d(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)a.K, (uint64_t)a.M,
                              (uint64_t)a.K * 2, 64u, 64u, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != WQ_OK) return s;
    if ((s = make_map_2d(&lm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L1, (uint64_t)R, (uint64_t)a.K, (uint64_t)R * 2,
                         (uint32_t)R, 64u, CU_TENSOR_MAP_SWIZZLE_NONE)) != WQ_OK)
        return s;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)mtiles, (unsigned)ks, 1);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = PL::kAlloc;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)ks;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, wq::lowrank_prepass_kernel<R>, xm, lm, t, a.M, a.K);
    if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(lowrank_prepass_kernel)");
    return check_launch("lowrank_prepass_kernel");
}

// Tokens per tensor-core tile: 256 or 240 (one MMA covers 128 weight rows x that many tokens,
// long enough to hide the per-group hand-off of the partial products), whichever needs fewer
// tile-waves x tokens on this many SMs (a last wave left mostly empty costs a whole wave); 128
// when there are few tokens.
int tc_tile_tokens(int64_t M, int64_t N, int sm_count) {
    if (M <= 128) return 128;
    const int64_t tiles_n = (N + wq::kTcBW - 1) / wq::kTcBW;
    int best = 256;
    int64_t best_cost = -1;
    for (int tt : {256, 240}) {
        const int64_t tiles = (M + tt - 1) / tt * tiles_n;
        const int64_t waves = (tiles + sm_count - 1) / sm_count;
        const int64_t cost = waves * tt;
        if (best_cost < 0 || cost < best_cost) { best = tt; best_cost = cost; }
    }
    return best;
}

wq_status tc_linear(const TcArgs &a, int sm_count, cudaStream_t st) {
    wq_status s = get_encoder();
    if (s != WQ_OK) return s;
    if (a.M > (int64_t)INT32_MAX || a.N > (int64_t)INT32_MAX || a.K > (int64_t)INT32_MAX)
        return fail(WQ_ERR_INVALID_ARG, "dimension above 2^31 on the tensor-core path");
    const int tt = tc_tile_tokens(a.M, a.N, sm_count);
    CUtensorMap xm, tm, lm;
    int l_tma = 0;
    if ((s = make_map_2d(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, (uint64_t)a.K, (uint64_t)a.M,
                         (uint64_t)a.K * 2, wq::kTcBK, (uint32_t)tt, CU_TENSOR_MAP_SWIZZLE_128B)) != WQ_OK)
        return s;
    // packed codes as [N][K*b/8] bytes: one group of 128 rows (16*b bytes each) per copy
    CUtensorMap pm;
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
                             (uint64_t)wq::kTStride * 2, wq::kTcBK, (uint32_t)tt, CU_TENSOR_MAP_SWIZZLE_128B)) != WQ_OK)
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
        case 3: return launch_tc_tt<3>(a, tt, xm, tm, lm, pm, l_tma, sm_count, st);
        case 4: return launch_tc_tt<4>(a, tt, xm, tm, lm, pm, l_tma, sm_count, st);
        case 5: return launch_tc_tt<5>(a, tt, xm, tm, lm, pm, l_tma, sm_count, st);
        case 6: return launch_tc_tt<6>(a, tt, xm, tm, lm, pm, l_tma, sm_count, st);
        default: return launch_tc_tt<7>(a, tt, xm, tm, lm, pm, l_tma, sm_count, st);
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

wq_status wq_dequantize(const uint8_t *packed, const float *scales, int64_t N, int64_t K, int bits, int group,
                        void *W_hat, wq_stream_t stream) {
    g_last_error[0] = 0;
    if (bits < 3 || bits > 7) return fail(WQ_ERR_UNSUPPORTED_BITS, "bits=%d", bits);
    if (group != 128) return fail(WQ_ERR_UNSUPPORTED_GROUP, "group=%d", group);
    if (N < 0 || K < 0) return fail(WQ_ERR_INVALID_ARG, "negative size N=%lld K=%lld", (long long)N, (long long)K);
    if (K % 128 != 0) return fail(WQ_ERR_INVALID_ARG, "K=%lld is not a multiple of 128", (long long)K);
    if (N == 0 || K == 0) return WQ_OK;
    if (!packed || !scales || !W_hat) return fail(WQ_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(packed) || !aligned16(scales) || !aligned16(W_hat))
        return fail(WQ_ERR_MISALIGNED, "packed/scales/W_hat must be 16-byte aligned");
    int dev;
    const DeviceInfo *info;
    wq_status s = current_device(&dev, &info);
    if (s != WQ_OK) return s;
    const int64_t n_groups = N * (K / 128);
    const int64_t per_block = 8 * (wq::kDeqThreads / 32);
    const int grid = (int)std::min<int64_t>((n_groups + per_block - 1) / per_block, (int64_t)info->sm_count * 8);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint16_t *out = static_cast<uint16_t *>(W_hat);
    switch (bits) {
        case 3: wq::dequantize_kernel<3><<<grid, wq::kDeqThreads, 0, st>>>(packed, scales, n_groups, out); break;
        case 4: wq::dequantize_kernel<4><<<grid, wq::kDeqThreads, 0, st>>>(packed, scales, n_groups, out); break;
        case 5: wq::dequantize_kernel<5><<<grid, wq::kDeqThreads, 0, st>>>(packed, scales, n_groups, out); break;
        case 6: wq::dequantize_kernel<6><<<grid, wq::kDeqThreads, 0, st>>>(packed, scales, n_groups, out); break;
        default: wq::dequantize_kernel<7><<<grid, wq::kDeqThreads, 0, st>>>(packed, scales, n_groups, out); break;
    }
    return check_launch("dequantize_kernel");
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

wq_status wq_quant_error_many(const wq_error_job *jobs, int n_jobs, int group, wq_stream_t stream) {
    g_last_error[0] = 0;
    if (group != 128) return fail(WQ_ERR_UNSUPPORTED_GROUP, "group=%d", group);
    if (n_jobs < 0) return fail(WQ_ERR_INVALID_ARG, "n_jobs=%d", n_jobs);
    if (n_jobs == 0) return WQ_OK;
    if (!jobs) return fail(WQ_ERR_INVALID_ARG, "NULL job array");
    for (int i = 0; i < n_jobs; ++i) {
        const wq_error_job &j = jobs[i];
        if (j.N < 0 || j.K < 0)
            return fail(WQ_ERR_INVALID_ARG, "job %d: negative size N=%lld K=%lld", i, (long long)j.N, (long long)j.K);
        if (j.K % 128 != 0) return fail(WQ_ERR_INVALID_ARG, "job %d: K=%lld is not a multiple of 128", i, (long long)j.K);
        if (!j.out || (j.N > 0 && j.K > 0 && !j.W)) return fail(WQ_ERR_INVALID_ARG, "job %d: NULL pointer", i);
        if ((reinterpret_cast<uintptr_t>(j.out) & 7u) != 0 || (j.W && !aligned16(j.W)))
            return fail(WQ_ERR_MISALIGNED, "job %d: W must be 16-byte and out 8-byte aligned", i);
    }
    int dev;
    const DeviceInfo *info;
    wq_status s = current_device(&dev, &info);
    if (s != WQ_OK) return s;
    return launch_error_many(jobs, n_jobs, info->sm_count, reinterpret_cast<cudaStream_t>(stream));
}

wq_status wq_quant_error(const void *W, int64_t N, int64_t K, int group, double *out, wq_stream_t stream) {
    const wq_error_job job{W, N, K, out};
    return wq_quant_error_many(&job, 1, group, stream);
}

wq_status wq_pd_search(const double *mse_table, const int64_t *n_params, int n_tensors, const int *bits, int n_bits,
                       double target_bpw, int n_iters, int n_restarts, const double *t_init, int *bits_out,
                       double *result) {
    g_last_error[0] = 0;
    if (n_tensors <= 0 || n_bits <= 0 || n_iters < 0 || n_restarts <= 0)
        return fail(WQ_ERR_INVALID_ARG, "n_tensors=%d n_bits=%d n_iters=%d n_restarts=%d", n_tensors, n_bits, n_iters,
                    n_restarts);
    if (!mse_table || !n_params || !bits || !t_init || !bits_out || !result)
        return fail(WQ_ERR_INVALID_ARG, "NULL pointer");
    for (int j = 0; j < n_bits; ++j)
        if (bits[j] < 1 || bits[j] > 16 || (j > 0 && bits[j] <= bits[j - 1]))
            return fail(WQ_ERR_INVALID_ARG, "candidate widths must be strictly increasing in 1..16");
    for (int i = 0; i < n_tensors; ++i)
        if (n_params[i] <= 0) return fail(WQ_ERR_INVALID_ARG, "tensor %d: n_params=%lld", i, (long long)n_params[i]);
    for (int64_t k = 0; k < (int64_t)n_tensors * n_bits; ++k)
        if (!(mse_table[k] >= 0.0) || std::isinf(mse_table[k]))
            return fail(WQ_ERR_INVALID_ARG, "mse_table[%lld] is not a finite non-negative number", (long long)k);
    if (!(target_bpw >= bits[0] && target_bpw <= bits[n_bits - 1]))
        return fail(WQ_ERR_INVALID_ARG, "target_bpw=%g outside the candidate widths", target_bpw);
    const wq::PdResult r = wq::pd_search_host(mse_table, n_params, n_tensors, bits, n_bits, target_bpw, n_iters,
                                              n_restarts, t_init, bits_out);
    result[0] = r.total_mse;
    result[1] = r.bpw;
    result[2] = (double)r.restart;
    return WQ_OK;
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
