// smallm.cuh -- small-M quantized linear (KS): streams the packed weight at HBM rate.
//
// y = x * dequant(W)^T (+ (x L1) L2) (+ bias) for up to 16 tokens per launch. The Per-group(128) article
// dequantizes a block's weights on the GPU (sec. 3.4) and then runs a bf16 matmul (sec.
// 5.3/5.4); for a handful of tokens that matmul only streams the weight, so this kernel
// never materializes dequant(W): it reads the packed codes once, straight into shared
// memory, and contracts them there.
//
// Work: the weight is cut into 16-row units (the M side of mma.m16n8k16) and 128-wide
// groups. A thread-block cluster of S CTAs (S = 1, 2 or 4) owns a contiguous range of row
// units, balanced to +-1 unit over the clusters of one wave (one CTA per SM); its CTAs
// split the K groups. Within a CTA the (row unit, group) items of each chunk are dealt to
// 11 consumer warps in group-major order, so a warp loads the x fragment of a group once and
// reuses it for every row unit it owns in that group, and every warp works on every chunk.
//
// Data movement: one producer warp streams chunks (gc groups of all the CTA's rows) into a
// ring of shared-memory stages with TMA tensor copies. The weight is read as a 2-D array of
// 32-bit words, one box {gc groups, 64, 32 or 16 rows} per copy, so that copies move
// kilobytes: a per-request cost makes copies of a few kilobytes stream at a third of HBM
// bandwidth, while 16 KB and larger ones reach ~5.6 TB/s. gc divides the CTA's K range when
// the split allows; otherwise the last chunk of a range uses one-group boxes. x arrives as
// one box {128 k, gc groups, all tokens} per chunk. The per-group steps of a pass arrive once
// by TMA (row stride a multiple of 16 bytes) or, failing that, by 4-byte asynchronous copies
// per chunk. Completion is tracked by the stage's mbarrier (transaction bytes plus one
// arrival per producer lane); consumers release a stage with one arrival per warp after every lane's
// proxy fence (their reads are generic-proxy, the next copy is async-proxy).
//
// Arithmetic: thread (g, c) of a warp holds rows g and g+8 of the unit and the 32
// consecutive codes [32c, 32c+32) of the group, 4*b contiguous bytes per row. Inside one
// MMA step s the k slots it feeds are mapped to k = 32c + 4s + {0,1} and 32c + 4s + {2,3}
// (the same map on the x side), so both operands are read in natural order. Codes enter
// the MMAs as the exact bf16 values 128 + code (bit pattern 0x4300 | code); the group's
// (128 + 2^(b-1)) * sum(x) is formed by eight more MMAs with a constant A operand and
// subtracted once per item, which leaves sum_k q x exactly as before rounding. Each
// group's fp32 product is scaled by the group's fp32 step and accumulated in fp32: the
// weight is never rounded.
//
// Reduction: the consumer warps' partial sums meet in a fixed tree through shared memory, then the
// S CTAs of a cluster add theirs through distributed shared memory (in rank order), add the
// low-rank branch and the bias, and round once to bf16. All orders are fixed: the result is
// deterministic. Every wait is bounded; a timeout raises the CTA's abort flag, which makes
// the remaining waits return at once, and every thread still reaches the same barriers.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "unpack.cuh"

namespace wq {

constexpr int kSmConsumerWarps = 11;  // + producer = 12 warps: 3 per SM sub-partition
constexpr int kSmThreads = (kSmConsumerWarps + 1) * 32;     // + one producer warp
constexpr int kSmMaxStages = 8;
constexpr int kSmMaxTok = 16;                                // tokens per launch
constexpr int kTStrideSm = 128;                              // row stride of [t_hi | t_lo]

template <int TOK> struct SmTok {
    static constexpr int kTiles = TOK / 8;                   // n8 token tiles per MMA step
    // row units per pass: each is a register block and one unrolled copy of the item code;
    // 6 measured faster than 12 (smaller code) even where it needs a second pass
    static constexpr int kRP = TOK <= 8 ? 6 : (TOK <= 16 ? 6 : 3);
    static constexpr int kNR = kRP * kTiles * 4;             // fp32 partials per thread
    static constexpr int kPStride = kRP * 16 + 1;            // part[] row stride (floats)
    static constexpr int kChains = TOK <= 16 ? 4 : 2;       // independent MMA accumulators per item
};

struct SmallMArgs {
    const uint16_t *x;        // M x K bf16 (read through the x tensor maps)
    const float *scales;      // N x K/128
    const uint16_t *bias;     // N or null
    const uint16_t *t;        // M x 128 bf16: [t_hi | t_lo] of x L1 (rank columns each), or null
    const uint16_t *L2;       // rank x N bf16 or null
    uint16_t *y;              // M x N bf16
    int64_t M, N, K;
    int rank;
    int S;                    // CTAs per cluster (K split)
    int n_clusters;
    int gc;                   // groups per chunk
    int stages;               // ring depth
    int srows;                // weight rows per stage (= scale rows)
    uint32_t stage_bytes;     // one ring stage: weight boxes | x box | steps
    uint32_t off_x, off_s;    // offsets inside a stage
    uint32_t off_tree, off_part, off_bar;   // dynamic shared memory layout
    int scale_tma;            // 1: a pass's steps arrive once, by TMA, into [rows][sbox] at off_sres
    int sbox;                 // groups per row in that region (a multiple of 4)
    uint32_t off_sres;
};

// ---------------------------------------------------------------- async copies
__device__ __forceinline__ void cp_async_4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// Arrive on the barrier once all of this thread's earlier cp.async copies have landed
// (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t remote_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ void consumer_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(kSmConsumerWarps * 32) : "memory");
}

// Bounded warp-wide wait on a barrier whose phase is published at cluster scope.
__device__ __forceinline__ bool warp_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort) {
    const int lane = threadIdx.x & 31;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const bool ok = mbar_try_wait_cluster(bar, parity);
        if (__all_sync(0xffffffffu, ok)) return true;
        if ((it & 63u) == 63u) {
            int stop = 0;
            if (lane == 0) {
                const uint64_t now = globaltimer_ns();
                if (t0 == 0) t0 = now;
                if (*abort) {
                    stop = 1;
                } else if (now - t0 > kWaitLimitNs) {
                    record_status(WQ_ERR_TIMEOUT);
                    *abort = 1;
                    stop = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) return false;
        }
    }
}

// 4*b bytes of packed codes (one thread's 32-code slice) from shared memory, plus a zero word.
template <int BITS>
__device__ __forceinline__ void lds_slice(const uint8_t *p, uint32_t (&w)[BITS + 1]) {
    if constexpr (BITS == 4) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BITS == 6) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const uint2 v = *reinterpret_cast<const uint2 *>(p + 8 * i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = *reinterpret_cast<const uint32_t *>(p + 4 * i);
    }
    w[BITS] = 0;
}

template <int BITS, int TOK>
__global__ void __launch_bounds__(kSmThreads, 1)
smallm_kernel(const __grid_constant__ CUtensorMap pm64, const __grid_constant__ CUtensorMap pm32,
              const __grid_constant__ CUtensorMap pm16, const __grid_constant__ CUtensorMap pm_tail,
              const __grid_constant__ CUtensorMap xm_full, const __grid_constant__ CUtensorMap xm_tail,
              const __grid_constant__ CUtensorMap sm_map, const SmallMArgs a) {
    constexpr int NT = SmTok<TOK>::kTiles;
    constexpr int RP = SmTok<TOK>::kRP;
    constexpr int NR = SmTok<TOK>::kNR;
    constexpr int PS = SmTok<TOK>::kPStride;
    constexpr int CH = SmTok<TOK>::kChains;
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = a.S;
    const uint32_t srank = (S > 1) ? cluster_ctarank() : 0u;
    const int cid = blockIdx.x / S;
    const int64_t U = (a.N + 15) / 16;
    const int64_t u0 = U * cid / a.n_clusters, u1 = U * (cid + 1) / a.n_clusters;
    const int Rc = (int)(u1 - u0);
    const int G = (int)(a.K / 128);
    const int g0 = (int)((int64_t)G * srank / S), g1 = (int)((int64_t)G * (srank + 1) / S);
    const int Gcta = g1 - g0;
    const int npass = (Rc + RP - 1) / RP;
    const int nch = (Gcta + a.gc - 1) / a.gc;
    constexpr uint32_t kGB = 16 * BITS;                        // bytes of one group of one row
    // bf16x2 (128 + 2^(b-1)) in both halves: the bias the unpacked codes carry
    constexpr uint32_t kBias2 = (uint32_t)(0x4300 + (1 << (BITS - 1))) * 0x10001u;

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + a.off_bar);
    uint64_t *empty = full + a.stages;
    uint64_t *pready = empty + a.stages, *pdone = pready + 1;
    uint64_t *sfull = pdone + 1, *sempty = sfull + 1;
    volatile int *abort = reinterpret_cast<volatile int *>(sempty + 1);
    const float *sres = reinterpret_cast<const float *>(smem + a.off_sres);
    const int g0s = g0 & ~3;                                   // first group of the resident step box
    float *tree = reinterpret_cast<float *>(smem + a.off_tree);
    float *part = reinterpret_cast<float *>(smem + a.off_part);

    if (warp == kSmConsumerWarps && lane == 0) {
        // descriptor fetches overlap the barrier set-up instead of stalling the first copies
        tma_prefetch_desc(&pm64);
        tma_prefetch_desc(&pm32);
        tma_prefetch_desc(&pm16);
        tma_prefetch_desc(&xm_full);
        if (a.scale_tma) tma_prefetch_desc(&sm_map);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&full[s], a.scale_tma ? 1 : 1 + 32);
            mbar_init(&empty[s], kSmConsumerWarps);
        }
        mbar_init(pready, 32 * S);
        mbar_init(pdone, 32 * S);
        mbar_init(sfull, 1);
        mbar_init(sempty, kSmConsumerWarps);
        *abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (S > 1) cluster_sync();       // every CTA's barriers exist before any remote arrival

    if (warp == kSmConsumerWarps) {
        // ------------------------------------------------------------ producer
        int armed[kSmMaxStages];
        for (int s = 0; s < kSmMaxStages; ++s) armed[s] = -1;
        uint32_t it = 0;
        int s_armed = -1;
        for (int p = 0; p < npass; ++p) {
            const int r0 = Rc * p / npass, r1 = Rc * (p + 1) / npass;
            const int Rp = r1 - r0;
            const int64_t n_base = (u0 + r0) * 16;
            const int rows_v = (int)min((int64_t)Rp * 16, (int64_t)(a.N - n_base));
            for (int j = 0; j < nch; ++j, ++it) {
                const int s = (int)(it % (uint32_t)a.stages);
                const uint32_t ph = (it / (uint32_t)a.stages) & 1u;
                const int gb = g0 + j * a.gc, gcnt = min(a.gc, g1 - gb);
                if (!warp_wait(&empty[s], ph ^ 1u, abort)) goto prod_done;
                uint8_t *st = smem + (size_t)s * a.stage_bytes;
                const bool tail = gcnt < a.gc;
                const uint32_t unit_bytes = 16u * (uint32_t)a.gc * kGB;    // one row unit's region
                armed[s] = (int)ph;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[s], (uint32_t)Rp * 16u * (uint32_t)gcnt * kGB +
                                                        (uint32_t)TOK * (uint32_t)gcnt * 256u);
                    if (!tail) {
                        tma_load_3d(st + a.off_x, &xm_full, &full[s], 0, gb, 0);
                        // row units in boxes of 4, 2 and 1 (64, 32, 16 rows of gc groups)
                        int r = 0;
                        for (; r + 4 <= Rp; r += 4)
                            tma_load_2d(st + (size_t)r * unit_bytes, &pm64, &full[s], gb * 4 * BITS, (int32_t)(n_base + 16 * r));
                        if (r + 2 <= Rp) {
                            tma_load_2d(st + (size_t)r * unit_bytes, &pm32, &full[s], gb * 4 * BITS, (int32_t)(n_base + 16 * r));
                            r += 2;
                        }
                        if (r < Rp)
                            tma_load_2d(st + (size_t)r * unit_bytes, &pm16, &full[s], gb * 4 * BITS, (int32_t)(n_base + 16 * r));
                    } else {
                        for (int q = 0; q < gcnt; ++q) {
                            tma_load_3d(st + a.off_x + (uint32_t)q * TOK * 256u, &xm_tail, &full[s], 0, gb + q, 0);
                            for (int r = 0; r < Rp; ++r)
                                tma_load_3d(st + (size_t)r * unit_bytes + (uint32_t)q * 16u * kGB, &pm_tail, &full[s], 0,
                                            gb + q, (int32_t)(n_base + 16 * r));
                        }
                    }
                }
                __syncwarp();
                if (!a.scale_tma) {
                    float *sc = reinterpret_cast<float *>(st + a.off_s);
                    for (int e = lane; e < rows_v * gcnt; e += 32) {
                        const int i = e / gcnt, gl = e - i * gcnt;     // consecutive lanes: one row's groups
                        cp_async_4(sc + gl * a.srows + i, a.scales + (n_base + i) * G + gb + gl);
                    }
                }
                if (!a.scale_tma) cp_async_arrive_noinc(&full[s]);
                if (j == 0 && a.scale_tma) {
                    // the pass's steps (after its first chunk): one box {sbox groups, 16 rows} per
                    // row unit, resident for the whole pass
                    if (p > 0 && !warp_wait(sempty, (uint32_t)(p - 1) & 1u, abort)) goto prod_done;
                    if (lane == 0) mbar_arrive_expect_tx(sfull, (uint32_t)Rp * 16u * (uint32_t)a.sbox * 4u);
                    s_armed = p & 1;
                    __syncwarp();
                    for (int r = lane; r < Rp; r += 32)
                        tma_load_2d(smem + a.off_sres + (size_t)r * 16 * a.sbox * 4, &sm_map, sfull, g0s,
                                    (int32_t)(n_base + 16 * r));
                }
            }
        }
    prod_done:
        if (*abort) {
            // wait (bounded) for the copies still in flight before the CTA can exit
            for (int s = 0; s < a.stages && s < kSmMaxStages; ++s) {
                int local = 0;
                if (armed[s] >= 0) (void)mbar_wait(&full[s], (uint32_t)armed[s], &local, 50ull * 1000ull * 1000ull);
            }
            int local = 0;
            if (s_armed >= 0) (void)mbar_wait(sfull, (uint32_t)s_armed, &local, 50ull * 1000ull * 1000ull);
        }
    } else {
        // ------------------------------------------------------------ consumers
        const int g = lane >> 2, c = lane & 3;
        uint32_t it = 0;
        for (int p = 0; p < npass; ++p) {
            const int r0 = Rc * p / npass, r1 = Rc * (p + 1) / npass;
            const int Rp = r1 - r0;
            const int64_t n_base = (u0 + r0) * 16;
            const int rows_v = (int)min((int64_t)Rp * 16, (int64_t)(a.N - n_base));
            float R[RP][NT][4];
#pragma unroll
            for (int r = 0; r < RP; ++r)
#pragma unroll
                for (int t = 0; t < NT; ++t) R[r][t][0] = R[r][t][1] = R[r][t][2] = R[r][t][3] = 0.0f;

            const bool s_ok = !a.scale_tma || warp_wait(sfull, (uint32_t)p & 1u, abort);
            for (int j = 0; j < nch; ++j, ++it) {
                const int s = (int)(it % (uint32_t)a.stages);
                const uint32_t ph = (it / (uint32_t)a.stages) & 1u;
                const bool ok = warp_wait(&full[s], ph, abort) && s_ok;
                const uint8_t *st = smem + (size_t)s * a.stage_bytes;
                const int gcnt = min(a.gc, Gcta - j * a.gc);
                const bool tail = gcnt < a.gc;
                // box layouts: full chunk [16 rows][gc][16b] per row unit and [TOK][gc][128] for x;
                // tail chunk one box per group: [16 rows][16b] and [TOK][128]
                const uint32_t unit_bytes = 16u * (uint32_t)a.gc * kGB;
                const uint32_t w_row = tail ? kGB : (uint32_t)a.gc * kGB, w_grp = tail ? 16u * kGB : kGB;
                const uint32_t x_tok = tail ? 256u : (uint32_t)a.gc * 256u, x_grp = tail ? (uint32_t)TOK * 256u : 256u;
                // this chunk's (group, row unit) items, group-major, dealt to the warps in
                // contiguous shares: every warp works on every chunk as it lands
                const int I = Rp * gcnt;
                const int i0 = I * warp / kSmConsumerWarps, i1 = I * (warp + 1) / kSmConsumerWarps;
                for (int gl = 0; ok && gl < gcnt; ++gl) {
                    const int gg = j * a.gc + gl;
                    const int ia = max(i0, gl * Rp), ib = min(i1, (gl + 1) * Rp);
                    if (ia >= ib) continue;
                    const int ra = ia - gl * Rp, rb = ib - gl * Rp;
                    // x fragment of the group: token 8t + g, words [16c, 16c + 16) of its 64
                    uint32_t X[NT][16];
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const uint4 *xp = reinterpret_cast<const uint4 *>(st + a.off_x + (uint32_t)(8 * t + g) * x_tok +
                                                                          (uint32_t)gl * x_grp + c * 64);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 v = xp[q];
                            X[t][4 * q] = v.x; X[t][4 * q + 1] = v.y; X[t][4 * q + 2] = v.z; X[t][4 * q + 3] = v.w;
                        }
                    }
                    // steps of row (16 r + row) for this group: resident [row][sbox] or per-chunk [gl][row]
                    // (128 + 2^(b-1)) * sum_k x[token][k] over the group, for every token column of
                    // the D fragment: the same MMA steps with a constant A operand
                    float corr[NT][4];
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        corr[t][0] = corr[t][1] = corr[t][2] = corr[t][3] = 0.0f;
#pragma unroll
                        for (int s8 = 0; s8 < 8; ++s8)
                            mma_16816_bf16(corr[t], kBias2, kBias2, kBias2, kBias2, X[t][2 * s8], X[t][2 * s8 + 1]);
                    }
                    const float *scs = a.scale_tma ? sres + (gg + g0 - g0s) : reinterpret_cast<const float *>(st + a.off_s) + gl * a.srows;
                    const int sst = a.scale_tma ? a.sbox : 1;
                    const uint8_t *wbase = st + (uint32_t)gl * w_grp + c * 4 * BITS;
#pragma unroll
                    for (int r = 0; r < RP; ++r) {
                        if (r < ra || r >= rb) continue;
                        uint32_t wa[BITS + 1], wb[BITS + 1];
                        lds_slice<BITS>(wbase + (uint32_t)r * unit_bytes + (uint32_t)g * w_row, wa);
                        lds_slice<BITS>(wbase + (uint32_t)r * unit_bytes + (uint32_t)(g + 8) * w_row, wb);
                        uint32_t Pa[16], Pb[16];
                        unpack_pairs_biased<BITS, 0, 4>(wa, Pa);
                        unpack_pairs_biased<BITS, 0, 4>(wb, Pb);
                        float acc[NT][CH][4];
#pragma unroll
                        for (int t = 0; t < NT; ++t)
#pragma unroll
                            for (int h = 0; h < CH; ++h) acc[t][h][0] = acc[t][h][1] = acc[t][h][2] = acc[t][h][3] = 0.0f;
#pragma unroll
                        for (int s8 = 0; s8 < 8; ++s8)
#pragma unroll
                            for (int t = 0; t < NT; ++t)
                                mma_16816_bf16(acc[t][s8 % CH], Pa[2 * s8], Pb[2 * s8], Pa[2 * s8 + 1], Pb[2 * s8 + 1],
                                               X[t][2 * s8], X[t][2 * s8 + 1]);
                        const float sa = scs[(r * 16 + g) * sst], sb = scs[(r * 16 + g + 8) * sst];
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                float sum = acc[t][0][k] - corr[t][k];
#pragma unroll
                                for (int h = 1; h < CH; ++h) sum += acc[t][h][k];
                                R[r][t][k] = fmaf(k < 2 ? sa : sb, sum, R[r][t][k]);
                            }
                        }
                    }
                }
                // release: every lane orders its reads (all consumed by now) before the next
                // async-proxy write; one arrival per warp keeps the barrier uncontended
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }

            // this thread's first output element of the pass: fetch its bias now, so the load
            // overlaps the reduction
            const int E = (int)a.M * rows_v;
            const int e0 = (int)((int64_t)E * srank / S), e1 = (int)((int64_t)E * (srank + 1) / S);
            float bias_first = 0.0f;
            if (a.bias && e0 + (int)threadIdx.x < e1) {
                const int ef = e0 + (int)threadIdx.x;
                bias_first = bf16_bits_to_f32(__ldg(a.bias + n_base + (ef - (ef / rows_v) * rows_v)));
            }
            if (a.scale_tma) {
                // this pass no longer reads the resident steps (generic reads before async writes)
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(sempty);
            }
            // -------------------------------------------------------- reduce the pass
            // 8 warps -> 1 through a fixed tree in shared memory
            float *Rf = &R[0][0][0];
            auto put = [&](int slot) {
#pragma unroll
                for (int i = 0; i < NR; ++i) tree[(slot * NR + i) * 32 + lane] = Rf[i];
            };
            auto add = [&](int slot) {
#pragma unroll
                for (int i = 0; i < NR; ++i) Rf[i] += tree[(slot * NR + i) * 32 + lane];
            };
            // warps [h, 2h) hand their sums to warps [0, h), h = 8, 4, 2, 1
#pragma unroll
            for (int h = 8; h >= 1; h /= 2) {
                if (warp >= h && warp < 2 * h) put(warp - h);
                consumer_bar();
                if (warp < h && warp + h < kSmConsumerWarps && h > 1) add(warp);
                if (h > 1) consumer_bar();
            }
            if (warp == 0) {
                add(0);
                // the CTAs of the cluster have finished reading part[] of the previous pass
                if (p > 0) (void)warp_wait_cluster(pdone, (uint32_t)(p - 1) & 1u, abort);
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    if (r >= Rp) continue;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const int tok = 8 * t + 2 * c, row = r * 16 + g;
                        part[tok * PS + row] = R[r][t][0];
                        part[(tok + 1) * PS + row] = R[r][t][1];
                        part[tok * PS + row + 8] = R[r][t][2];
                        part[(tok + 1) * PS + row + 8] = R[r][t][3];
                    }
                }
                __syncwarp();
                // publish: every lane arrives on the pready barrier of every CTA in the cluster
                if (S > 1) {
                    for (int q = 0; q < S; ++q) mbar_arrive_cluster(map_cluster_smem(smem_u32(pready), (uint32_t)q));
                } else {
                    mbar_arrive(pready);
                }
            }
            const bool ready = (S > 1) ? warp_wait_cluster(pready, (uint32_t)p & 1u, abort)
                                       : warp_wait(pready, (uint32_t)p & 1u, abort);
            // -------------------------------------------------------- finalize a 1/S share
            const uint32_t part_addr = smem_u32(part);
            for (int e = e0 + (int)threadIdx.x; ready && e < e1; e += kSmConsumerWarps * 32) {
                const int m = e / rows_v, i = e - m * rows_v;
                const uint32_t off = 4u * (uint32_t)(m * PS + i);
                float v = 0.0f;
                if (S > 1) {
                    for (int q = 0; q < S; ++q) v += ld_cluster_f32(map_cluster_smem(part_addr + off, (uint32_t)q));
                } else {
                    v = part[m * PS + i];
                }
                const int64_t n = n_base + i;
                if (a.rank > 0) {
                    const uint16_t *tm = a.t + (int64_t)m * kTStrideSm;
                    float lr = 0.0f;
                    for (int jr = 0; jr < a.rank; ++jr) {
                        const float tv = bf16_bits_to_f32(tm[jr]) + bf16_bits_to_f32(tm[a.rank + jr]);
                        lr = fmaf(tv, bf16_bits_to_f32(__ldg(a.L2 + (int64_t)jr * a.N + n)), lr);
                    }
                    v += lr;
                }
                if (a.bias) v += (e == e0 + (int)threadIdx.x) ? bias_first : bf16_bits_to_f32(__ldg(a.bias + n));
                a.y[(int64_t)m * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            }
            consumer_bar();
            if (warp == 0) {
                if (S > 1) {
                    for (int q = 0; q < S; ++q) mbar_arrive_cluster(map_cluster_smem(smem_u32(pdone), (uint32_t)q));
                } else {
                    mbar_arrive(pdone);
                }
            }
        }
    }
    __syncthreads();
    if (S > 1) cluster_sync();       // no CTA leaves while another may still read its part[]
}

}  // namespace wq
