// smallm.cuh -- small-M quantized linear (KS): streams the packed weight at HBM rate.
//
// y = x * dequant(W)^T (+ (x L1) L2) (+ bias) for up to 16 tokens per launch. The Per-group(128)
// article dequantizes a block's weights on the GPU (sec. 3.4) and then runs a bf16 matmul
// (sec. 5.3/5.4); for a handful of tokens that matmul only streams the weight, so this kernel
// never materializes dequant(W): it reads the packed codes once and contracts them on the
// fly.
//
// Work: the weight is cut into 16-row units (the M side of mma.m16n8k16) and 128-wide
// groups. A thread-block cluster of S CTAs (S = 1, 2, 4 or 8; one CTA per SM) owns a
// contiguous range of units, balanced to +-1 unit over the clusters; its CTAs split the K
// groups. Inside a CTA each warp owns blocks of RB units (RB fixed per launch) and a range
// of the CTA's groups (when there are fewer blocks than warps, several warps share a block,
// each with its own groups), and walks them one group at a time: the x fragment of a group
// is loaded once for all units of the block, and the units' MMA chains are independent, so
// they interleave.
//
// Data movement: every warp streams its own items (one group of one block) through a
// private ring of D slots in shared memory: the codes of item i are read into registers,
// then the slot is refilled with item i + D while item i is computed.
// Lane 0 of the warp fills a slot with one TMA tile copy per unit (16 rows x 16*b bytes,
// rows past N zero-filled) that completes on the slot's mbarrier; the warp waits on that
// barrier only. There is no producer warp and no barrier between warps until the final
// reduction. At the start the CTA copies into shared memory, once, with asynchronous copies
// issued ahead of the rings' first slots: the steps of its rows and groups and the token
// rows of x for its groups (each group's 16-byte chunks placed in the order the fragments
// are read in); they complete on a staging mbarrier that each warp waits on before its first
// item. With a low-rank branch the L2 columns of its rows follow, needed only at the finish.
//
// Arithmetic: thread (g, c) of a warp holds rows g and g+8 of the unit and the 32
// consecutive codes [32c, 32c+32) of the group, 4*b contiguous bytes per row; its x values
// for those k sit in 4 chunks of 16 bytes, stored so that the 4 lanes of a row read
// consecutive chunks (for 4 bits the fragment is permuted in registers into the codes' k
// order). Codes enter the MMAs as the exact bf16 values 128 + code (bit pattern
// 0x4300 | code); the group's (128 + 2^(b-1)) * sum(x) is removed from the MMA result, the
// sum taken per token by MMAs of the x fragment against an all-ones operand (8 per group,
// shared by the block's units). Each group's fp32 product is scaled by the group's fp32
// step and accumulated in fp32: the weight is never rounded.
//
// Reduction: warps that share a block add their partial sums in a fixed order through
// shared memory, then the S CTAs of a cluster add theirs through distributed shared memory
// (in rank order), add the low-rank branch and the bias, and round once to bf16. The
// low-rank input t = x L1 is written by a prepass launched just before this kernel; this
// kernel is launched as its programmatic dependent, streams the weight while the prepass
// runs, and waits for it only before the finish. All orders are fixed: the result is
// deterministic. Every wait on a slot is bounded: past the limit the kernel records
// WQ_ERR_TIMEOUT, lets the copies it issued land (again bounded) and finishes.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "unpack.cuh"

namespace wq {

constexpr int kSmMaxTok = 16;                                // tokens per launch
constexpr int kTStrideSm = 128;                              // row stride of [t_hi | t_lo]
constexpr int kSmMaxRB = 4;                                  // units per warp block (8 tokens)
template <int TOK> constexpr int sm_max_rb() { return TOK > 8 ? 3 : kSmMaxRB; }   // within the registers
constexpr int kSmMaxD = 4;                                   // ring slots per warp

template <int TOK> struct SmCfg {
    static constexpr int kWarps = 12;
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kNT = TOK / 8;                      // n8 token tiles per MMA step
    static constexpr int kCH = 2;                            // independent MMA accumulators per item
};

struct SmallMArgs {
    const uint16_t *x;        // M x K bf16
    const float *scales;      // N x K/128
    const uint16_t *bias;     // N or null
    const uint16_t *t;        // M x 128 bf16: [t_hi | t_lo] of x L1 (rank columns each), or null
    const uint16_t *L2;       // rank x N bf16 or null
    uint16_t *y;              // M x N bf16
    int64_t M, N, K;
    int rank;
    int S;                    // CTAs per cluster (K split)
    int n_clusters;
    int RB;                   // units per warp block (the kernel's template argument)
    int GW;                   // warps per block (group splits) when blocks < warps
    int D;                    // ring slots per warp (2..kSmMaxD)
    int rows_max;             // rows of the largest cluster range (units * 16)
    int rows_pad;             // rows_max + 16 * (RB - 1): row stride of the staged steps
    int gmax;                 // groups of the largest CTA share
    uint32_t x_stride;        // bytes per token row of the staged x (gmax * 256 + 64)
    uint32_t slot_bytes;      // one ring slot: RB units x 16 rows x 16b bytes of codes
    uint32_t off_zero;        // 256 zero bytes (the x of tokens past M), at 64 mod 128
    uint32_t off_st, off_l2, off_ring, off_part;
    uint32_t off_bar;         // W x D ring mbarriers, the staging mbarrier, the CTA's abort word
    int l2_staged;            // 1 when L2 is staged (rows of 16-byte multiples: N % 8 == 0)
};

// ---------------------------------------------------------------- asynchronous copies
// 16 bytes global -> shared through L2 only; src_bytes = 0 writes zeros (nothing is read).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// One arrival on the mbarrier once all of this thread's earlier cp.async copies have landed
// (counted in the barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Waits for a slot phase with a plain time limit and no abort flag (used only to let the
// copies already issued land before a kernel that gave up finishes).
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > kWaitLimitNs / 10) return;
}

// Shared-memory loads at 32-bit shared addresses (ordered after the barrier waits before them).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

// 4*b bytes of packed codes (one thread's 32-code slice) from shared memory, plus a zero word.
template <int BITS>
__device__ __forceinline__ void lds_slice(uint32_t a, uint32_t (&w)[BITS + 1]) {
    if constexpr (BITS == 4) {
        const uint4 v = lds128(a);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BITS == 6) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const uint2 v = lds64(a + 8 * i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = lds32(a + 4 * i);
    }
    w[BITS] = 0;
}

template <int BITS, int TOK, int RB>
__global__ void __launch_bounds__(SmCfg<TOK>::kThreads, 1)
smallm_kernel(const __grid_constant__ CUtensorMap pmap, const SmallMArgs a) {
    constexpr int W = SmCfg<TOK>::kWarps;
    constexpr int NT = SmCfg<TOK>::kNT;
    constexpr int CH = SmCfg<TOK>::kCH;
    constexpr uint32_t kGB = 16 * BITS;                        // bytes of one group of one row
    constexpr uint32_t kUnitBytes = 16 * kGB;                  // one unit's codes of one group
    constexpr float kBiasF = 128.0f + (float)(1 << (BITS - 1)); // the bias the unpacked codes carry
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g_l = lane >> 2, c_l = lane & 3;
    const int S = a.S;
    const uint32_t srank = (S > 1) ? cluster_ctarank() : 0u;
    const int cid = blockIdx.x / S;
    const int64_t U = (a.N + 15) / 16;
    const int64_t u0 = U * cid / a.n_clusters, u1 = U * (cid + 1) / a.n_clusters;
    const int Uc = (int)(u1 - u0);
    const int G = (int)(a.K / 128);
    const int g0 = (int)((int64_t)G * srank / S), g1 = (int)((int64_t)G * (srank + 1) / S);
    const int Gc = g1 - g0;
    const int rows_c = Uc * 16;
    const int64_t n_base = u0 * 16;
    const int M = (int)a.M;                                     // 1..TOK
    float *st = reinterpret_cast<float *>(smem + a.off_st);     // [gmax][rows_pad] steps
    float *part = reinterpret_cast<float *>(smem + a.off_part);
    const int part_stride = TOK * a.rows_max;                   // floats per group split
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + a.off_bar) + warp * a.D;
    uint64_t *stage_bar = reinterpret_cast<uint64_t *>(smem + a.off_bar) + W * a.D;        // after the rings' barriers
    int *s_abort = reinterpret_cast<int *>(stage_bar + 1);
    uint8_t *ring = smem + a.off_ring + (uint32_t)warp * (uint32_t)a.D * a.slot_bytes;

    // ---------------------------------------------------------------- this warp's items
    // with at least as many blocks as warps, warp w takes blocks w, w + W, ... over all the
    // CTA's groups; otherwise warp w takes block w % NB and group split w / NB of GW
    const int NB = (Uc + RB - 1) / RB;
    const bool shared_blocks = NB < W;
    const int split = shared_blocks ? warp / NB : 0;
    const bool active = shared_blocks ? (warp < NB * a.GW) : true;
    const int gs0 = shared_blocks ? Gc * split / a.GW : 0, gs1 = shared_blocks ? Gc * (split + 1) / a.GW : Gc;
    const int ng = gs1 - gs0;
    const int ub0 = shared_blocks ? (warp % NB) * RB : warp * RB;
    const int ub_step = W * RB;
    // (a warp whose group share is empty still writes zeros for its block)
    const int nblk = !active ? 0 : (shared_blocks ? 1 : (Uc - ub0 + ub_step - 1) / ub_step);
    const int n_items = nblk * max(ng, 0);

    if (threadIdx.x == 0) {
        *s_abort = 0;
        mbar_init(stage_bar, W * 32 + 1);
    }
    if (lane == 0)
        for (int s = 0; s < a.D; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
    __syncthreads();                                           // barriers ready before any arrival

    // item i (block i / ng, group i % ng) -> slot i % D, issued by lane 0 in item order; the
    // issue position (slot, TMA coordinates, units in the block) is tracked incrementally
    int pf_i = 0, pf_s = 0, pf_gl = gs0;
    int32_t pf_x = (g0 + gs0) * (int32_t)kGB, pf_y = (int32_t)(n_base + (int64_t)ub0 * 16);
    int pf_nr = min(RB, Uc - ub0);
    // every lane keeps the (warp-uniform) issue position; lane 0 issues the copies
    auto issue_next = [&]() {
        if (lane == 0) {
            fence_proxy_async_smem();                            // earlier reads of the slot first
            uint8_t *dst = ring + (uint32_t)pf_s * a.slot_bytes;
            mbar_arrive_expect_tx(&bars[pf_s], (uint32_t)pf_nr * kUnitBytes);
#pragma unroll
            for (int r = 0; r < RB; ++r)
                if (r < pf_nr) tma_load_2d(dst + r * kUnitBytes, &pmap, &bars[pf_s], pf_x, pf_y + 16 * r);
        }
        ++pf_i;
        if (++pf_s == a.D) pf_s = 0;
        pf_x += (int32_t)kGB;
        if (++pf_gl == gs1) {
            pf_gl = gs0;
            pf_x = (g0 + gs0) * (int32_t)kGB;
            pf_y += 16 * ub_step;
            pf_nr = min(RB, Uc - (pf_y - (int32_t)n_base) / 16);
        }
    };
    // ---------------------------------------------------------------- stage steps and x
    // Asynchronous copies, issued before the rings' first slots so that they land first. The
    // steps of the CTA's rows and groups go to [group][row]; chunk 4c + q of each group of a
    // token row of x (lane c's x, part q) goes to position 4q + c, so that the 4 lanes of a
    // row read consecutive chunks. Each thread's copies complete on the staging barrier (one
    // arrival per thread, and one from thread 0 after it has zeroed the x row used for
    // tokens past M), which every warp waits on before its first item: there is no CTA-wide
    // barrier before the streaming.
    {
        // element e = threadIdx.x + k * W * 32 of each copy list; its (row, column) is advanced
        // by the constant step instead of divided out each time
        const int rows_v = (int)min((int64_t)rows_c, a.N - n_base);
        const uint32_t ss = smem_u32(st);
        {
            const int di = W * 32 / Gc, dgl = W * 32 - di * Gc;
            int i = (int)threadIdx.x / Gc, gl = (int)threadIdx.x - i * Gc;
            while (i < rows_v) {
                cp_async_4(ss + 4u * (uint32_t)(gl * a.rows_pad + i), a.scales + (n_base + i) * G + g0 + gl, 4u);
                i += di;
                gl += dgl;
                if (gl >= Gc) { gl -= Gc; ++i; }
            }
        }
        {
            const int chunks = Gc * 16;                        // 16-byte chunks per token row
            const int dt = W * 32 / chunks, dj = W * 32 - dt * chunks;
            int tok = (int)threadIdx.x / chunks, jj = (int)threadIdx.x - tok * chunks;
            while (tok < M) {
                const int j = jj & 15;
                cp_async_16(smem_u32(smem) + (uint32_t)tok * a.x_stride + 16u * (uint32_t)((jj & ~15) + 4 * (j & 3) + (j >> 2)),
                            a.x + (int64_t)tok * a.K + (int64_t)g0 * 128 + 8 * jj, 16u);
                tok += dt;
                jj += dj;
                if (jj >= chunks) { jj -= chunks; ++tok; }
            }
        }
        cp_async_arrive_noinc(stage_bar);
        if (threadIdx.x == 0) {
#pragma unroll
            for (int q = 0; q < 16; ++q) reinterpret_cast<uint4 *>(smem + a.off_zero)[q] = make_uint4(0, 0, 0, 0);
            mbar_arrive(stage_bar);
        }
    }
    if (lane == 0) tma_prefetch_desc(&pmap);
    while (pf_i < n_items && pf_i < a.D) issue_next();
    // L2 columns [n_base, n_base + rows_c) of every rank row (zeros past N), needed only at the
    // finish: their own copy group, waited for after the streaming
    if (a.l2_staged) {
        const int per_row = rows_c / 8;
        const uint32_t ls = smem_u32(smem + a.off_l2);
        for (int jr = warp; jr < a.rank; jr += W) {
            for (int cj = lane; cj < per_row; cj += 32) {
                const int64_t n = n_base + 8 * cj;
                const bool ok = n < a.N;
                cp_async_16(ls + 2u * (uint32_t)(jr * a.rows_max + 8 * cj), ok ? a.L2 + (int64_t)jr * a.N + n : a.L2,
                            ok ? 16u : 0u);
            }
        }
    }
    cp_async_commit();

    // ---------------------------------------------------------------- stream and contract
    // Shared-memory addresses of this lane's reads, advanced item by item. The x fragment of
    // lane (g, c) for token tile t: token 8t + g (the zero row past M); chunk 4q + c of a
    // group holds its words [4q, 4q + 4).
    uint32_t x_lane[NT], x_step[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int tok = 8 * t + g_l;
        x_lane[t] = smem_u32(smem) + (tok < M ? (uint32_t)tok * a.x_stride : a.off_zero) + 16u * c_l;
        x_step[t] = tok < M ? 256u : 0u;
    }
    const uint32_t slot_bytes = a.slot_bytes, ring_u = smem_u32(ring), ring_end = ring_u + (uint32_t)a.D * slot_bytes;
    const uint32_t code_lane = (uint32_t)g_l * kGB + (uint32_t)c_l * 4u * BITS;   // row g, lane c's slice
    const uint32_t st_step = 4u * (uint32_t)a.rows_pad;                           // one group of steps
    const BiasedConsts<BITS> kc;
    volatile int *abort = s_abort;
    int i = 0, cs = 0;                                          // item, its slot (i % D)
    uint32_t cph = 0;                                           // its slot's phase parity ((i / D) & 1)
    uint32_t slot_u = ring_u;                                   // its slot's address
    bool ok = n_items == 0 || warp_wait(stage_bar, 0u, abort);
    for (int b = 0; b < nblk && ok; ++b) {
        const int ub = ub0 + b * ub_step;
        float R[RB][NT][4];
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int t = 0; t < NT; ++t) R[r][t][0] = R[r][t][1] = R[r][t][2] = R[r][t][3] = 0.0f;
        uint32_t x_u[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) x_u[t] = x_lane[t] + (uint32_t)gs0 * x_step[t];
        uint32_t st_u = smem_u32(st) + (uint32_t)gs0 * st_step + 4u * (uint32_t)(ub * 16 + g_l);
        for (int gl = gs0; gl < gs1; ++gl) {
            if (!warp_wait(&bars[cs], cph, abort)) { ok = false; break; }
            ++i;
            if (++cs == a.D) { cs = 0; cph ^= 1u; }
            // the slot's codes (all units) go to registers first, so that lane 0 refills the
            // slot with item i + D before the arithmetic starts
            uint32_t wa[RB][BITS + 1], wb[RB][BITS + 1];
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                lds_slice<BITS>(slot_u + code_lane + 16u * kGB * r, wa[r]);
                lds_slice<BITS>(slot_u + code_lane + 16u * kGB * r + 8u * kGB, wb[r]);
            }
            slot_u += slot_bytes;
            if (slot_u == ring_end) slot_u = ring_u;
            __syncwarp();                                       // every lane has read the slot
            if (pf_i < n_items) issue_next();
            // x fragment (in the codes' k order) and the group's correction
            // -(128 + 2^(b-1)) * sum_k x, the sum by MMAs against an all-ones operand
            uint32_t X[NT][16];
            float corr[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 v = lds128(x_u[t] + 64u * q);
                    if constexpr (BiasedOrder<BITS>::kPermuted) v = permute_x8(v);
                    X[t][4 * q] = v.x; X[t][4 * q + 1] = v.y; X[t][4 * q + 2] = v.z; X[t][4 * q + 3] = v.w;
                }
                x_u[t] += x_step[t];
                float on[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
                constexpr uint32_t kOnes = 0x3F803F80u;            // bf16 pair (1, 1)
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8)
                    mma_16816_bf16(on[s8 & 1], kOnes, kOnes, kOnes, kOnes, X[t][2 * s8], X[t][2 * s8 + 1]);
#pragma unroll
                for (int k = 0; k < 4; ++k) corr[t][k] = -kBiasF * (on[0][k] + on[1][k]);
            }
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const float sa = __uint_as_float(lds32(st_u + 64u * r)), sb = __uint_as_float(lds32(st_u + 64u * r + 32u));
                float acc[NT][CH][4];
#pragma unroll
                for (int t = 0; t < NT; ++t) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) acc[t][0][k] = corr[t][k];
#pragma unroll
                    for (int h = 1; h < CH; ++h) acc[t][h][0] = acc[t][h][1] = acc[t][h][2] = acc[t][h][3] = 0.0f;
                }
                static_for<4>([&](auto bb) {
                    constexpr int blk = decltype(bb)::value;
                    uint32_t pa[4], pb[4];
                    unpack_pairs_biased<BITS, blk, 1>(wa[r], pa, kc);
                    unpack_pairs_biased<BITS, blk, 1>(wb[r], pb, kc);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int s8 = 2 * blk + h;
#pragma unroll
                        for (int t = 0; t < NT; ++t)
                            mma_16816_bf16(acc[t][s8 % CH], pa[2 * h], pb[2 * h], pa[2 * h + 1], pb[2 * h + 1],
                                           X[t][2 * s8], X[t][2 * s8 + 1]);
                    }
                });
#pragma unroll
                for (int t = 0; t < NT; ++t) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float sum = acc[t][0][k];
#pragma unroll
                        for (int h = 1; h < CH; ++h) sum += acc[t][h][k];
                        R[r][t][k] = fmaf(k < 2 ? sa : sb, sum, R[r][t][k]);
                    }
                }
            }
            st_u += st_step;
        }
        if (!ok) break;
        // this block's partial sums -> part[split][token][row of the cluster range]
        const int nr = min(RB, Uc - ub);
        float *ps = part + split * part_stride;
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            if (r >= nr) break;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int tok = 8 * t + 2 * c_l, row = (ub + r) * 16 + g_l;
                ps[tok * a.rows_max + row] = R[r][t][0];
                ps[(tok + 1) * a.rows_max + row] = R[r][t][1];
                ps[tok * a.rows_max + row + 8] = R[r][t][2];
                ps[(tok + 1) * a.rows_max + row + 8] = R[r][t][3];
            }
        }
    }
    if (!ok && lane == 0) {   // (the issue position is the same in every lane)
        // gave up: let the copies already issued land before the shared memory is released
        for (int j = i; j < pf_i; ++j) {
            mbar_drain(&bars[cs], cph);
            if (++cs == a.D) { cs = 0; cph ^= 1u; }
        }
    }
    cp_async_wait<0>();                                        // the staged L2 columns
    __syncwarp();
    __syncthreads();
    // ---------------------------------------------------------------- CTA reduction (fixed order)
    if (shared_blocks && a.GW > 1) {
        for (int e = threadIdx.x; e < M * rows_c; e += W * 32) {
            const int tok = e / rows_c, row = e - tok * rows_c;
            float v = part[tok * a.rows_max + row];
            for (int j = 1; j < a.GW; ++j) v += part[j * part_stride + tok * a.rows_max + row];
            part[tok * a.rows_max + row] = v;
        }
        __syncthreads();
    }
    if (S > 1) cluster_sync();
    // ---------------------------------------------------------------- low-rank input
    // t = x L1 comes from the launch before this one, which may still be running: wait for
    // it, then hold t_hi + t_lo per token and rank column in fp32 where the rings were
    float *ts = reinterpret_cast<float *>(smem + a.off_ring);
    if (a.rank > 0) {
        grid_dependency_wait();
        for (int e = threadIdx.x; e < M * a.rank; e += W * 32) {
            const int m = e / a.rank, jr = e - m * a.rank;
            const uint16_t *tm = a.t + (int64_t)m * kTStrideSm;
            ts[e] = bf16_bits_to_f32(tm[jr]) + bf16_bits_to_f32(tm[a.rank + jr]);
        }
        __syncthreads();
    }
    // ---------------------------------------------------------------- finalize a 1/S share
    // Each thread finishes kFin outputs at a time so that their partial-sum loads overlap.
    constexpr int kFin = 4;
    const int rows_v = (int)min((int64_t)rows_c, a.N - n_base);
    const int E = M * rows_v;
    const int e0 = (int)((int64_t)E * srank / S), e1 = (int)((int64_t)E * (srank + 1) / S);
    const uint32_t part_addr = smem_u32(part);
    const uint16_t *l2s = reinterpret_cast<const uint16_t *>(smem + a.off_l2);
    for (int eb = e0 + (int)threadIdx.x; eb < e1; eb += kFin * W * 32) {
        float v[kFin];
        int mm[kFin], ii[kFin];
#pragma unroll
        for (int u = 0; u < kFin; ++u) {
            const int e = eb + u * W * 32;
            mm[u] = e < e1 ? e / rows_v : 0;
            ii[u] = e < e1 ? e - mm[u] * rows_v : 0;
            v[u] = 0.0f;
        }
        if (S > 1) {
            for (int q = 0; q < S; ++q) {
#pragma unroll
                for (int u = 0; u < kFin; ++u)
                    if (eb + u * W * 32 < e1)
                        v[u] += ld_cluster_f32(map_cluster_smem(part_addr + 4u * (uint32_t)(mm[u] * a.rows_max + ii[u]),
                                                                (uint32_t)q));
            }
        } else {
#pragma unroll
            for (int u = 0; u < kFin; ++u)
                if (eb + u * W * 32 < e1) v[u] = part[mm[u] * a.rows_max + ii[u]];
        }
#pragma unroll
        for (int u = 0; u < kFin; ++u) {
            if (eb + u * W * 32 >= e1) break;
            const int64_t n = n_base + ii[u];
            float acc = v[u];
            if (a.rank > 0) {
                const float *tm = ts + mm[u] * a.rank;
                float lr = 0.0f;
                if (a.l2_staged) {
                    for (int jr = 0; jr < a.rank; ++jr)
                        lr = fmaf(tm[jr], bf16_bits_to_f32(l2s[jr * a.rows_max + ii[u]]), lr);
                } else {
                    for (int jr = 0; jr < a.rank; ++jr)
                        lr = fmaf(tm[jr], bf16_bits_to_f32(__ldg(a.L2 + (int64_t)jr * a.N + n)), lr);
                }
                acc += lr;
            }
            if (a.bias) acc += bf16_bits_to_f32(__ldg(a.bias + n));
            a.y[(int64_t)mm[u] * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
        }
    }
    if (S > 1) cluster_sync();       // no CTA leaves while another may still read its part[]
}

}  // namespace wq
