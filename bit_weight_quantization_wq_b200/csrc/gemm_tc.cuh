// gemm_tc.cuh -- large-M fused dequant-GEMM on the 5th-generation tensor cores (KL).
//
//   y = x * dequant(W)^T + (x L1) L2 + bias,   dequant(code) = (code - 2^(b-1)) * step
//
// The Per-group(128) article dequantizes each block's weights on the GPU (sec. 3.4) and
// then runs a bf16 matmul, noting it has no low-bit matmul kernel (sec. 5.3, 5.4); the
// SVDQuant article adds a 16-bit low-rank branch computed next to the quantized residual
// ("Technical principles", "Engineering highlights"). Here the weight is never
// dequantized to memory, and never rounded: the tensor cores multiply the exact integer
// codes q = code - 2^(b-1) (exact in bf16) by x, one 128-wide group at a time, and each
// group's fp32 partial product is scaled by its fp32 step and added to the result:
//
//   y[m][n] = sum_g step[n][g] * ( sum_{k in g} q[n][k] x[m][k] )  (+ low-rank, + bias)
//
// Orientation: D = W_q x^T, so TMEM lanes are weight rows and columns are tokens; the
// per-group step is then one scalar per lane.
// One persistent CTA per SM walks 128 x 128 tiles (128 weight rows x 128 tokens).
// TMEM (512 columns): T0, T1 = per-group partials (double-buffered, 128 columns each) and
// 8 stages of codes (32 columns = 64 k each).
// Warp roles (512 threads):
//   warp 0      TMA producer of x tiles (128 tokens x 64 k bf16, 128B swizzle, 16 KB/stage)
//   warps 1, 3  warp 1 allocates TMEM; one thread of each issues tcgen05.mma (A = codes from
//               TMEM, B = x from shared memory, M=128 N=128 K=16) for alternate units
//   warp 2      TMA producer of packed-weight tiles (128 rows x one group, 16*b bytes a row)
//   warps 4-7   unpack: one weight row per thread; bf16 pairs of exact q written to the A
//               stage with tcgen05.st
//   warps 8-15  promotion: R += step * T per group (fp32, two lanes per instruction) with R in
//               registers (two warps per TMEM lane quarter, 64 columns each), then the epilogue
//               (+ bias, round once to bf16, store y)
// Synchronization is per unit (one 128-k group, or the low-rank unit), not per k stage: the
// single MMA-issuing thread pays ~140 cycles per mbarrier wait, so it waits once per unit on
// ready[slot], which completes when the unit's x tiles have landed (TMA transaction bytes),
// its codes are in TMEM (4 unpack warps) and its T buffer is free (8 promotion warps); one
// commit per unit releases the slot (consumed[slot]) and another hands T to the promotion.
// Low-rank branch: one more unit per tile with B = [t_hi | t_lo] (t = x L1 split into two
// bf16 terms by lowrank_prepass_kernel) and A = [L2^T | L2^T] (bf16 from global), promoted
// with scale 1 into the same R; the split keeps t's rounding out of the result.
//
// Every wait is bounded (see common.cuh). On a timeout the roles stop, the producer waits
// (bounded) for its copies in flight, the MMA thread for its MMAs, and TMEM is freed.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "unpack.cuh"

namespace wq {

constexpr int kTcBW = 128;                // weight rows per tile (MMA M)
constexpr int kTcBT = 128;                // tokens per tile (MMA N)
constexpr int kTcBK = 64;                 // k per x stage / A stage
constexpr int kTcSlots = 4;               // units in flight (each: 2 x stages + 2 code stages)
constexpr int kTcStagesX = 2 * kTcSlots;
constexpr int kTcStagesA = 2 * kTcSlots;
constexpr int kTcThreads = 512;
constexpr int kTcUnpackWarp0 = 4;
constexpr int kTcPromoteWarp0 = 8;
constexpr int kTcPromoteWarps = 8;
constexpr uint32_t kTcTmemCols = 512;
constexpr uint32_t kTmemT0 = 0, kTmemA = 256;
constexpr int kTStride = 128;             // row stride (elements) of the low-rank [t_hi | t_lo] buffer

template <int BITS> struct TcStagesP { static constexpr int value = BITS <= 4 ? 8 : 5; };

template <int BITS>
struct TcLayout {
    static constexpr int kSP = TcStagesP<BITS>::value;
    static constexpr uint32_t kXBytes = kTcBT * kTcBK * 2;          // 16 KB
    static constexpr uint32_t kPBytes = kTcBW * 16 * BITS;          // 128 rows x one group
    static constexpr uint32_t kOffX = 0;
    static constexpr uint32_t kOffP = kOffX + kTcStagesX * kXBytes;
    static constexpr uint32_t kOffL = kOffP + kSP * kPBytes;       // low-rank L2 tile [rank][128] bf16
    static constexpr uint32_t kLBytes = 64 * kTcBW * 2;
    static constexpr uint32_t kOffBar = kOffL + kLBytes;
    static constexpr uint32_t kNumBars = 2 * kTcSlots + 2 * kSP + 2 + 2 + 2;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kBytes = kOffMisc + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;               // slack to align the base to 1024 B
};

struct TcParams {
    const float *scales;      // N x K/128
    const uint16_t *L2;       // rank x N bf16 or null
    const uint16_t *bias;     // N bf16 or null
    uint16_t *y;              // M x N bf16
    int64_t M, N, K;
    int rank;
    int tiles_m, tiles_n;
    int l_tma;                // 1: the low-rank L2 tile of each weight tile arrives by TMA (l_map)
};

// k stages (64 wide) of the low-rank unit: [t_hi | t_lo] has 2 * rank columns.
__host__ __device__ constexpr int lowrank_stages(int rank) { return (2 * rank + kTcBK - 1) / kTcBK; }

template <int BITS>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_linear_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap p_map,
                 const __grid_constant__ CUtensorMap t_map, const __grid_constant__ CUtensorMap l_map,
                 const TcParams p) {
    using L = TcLayout<BITS>;
    constexpr int SP = L::kSP;
    constexpr int NWG = 4 * BITS + 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *ready = bars, *consumed = ready + kTcSlots;
    uint64_t *p_full = consumed + kTcSlots, *p_empty = p_full + SP;
    uint64_t *t_full = p_empty + SP, *drain = t_full + 2;      // drain[2]: one per MMA thread
    uint64_t *l_full = drain + 2, *l_empty = l_full + 1;        // low-rank L2 tile handoff
    const uint16_t *l_tile = reinterpret_cast<const uint16_t *>(smem + L::kOffL);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        // ready: x producer (1, plus transaction bytes) + 4 unpack warps + the promotion warps
        for (int i = 0; i < kTcSlots; ++i) { mbar_init(&ready[i], 1 + 4 + kTcPromoteWarps); mbar_init(&consumed[i], 1); }
        for (int i = 0; i < SP; ++i) { mbar_init(&p_full[i], 1); mbar_init(&p_empty[i], 4 * 32); }
        for (int i = 0; i < 2; ++i) mbar_init(&t_full[i], 1);
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        mbar_init(l_full, 1);
        mbar_init(l_empty, 4 * 32);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int G = (int)(p.K / 128);
    const int U = G + (p.rank > 0 ? 1 : 0);          // units per tile: groups (+ low-rank)
    const int tiles = p.tiles_m * p.tiles_n;

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------- x / t producer
        tma_prefetch_desc(&x_map);
        tma_prefetch_desc(&t_map);
        int armed[kTcSlots];
        for (int i = 0; i < kTcSlots; ++i) armed[i] = -1;
        uint32_t unit = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int mt = tile % p.tiles_m;
            for (int u = 0; u < U; ++u, ++unit) {
                const uint32_t slot = unit % kTcSlots, ph = (unit / kTcSlots) & 1;
                const int nst = (u < G) ? 2 : lowrank_stages(p.rank);
                if (!mbar_wait(&consumed[slot], ph ^ 1, abort)) goto x_done;
                mbar_arrive_expect_tx(&ready[slot], nst * L::kXBytes);
                armed[slot] = (int)ph;
                for (int st = 0; st < nst; ++st) {
                    uint8_t *dst = smem + L::kOffX + (slot * 2 + st) * L::kXBytes;
                    if (u < G) tma_load_2d(dst, &x_map, &ready[slot], (2 * u + st) * kTcBK, mt * kTcBT);
                    else tma_load_2d(dst, &t_map, &ready[slot], st * kTcBK, mt * kTcBT);
                }
            }
        }
    x_done:
        // wait (bounded) for the copies still in flight: a slot's phase cannot complete without
        // them, so poll the transaction count through the phase of the last armed unit
        for (int i = 0; i < kTcSlots; ++i) {
            int local = 0;
            if (armed[i] >= 0 && *abort) (void)mbar_wait(&ready[i], (uint32_t)armed[i], &local, 50ull * 1000ull * 1000ull);
        }
    } else if (warp == 2 && lane == 0) {
        // ---------------------------------------------------------- packed-weight producer
        tma_prefetch_desc(&p_map);
        int armed[SP];
        for (int i = 0; i < SP; ++i) armed[i] = -1;
        if (p.l_tma) tma_prefetch_desc(&l_map);
        uint32_t s = 0, ph = 0, lph = 0;
        int l_armed = -1;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int nt = tile / p.tiles_m;
            for (int g = 0; g < G; ++g) {
                if (!mbar_wait(&p_empty[s], ph ^ 1, abort)) goto p_done;
                mbar_arrive_expect_tx(&p_full[s], L::kPBytes);
                armed[s] = (int)ph;
                tma_load_2d(smem + L::kOffP + s * L::kPBytes, &p_map, &p_full[s], g * 16 * BITS, nt * kTcBW);
                if (++s == SP) { s = 0; ph ^= 1; }
            }
            if (p.l_tma) {
                // this tile's L2 columns, [rank][128 rows]; the tile's low-rank unit comes after all
                // its groups, so the copy issued here lands long before it is read
                if (!mbar_wait(l_empty, lph ^ 1, abort)) goto p_done;
                mbar_arrive_expect_tx(l_full, (uint32_t)p.rank * kTcBW * 2);
                l_armed = (int)lph;
                tma_load_2d(smem + L::kOffL, &l_map, l_full, nt * kTcBW, 0);
                lph ^= 1;
            }
        }
    p_done:
        for (int i = 0; i < SP; ++i) {
            int local = 0;
            if (armed[i] >= 0) (void)mbar_wait(&p_full[i], (uint32_t)armed[i], &local);
        }
        if (l_armed >= 0) {
            int local = 0;
            (void)mbar_wait(l_full, (uint32_t)l_armed, &local);
        }
    } else if ((warp == 1 || warp == 3) && lane == 0) {
        // ---------------------------------------------------------- MMA issuers
        // Two threads issue: warp 1 the even units (into T0), warp 3 the odd units (into T1).
        // An MMA issue occupies the issuing thread for ~85 cycles and each unit also costs a
        // barrier wait and two commits; a second issuer overlaps that with the other's MMAs.
        const uint32_t mine = (warp == 1) ? 0u : 1u;
        constexpr uint32_t idesc = umma_idesc_bf16(kTcBW, kTcBT);
        uint32_t unit = 0;
        const uint32_t x_base = smem_u32(smem + L::kOffX);
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            for (int u = 0; u < U; ++u, ++unit) {
                if ((unit & 1u) != mine) continue;
                const uint32_t slot = unit % kTcSlots, ph = (unit / kTcSlots) & 1, tb = unit & 1;
                if (!mbar_wait(&ready[slot], ph, abort)) goto m_done;
                tc_fence_after();
                const uint32_t d = tmem + kTmemT0 + tb * kTcBT;
                const int nst = (u < G) ? 2 : lowrank_stages(p.rank);
                for (int st = 0; st < nst; ++st) {
                    const int nk = (u < G) ? kTcBK / 16 : min(kTcBK, 2 * p.rank - st * kTcBK) / 16;
                    const uint32_t a = tmem + kTmemA + (slot * 2 + st) * (kTcBK / 2);
                    const uint32_t b_base = x_base + (slot * 2 + st) * L::kXBytes;
                    for (int k = 0; k < nk; ++k) {
                        const uint64_t bd = umma_desc_sw128(b_base + k * 32, 1024);
                        umma_bf16_ts(d, a + k * 8, bd, idesc, (st > 0 || k > 0) ? 1u : 0u);
                    }
                }
                umma_commit(&consumed[slot]);
                umma_commit(&t_full[tb]);
            }
        }
    m_done:
        {
            // every MMA issued by this thread completes before TMEM is released
            umma_commit(&drain[mine]);
            int local = 0;
            (void)mbar_wait(&drain[mine], 0, &local);
        }
    } else if (warp >= kTcUnpackWarp0 && warp < kTcPromoteWarp0) {
        // ---------------------------------------------------------- unpack codes into TMEM
        const int quarter = warp & 3;
        const int row_local = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        uint32_t sp = 0, pp = 0, unit = 0, lph = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int nt = tile / p.tiles_m;
            const int64_t n = (int64_t)nt * kTcBW + row_local;
            const bool row_ok = n < p.N;
            for (int u = 0; u < U; ++u, ++unit) {
                const uint32_t slot = unit % kTcSlots, ph = (unit / kTcSlots) & 1;
                const uint32_t a_addr = tmem + lane_addr + kTmemA + slot * 2 * (kTcBK / 2);
                if (u < G) {
                    if (!warp_wait(&p_full[sp], pp, abort)) goto u_done;
                    uint32_t w[NWG];
                    {
                        const uint4 *src = reinterpret_cast<const uint4 *>(smem + L::kOffP + sp * L::kPBytes +
                                                                            row_local * 16 * BITS);
#pragma unroll
                        for (int i = 0; i < BITS; ++i) {
                            const uint4 v = src[i];
                            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
                        }
                        w[4 * BITS] = 0;
                    }
                    // Every consuming thread releases the stage itself (arrival count 128), after a
                    // proxy fence: its loads are generic-proxy reads and the producer's next copy
                    // is an async-proxy write, so the reads are ordered before the release across
                    // proxies. (One lane's arrive after a warp sync let the next copy land while
                    // other lanes' loads were in flight.)
                    fence_proxy_async_smem();
                    mbar_arrive(&p_empty[sp]);
                    if (++sp == SP) { sp = 0; pp ^= 1; }
                    uint32_t q0[32], q1[32];
                    unpack_pairs<BITS, 0, 8>(w, q0);
                    unpack_pairs<BITS, 8, 8>(w, q1);
                    if (!warp_wait(&consumed[slot], ph ^ 1, abort)) goto u_done;
                    tc_fence_after();        // order the stores after the MMAs that read this slot
                    tmem_st_32x32b_x32(a_addr, q0);
                    tmem_st_32x32b_x32(a_addr + kTcBK / 2, q1);
                } else {
                    // low-rank unit: A[n][k] = L2[k mod rank][n] for k < 2 rank (both halves of
                    // [t_hi | t_lo] meet the same L2), zero beyond; from the shared-memory tile
                    // when it came by TMA, else straight from global memory
                    if (p.l_tma && !warp_wait(l_full, lph, abort)) goto u_done;
                    if (!warp_wait(&consumed[slot], ph ^ 1, abort)) goto u_done;
                    tc_fence_after();
                    const int nst = lowrank_stages(p.rank);
                    for (int st = 0; st < nst; ++st) {
                        uint32_t q[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int k = st * kTcBK + 2 * i;
                            uint32_t v = 0;
                            if (k < 2 * p.rank) {
                                const int j = k < p.rank ? k : k - p.rank;
                                if (p.l_tma) {
                                    v = (uint32_t)l_tile[j * kTcBW + row_local] | ((uint32_t)l_tile[(j + 1) * kTcBW + row_local] << 16);
                                } else if (row_ok) {
                                    v = (uint32_t)__ldg(p.L2 + (int64_t)j * p.N + n) |
                                        ((uint32_t)__ldg(p.L2 + (int64_t)(j + 1) * p.N + n) << 16);
                                }
                            }
                            q[i] = v;
                        }
                        tmem_st_32x32b_x32(a_addr + st * (kTcBK / 2), q);
                    }
                    if (p.l_tma) {
                        // the tile is read: release it to the next tile's copy (per lane, after the
                        // proxy fence, as for the packed stages)
                        fence_proxy_async_smem();
                        mbar_arrive(l_empty);
                        lph ^= 1;
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ready[slot]);
            }
        }
    u_done:;
    } else if (warp >= kTcPromoteWarp0) {
        // ---------------------------------------------------------- promotion + epilogue
        const int quarter = warp & 3;
        const int colh = (warp - kTcPromoteWarp0) >> 2;            // which 64 token columns
        const int row_local = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        constexpr int kPre = 4;                                     // scale prefetch distance
        // both T buffers start free: count this warp's release for units 0 and 1
        if (lane == 0) { mbar_arrive(&ready[0]); mbar_arrive(&ready[1]); }
        uint32_t unit = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int mt = tile % p.tiles_m, nt = tile / p.tiles_m;
            const int64_t n = (int64_t)nt * kTcBW + row_local;
            const bool row_ok = n < p.N;
            const float *srow = p.scales + (row_ok ? n : 0) * (int64_t)G;
            float sq[kPre];
#pragma unroll
            for (int i = 0; i < kPre; ++i) sq[i] = (row_ok && i < G) ? __ldg(srow + i) : 0.0f;
            float R[64];
            for (int u = 0; u < U; ++u, ++unit) {
                float s = 1.0f;
                if (u < G) {
                    s = sq[0];
#pragma unroll
                    for (int i = 0; i + 1 < kPre; ++i) sq[i] = sq[i + 1];
                    sq[kPre - 1] = (row_ok && u + kPre < G) ? __ldg(srow + u + kPre) : 0.0f;
                }
                const uint32_t tb = unit & 1, tph = (unit >> 1) & 1;
                if (!warp_wait(&t_full[tb], tph, abort)) goto pr_done;
                tc_fence_after();
                const uint32_t t_addr = tmem + lane_addr + kTmemT0 + tb * kTcBT + colh * 64;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t tv[32];
                    tmem_ld_32x32b_x32(t_addr + 32 * hf, tv);
                    tmem_wait_ld();
                    if (hf == 1) {
                        // both halves of T are in registers: hand the buffer back to the MMA
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ready[(unit + 2) % kTcSlots]);
                    }
                    if (u == 0) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) R[32 * hf + i] = __uint_as_float(tv[i]) * s;
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; i += 2)
                            ffma2(R[32 * hf + i], R[32 * hf + i + 1], __uint_as_float(tv[i]), __uint_as_float(tv[i + 1]),
                                  s, s, R[32 * hf + i], R[32 * hf + i + 1]);
                    }
                }
            }
            // ------------------------------------------------------ epilogue
            if (row_ok) {
                const float bn = p.bias ? bf16_bits_to_f32(__ldg(p.bias + n)) : 0.0f;
                const int64_t m0 = (int64_t)mt * kTcBT + colh * 64;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    if (m0 + j < p.M)
                        p.y[(m0 + j) * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(R[j] + bn));
                }
            }
        }
    pr_done:;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

// ---------------------------------------------------------------------------------------
// t = x L1 (M x R, R = rank 16..64) as two bf16 terms, t_hi = bf16(t) in columns [0, R) and
// t_lo = bf16(t - t_hi) in [R, 2R), row stride kTStride = 128 (the rest zero), so that
// 64-wide TMA boxes cover a row exactly.
// x is read once; tensor cores via mma.m16n8k16.
// grid (ceil(M/64), KS) with clusters of KS CTAs along K; a CTA owns 64 tokens (4 warps x
// 16) and 1/KS of K; partial sums are added through distributed shared memory.
// Inside a thread, k is taken in the order that makes its x loads contiguous (16
// consecutive k per row per 64-k stage); the L1 fragments are fetched with
// ldmatrix.trans from row addresses in the same order.
template <int R>
__global__ void __launch_bounds__(128)
lowrank_prepass_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ L1,
                       uint16_t *__restrict__ t, int64_t M, int64_t K) {
    constexpr int kLd = R + 8;                          // padded smem row (elements)
    __shared__ __align__(16) uint16_t l1s[2][64 * kLd];
    __shared__ __align__(16) float part[64 * R];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const uint32_t KS = gridDim.y, split = cluster_ctarank();
    const int64_t m0 = (int64_t)blockIdx.x * 64;
    const int64_t nkb = K / 64;
    const int64_t kb0 = nkb * split / KS, kb1 = nkb * (split + 1) / KS;
    const int64_t ra = m0 + warp * 16 + g, rb = ra + 8;
    float acc[R / 8][4];
#pragma unroll
    for (int j = 0; j < R / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;

    auto load_l1 = [&](int buf, int64_t kb) {
        constexpr int chunks = 64 * R / 8;              // 16-byte chunks of the 64 x R slab
        for (int i = tid; i < chunks; i += 128) {
            const int kr = i / (R / 8), cj = i % (R / 8);
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(L1 + (kb * 64 + kr) * R) + cj);
            *reinterpret_cast<uint4 *>(&l1s[buf][kr * kLd + cj * 8]) = v;
        }
    };
    auto load_x = [&](int64_t kb, uint4 (&xa)[2], uint4 (&xb)[2]) {
        const int64_t k = kb * 64 + 16 * c;
        if (ra < M) { xa[0] = __ldg(reinterpret_cast<const uint4 *>(x + ra * K + k)); xa[1] = __ldg(reinterpret_cast<const uint4 *>(x + ra * K + k + 8)); }
        else xa[0] = xa[1] = make_uint4(0, 0, 0, 0);
        if (rb < M) { xb[0] = __ldg(reinterpret_cast<const uint4 *>(x + rb * K + k)); xb[1] = __ldg(reinterpret_cast<const uint4 *>(x + rb * K + k + 8)); }
        else xb[0] = xb[1] = make_uint4(0, 0, 0, 0);
    };

    uint4 xa[2], xb[2], na[2], nb[2];
    if (kb0 < kb1) {
        load_l1(0, kb0);
        load_x(kb0, xa, xb);
    }
    __syncthreads();
    for (int64_t kb = kb0; kb < kb1; ++kb) {
        const int buf = (int)((kb - kb0) & 1);
        if (kb + 1 < kb1) {
            load_l1(buf ^ 1, kb + 1);
            load_x(kb + 1, na, nb);
        }
        const uint32_t aw[8] = {xa[0].x, xa[0].y, xa[0].z, xa[0].w, xa[1].x, xa[1].y, xa[1].z, xa[1].w};
        const uint32_t bw[8] = {xb[0].x, xb[0].y, xb[0].z, xb[0].w, xb[1].x, xb[1].y, xb[1].z, xb[1].w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            // k-slot q of this step <-> actual k = 16 (q%8 / 2) + 4 s + 2 (q / 8) + (q % 2)
            const int q = lane & 15;
            const int kr = 16 * ((q & 7) >> 1) + 4 * s + 2 * (q >> 3) + (q & 1);
#pragma unroll
            for (int jt = 0; jt < R / 8; jt += 2) {
                uint32_t b0, b1, b2, b3;
                const int col = jt * 8 + (lane >> 4) * 8;
                const uint32_t addr = smem_u32(&l1s[buf][kr * kLd + (col < R ? col : jt * 8)]);
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3) : "r"(addr));
                mma_16816_bf16(acc[jt], aw[2 * s], bw[2 * s], aw[2 * s + 1], bw[2 * s + 1], b0, b1);
                if (jt + 1 < R / 8)
                    mma_16816_bf16(acc[jt + 1], aw[2 * s], bw[2 * s], aw[2 * s + 1], bw[2 * s + 1], b2, b3);
            }
        }
        __syncthreads();
        if (kb + 1 < kb1) {
            xa[0] = na[0]; xa[1] = na[1]; xb[0] = nb[0]; xb[1] = nb[1];
        }
    }
    // partial sums -> shared memory [token][j]
#pragma unroll
    for (int jt = 0; jt < R / 8; ++jt) {
        const int tl = warp * 16 + g, j = jt * 8 + 2 * c;
        part[tl * R + j] = acc[jt][0];
        part[tl * R + j + 1] = acc[jt][1];
        part[(tl + 8) * R + j] = acc[jt][2];
        part[(tl + 8) * R + j + 1] = acc[jt][3];
    }
    __syncthreads();
    cluster_sync();
    const int E = 64 * R;
    const int e0 = (int)((int64_t)E * split / KS), e1 = (int)((int64_t)E * (split + 1) / KS);
    const uint32_t base = smem_u32(part);
    for (int e = e0 + tid; e < e1; e += 128) {
        float v = 0.0f;
        for (uint32_t r = 0; r < KS; ++r) v += ld_cluster_f32(map_cluster_smem(base + 4u * e, r));
        const int64_t m = m0 + e / R;
        if (m < M) {
            // two bf16 terms: t_hi = bf16(t) in column j, t_lo = bf16(t - t_hi) in column R + j
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
            t[m * kTStride + e % R] = __bfloat16_as_ushort(hi);
            t[m * kTStride + R + e % R] = __bfloat16_as_ushort(lo);
        }
    }
    if constexpr (2 * R < kTStride) {
        // zero the padding columns so that the whole row is defined
        constexpr int kPad = kTStride - 2 * R;
        if (split == 0) {
            for (int i = tid; i < 64 * kPad; i += 128) {
                const int64_t m = m0 + i / kPad;
                if (m < M) t[m * kTStride + 2 * R + i % kPad] = 0;
            }
        }
    }
    cluster_sync();
}

}  // namespace wq
