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
// One persistent CTA per SM walks tiles of 128 weight rows x TT tokens (TT = 256 or 240,
// whichever leaves the last wave of tiles fuller, or 128 for few tokens), weight tiles fastest, so a wave of CTAs shares one token tile of x in L2 and
// the (4-8x smaller) packed weight stays L2-resident across token tiles.
// Shared memory: a ring of kStages 64-k stages, each holding the x tile (TT tokens x 64 k,
// bf16, 128-byte swizzle, by TMA) and the code tile (128 rows x 64 k exact bf16 q, the same
// swizzled layout, written by the unpack warps). TMEM (512 columns): T0 at column 0 and T1 at
// column 256 = the per-group partial products (double-buffered, TT columns each).
// One unit = one 128-k group (two stages) or the low-rank unit. Per unit, one MMA-issuing
// thread waits for T to be free and for each stage to be full, issues M=128 N=TT K=16 MMAs
// (A = codes, B = x, both from shared memory), releases each stage with a commit and hands T
// to the promotion with another. With TT = 256 one unit is ~1100 tensor cycles, long enough
// to hide the promotion's hand-off of the other T buffer.
// Warp roles (512 threads; registers re-split per warpgroup with setmaxnreg, 48/96/184,
// summing to the 128 per thread the block is launched with):
//   warp 0      TMA producer of the x tiles (and of t = x L1 for the low-rank unit)
//   warps 1, 3  warp 1 allocates TMEM; one thread of each issues the MMAs of alternate units
//   warp 2      TMA producer of the tile's [rank][128] block of L2 (when N % 8 == 0)
//   warps 4-7   unpack: one weight row per thread, packed group straight from global memory
//               (two groups in flight in registers) to exact bf16 q pairs in the code tile
//   warps 8-15  promotion: R += step * T per group (fp32, two lanes per instruction) with R in
//               registers (two warps per TMEM lane quarter, TT/2 columns each), then the
//               epilogue (+ bias, round once to bf16, store y)
// Low-rank branch: one more unit per tile with B = [t_hi | t_lo] (t = x L1 split into two
// bf16 terms by lowrank_prepass_kernel) and A = [L2^T | L2^T], promoted with scale 1 into the
// same R; the split keeps t's rounding out of the result.
//
// Every wait is bounded (see common.cuh). On a timeout the roles stop, the producers wait
// (bounded) for their copies in flight, the MMA threads for their MMAs, and TMEM is freed.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "unpack.cuh"

namespace wq {

constexpr int kTcBW = 128;                // weight rows per tile (MMA M)
constexpr int kTcBK = 64;                 // k per shared-memory stage (one 128-byte swizzled row)
constexpr int kTcThreads = 512;
constexpr uint32_t kTcTmemCols = 512;
constexpr int kTStride = 128;             // row stride (elements) of the low-rank [t_hi | t_lo] buffer
// registers per thread of each warpgroup after setmaxnreg: producers/MMA, unpack, promotion x 2;
// 128 * (48 + 96 + 2 * 184) = 512 threads * 128, the block's allocation at launch
constexpr int kTcRegsWg0 = 48, kTcRegsWg1 = 96, kTcRegsPromote = 184, kTcRegsLaunch = 128;
static_assert(kTcRegsWg0 + kTcRegsWg1 + 2 * kTcRegsPromote == 4 * kTcRegsLaunch, "register split");

template <int TT>
struct TcLayout {
    static constexpr int kStages = TT > 128 ? 4 : 6;
    static constexpr uint32_t kXBytes = TT * kTcBK * 2;             // 32 KB (TT = 256)
    static constexpr uint32_t kABytes = kTcBW * kTcBK * 2;          // 16 KB
    static constexpr uint32_t kOffX = 0;
    static constexpr uint32_t kOffA = kOffX + kStages * kXBytes;
    static constexpr uint32_t kOffL = kOffA + kStages * kABytes;    // low-rank L2 tile [rank][128] bf16
    static constexpr uint32_t kLBytes = 64 * kTcBW * 2;
    static constexpr uint32_t kOffBar = kOffL + kLBytes;
    // full[S], empty[S], p_full[S], t_full[2], t_empty[2], l_full, l_empty, drain[2]
    static constexpr uint32_t kNumBars = 3 * kStages + 8;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kBytes = kOffMisc + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;               // slack to align the base to 1024 B
};

struct TcParams {
    const uint8_t *packed;    // N x K*b/8
    const float *scales;      // N x K/128
    const uint16_t *L2;       // rank x N bf16 or null
    const uint16_t *bias;     // N bf16 or null
    uint16_t *y;              // M x N bf16
    int64_t M, N, K;
    int64_t row_bytes;        // K * b / 8
    int rank;
    int tiles_m, tiles_n;
    int l_tma;                // 1: the low-rank L2 tile of each weight tile arrives by TMA (l_map)
};

// k stages (64 wide) of the low-rank unit: [t_hi | t_lo] has 2 * rank columns.
__host__ __device__ constexpr int lowrank_stages(int rank) { return (2 * rank + kTcBK - 1) / kTcBK; }

template <int N> __device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N> __device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Named barrier 1 over the 128 unpack threads that also ORs a predicate across them: every
// thread gets the same answer.
__device__ __forceinline__ bool unpack_bar_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "barrier.cta.red.or.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)pred) : "memory");
    return r != 0;
}

// Byte offset of 16-byte chunk c (0..7) of row r in a tile of 128-byte rows stored in the
// canonical K-major 128-byte-swizzle layout (8-row blocks of 1024 bytes, chunk index XOR
// row mod 8) -- the layout TMA writes with CU_TENSOR_MAP_SWIZZLE_128B and the MMA reads.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t r, uint32_t c) {
    return (r >> 3) * 1024u + (r & 7u) * 128u + ((c ^ (r & 7u)) << 4);
}

template <int BITS, int TT>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_linear_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap t_map,
                 const __grid_constant__ CUtensorMap l_map, const __grid_constant__ CUtensorMap p_map,
                 const TcParams p) {
    using L = TcLayout<TT>;
    constexpr int S = L::kStages;
    constexpr int NWG = 4 * BITS + 1;
    constexpr int kHalf = TT / 2;                 // promotion columns per warp
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *full = bars, *empty = full + S, *p_full = empty + S;
    uint64_t *t_full = p_full + S, *t_empty = t_full + 2;
    uint64_t *l_full = t_empty + 2, *l_empty = l_full + 1;
    uint64_t *drain = l_empty + 1;                               // drain[2]: one per MMA thread
    const uint16_t *l_tile = reinterpret_cast<const uint16_t *>(smem + L::kOffL);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1 + 4);          // x producer (+ transaction bytes) + 4 unpack warps
            mbar_init(&empty[i], 1);             // the commit of the MMAs that read the stage
            mbar_init(&p_full[i], 1);            // packed group tile landed in this stage (TMA bytes)
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&t_full[i], 1);
            mbar_init(&t_empty[i], 8);           // the 8 promotion warps
        }
        mbar_init(l_full, 1);
        mbar_init(l_empty, 4);
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
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
    const int nlr = p.rank > 0 ? lowrank_stages(p.rank) : 0;
    const int U = G + (p.rank > 0 ? 1 : 0);          // units per tile: groups (+ low-rank)
    const int tiles = p.tiles_m * p.tiles_n;
    const int wg = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 7), 0);   // warp-uniform role

    if (wg == 0) {
        regs_dec<kTcRegsWg0>();
        if (warp == 0 && lane == 0) {
            // ------------------------------------------------------ x / t producer
            tma_prefetch_desc(&x_map);
            tma_prefetch_desc(&t_map);
            int armed[S];
            for (int i = 0; i < S; ++i) armed[i] = -1;
            uint32_t q = 0;
            for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
                const int mt = tile / p.tiles_n;
                for (int u = 0; u < U; ++u) {
                    const int nst = (u < G) ? 2 : nlr;
                    for (int st = 0; st < nst; ++st, ++q) {
                        const uint32_t s = q % S, ph = (q / S) & 1;
                        if (!mbar_wait(&empty[s], ph ^ 1, abort)) goto x_done;
                        mbar_arrive_expect_tx(&full[s], L::kXBytes);
                        armed[s] = (int)ph;
                        uint8_t *dst = smem + L::kOffX + s * L::kXBytes;
                        if (u < G) tma_load_2d(dst, &x_map, &full[s], (2 * u + st) * kTcBK, mt * TT);
                        else tma_load_2d(dst, &t_map, &full[s], st * kTcBK, mt * TT);
                    }
                }
            }
        x_done:
            // wait (bounded) for the copies still in flight: a stage's phase cannot complete
            // without them, so poll the transaction count through the last armed phase
            for (int i = 0; i < S; ++i) {
                int local = 0;
                if (armed[i] >= 0 && *abort) (void)mbar_wait(&full[i], (uint32_t)armed[i], &local, 50ull * 1000ull * 1000ull);
            }
        } else if (warp == 2 && lane == 0) {
            // ------------------------------------------------------ packed-code and L2 tile producer
            // A group's packed tile (128 rows x 16*b bytes, <= 14 KB) lands in the code buffer of
            // the unit's second stage, where the unpack warps read it before overwriting it with
            // that stage's codes; the tile's L2 block goes to its own buffer once per tile.
            tma_prefetch_desc(&p_map);
            if (p.l_tma && p.rank > 0) tma_prefetch_desc(&l_map);
            int armed[S];
            for (int i = 0; i < S; ++i) armed[i] = -1;
            int l_armed = -1;
            // p_full[s] is armed only when stage s is a group's second stage, which is not every
            // use of s (a one-stage low-rank unit shifts the pairing), so its phase is counted
            // per stage: bit s of pph
            uint32_t q = 0, lph = 0, pph = 0;
            for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
                const int nt = tile % p.tiles_n;
                for (int u = 0; u < G; ++u, q += 2) {
                    const uint32_t s1 = (q + 1) % S, ph1 = ((q + 1) / S) & 1;
                    if (!mbar_wait(&empty[s1], ph1 ^ 1, abort)) goto p_done;
                    mbar_arrive_expect_tx(&p_full[s1], (uint32_t)kTcBW * 16u * BITS);
                    armed[s1] = (int)((pph >> s1) & 1u);
                    pph ^= 1u << s1;
                    tma_load_2d(smem + L::kOffA + s1 * L::kABytes, &p_map, &p_full[s1], u * 16 * BITS, nt * kTcBW);
                }
                if (p.rank > 0) {
                    q += nlr;
                    if (p.l_tma) {
                        if (!mbar_wait(l_empty, lph ^ 1, abort)) goto p_done;
                        mbar_arrive_expect_tx(l_full, (uint32_t)p.rank * kTcBW * 2);
                        l_armed = (int)lph;
                        tma_load_2d(smem + L::kOffL, &l_map, l_full, nt * kTcBW, 0);
                        lph ^= 1;
                    }
                }
            }
        p_done:
            for (int i = 0; i < S; ++i) {
                int local = 0;
                if (armed[i] >= 0) (void)mbar_wait(&p_full[i], (uint32_t)armed[i], &local, 50ull * 1000ull * 1000ull);
            }
            if (l_armed >= 0) {
                int local = 0;
                (void)mbar_wait(l_full, (uint32_t)l_armed, &local, 50ull * 1000ull * 1000ull);
            }
        } else if ((warp == 1 || warp == 3) && lane == 0) {
            // ------------------------------------------------------ MMA issuers
            // Two threads issue: warp 1 the even units (into T0), warp 3 the odd units (into T1).
            const uint32_t mine = (warp == 1) ? 0u : 1u;
            constexpr uint32_t idesc = umma_idesc_bf16(kTcBW, TT);
            const uint32_t x_base = smem_u32(smem + L::kOffX), a_base = smem_u32(smem + L::kOffA);
            uint32_t q = 0, unit = 0;
            for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
                for (int u = 0; u < U; ++u, ++unit) {
                    const int nst = (u < G) ? 2 : nlr;
                    if ((unit & 1u) != mine) { q += nst; continue; }
                    const uint32_t tb = unit & 1;
                    if (!mbar_wait(&t_empty[tb], ((unit >> 1) & 1) ^ 1, abort)) goto m_done;
                    tc_fence_after();
                    const uint32_t d = tmem + tb * 256u;
                    for (int st = 0; st < nst; ++st, ++q) {
                        const uint32_t s = q % S, ph = (q / S) & 1;
                        if (!mbar_wait(&full[s], ph, abort)) goto m_done;
                        tc_fence_after();
                        const int nk = (u < G) ? kTcBK / 16 : min(kTcBK, 2 * p.rank - st * kTcBK) / 16;
                        const uint32_t xa = x_base + s * L::kXBytes, aa = a_base + s * L::kABytes;
                        for (int k = 0; k < nk; ++k)
                            umma_bf16(d, umma_desc_sw128(aa + k * 32, 1024), umma_desc_sw128(xa + k * 32, 1024), idesc,
                                      (st > 0 || k > 0) ? 1u : 0u);
                        umma_commit(&empty[s]);
                    }
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
        }
    } else if (wg == 1) {
        regs_dec<kTcRegsWg1>();
        // ---------------------------------------------------------- unpack codes into shared memory
        const int row_local = threadIdx.x - 128;
        const uint32_t a_base = smem_u32(smem + L::kOffA);
        uint32_t q = 0, lph = 0, pph = 0;     // pph: per-stage phase bits of p_full (see the producer)
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int nt = tile % p.tiles_n;
            const int64_t n = (int64_t)nt * kTcBW + row_local;
            const bool row_ok = n < p.N;        // (rows past N arrive as zeros and are never stored)
            for (int g = 0; g < G; ++g) {
                const uint32_t s0 = q % S, ph0 = (q / S) & 1;
                const uint32_t s1 = (q + 1) % S;
                q += 2;
                // this row's packed group, from the tile the producer put in stage s1's code buffer
                const bool got = warp_wait(&p_full[s1], (pph >> s1) & 1u, abort);
                pph ^= 1u << s1;
                uint32_t w[NWG];
                w[4 * BITS] = 0;
                if (got) {
                    const uint8_t *src = smem + L::kOffA + s1 * L::kABytes + row_local * (16 * BITS);
#pragma unroll
                    for (int i = 0; i < BITS; ++i) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(src + 16 * i);
                        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
                    }
                }
                const bool ready = got && warp_wait(&empty[s0], ph0 ^ 1, abort);
                // every unpack thread has its row in registers before any code overwrites the
                // tile; the barrier also votes, so that the four warps stop together when a wait
                // gave up (a warp that left alone would strand the others at the next barrier)
                if (unpack_bar_any(!ready)) goto u_done;
                static_for<2>([&](auto st_) {
                    constexpr int st = decltype(st_)::value;
                    const uint32_t s = st == 0 ? s0 : s1;
                    const uint32_t base = a_base + s * L::kABytes;
                    static_for<8>([&](auto c_) {
                        constexpr int c = decltype(c_)::value;
                        uint32_t o[4];
                        unpack_pairs<BITS, st * 8 + c, 1>(w, o);
                        st_shared_v4(base + sw128_offset(row_local, c), o[0], o[1], o[2], o[3]);
                    });
                    // the MMA reads the tile through the async proxy
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[s]);
                });
            }
            if (p.rank > 0) {
                // low-rank unit: A[n][k] = L2[k mod rank][n] for k < 2 rank (both halves of
                // [t_hi | t_lo] meet the same L2), zero beyond; from the shared-memory tile when
                // it came by TMA, else straight from global memory
                if (p.l_tma && !warp_wait(l_full, lph, abort)) goto u_done;
                for (int st = 0; st < nlr; ++st, ++q) {
                    const uint32_t s = q % S, ph = (q / S) & 1;
                    if (!warp_wait(&empty[s], ph ^ 1, abort)) goto u_done;
                    const uint32_t base = a_base + s * L::kABytes;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = st * kTcBK + c * 8 + 2 * e;
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
                            o[e] = v;
                        }
                        st_shared_v4(base + sw128_offset(row_local, c), o[0], o[1], o[2], o[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[s]);
                }
                if (p.l_tma) {
                    // the L2 tile is read: release it to the next tile's copy (generic reads before
                    // the next async-proxy write)
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(l_empty);
                    lph ^= 1;
                }
            }
        }
    u_done:;
    } else {
        regs_inc<kTcRegsPromote>();
        // ---------------------------------------------------------- promotion + epilogue
        const int quarter = warp & 3;
        const int colh = (warp - 8) >> 2;                          // which TT/2 token columns
        const int row_local = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        constexpr int kPre = 4;                                     // scale prefetch distance
        uint32_t unit = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int mt = tile / p.tiles_n, nt = tile % p.tiles_n;
            const int64_t n = (int64_t)nt * kTcBW + row_local;
            const bool row_ok = n < p.N;
            const float *srow = p.scales + (row_ok ? n : 0) * (int64_t)G;
            float sq[kPre];
#pragma unroll
            for (int i = 0; i < kPre; ++i) sq[i] = (row_ok && i < G) ? __ldg(srow + i) : 0.0f;
            float R[kHalf];
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
                const uint32_t t_addr = tmem + lane_addr + tb * 256u + colh * kHalf;
                // this warp's kHalf columns in chunks of 32 (then one chunk of the remaining
                // multiple of 8); T is handed back once the last chunk is in registers
                constexpr int kFull = kHalf / 32, kRest = kHalf % 32, kChunks = kFull + (kRest ? 1 : 0);
                static_for<kChunks>([&](auto hc) {
                    constexpr int hf = decltype(hc)::value;
                    constexpr int width = hf < kFull ? 32 : kRest;
                    uint32_t tv[32];
                    if constexpr (width == 32) {
                        tmem_ld_32x32b_x32(t_addr + 32 * hf, tv);
                    } else {
#pragma unroll
                        for (int e = 0; e < width / 8; ++e) tmem_ld_32x32b_x8(t_addr + 32 * hf + 8 * e, tv + 8 * e);
                    }
                    tmem_wait_ld();
                    if (hf == kChunks - 1) {
                        // all of this warp's T columns are in registers: hand the buffer back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&t_empty[tb]);
                    }
                    if (u == 0) {
#pragma unroll
                        for (int i = 0; i < width; ++i) R[32 * hf + i] = __uint_as_float(tv[i]) * s;
                    } else {
#pragma unroll
                        for (int i = 0; i < width; i += 2)
                            ffma2(R[32 * hf + i], R[32 * hf + i + 1], __uint_as_float(tv[i]), __uint_as_float(tv[i + 1]),
                                  s, s, R[32 * hf + i], R[32 * hf + i + 1]);
                    }
                });
            }
            // ------------------------------------------------------ epilogue
            if (row_ok) {
                const float bn = p.bias ? bf16_bits_to_f32(__ldg(p.bias + n)) : 0.0f;
                const int64_t m0 = (int64_t)mt * TT + colh * kHalf;
#pragma unroll
                for (int j = 0; j < kHalf; ++j) {
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
// x is read once, at close to HBM rate; tensor cores via mma.m16n8k16.
// grid (ceil(M/64), KS) with clusters of KS (<= 16) CTAs along K; a CTA owns 64 tokens (4
// warps x 16) and 1/KS of K, which it streams in 64-k blocks through a ring of kPreStages
// stages: per stage one TMA tile of x (64 tokens x 64 k, 128-byte swizzle) and one of L1
// (64 k x R), 4 or 6 stages. Thread 0 refills a stage once the four warps have released it. The A
// fragments come from the x tile with ldmatrix, the B fragments from the L1 tile with
// ldmatrix.trans; the KS partial sums are added through distributed shared memory.
constexpr int kPreMaxKS = 16;

template <int R> struct PreLayout {
    static constexpr int kStages = R > 32 ? 4 : 6;                  // two CTAs per SM
    static constexpr uint32_t kXBytes = 64 * 64 * 2;               // 8 KB, 1024-aligned
    static constexpr uint32_t kLBytes = 64 * R * 2;                // 2..8 KB
    static constexpr uint32_t kStageBytes = kXBytes + ((kLBytes + 1023) / 1024) * 1024;
    static constexpr uint32_t kOffPart = kStages * kStageBytes;    // [64][R] fp32
    static constexpr uint32_t kOffBar = kOffPart + 64 * R * 4;     // full[S], empty[S], abort
    static constexpr uint32_t kBytes = kOffBar + 2 * kStages * 8 + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;              // room to align the base to 1024
};

template <int R>
__global__ void __launch_bounds__(128)
lowrank_prepass_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap l1_map,
                       uint16_t *__restrict__ t, int64_t M, int64_t K) {
    using L = PreLayout<R>;
    constexpr int S = L::kStages;
    extern __shared__ __align__(1024) uint8_t pre_raw[];
    uint8_t *smem = pre_raw + ((1024u - (smem_u32(pre_raw) & 1023u)) & 1023u);   // 1024-aligned for the swizzle
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const uint32_t KS = gridDim.y, split = cluster_ctarank();
    const int64_t m0 = (int64_t)blockIdx.x * 64;
    const int64_t nkb = K / 64;
    const int kb0 = (int)(nkb * split / KS), kb1 = (int)(nkb * (split + 1) / KS);
    const int nb = kb1 - kb0;
    float *part = reinterpret_cast<float *>(smem + L::kOffPart);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar), *empty = full + S;
    volatile int *abort = reinterpret_cast<int *>(empty + S);
    grid_launch_dependents();                           // the consumer of t waits for this grid's end

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 4);
        }
        *abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&x_map);
        tma_prefetch_desc(&l1_map);
    }
    __syncthreads();
    // block i of the share -> stage i % S (thread 0)
    auto issue = [&](int i) {
        const uint32_t s = (uint32_t)(i % S);
        uint8_t *st = smem + s * L::kStageBytes;
        mbar_arrive_expect_tx(&full[s], L::kXBytes + L::kLBytes);
        tma_load_2d(st, &x_map, &full[s], (kb0 + i) * 64, (int32_t)m0);
        tma_load_2d(st + L::kXBytes, &l1_map, &full[s], 0, (kb0 + i) * 64);
    };
    if (tid == 0)
        for (int i = 0; i < S - 1 && i < nb; ++i) issue(i);

    float acc[R / 8][4];
#pragma unroll
    for (int j = 0; j < R / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    // ldmatrix row of this lane: A (x tile, swizzled): token 16 warp + (lane & 15), chunk half
    // lane >> 4; B (L1 tile): k row (lane & 7) + 8 ((lane >> 3) & 1), column block lane >> 4
    const uint32_t a_row = (uint32_t)(warp * 16 + (lane & 15)), a_half = (uint32_t)(lane >> 4);
    const uint32_t b_row = (uint32_t)((lane & 7) + 8 * ((lane >> 3) & 1)), b_col = (uint32_t)(lane >> 4);
    bool ok = true;
    for (int i = 0; i < nb; ++i) {
        if (tid == 0 && i + S - 1 < nb) {
            // stage (i - 1) % S is free once all four warps have released block i - 1
            const int j = i + S - 1;
            if (j >= S && !mbar_wait(&empty[j % S], (uint32_t)((j / S) - 1) & 1u, abort)) ok = false;
            if (ok) issue(j);
        }
        const uint32_t s = (uint32_t)(i % S);
        if (!warp_wait(&full[s], (uint32_t)(i / S) & 1u, abort)) { ok = false; break; }
        const uint32_t xs = smem_u32(smem + s * L::kStageBytes), ls = xs + L::kXBytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t a0, a1, a2, a3;
            const uint32_t aaddr = xs + sw128_offset(a_row, 2u * ks + a_half);
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3) : "r"(aaddr));
#pragma unroll
            for (int jt = 0; jt < R / 8; jt += 2) {
                uint32_t b0, b1, b2, b3;
                const uint32_t col = (uint32_t)jt * 8u + b_col * 8u;
                const uint32_t baddr = ls + ((uint32_t)(16 * ks) + b_row) * (R * 2u) + 2u * (col < (uint32_t)R ? col : (uint32_t)jt * 8u);
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3) : "r"(baddr));
                mma_16816_bf16(acc[jt], a0, a1, a2, a3, b0, b1);
                if (jt + 1 < R / 8) mma_16816_bf16(acc[jt + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);          // this warp has read the stage
    }
    if (!ok && tid == 0) {
        // gave up: let the copies already issued land before the shared memory is released
        for (int i = 0; i < nb && i < S; ++i) {
            int local = 0;
            (void)mbar_wait(&full[(nb - 1 - i) % S], (uint32_t)((nb - 1 - i) / S) & 1u, &local, 50ull * 1000ull * 1000ull);
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
        // the KS partials in rank order, loaded four at a time
        float v = 0.0f;
        for (int r0 = 0; r0 < (int)KS; r0 += 4) {
            float pv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
                pv[r] = r0 + r < (int)KS ? ld_cluster_f32(map_cluster_smem(base + 4u * e, (uint32_t)(r0 + r))) : 0.0f;
#pragma unroll
            for (int r = 0; r < 4; ++r) v += pv[r];
        }
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
