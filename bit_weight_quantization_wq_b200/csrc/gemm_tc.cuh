// gemm_tc.cuh -- large-M fused dequant-GEMM on the 5th-generation tensor cores (KL).
//
//   y = x * dequant(W)^T + (x L1) L2 + bias
//
// The Per-group(128) article dequantizes each block's weights on the GPU (sec. 3.4) and
// then runs a bf16 matmul, noting it has no low-bit matmul kernel (sec. 5.3, 5.4); the
// SVDQuant article adds a 16-bit low-rank branch computed next to the quantized residual
// ("Technical principles", "Engineering highlights"). Here the dequantization happens in
// registers inside the GEMM: the bf16 weight is never written to global memory.
//
// One persistent CTA per SM walks 256 x 256 output tiles (256 tokens x 256 weight rows).
// Warp roles (384 threads):
//   warp 0     TMA producer of x tiles (256 tokens x 64 k bf16, 128B-swizzled, 32 KB/stage)
//   warp 1     TMEM allocator and the single MMA-issuing thread: per 64-k stage, 4 k-steps of
//              two tcgen05.mma M=128 N=256 K=16 (one per token half) into two fp32 TMEM
//              accumulators (2 x 256 columns = all 512)
//   warp 2     TMA producer of packed-weight tiles (256 rows x one 128-code group)
//   warps 4-11 dequantizers, one weight row per thread: unpack 8 codes at a time from the
//              packed tile, dequantize in fp32 ((code - 2^(b-1)) * step as one FMA on the
//              exponent-trick value 1 + code/128), round to bf16 and store the 128B-swizzled
//              K-major B operand the MMA reads; after the k loop they run the epilogue
//              (tcgen05.ld, + bias, round to bf16, store y).
// Low-rank branch: y = [x, t] [deq(W)^T ; L2] with t = bf16(x L1) (M x rank, computed by
// lowrank_prepass_kernel), so it is one more k stage into the same accumulators.
//
// Every wait is bounded (see common.cuh). On a timeout the roles stop, the producers wait
// (bounded) for their copies in flight, the MMA thread for its MMAs, and TMEM is freed.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "smallm.cuh"

namespace wq {

constexpr int kTcBM = 256;
constexpr int kTcBN = 256;
constexpr int kTcBK = 64;
constexpr int kTcStagesA = 3;
constexpr int kTcStagesB = 2;
constexpr int kTcStagesP = 2;
constexpr int kTcThreads = 384;
constexpr int kTcFirstDequantWarp = 4;
constexpr int kTcDequantWarps = 8;
constexpr uint32_t kTcTmemCols = 512;
constexpr int kTStride = 64;              // row stride (elements) of the low-rank t buffer

template <int BITS>
struct TcLayout {
    static constexpr uint32_t kABytes = kTcBM * kTcBK * 2;
    static constexpr uint32_t kBBytes = kTcBN * kTcBK * 2;
    static constexpr uint32_t kPBytes = kTcBN * 16 * BITS;
    static constexpr uint32_t kOffA = 0;
    static constexpr uint32_t kOffB = kOffA + kTcStagesA * kABytes;
    static constexpr uint32_t kOffP = kOffB + kTcStagesB * kBBytes;
    static constexpr uint32_t kOffBar = kOffP + kTcStagesP * kPBytes;
    static constexpr uint32_t kNumBars = 2 * kTcStagesA + 2 * kTcStagesB + 2 * kTcStagesP + 3;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kBytes = kOffMisc + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;     // slack to align the base to 1024 B
};

struct TcParams {
    const float *scales;      // N x K/128
    const uint16_t *L2;       // rank x N bf16 or null
    const uint16_t *bias;     // N bf16 or null
    uint16_t *y;              // M x N bf16
    int64_t M, N, K;
    int rank;
    int tiles_m, tiles_n;
};

template <int I> struct Int { static constexpr int value = I; };
template <int N, int I = 0, class F>
__device__ __forceinline__ void static_for(F &&f) {
    if constexpr (I < N) {
        f(Int<I>{});
        static_for<N, I + 1>(f);
    }
}

// Big-endian 8-code block BLK (b bytes at byte offset BLK*b) of a group held as words.
template <int BITS, int BLK, int NW>
__device__ __forceinline__ void tc_block_be(const uint32_t (&w)[NW], uint32_t &lo, uint32_t &hi) {
    constexpr int o = BLK * BITS;
    if constexpr (BITS == 3) {
        lo = be32<o, NW>(w) >> 8;
        hi = 0;
    } else if constexpr (BITS == 4) {
        lo = be32<o, NW>(w);
        hi = 0;
    } else {
        lo = be32<o + BITS - 4, NW>(w);
        hi = be32<o, NW>(w) >> (8 * (8 - BITS));
    }
}

// Code I of a big-endian block as the fp32 value 1 + code/128 (code placed at mantissa bit 16).
template <int BITS, int I>
__device__ __forceinline__ float tc_code_f32(uint32_t lo, uint32_t hi) {
    constexpr int sh = BITS * (7 - I);
    constexpr uint32_t m = ((1u << BITS) - 1u) << 16;
    uint32_t v;
    if constexpr (sh >= 48) v = hi >> (sh - 48);
    else if constexpr (sh >= 16) v = __funnelshift_r(lo, hi, sh - 16);
    else v = lo << (16 - sh);
    return __uint_as_float((v & m) | 0x3F800000u);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// All 32 lanes wait on a barrier phase; the give-up decision is taken by lane 0 so that the
// warp leaves together.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    const int lane = threadIdx.x & 31;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const bool ok = mbar_try_wait(bar, parity);
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

template <int BITS>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_linear_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap p_map,
                 const __grid_constant__ CUtensorMap t_map, const TcParams p) {
    using L = TcLayout<BITS>;
    constexpr int SA = kTcStagesA, SB = kTcStagesB, SP = kTcStagesP;
    constexpr int kHalf = 1 << (BITS - 1);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *a_full = bars, *a_empty = a_full + SA;
    uint64_t *b_full = a_empty + SA, *b_empty = b_full + SB;
    uint64_t *p_full = b_empty + SB, *p_empty = p_full + SP;
    uint64_t *acc_full = p_empty + SP, *acc_empty = acc_full + 1, *drain = acc_empty + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < SA; ++i) { mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 1); }
        for (int i = 0; i < SB; ++i) { mbar_init(&b_full[i], kTcDequantWarps); mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < SP; ++i) { mbar_init(&p_full[i], 1); mbar_init(&p_empty[i], kTcDequantWarps); }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kTcDequantWarps);
        mbar_init(drain, 1);
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

    const int KBm = (int)(p.K / kTcBK);              // k stages of the quantized weight
    const int KB = KBm + (p.rank > 0 ? 1 : 0);       // + the low-rank stage
    const int G = (int)(p.K / 128);
    const int tiles = p.tiles_m * p.tiles_n;

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------- x / t producer
        tma_prefetch_desc(&x_map);
        tma_prefetch_desc(&t_map);
        int armed[SA];
        for (int i = 0; i < SA; ++i) armed[i] = -1;
        uint32_t s = 0, ph = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int mt = tile % p.tiles_m;
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(&a_empty[s], ph ^ 1, abort)) goto a_done;
                mbar_arrive_expect_tx(&a_full[s], L::kABytes);
                armed[s] = (int)ph;
                uint8_t *dst = smem + L::kOffA + s * L::kABytes;
                if (kb < KBm) tma_load_2d(dst, &x_map, &a_full[s], kb * kTcBK, mt * kTcBM);
                else tma_load_2d(dst, &t_map, &a_full[s], 0, mt * kTcBM);
                if (++s == SA) { s = 0; ph ^= 1; }
            }
        }
    a_done:
        for (int i = 0; i < SA; ++i) {
            int local = 0;
            if (armed[i] >= 0) (void)mbar_wait(&a_full[i], (uint32_t)armed[i], &local);
        }
    } else if (warp == 2 && lane == 0) {
        // ---------------------------------------------------------- packed-weight producer
        tma_prefetch_desc(&p_map);
        int armed[SP];
        for (int i = 0; i < SP; ++i) armed[i] = -1;
        uint32_t s = 0, ph = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int nt = tile / p.tiles_m;
            for (int g = 0; g < G; ++g) {
                if (!mbar_wait(&p_empty[s], ph ^ 1, abort)) goto p_done;
                mbar_arrive_expect_tx(&p_full[s], L::kPBytes);
                armed[s] = (int)ph;
                tma_load_2d(smem + L::kOffP + s * L::kPBytes, &p_map, &p_full[s], g * 16 * BITS, nt * kTcBN);
                if (++s == SP) { s = 0; ph ^= 1; }
            }
        }
    p_done:
        for (int i = 0; i < SP; ++i) {
            int local = 0;
            if (armed[i] >= 0) (void)mbar_wait(&p_full[i], (uint32_t)armed[i], &local);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = umma_idesc_bf16(128, kTcBN);
        uint32_t sa = 0, pa = 0, sb = 0, pb = 0, acc_ph = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            if (!mbar_wait(acc_empty, acc_ph ^ 1, abort)) goto m_done;
            acc_ph ^= 1;
            tc_fence_after();
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(&a_full[sa], pa, abort)) goto m_done;
                if (!mbar_wait(&b_full[sb], pb, abort)) goto m_done;
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + L::kOffA + sa * L::kABytes);
                const uint32_t b_base = smem_u32(smem + L::kOffB + sb * L::kBBytes);
                const int nk = (kb < KBm) ? kTcBK / 16 : p.rank / 16;
                for (int k = 0; k < nk; ++k) {
                    const uint64_t bd = umma_desc_sw128(b_base + k * 32, 1024);
                    const uint64_t ad0 = umma_desc_sw128(a_base + k * 32, 1024);
                    const uint64_t ad1 = umma_desc_sw128(a_base + 128 * 128 + k * 32, 1024);
                    const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
                    umma_bf16(tmem, ad0, bd, idesc, acc);
                    umma_bf16(tmem + kTcBN, ad1, bd, idesc, acc);
                }
                umma_commit(&a_empty[sa]);
                umma_commit(&b_empty[sb]);
                if (++sa == SA) { sa = 0; pa ^= 1; }
                if (++sb == SB) { sb = 0; pb ^= 1; }
            }
            umma_commit(acc_full);
        }
    m_done:
        {
            // every MMA issued by this thread completes before TMEM is released
            umma_commit(drain);
            int local = 0;
            (void)mbar_wait(drain, 0, &local);
        }
    } else if (warp >= kTcFirstDequantWarp) {
        // ---------------------------------------------------------- dequant + epilogue
        const int e = warp - kTcFirstDequantWarp;
        const int nl = e * 32 + lane;                    // weight row inside the tile
        const int quarter = warp & 3;                    // TMEM lanes this warp may access
        const int half = e >> 2;                         // token half = accumulator
        uint32_t sp = 0, pp = 0, sb = 0, pb = 0, acc_ph = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            const int mt = tile % p.tiles_m, nt = tile / p.tiles_m;
            const int64_t n = (int64_t)nt * kTcBN + nl;
            const bool row_ok = n < p.N;
            const float *srow = p.scales + (row_ok ? n : 0) * (int64_t)G;
            float step_next = row_ok ? __ldg(srow) : 0.0f;
            for (int g = 0; g < G; ++g) {
                const float step = step_next;
                if (g + 1 < G) step_next = row_ok ? __ldg(srow + g + 1) : 0.0f;
                if (!warp_wait(&p_full[sp], pp, abort)) goto d_done;
                uint32_t w[4 * BITS + 1];
                {
                    const uint4 *src = reinterpret_cast<const uint4 *>(smem + L::kOffP + sp * L::kPBytes + nl * 16 * BITS);
#pragma unroll
                    for (int i = 0; i < BITS; ++i) {
                        const uint4 v = src[i];
                        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
                    }
                    w[4 * BITS] = 0;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_empty[sp]);
                if (++sp == SP) { sp = 0; pp ^= 1; }
                // dequant = (c - 2^(b-1)) * step = f * S - T with f = 1 + c/128, S = 128 step
                const float S = __fmul_rn(step, 128.0f);
                const float T = __fmul_rn(S, 1.0f + (float)kHalf / 128.0f);
                const int sw = nl & 7;
                bool ok = true;
                static_for<2>([&](auto hh) {
                    constexpr int h = decltype(hh)::value;
                    if (!ok) return;
                    if (!warp_wait(&b_empty[sb], pb ^ 1, abort)) { ok = false; return; }
                    uint8_t *row = smem + L::kOffB + sb * L::kBBytes + (nl >> 3) * 1024 + (nl & 7) * 128;
                    static_for<8>([&](auto cc) {
                        constexpr int c = decltype(cc)::value;
                        uint32_t lo, hi;
                        tc_block_be<BITS, 8 * h + c>(w, lo, hi);
                        float f[8];
                        static_for<8>([&](auto ii) {
                            constexpr int i = decltype(ii)::value;
                            f[i] = fmaf(tc_code_f32<BITS, i>(lo, hi), S, -T);
                        });
                        uint4 o;
                        o.x = pack_bf16x2(f[0], f[1]);
                        o.y = pack_bf16x2(f[2], f[3]);
                        o.z = pack_bf16x2(f[4], f[5]);
                        o.w = pack_bf16x2(f[6], f[7]);
                        *reinterpret_cast<uint4 *>(row + ((c ^ sw) << 4)) = o;
                    });
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&b_full[sb]);
                    if (++sb == SB) { sb = 0; pb ^= 1; }
                });
                if (!ok) goto d_done;
            }
            if (p.rank > 0) {
                // low-rank stage: B[n][j] = L2[j][n] for j < rank, zero up to 64
                if (!warp_wait(&b_empty[sb], pb ^ 1, abort)) goto d_done;
                uint8_t *row = smem + L::kOffB + sb * L::kBBytes + (nl >> 3) * 1024 + (nl & 7) * 128;
                const int sw = nl & 7;
                for (int c = 0; c < 8; ++c) {
                    uint32_t v[4] = {0u, 0u, 0u, 0u};
                    if (row_ok && 8 * c < p.rank) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint32_t a = __ldg(p.L2 + (int64_t)(8 * c + 2 * i) * p.N + n);
                            const uint32_t b = __ldg(p.L2 + (int64_t)(8 * c + 2 * i + 1) * p.N + n);
                            v[i] = a | (b << 16);
                        }
                    }
                    *reinterpret_cast<uint4 *>(row + ((c ^ sw) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&b_full[sb]);
                if (++sb == SB) { sb = 0; pb ^= 1; }
            }
            // ------------------------------------------------------ epilogue
            if (!warp_wait(acc_full, acc_ph, abort)) goto d_done;
            acc_ph ^= 1;
            tc_fence_after();
            {
                const int64_t m = (int64_t)mt * kTcBM + half * 128 + quarter * 32 + lane;
                const bool vec = (p.N % 8) == 0;
                for (int cc = 0; cc < kTcBN / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + half * kTcBN + cc * 32, r);
                    tmem_wait_ld();
                    const int64_t nb = (int64_t)nt * kTcBN + cc * 32;
                    if (m < p.M) {
                        uint16_t *yrow = p.y + m * p.N;
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            float v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[j + i]);
                            const int64_t n0 = nb + j;
                            if (vec && n0 + 8 <= p.N) {
                                if (p.bias) {
                                    const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(p.bias + n0));
                                    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                                    for (int i = 0; i < 4; ++i) {
                                        v[2 * i] += bf16_bits_to_f32(bw[i] & 0xFFFFu);
                                        v[2 * i + 1] += bf16_bits_to_f32(bw[i] >> 16);
                                    }
                                }
                                uint4 o;
                                o.x = pack_bf16x2(v[0], v[1]);
                                o.y = pack_bf16x2(v[2], v[3]);
                                o.z = pack_bf16x2(v[4], v[5]);
                                o.w = pack_bf16x2(v[6], v[7]);
                                *reinterpret_cast<uint4 *>(yrow + n0) = o;
                            } else {
                                for (int i = 0; i < 8; ++i) {
                                    if (n0 + i < p.N) {
                                        float a = v[i];
                                        if (p.bias) a += bf16_bits_to_f32(__ldg(p.bias + n0 + i));
                                        yrow[n0 + i] = __bfloat16_as_ushort(__float2bfloat16_rn(a));
                                    }
                                }
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
        }
    d_done:;
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
// t = bf16(x L1): M x R (R = rank, 16..64), stored with a row stride of kTStride = 64
// elements (columns R..63 zero) so that one 64-wide TMA box covers a row exactly.
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
        if (m < M) t[m * kTStride + e % R] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
    if constexpr (R < kTStride) {
        // zero the padding columns so that the whole 64-wide row is defined
        constexpr int kPad = kTStride - R;
        if (split == 0) {
            for (int i = tid; i < 64 * kPad; i += 128) {
                const int64_t m = m0 + i / kPad;
                if (m < M) t[m * kTStride + R + i % kPad] = 0;
            }
        }
    }
    cluster_sync();
}

}  // namespace wq
