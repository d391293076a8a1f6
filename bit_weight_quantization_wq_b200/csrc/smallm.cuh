// smallm.cuh -- small-M quantized linear (KS): streams the packed weight at HBM rate.
//
// y = x * dequant(W)^T (+ (x L1) L2) (+ bias) for few tokens. The Per-group(128) article
// dequantizes a block's weights on the GPU (sec. 3.4) and then runs a bf16 matmul (sec.
// 5.3/5.4); for a handful of tokens that matmul only streams the weight, so this kernel
// never materializes dequant(W): it reads the packed codes once and contracts them
// directly.
//
// Structure
//   * grid (ceil(N/64), S, ceil(M / (8*NT))); a CTA owns 64 weight rows (4 warps x 16),
//     a contiguous 1/S share of the K groups and up to 8*NT tokens. The S CTAs that share
//     a row slab form one thread-block cluster and add their partial sums through
//     distributed shared memory (no global workspace, one launch).
//   * every thread issues all loads of its share of packed codes up front (up to PF groups)
//     so that each SM keeps ~100 KB of HBM reads in flight.
//   * tensor cores on the integer codes: with the row slab as the 16-row A operand of
//     mma.m16n8k16 and tokens as the 8-column B operand, a thread needs 32 consecutive codes
//     of two rows per group: exactly one contiguous 4*b-byte slice of each row's packed
//     group. Codes become bf16 by the exponent trick bf16(0x4300 | c) = 128 + c (exact for
//     c < 128), so the MMA sums (128 + 2^(b-1) + q) x; the per-group correction
//     (128 + 2^(b-1)) * sum(x) and the group's step are applied in fp32 after the group's
//     8 MMAs.
//   * the order of k inside a thread's 32-code slice is free (the same permutation is
//     applied to x when it is staged in shared memory), so codes are taken in pairs that
//     are cheap to extract: for 4 bits, nibbles 16 bits apart; for 3/5/6/7 bits, code i and
//     code i+8, which sit at the same bit phase b bytes apart.
#pragma once

#include "common.cuh"

namespace wq {

constexpr int kSmallThreads = 128;   // 4 warps
constexpr int kSmallRows = 64;       // weight rows per CTA

// chunk-local code indices of pair p (0..15) in a thread's 32-code slice
__host__ __device__ constexpr int pair_lo(int bits, int p) {
    return bits == 4 ? 8 * (p / 4) + (p % 4) : (p < 8 ? p : 16 + (p - 8));
}
__host__ __device__ constexpr int pair_hi(int bits, int p) {
    return pair_lo(bits, p) + (bits == 4 ? 4 : 8);
}
__host__ __device__ constexpr int small_prefetch(int bits) { return bits <= 4 ? 8 : 4; }

// Big-endian 32-bit window of bytes [k0, k0+4) of a little-endian word array.
template <int K0, int NW>
__device__ __forceinline__ uint32_t be32(const uint32_t (&w)[NW]) {
    constexpr int s = K0 % 4;
    constexpr uint32_t sel = (uint32_t)(s + 3) | ((uint32_t)(s + 2) << 4) |
                             ((uint32_t)(s + 1) << 8) | ((uint32_t)s << 12);
    return __byte_perm(w[K0 / 4], w[K0 / 4 + 1], sel);
}

// Code i (0..7) of a big-endian 8-code block held as hi:lo.
template <int BITS, int I>
__device__ __forceinline__ uint32_t block_code(uint32_t lo, uint32_t hi) {
    constexpr int sh = BITS * (7 - I);
    if constexpr (sh >= 32) return hi >> (sh - 32);
    else if constexpr (sh == 0) return lo;
    else return __funnelshift_r(lo, hi, sh);
}

template <int BITS, int BLK, int NW>
__device__ __forceinline__ void block_be(const uint32_t (&w)[NW], uint32_t &lo, uint32_t &hi) {
    constexpr int o = BLK * BITS;
    if constexpr (BITS == 3) {
        lo = be32<o, NW>(w) >> 8;
        hi = 0;
    } else {
        lo = be32<o + BITS - 4, NW>(w);
        hi = be32<o, NW>(w) >> (8 * (8 - BITS));
    }
}

template <int BITS, int P>
__device__ __forceinline__ uint32_t make_pair(const uint32_t (&lo)[4], const uint32_t (&hi)[4]) {
    constexpr uint32_t m = (1u << BITS) - 1;
    constexpr int i = P % 8, ba = (P < 8) ? 0 : 2;
    const uint32_t a = block_code<BITS, i>(lo[ba], hi[ba]);
    const uint32_t b = block_code<BITS, i>(lo[ba + 1], hi[ba + 1]);
    return (__byte_perm(a, b, 0x5410) & (m | (m << 16))) | 0x43004300u;
}

template <int BITS, int P = 0>
__device__ __forceinline__ void make_pairs(const uint32_t (&lo)[4], const uint32_t (&hi)[4],
                                           uint32_t (&out)[16]) {
    if constexpr (P < 16) {
        out[P] = make_pair<BITS, P>(lo, hi);
        make_pairs<BITS, P + 1>(lo, hi, out);
    }
}

// Words per 32-code slice (4*BITS bytes) plus one zero word of padding.
template <int BITS> struct Slice { static constexpr int kWords = BITS + 1; };

// 16 bf16x2 pairs (128 + code) of one 32-code slice, in pair order.
template <int BITS>
__device__ __forceinline__ void unpack_slice(const uint32_t (&w)[Slice<BITS>::kWords], uint32_t (&P)[16]) {
    if constexpr (BITS == 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            P[4 * q + 0] = ((w[q] >> 4) & 0x000F000Fu) | 0x43004300u;
            P[4 * q + 1] = (w[q] & 0x000F000Fu) | 0x43004300u;
            P[4 * q + 2] = ((w[q] >> 12) & 0x000F000Fu) | 0x43004300u;
            P[4 * q + 3] = ((w[q] >> 8) & 0x000F000Fu) | 0x43004300u;
        }
    } else {
        uint32_t lo[4], hi[4];
        block_be<BITS, 0>(w, lo[0], hi[0]);
        block_be<BITS, 1>(w, lo[1], hi[1]);
        block_be<BITS, 2>(w, lo[2], hi[2]);
        block_be<BITS, 3>(w, lo[3], hi[3]);
        make_pairs<BITS>(lo, hi, P);
    }
}

template <int BITS>
__device__ __forceinline__ void load_slice(const uint8_t *p, uint32_t (&w)[Slice<BITS>::kWords]) {
    if constexpr (BITS == 4) {
        const uint4 v = ldg_stream_v4(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BITS == 6) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const uint2 v = ldg_stream_v2(p + 8 * i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = ldg_stream_u32(p + 4 * i);
    }
    w[BITS] = 0;
}

__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct SmallMArgs {
    const uint16_t *x;        // M x K bf16
    const uint8_t *packed;    // N x K*bits/8
    const float *scales;      // N x K/128
    const uint16_t *bias;     // N or null
    const float *t;           // M x rank fp32 (x L1) or null
    const uint16_t *L2;       // rank x N bf16 or null
    uint16_t *y;              // M x N bf16
    int64_t M, N, K;
    int rank;
};

template <int NT>
__host__ __device__ constexpr size_t small_smem_bytes(int pf) {
    // xs: pf groups x (8 NT tokens) x 256 B; sx partials: pf x 8NT x 4 fp32; part: 8NT x 64 fp32
    return (size_t)pf * 8 * NT * 256 + (size_t)pf * 8 * NT * 16 + (size_t)8 * NT * kSmallRows * 4;
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kSmallThreads)
smallm_kernel(SmallMArgs a) {
    constexpr int PF = small_prefetch(BITS);
    constexpr int NTOK = 8 * NT;
    constexpr int NWD = Slice<BITS>::kWords;
    constexpr float kCorr = (float)(128 + (1 << (BITS - 1)));
    extern __shared__ __align__(16) uint8_t smem[];
    uint4 *xs = reinterpret_cast<uint4 *>(smem);                                // [PF][4][NTOK][4]
    float *sxp = reinterpret_cast<float *>(smem + (size_t)PF * NTOK * 256);     // [PF][NTOK][4]
    float *part = sxp + PF * NTOK * 4;                                          // [NTOK][64]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3;
    const uint32_t S = gridDim.y;
    const uint32_t split = cluster_ctarank();
    const int64_t n0 = (int64_t)blockIdx.x * kSmallRows;
    const int64_t m0 = (int64_t)blockIdx.z * NTOK;
    const int64_t G = a.K / 128;
    const int64_t gs = G * split / S, ge = G * (split + 1) / S;
    const int64_t row0 = n0 + warp * 16 + g, row1 = row0 + 8;
    const int64_t row_bytes = a.K * BITS / 8;

    float total[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) total[nt][i] = 0.0f;

    for (int64_t gb = gs; gb < ge; gb += PF) {
        const int nb = (int)min((int64_t)PF, ge - gb);
        // 1. issue the packed-code loads of this batch (both rows) and their scales
        uint32_t wd[PF][2][NWD];
        float sc[PF][2];
#pragma unroll
        for (int gl = 0; gl < PF; ++gl) {
            if (gl < nb) {
                const int64_t off = (gb + gl) * 16 * BITS + c * 4 * BITS;
                if (row0 < a.N) load_slice<BITS>(a.packed + row0 * row_bytes + off, wd[gl][0]);
                else for (int i = 0; i < NWD; ++i) wd[gl][0][i] = 0;
                if (row1 < a.N) load_slice<BITS>(a.packed + row1 * row_bytes + off, wd[gl][1]);
                else for (int i = 0; i < NWD; ++i) wd[gl][1][i] = 0;
                sc[gl][0] = (row0 < a.N) ? __ldg(a.scales + row0 * G + gb + gl) : 0.0f;
                sc[gl][1] = (row1 < a.N) ? __ldg(a.scales + row1 * G + gb + gl) : 0.0f;
            }
        }
        // 2. stage x for the batch in pair order; one unit = (group, token, quarter)
        const int units = nb * NTOK * 4;
        for (int u = tid; u < units; u += kSmallThreads) {
            const int gl = u / (NTOK * 4), n = (u >> 2) % NTOK, q = u & 3;
            const int64_t m = m0 + n;
            uint32_t xw[16];
            float psum = 0.0f;
            if (m < a.M) {
                const uint4 *src = reinterpret_cast<const uint4 *>(a.x + m * a.K + (gb + gl) * 128 + q * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 v = __ldg(src + i);
                    xw[4 * i] = v.x; xw[4 * i + 1] = v.y; xw[4 * i + 2] = v.z; xw[4 * i + 3] = v.w;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    psum += bf16_bits_to_f32(xw[i] & 0xFFFFu) + bf16_bits_to_f32(xw[i] >> 16);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) xw[i] = 0;
            }
            uint32_t pr[16];
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const int lo = pair_lo(BITS, p), hi = pair_hi(BITS, p);
                const uint32_t sel = ((lo & 1) ? 0x32u : 0x10u) | (((hi & 1) ? 0x76u : 0x54u) << 8);
                pr[p] = __byte_perm(xw[lo >> 1], xw[hi >> 1], sel);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                xs[((gl * 4 + j) * NTOK + n) * 4 + q] =
                    make_uint4(pr[4 * j], pr[4 * j + 1], pr[4 * j + 2], pr[4 * j + 3]);
            sxp[(gl * NTOK + n) * 4 + q] = psum;
        }
        __syncthreads();
        // 3. contract: 8 MMAs per (group, token tile), then the fp32 rescale
#pragma unroll
        for (int gl = 0; gl < PF; ++gl) {
            if (gl < nb) {
                uint32_t P0[16], P1[16];
                unpack_slice<BITS>(wd[gl][0], P0);
                unpack_slice<BITS>(wd[gl][1], P1);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 e = xs[((gl * 4 + j) * NTOK + nt * 8 + g) * 4 + c];
                        mma_16816_bf16(acc, P0[4 * j], P1[4 * j], P0[4 * j + 1], P1[4 * j + 1], e.x, e.y);
                        mma_16816_bf16(acc, P0[4 * j + 2], P1[4 * j + 2], P0[4 * j + 3], P1[4 * j + 3], e.z, e.w);
                    }
                    const float *sp0 = sxp + (gl * NTOK + nt * 8 + 2 * c) * 4;
                    const float sx0 = (sp0[0] + sp0[1]) + (sp0[2] + sp0[3]);
                    const float sx1 = (sp0[4] + sp0[5]) + (sp0[6] + sp0[7]);
                    total[nt][0] = fmaf(sc[gl][0], acc[0] - kCorr * sx0, total[nt][0]);
                    total[nt][1] = fmaf(sc[gl][0], acc[1] - kCorr * sx1, total[nt][1]);
                    total[nt][2] = fmaf(sc[gl][1], acc[2] - kCorr * sx0, total[nt][2]);
                    total[nt][3] = fmaf(sc[gl][1], acc[3] - kCorr * sx1, total[nt][3]);
                }
            }
        }
        __syncthreads();
    }

    // 4. partial sums to shared memory, [token][row]
    const int rl0 = warp * 16 + g;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int t0 = nt * 8 + 2 * c;
        part[t0 * kSmallRows + rl0] = total[nt][0];
        part[(t0 + 1) * kSmallRows + rl0] = total[nt][1];
        part[t0 * kSmallRows + rl0 + 8] = total[nt][2];
        part[(t0 + 1) * kSmallRows + rl0 + 8] = total[nt][3];
    }
    __syncthreads();
    cluster_sync();

    // 5. each CTA of the cluster reduces a share of the slab across the S partials,
    //    adds the low-rank branch and the bias, rounds once to bf16 and stores
    const int E = NTOK * kSmallRows;
    const int e0 = (int)((int64_t)E * split / S), e1 = (int)((int64_t)E * (split + 1) / S);
    const uint32_t part_addr = smem_u32(part);
    for (int e = e0 + tid; e < e1; e += kSmallThreads) {
        const int tok = e / kSmallRows, rl = e % kSmallRows;
        const int64_t m = m0 + tok, n = n0 + rl;
        float v = 0.0f;
        for (uint32_t r = 0; r < S; ++r) v += ld_cluster_f32(map_cluster_smem(part_addr + 4u * e, r));
        if (m < a.M && n < a.N) {
            if (a.rank > 0) {
                const float *tm = a.t + m * a.rank;
                float lr = 0.0f;
                for (int j = 0; j < a.rank; ++j)
                    lr = fmaf(tm[j], bf16_bits_to_f32(__ldg(a.L2 + (int64_t)j * a.N + n)), lr);
                v += lr;
            }
            if (a.bias) v += bf16_bits_to_f32(__ldg(a.bias + n));
            a.y[m * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        }
    }
    cluster_sync();
}

// t = x L1 in fp32 for few tokens: grid (M, ceil(rank/32)), 256 threads; warp w sums a
// 1/8 share of K for the 32 low-rank columns its lanes own, then the 8 shares are added.
__global__ void __launch_bounds__(256)
lowrank_small_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ L1, float *__restrict__ t,
                     int64_t K, int rank) {
    __shared__ float red[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t m = blockIdx.x;
    const int j = blockIdx.y * 32 + lane;
    const int64_t k0 = K * warp / 8, k1 = K * (warp + 1) / 8;
    float acc = 0.0f;
    if (j < rank)
        for (int64_t k = k0; k < k1; ++k)
            acc = fmaf(bf16_bits_to_f32(__ldg(x + m * K + k)), bf16_bits_to_f32(__ldg(L1 + k * rank + j)), acc);
    red[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && j < rank) {
        float s = 0.0f;
        for (int w = 0; w < 8; ++w) s += red[w][lane];
        t[m * rank + j] = s;
    }
}

}  // namespace wq
