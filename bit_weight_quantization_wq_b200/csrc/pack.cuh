// pack.cuh -- quantize + pack kernel (KP).
//
// Per-group(128) symmetric quantization and multi-bit packing, per the Per-group(128)
// mixed-precision article (Wan-Dancer-14B), sec. 3.1 (abs_max * 1.01, step = 2 abs_max /
// (2^b - 1), q = round(w / step) clamped) and sec. 3.3 (code = q + 2^(b-1), 8 codes ->
// b bytes, first code in the most significant bits).
//
// Layout: the W rows are contiguous 128-element groups, so group G = n * (K/128) + g sits
// at bf16 offset 128 G, its packed bytes at 16*b*G and its scale at G. The kernel is a flat
// grid-stride loop over groups: four lanes own one group, each lane 32 consecutive weights
// (64 bytes) and therefore exactly 4*b output bytes (b whole words). A warp takes 16 groups
// at a time (pack_block); quantize_pack_many_kernel runs the same blocks over the groups of
// up to 64 tensors of one width, one launch for all of them.
//
// The kernel is HBM-bound only if it stays under ~8 instructions per weight, so every step
// is chosen for its instruction count:
//   * abs_max: bf16x2 max of magnitudes (max.xorsign.abs) over the lane's 16 words, then
//     two shuffles across the group's four lanes;
//   * step = RN(2s / (2^b - 1)) by one-correction division with the correctly rounded
//     constant y = RN(1/L): q0 = RN(2s y), r = 2s - L q0 (exact by fma),
//     step = RN(q0 + r y). This is Markstein's correction step; it was checked to equal the
//     IEEE quotient for every bf16 abs_max whose 2s lies in [2^-120, 2^120] and every L in
//     {7, 15, 31, 63, 127}. Outside that range the kernel divides.
//   * quantize two weights per instruction with the packed fp32 pair operations of sm_100
//     (mul/add/sub .f32x2);
//   * codes are formed by the fp32 adder itself (see "Codes" below) and packed with shifts,
//     byte permutes and one 16-byte (4-bit) or b 4-byte stores per lane.
//
// Exactness: q must equal round_half_even(fl32(w / step)). The kernel multiplies by the
// correctly rounded reciprocal and recomputes with an IEEE division only when the product
// lies within 4e-5 of a half-integer. Why that suffices: with inv = RN(1/step),
// r' = RN(w * inv) = (w/step)(1 + d1)(1 + d2), |d1|, |d2| <= 2^-24, while
// RN(w / step) = (w/step)(1 + d3). For |w/step| < 64 (always true, b <= 7) the two differ
// by less than 64 * 3 * 2^-24 < 1.2e-5, so outside the 4e-5 window both round to the same
// integer.
//
// Codes: for a weight pair (a, b) = elements (2i, 2i+1), t_a = RN(r_a + 1.5 * 2^23) and
// t_b = RN(r_b + 2^23 + o (2^b + 1)), o = 2^(b-1). Both constants are even and both sums lie
// in [2^23, 2^24), where fp32 spacing is 1, so each add rounds r to the nearest integer with
// ties to even: t_a = 1.5 * 2^23 + q_a, t_b = 2^23 + o (2^b + 1) + q_b exactly. Then
// fma(t_a - 1.5 * 2^23, 2^b, t_b) = 2^23 + (q_a + o) 2^b + (q_b + o) is exact, so the low 2b
// mantissa bits of that float are the two codes, first code high: the pair field of the
// MSB-first bitstream.
//
// Clamp: the page clamps q to +-(2^(b-1) - 1). The clamp never binds: |w| <= abs_max and
// abs_max / step <= (2^b - 1) / 2.02 (1 + 2^-22) < 2^(b-1) - 1/2 for b = 3..7, so |q| <=
// 2^(b-1) - 1 always (checked for every bf16 abs_max on the CPU). The kernel therefore has
// no clamp. Weights must be finite; a group holding inf or NaN gets unspecified codes.
#pragma once

#include "common.cuh"

namespace wq {

constexpr int kPackThreads = 128;       // with 6 CTAs per SM (<= 80 registers): 24 warps of loads in flight
constexpr int kPackUnroll = 2;          // 8-group blocks per warp per loop iteration
constexpr int kPackGroupsPerWarp = 8 * kPackUnroll;

__device__ __forceinline__ uint32_t bf16x2_maxabs(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2(float a, float b) {
    return (uint64_t)__float_as_uint(a) | ((uint64_t)__float_as_uint(b) << 32);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// abs_max of the group held by four consecutive lanes (32 bf16 weights, as 16 words, each):
// a bf16x2 max-of-magnitudes tree, then two shuffles across the four lanes.
__device__ __forceinline__ float group_abs_max(const uint32_t (&w)[16]) {
    uint32_t m8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m8[i] = bf16x2_maxabs(w[2 * i], w[2 * i + 1]);
#pragma unroll
    for (int i = 0; i < 4; ++i) m8[i] = bf16x2_maxabs(m8[i], m8[i + 4]);
    m8[0] = bf16x2_maxabs(m8[0], m8[2]);
    m8[1] = bf16x2_maxabs(m8[1], m8[3]);
    const uint32_t m2 = bf16x2_maxabs(m8[0], m8[1]) & 0x7FFF7FFFu;
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
    return __uint_as_float(m << 16);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// step = RN(2 RN(abs_max * 1.01) / (2^b - 1)) of one group (see the header comment).
template <int BITS>
__device__ __forceinline__ float group_step(float abs_max) {
    constexpr float kL = (float)((1 << BITS) - 1);
    constexpr float kInvL = 1.0f / kL;                              // RN(1/L), folded by the compiler
    const float two = __fmul_rn(2.0f, __fmul_rn(abs_max, 1.01f));
    if (two >= 7.52316384526264e-37f && two <= 1.329227995784916e36f) {   // [2^-120, 2^120]
        const float q0 = __fmul_rn(two, kInvL);
        const float r = __fmaf_rn(-q0, kL, two);
        return __fmaf_rn(r, kInvL, q0);
    }
    return __fdiv_rn(two, kL);
}

template <int BITS>
__host__ __device__ constexpr int pack_stage_words() { return BITS == 4 ? 1 : kPackGroupsPerWarp * 4 * BITS; }

// One warp quantizes and packs the kPackGroupsPerWarp groups [g0, g0 + 16) of one tensor
// (groups at or past n_groups are skipped). Widths other than 4 write each lane's b words
// either straight to memory (DIRECT: b 4-byte stores per lane, which the L2 merges into
// whole lines) or through stage_w, the warp's pack_stage_words<BITS>() words of shared
// memory (16-byte aligned), as 16-byte stores; the staged form needs fewer registers.
template <int BITS, bool DIRECT>
__device__ __forceinline__ void pack_block(const uint16_t *__restrict__ W, int64_t n_groups,
                                           uint8_t *__restrict__ packed, float *__restrict__ scales,
                                           int64_t g0, uint32_t *stage_w, int lane) {
    constexpr int kOff = 1 << (BITS - 1);
    constexpr int kGroupBytes = 16 * BITS;
    constexpr int U = kPackUnroll;
    constexpr int GW = kPackGroupsPerWarp;
    constexpr float kMagicA = 12582912.0f;                          // 1.5 * 2^23
    constexpr float kMagicB = 8388608.0f + (float)(kOff * ((1 << BITS) + 1));
    constexpr float kPow = (float)(1 << BITS);
    constexpr uint32_t kMask2 = (1u << (2 * BITS)) - 1u;
    const int gi = lane >> 2, l4 = lane & 3;

    uint32_t w[U][16];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t g = g0 + 8 * u + gi;
        const uint16_t *src = W + g * 128 + l4 * 32;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = (g < n_groups) ? ldg_nc_v4(src + 8 * i) : make_uint4(0, 0, 0, 0);
            w[u][4 * i] = v.x; w[u][4 * i + 1] = v.y; w[u][4 * i + 2] = v.z; w[u][4 * i + 3] = v.w;
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t g = g0 + 8 * u + gi;
        // ---- abs_max of the group (bf16 magnitudes; the max tree keeps only |.|), then the step
        const float step = group_step<BITS>(group_abs_max(w[u]));
        float inv = (step == 0.0f) ? 0.0f : __frcp_rn(step);
        bool near = !(inv <= 3.402823466e38f);           // 1/step overflowed: divide always
        if (near) inv = 0.0f;
        // ---- quantize, two weights per instruction
        const uint64_t inv2 = f2(inv, inv), magic = f2(kMagicA, kMagicB);
        // pair fields: the low 2b bits of F[i] = code(2i) << b | code(2i+1)
        uint32_t F[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint64_t x2 = (uint64_t)(w[u][i] << 16) | ((uint64_t)(w[u][i] & 0xFFFF0000u) << 32);
            const uint64_t r2 = mul2(x2, inv2);
            const uint64_t t2 = add2(r2, magic);
            const uint64_t q2 = sub2(t2, magic);
            const uint64_t e2 = sub2(r2, q2);
            near |= (fabsf(f2_lo(e2)) > 0.49996f) | (fabsf(f2_hi(e2)) > 0.49996f);
            F[i] = __float_as_uint(__fmaf_rn(f2_lo(q2), kPow, f2_hi(t2)));
        }
        if (near) {
            // rare: a product close to a half-integer (or a huge 1/step): IEEE division
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float xa = __uint_as_float(w[u][i] << 16), xb = __uint_as_float(w[u][i] & 0xFFFF0000u);
                const float ra = (step == 0.0f) ? 0.0f : __fdiv_rn(xa, step);
                const float rb = (step == 0.0f) ? 0.0f : __fdiv_rn(xb, step);
                const float qa = __fsub_rn(__fadd_rn(ra, kMagicA), kMagicA);
                F[i] = __float_as_uint(__fmaf_rn(qa, kPow, __fadd_rn(rb, kMagicB)));
            }
        }
        if (l4 == 0 && g < n_groups) scales[g] = step;
        if constexpr (BITS == 4) {
            // a pair field is one whole byte (bits 8..22 of the float are zero)
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                o[k] = __byte_perm(__byte_perm(F[4 * k], F[4 * k + 1], 0x0040u),
                                   __byte_perm(F[4 * k + 2], F[4 * k + 3], 0x0040u), 0x5410u);
            if (g < n_groups)
                *reinterpret_cast<uint4 *>(packed + g * kGroupBytes + l4 * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        } else {
            // quad fields (4 codes, 4b bits), placed into the 32b-bit stream number whose
            // most significant bits hold the first code; memory order is big-endian
            uint32_t Nw[BITS];
#pragma unroll
            for (int k = 0; k < BITS; ++k) Nw[k] = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t T = ((F[2 * j] & kMask2) << (2 * BITS)) | (F[2 * j + 1] & kMask2);
                const int o = 4 * BITS * (7 - j), wd = o / 32, sh = o % 32;
                Nw[wd] |= T << sh;
                if (sh + 4 * BITS > 32) Nw[wd + 1] |= T >> (32 - sh);
            }
            if constexpr (DIRECT) {
                if (g < n_groups) {
                    uint32_t *dst = reinterpret_cast<uint32_t *>(packed + g * kGroupBytes + l4 * 4 * BITS);
#pragma unroll
                    for (int k = 0; k < BITS; ++k) dst[k] = __byte_perm(Nw[BITS - 1 - k], 0, 0x0123u);
                }
            } else {
                uint32_t *dst = stage_w + (8 * u + gi) * 4 * BITS + l4 * BITS;
#pragma unroll
                for (int k = 0; k < BITS; ++k) dst[k] = __byte_perm(Nw[BITS - 1 - k], 0, 0x0123u);
            }
        }
    }
    if constexpr (BITS != 4 && !DIRECT) {
        __syncwarp();
        const int64_t valid = min((int64_t)GW, n_groups - g0);
        const int chunks = (int)(valid * kGroupBytes / 16);
        uint4 *out = reinterpret_cast<uint4 *>(packed + g0 * kGroupBytes);
        for (int c = lane; c < chunks; c += 32) out[c] = reinterpret_cast<const uint4 *>(stage_w)[c];
        __syncwarp();
    }
}

// One tensor: a flat grid-stride loop over its groups.
template <int BITS>
__global__ void __launch_bounds__(kPackThreads, 6)
quantize_pack_kernel(const uint16_t *__restrict__ W, int64_t n_groups,
                     uint8_t *__restrict__ packed, float *__restrict__ scales) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t warp_id = (int64_t)blockIdx.x * (kPackThreads / 32) + warp;
    const int64_t n_warps = (int64_t)gridDim.x * (kPackThreads / 32);
    for (int64_t g0 = warp_id * kPackGroupsPerWarp; g0 < n_groups; g0 += n_warps * kPackGroupsPerWarp)
        pack_block<BITS, true>(W, n_groups, packed, scales, g0, nullptr, lane);
}

// Many tensors of one width in one launch (the mixed-precision article quantizes a whole
// model tensor by tensor, each at its own width: one launch per tensor would pay a grid's
// fill and drain per tensor). Segment i's groups occupy the virtual range
// [vbegin[i], vbegin[i+1]), its group count rounded up to a multiple of kPackGroupsPerWarp,
// so a warp's block of groups never straddles two tensors.
constexpr int kPackMaxSegs = 64;
struct PackSegments {
    int n;                                   // segments in this launch, 1..kPackMaxSegs
    int64_t vbegin[kPackMaxSegs + 1];        // vbegin[n] = end of the virtual range
    int64_t n_groups[kPackMaxSegs];
    const uint16_t *W[kPackMaxSegs];
    uint8_t *packed[kPackMaxSegs];
    float *scales[kPackMaxSegs];
};

template <int BITS>
__global__ void __launch_bounds__(kPackThreads, 6)
quantize_pack_many_kernel(const __grid_constant__ PackSegments segs) {
    __shared__ __align__(16) uint32_t stage[kPackThreads / 32][pack_stage_words<BITS>()];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t warp_id = (int64_t)blockIdx.x * (kPackThreads / 32) + warp;
    const int64_t n_warps = (int64_t)gridDim.x * (kPackThreads / 32);
    const int64_t v_end = segs.vbegin[segs.n];
    // the block's segment: a warp's blocks only move forward, so its segment index (the same in
    // every lane) advances past the segments that end at or before the block
    int s = 0;
    for (int64_t v0 = warp_id * kPackGroupsPerWarp; v0 < v_end; v0 += n_warps * kPackGroupsPerWarp) {
        while (s + 1 < segs.n && segs.vbegin[s + 1] <= v0) ++s;
        pack_block<BITS, false>(segs.W[s], segs.n_groups[s], segs.packed[s], segs.scales[s], v0 - segs.vbegin[s],
                                stage[warp], lane);
    }
}


}  // namespace wq
