// pack.cuh -- quantize + pack kernel (KP).
//
// Per-group(128) symmetric quantization and multi-bit packing, per the Per-group(128)
// mixed-precision article (Wan-Dancer-14B), sec. 3.1 (abs_max * 1.01, step = 2 abs_max /
// (2^b - 1), q = round(w / step) clamped) and sec. 3.3 (code = q + 2^(b-1), 8 codes ->
// b bytes, first code in the most significant bits).
//
// Layout: the W rows are contiguous 128-element groups, so group G = n * (K/128) + g sits
// at bf16 offset 128 G, its packed bytes at 16*b*G and its scale at G. The kernel is a flat
// grid-stride loop over groups: a half-warp owns one group, each lane 8 weights (one 16-byte
// load) and therefore exactly b output bytes.
//
// Exactness: q must equal round_half_even(fl32(w / step)). The kernel multiplies by the
// correctly rounded reciprocal and recomputes with an IEEE division only when the product
// lies within 4e-5 of a half-integer. Why that suffices: with inv = RN(1/step),
// r' = RN(w * inv) = (w/step)(1 + d1)(1 + d2), |d1|, |d2| <= 2^-24, while
// RN(w / step) = (w/step)(1 + d3). For |w/step| < 64 (always true, b <= 7) the two differ
// by less than 64 * 3 * 2^-24 < 1.2e-5, so outside the 4e-5 window both round to the same
// integer. Rounding to the nearest integer uses the 1.5 * 2^23 magic constant (an fp32 add
// rounds to nearest even at that magnitude), valid for |r| < 2^22.
#pragma once

#include "common.cuh"

namespace wq {

constexpr int kPackThreads = 256;
constexpr int kPackUnroll = 4;          // group pairs per warp per loop iteration

template <int BITS>
__global__ void __launch_bounds__(kPackThreads)
quantize_pack_kernel(const uint16_t *__restrict__ W, int64_t n_groups,
                     uint8_t *__restrict__ packed, float *__restrict__ scales) {
    constexpr int kLevels = (1 << BITS) - 1;
    constexpr int kQmax = kLevels / 2;
    constexpr int kOffset = 1 << (BITS - 1);
    constexpr int kGroupBytes = 16 * BITS;
    constexpr int U = kPackUnroll;
    constexpr int kWarpBytes = 2 * U * kGroupBytes;
    constexpr float kMagic = 12582912.0f;               // 1.5 * 2^23
    constexpr int kMagicBits = 0x4B400000;
    __shared__ __align__(16) uint8_t stage[kPackThreads / 32][kWarpBytes];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane >> 4, l16 = lane & 15;
    uint8_t *st = stage[warp];
    const int64_t warp_id = (int64_t)blockIdx.x * (kPackThreads / 32) + warp;
    const int64_t n_warps = (int64_t)gridDim.x * (kPackThreads / 32);

    for (int64_t g0 = warp_id * 2 * U; g0 < n_groups; g0 += n_warps * 2 * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t g = g0 + 2 * u + half;
            v[u] = (g < n_groups) ? ldg_stream_v4(W + g * 128 + l16 * 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t g = g0 + 2 * u + half;
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            // abs_max of the group: bf16 magnitudes compare like 15-bit integers
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
            const float abs_max = __uint_as_float(m << 16);
            const float s = __fmul_rn(abs_max, 1.01f);
            const float step = __fdiv_rn(__fmul_rn(2.0f, s), (float)kLevels);
            const bool zero = (step == 0.0f);
            float inv = zero ? 0.0f : __frcp_rn(step);
            const bool slow = !(inv <= 3.402823466e38f);    // 1/step overflowed: divide always
            if (slow) inv = 0.0f;

            uint64_t stream = 0;                            // 8 codes, first code highest
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t h = (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu);
                const float x = __uint_as_float(h << 16);
                float r = __fmul_rn(x, inv);
                float t = __fadd_rn(r, kMagic);
                const float e = __fsub_rn(r, __fadd_rn(t, -kMagic));
                if (slow || fabsf(e) > 0.49996f) {
                    r = __fdiv_rn(x, step);
                    t = __fadd_rn(r, kMagic);
                }
                int q = __float_as_int(t) - kMagicBits;
                q = min(max(q, -kQmax), kQmax);
                stream = (stream << BITS) | (uint32_t)(q + kOffset);
            }
            // this lane's BITS bytes, most significant first, at its place in the group
            uint8_t *dst = st + (2 * u + half) * kGroupBytes + l16 * BITS;
            if constexpr (BITS == 4) {
                *reinterpret_cast<uint32_t *>(dst) = __byte_perm((uint32_t)stream, 0, 0x0123);
            } else {
#pragma unroll
                for (int j = 0; j < BITS; ++j) dst[j] = (uint8_t)(stream >> (8 * (BITS - 1 - j)));
            }
            if (l16 == 0 && g < n_groups) scales[g] = step;
        }
        __syncwarp();
        const int64_t valid = min((int64_t)(2 * U), n_groups - g0);
        const int chunks = (int)(valid * kGroupBytes / 16);
        uint4 *out = reinterpret_cast<uint4 *>(packed + g0 * kGroupBytes);
        for (int c = lane; c < chunks; c += 32) out[c] = reinterpret_cast<const uint4 *>(st)[c];
        __syncwarp();
    }
}

}  // namespace wq
