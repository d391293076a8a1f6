// unpack.cuh -- packed b-bit codes -> exact bf16 values of q = code - 2^(b-1), in natural
// k order, two codes per 32-bit word (the operand format of the bf16 tensor-core MMAs).
//
// Packing (Per-group(128) article, sec. 3.3): the codes of a row form one bitstream, first
// code in the most significant bits; 8 codes fill exactly b bytes, so an 8-code "block"
// starts at byte 8*j*b/8 = j*b of the stream. Codes become bf16 by the exponent trick:
// the bit pattern 0x4300 | c is the bf16 number 128 + c for c < 128, and one bf16x2
// subtraction of 128 + 2^(b-1) then gives q exactly (|q| < 64 is exact in bf16).
#pragma once

#include "common.cuh"

namespace wq {

template <int I> struct Int { static constexpr int value = I; };
template <int N, int I = 0, class F>
__device__ __forceinline__ void static_for(F &&f) {
    if constexpr (I < N) {
        f(Int<I>{});
        static_for<N, I + 1>(f);
    }
}

// Big-endian 32-bit window of bytes [K0, K0+4) of a little-endian word array.
template <int K0, int NW>
__device__ __forceinline__ uint32_t be32(const uint32_t (&w)[NW]) {
    constexpr int s = K0 % 4;
    constexpr uint32_t sel = (uint32_t)(s + 3) | ((uint32_t)(s + 2) << 4) |
                             ((uint32_t)(s + 1) << 8) | ((uint32_t)s << 12);
    return __byte_perm(w[K0 / 4], w[K0 / 4 + 1], sel);
}

// Big-endian 8-code block BLK (b bytes at byte offset BLK*b) of a stream held as words,
// returned as hi:lo with the block's last code in the low bits of lo.
template <int BITS, int BLK, int NW>
__device__ __forceinline__ void block8_be(const uint32_t (&w)[NW], uint32_t &lo, uint32_t &hi) {
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

// PTX prmt in its default mode: selector nibble bits 2:0 pick one of the 8 source bytes and
// bit 3 replaces it by copies of that byte's sign bit (zero for bytes below 0x80). The CUDA
// __byte_perm intrinsic ignores bit 3, hence the inline form.
__device__ __forceinline__ uint32_t prmt_sx(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Blocks [BLK0, BLK0 + NBLK) of a stream held as NW little-endian words -> 4*NBLK bf16x2
// words of exact q: word i holds codes 2i (low half) and 2i+1 (high half) of the range.
// The array needs one word beyond the last block's bytes (zero or anything).
template <int BITS, int BLK0, int NBLK, int NW>
__device__ __forceinline__ void unpack_pairs(const uint32_t (&w)[NW], uint32_t (&out)[4 * NBLK]) {
    constexpr uint32_t kOff = 0x43004300u;                          // bf16 128 in each half
    const __nv_bfloat162 corr = __floats2bfloat162_rn(128.0f + (1 << (BITS - 1)), 128.0f + (1 << (BITS - 1)));
    if constexpr (BITS == 4) {
        // one word per block; byte j of a word = (code 2j << 4) | code 2j+1
#pragma unroll
        for (int i = 0; i < NBLK; ++i) {
            const uint32_t v = w[BLK0 + i];
            const uint32_t hiN = (v >> 4) & 0x0F0F0F0Fu, loN = v & 0x0F0F0F0Fu;
            // (hi nibble of byte j) | (lo nibble of byte j) << 16; the sign-replicating
            // selector nibbles (8 + byte) give the zero high bytes
            const uint32_t pp[4] = {prmt_sx(hiN, loN, 0xC480u) + kOff, prmt_sx(hiN, loN, 0xD591u) + kOff,
                                    prmt_sx(hiN, loN, 0xE6A2u) + kOff, prmt_sx(hiN, loN, 0xF7B3u) + kOff};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __nv_bfloat162 t = *reinterpret_cast<const __nv_bfloat162 *>(&pp[j]);
                t = __hsub2(t, corr);
                out[4 * i + j] = *reinterpret_cast<uint32_t *>(&t);
            }
        }
    } else {
        constexpr uint32_t m = (1u << BITS) - 1u;
        static_for<NBLK>([&](auto bb) {
            constexpr int blk = decltype(bb)::value;
            uint32_t lo, hi;
            block8_be<BITS, BLK0 + blk>(w, lo, hi);
            static_for<4>([&](auto pq) {
                constexpr int pr = decltype(pq)::value;
                constexpr int sh = 2 * BITS * (3 - pr);
                uint32_t G;
                if constexpr (sh >= 32) G = hi >> (sh - 32);
                else if constexpr (sh == 0) G = lo;
                else G = __funnelshift_r(lo, hi, sh);
                // G bits [0,b) = code 2pr+1, [b,2b) = code 2pr: low half <- G >> b, high half <- G
                uint32_t r = (__byte_perm(G >> BITS, G, 0x5410u) & (m | (m << 16))) | kOff;
                __nv_bfloat162 t = *reinterpret_cast<const __nv_bfloat162 *>(&r);
                t = __hsub2(t, corr);
                out[4 * blk + pr] = *reinterpret_cast<uint32_t *>(&t);
            });
        });
    }
}

// As unpack_pairs, but each half is the bf16 value 128 + code (no subtraction): the caller
// removes (128 + 2^(b-1)) * sum(x) once per group instead of once per code pair.
//
// 4 bits: the pairs come out in a permuted k order. Byte j of a block word is
// (code 2j << 4) | code 2j+1, so one mask keeps one nibble of each 16-bit half: bits [0,4)
// and [16,20) hold codes 1 and 5, and shifts by 4, 8 and 12 bring codes (0,4), (3,7) and
// (2,6) there. Word i of the block's output holds the pair (i, i+4), which is exact bf16
// 128 + code with the constant 0x4300 in each half: three shifts and four mask-and-or
// operations per 8 codes. The x operand of the MMA then takes the same order: see
// permute_x8. Other widths return pairs in natural order (word i = codes 2i, 2i+1).
template <int BITS> struct BiasedOrder { static constexpr bool kPermuted = (BITS == 4); };

// (a & b) | c in one instruction; b and c are registers, so the two constants of the biased
// unpack do not become two immediates of two instructions.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// The two constants of the biased unpack for width BITS, held in registers: the per-half
// code mask and the bf16 exponent pattern 0x4300 in each half.
template <int BITS> struct BiasedConsts {
    uint32_t mask, one;
    __device__ __forceinline__ BiasedConsts() {
        constexpr uint32_t m = (1u << (BITS == 4 ? 4 : BITS)) - 1u;
        mask = m | (m << 16);
        one = 0x43004300u;
        asm volatile("" : "+r"(mask), "+r"(one));       // keep them in registers
    }
};

template <int BITS, int BLK0, int NBLK, int NW>
__device__ __forceinline__ void unpack_pairs_biased(const uint32_t (&w)[NW], uint32_t (&out)[4 * NBLK],
                                                    const BiasedConsts<BITS> &k) {
    if constexpr (BITS == 4) {
#pragma unroll
        for (int i = 0; i < NBLK; ++i) {
            const uint32_t v = w[BLK0 + i];
            out[4 * i + 0] = and_or(v >> 4, k.mask, k.one);     // codes 0, 4
            out[4 * i + 1] = and_or(v, k.mask, k.one);          // codes 1, 5
            out[4 * i + 2] = and_or(v >> 12, k.mask, k.one);    // codes 2, 6
            out[4 * i + 3] = and_or(v >> 8, k.mask, k.one);     // codes 3, 7
        }
    } else {
        static_for<NBLK>([&](auto bb) {
            constexpr int blk = decltype(bb)::value;
            uint32_t lo, hi;
            block8_be<BITS, BLK0 + blk>(w, lo, hi);
            static_for<4>([&](auto pq) {
                constexpr int pr = decltype(pq)::value;
                constexpr int sh = 2 * BITS * (3 - pr);
                uint32_t G;
                if constexpr (sh >= 32) G = hi >> (sh - 32);
                else if constexpr (sh == 0) G = lo;
                else G = __funnelshift_r(lo, hi, sh);
                out[4 * blk + pr] = and_or(__byte_perm(G >> BITS, G, 0x5410u), k.mask, k.one);
            });
        });
    }
}

// Eight bf16 values x0..x7 (four words, natural order) -> the order the 4-bit biased pairs
// take: words (x0, x4), (x1, x5), (x2, x6), (x3, x7).
__device__ __forceinline__ uint4 permute_x8(const uint4 v) {
    return make_uint4(__byte_perm(v.x, v.z, 0x5410u), __byte_perm(v.x, v.z, 0x7632u),
                      __byte_perm(v.y, v.w, 0x5410u), __byte_perm(v.y, v.w, 0x7632u));
}

// mma.m16n8k16, bf16 inputs, fp32 accumulate in place.
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

}  // namespace wq
