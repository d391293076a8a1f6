// dequant.cuh -- standalone dequantize (KD): packed codes + steps -> the bf16 weight.
//
// The Per-group(128) article's own forward path (sec. 3.4, dequantize_on_gpu): unpack the
// stored codes, subtract the offset 2^(b-1), multiply by the group's fp32 step, and hand the
// result to the layer's bf16 matmul (sec. 5.3, 5.4: there is no low-bit matmul kernel). The
// output is W_hat[n][k] = bf16(fl32(q * step)): the weight that bf16 matmul sees. The fused
// wq_linear never materializes it; this kernel is that path's dequantize step, for callers
// that want the weight itself (and for measuring the fused kernel against the two-step path).
//
// Layout as wq_quantize_pack writes it: group G of the whole matrix (row-major groups) is 16*b
// packed bytes at 16*b*G and one step at G. A flat grid-stride loop over groups, four lanes
// per group, 32 codes per lane (4*b bytes in, 64 bytes out); codes -> exact q (bf16 pairs, as
// the GEMMs' unpack) -> fp32 -> times the step -> bf16.
#pragma once

#include "common.cuh"
#include "unpack.cuh"

namespace wq {

constexpr int kDeqThreads = 256;

template <int BITS>
__global__ void __launch_bounds__(kDeqThreads)
dequantize_kernel(const uint8_t *__restrict__ packed, const float *__restrict__ scales, int64_t n_groups,
                  uint16_t *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int gi = lane >> 2, l4 = lane & 3;
    const int64_t warp_id = ((int64_t)blockIdx.x * kDeqThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kDeqThreads) >> 5;
    for (int64_t g0 = warp_id * 8; g0 < n_groups; g0 += n_warps * 8) {
        const int64_t g = g0 + gi;
        if (g >= n_groups) continue;
        // this lane's 4*b bytes: codes [32 l4, 32 l4 + 32) of the group
        const uint8_t *src = packed + g * (16 * BITS) + l4 * (4 * BITS);
        uint32_t w[BITS + 1];
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(src) + i);
        w[BITS] = 0;
        const float step = __ldg(scales + g);
        uint32_t q[16];
        unpack_pairs<BITS, 0, 4>(w, q);
        uint32_t o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float lo = __fmul_rn(__uint_as_float(q[i] << 16), step);
            const float hi = __fmul_rn(__uint_as_float(q[i] & 0xFFFF0000u), step);
            o[i] = pack_bf16x2(lo, hi);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + g * 128 + l4 * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
}

}  // namespace wq
