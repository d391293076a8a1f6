// error.cuh -- quantization error table (KE): for each weight tensor, the sum over its
// weights of (w - dequant(quantize_b(w)))^2 at every width b = 3..7, and the sum of w^2.
//
// The Per-group(128) article chooses one bit width per tensor (sec. 3.2, PD-guided mixed
// precision) by minimizing sum_i ||W_i - Q_{b_i}(W_i)||_F^2 under a bits-per-weight budget;
// the search needs that error for every tensor at every candidate width (its mse_table).
// This kernel produces the table in one pass over each weight: per group the abs_max is
// shared by the five widths, and each width's codes are the ones wq_quantize_pack would store
// (the same step, the same rounding: reciprocal product, IEEE division within 4e-5 of a
// half-integer), so dequant(code) = q * step is exactly the value a dequantizing reader gets.
// The squared differences are formed and summed in fp64 (w - q*step is exact there);
// partial sums meet in fp64 atomics, so the last bits of a sum depend on the order in which
// warps finish.
#pragma once

#include "common.cuh"
#include "pack.cuh"

namespace wq {

constexpr int kErrThreads = 128;
constexpr int kErrMaxSegs = 64;
constexpr int kErrOut = 6;                 // sums per tensor: b = 3, 4, 5, 6, 7, then sum w^2

struct ErrSegments {
    int n;                                 // tensors in this launch, 1..kErrMaxSegs
    int64_t vbegin[kErrMaxSegs + 1];       // virtual group ranges, each rounded up to 8 groups
    int64_t n_groups[kErrMaxSegs];
    const uint16_t *W[kErrMaxSegs];
    double *out[kErrMaxSegs];              // kErrOut doubles each, zeroed before the launch
};

// Squared quantization error of one lane's 32 weights (16 bf16 pairs) at one width.
template <int BITS>
__device__ __forceinline__ double lane_sse(const uint32_t (&w)[16], float abs_max) {
    const float step = group_step<BITS>(abs_max);
    const float inv = (step == 0.0f) ? 0.0f : __frcp_rn(step);
    const bool huge = !(inv <= 3.402823466e38f);       // 1/step overflowed: divide always
    double sse = 0.0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float x = __uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
        const float r = huge ? 0.0f : __fmul_rn(x, inv);
        float q = __fsub_rn(__fadd_rn(r, 12582912.0f), 12582912.0f);     // nearest integer, ties to even
        if (huge || fabsf(__fsub_rn(r, q)) > 0.49996f) {
            const float rd = (step == 0.0f) ? 0.0f : __fdiv_rn(x, step);
            q = __fsub_rn(__fadd_rn(rd, 12582912.0f), 12582912.0f);
        }
        const double e = (double)x - (double)__fmul_rn(q, step);
        sse = __fma_rn(e, e, sse);
    }
    return sse;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void zero_error_outputs_kernel(const __grid_constant__ ErrSegments segs) {
    const int i = threadIdx.x;
    if (i < segs.n * kErrOut) segs.out[i / kErrOut][i % kErrOut] = 0.0;
}

// A flat grid-stride loop over the virtual group range of all the launch's tensors: a warp
// takes 8 groups at a time (four lanes per group, 32 weights per lane), keeps its sums in
// registers while it stays on one tensor and adds them to that tensor's outputs when it moves
// on (one atomic per sum per warp and tensor).
__global__ void __launch_bounds__(kErrThreads)
quant_error_many_kernel(const __grid_constant__ ErrSegments segs) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t warp_id = (int64_t)blockIdx.x * (kErrThreads / 32) + warp;
    const int64_t n_warps = (int64_t)gridDim.x * (kErrThreads / 32);
    const int64_t v_end = segs.vbegin[segs.n];
    const int gi = lane >> 2, l4 = lane & 3;
    double acc[kErrOut];
#pragma unroll
    for (int j = 0; j < kErrOut; ++j) acc[j] = 0.0;
    int cur = -1;
    auto flush = [&](int s) {
#pragma unroll
        for (int j = 0; j < kErrOut; ++j) {
            const double v = warp_sum_f64(acc[j]);
            if (lane == 0) atomicAdd(segs.out[s] + j, v);
            acc[j] = 0.0;
        }
    };
    for (int64_t v0 = warp_id * 8; v0 < v_end; v0 += n_warps * 8) {
        // the block's tensor = the number of tensors that end at or before v0 (warp-uniform)
        int s = 0;
#pragma unroll
        for (int base = 0; base < kErrMaxSegs; base += 32) {
            const int j = base + lane;
            s += __popc(__ballot_sync(0xffffffffu, j < segs.n && segs.vbegin[j + 1] <= v0));
        }
        if (s != cur) {
            if (cur >= 0) flush(cur);
            cur = s;
        }
        const int64_t g = v0 - segs.vbegin[s] + gi;
        const bool ok = g < segs.n_groups[s];
        uint32_t w[16];
        const uint16_t *src = segs.W[s] + g * 128 + l4 * 32;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = ok ? ldg_nc_v4(src + 8 * i) : make_uint4(0, 0, 0, 0);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
        const float am = group_abs_max(w);
        acc[0] += lane_sse<3>(w, am);
        acc[1] += lane_sse<4>(w, am);
        acc[2] += lane_sse<5>(w, am);
        acc[3] += lane_sse<6>(w, am);
        acc[4] += lane_sse<7>(w, am);
        double sq = 0.0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const double x = (double)__uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
            sq = __fma_rn(x, x, sq);
        }
        acc[5] += sq;
    }
    if (cur >= 0) flush(cur);
}

}  // namespace wq
