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
// groups. Inside a CTA each warp owns a block of up to four units and a range of the CTA's
// groups (when there are fewer blocks than warps, several warps share a block, each with its
// own groups), and walks it one group at a time: the x fragment of a group is loaded once
// for all units of the block, and the units' MMA chains are independent, so they interleave.
//
// Data movement: every warp streams its own groups. One ring slot holds one group of the
// block (16 rows x 16*b bytes per unit), copied with 16-byte asynchronous copies into a
// private ring of D slots in shared memory, D - 1 groups ahead of the one being computed;
// the warp waits on its own copy groups only. There is no producer warp and no barrier
// between warps until the final reduction. At the start the CTA copies into shared memory,
// once, with asynchronous copies that are in flight together with the ring's first slots:
// the token rows of x for its groups (padded stride), the steps of all its rows and groups
// and, with a low-rank branch, the L2 columns of its rows; then it sums every staged group of
// x per token.
//
// Arithmetic: thread (g, c) of a warp holds rows g and g+8 of the unit and the 32
// consecutive codes [32c, 32c+32) of the group, 4*b contiguous bytes per row. Inside one
// MMA step s the k slots it feeds are mapped to k = 32c + 4s + {0,1} and 32c + 4s + {2,3}
// (the same map on the x side), so both operands are read in natural order. Codes enter
// the MMAs as the exact bf16 values 128 + code (bit pattern 0x4300 | code); the group's
// (128 + 2^(b-1)) * sum(x), from the per-token group sums computed at the start, is
// subtracted once per item. Each
// group's fp32 product is scaled by the group's fp32 step and accumulated in fp32: the
// weight is never rounded.
//
// Reduction: warps that share a block add their partial sums in a fixed order through
// shared memory, then the S CTAs of a cluster add theirs through distributed shared memory
// (in rank order), add the low-rank branch and the bias, and round once to bf16. The
// low-rank input t = x L1 is written by a prepass launched just before this kernel; this
// kernel is launched as its programmatic dependent, streams the weight while the prepass
// runs, and waits for it only before the finish. All orders
// are fixed: the result is deterministic. The kernel has no waits on other threads' progress
// except __syncthreads and the cluster barrier, which every thread reaches.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "unpack.cuh"

namespace wq {

constexpr int kSmMaxTok = 16;                                // tokens per launch
constexpr int kTStrideSm = 128;                              // row stride of [t_hi | t_lo]
constexpr int kSmMaxRB = 4;                                  // units per warp block
constexpr int kSmMaxD = 6;                                   // ring slots per warp

template <int TOK> struct SmCfg {
    static constexpr int kWarps = 12;
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kNT = TOK / 8;                      // n8 token tiles per MMA step
    static constexpr int kCH = 2;                            // independent MMA accumulators per item
};

struct SmallMArgs {
    const uint16_t *x;        // M x K bf16
    const uint8_t *packed;    // N x K*b/8
    const float *scales;      // N x K/128
    const uint16_t *bias;     // N or null
    const uint16_t *t;        // M x 128 bf16: [t_hi | t_lo] of x L1 (rank columns each), or null
    const uint16_t *L2;       // rank x N bf16 or null
    uint16_t *y;              // M x N bf16
    int64_t M, N, K;
    int64_t row_bytes;        // K * b / 8
    int rank;
    int S;                    // CTAs per cluster (K split)
    int n_clusters;
    int RB, GW;               // units per warp block; warps per block (group splits) when blocks < warps
    int D;                    // ring slots per warp (2..kSmMaxD)
    int rows_max;             // rows of the largest cluster range (units * 16)
    int gmax;                 // groups of the largest CTA share (row stride of the staged sums and steps)
    uint32_t x_stride;        // bytes per token row of the staged x (gmax * 256 + 64)
    uint32_t slot_bytes;      // one ring slot: RB units x 16 rows x 16b bytes of codes
    uint32_t off_sx, off_st, off_ring, off_part;
    uint32_t off_l2;          // staged L2 columns of the cluster's rows, [rank][rows_max] bf16
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
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_dyn(int pending) {
    // the ring depth is a launch parameter; wait_group takes an immediate
    switch (pending) {
        case 0: cp_async_wait<0>(); break;
        case 1: cp_async_wait<1>(); break;
        case 2: cp_async_wait<2>(); break;
        case 3: cp_async_wait<3>(); break;
        case 4: cp_async_wait<4>(); break;
        default: cp_async_wait<5>(); break;
    }
}

// 4*b bytes of packed codes (one thread's 32-code slice) from shared memory, plus a zero word.
template <int BITS>
__device__ __forceinline__ void lds_slice(const uint8_t *p, uint32_t (&w)[BITS + 1]) {
    if constexpr (BITS == 4) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BITS == 6) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const uint2 v = *reinterpret_cast<const uint2 *>(p + 8 * i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = *reinterpret_cast<const uint32_t *>(p + 4 * i);
    }
    w[BITS] = 0;
}

template <int BITS, int TOK>
__global__ void __launch_bounds__(SmCfg<TOK>::kThreads, 1)
smallm_kernel(const SmallMArgs a) {
    constexpr int W = SmCfg<TOK>::kWarps;
    constexpr int NT = SmCfg<TOK>::kNT;
    constexpr int CH = SmCfg<TOK>::kCH;
    constexpr uint32_t kGB = 16 * BITS;                        // bytes of one group of one row
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
    float *sx = reinterpret_cast<float *>(smem + a.off_sx);     // [TOK][gmax] group sums of x
    float *st = reinterpret_cast<float *>(smem + a.off_st);     // [rows_max][gmax] steps
    float *part = reinterpret_cast<float *>(smem + a.off_part);
    const int part_stride = TOK * a.rows_max;                   // floats per group split
    const uint32_t ring = smem_u32(smem + a.off_ring) + (uint32_t)warp * (uint32_t)a.D * a.slot_bytes;

    // ---------------------------------------------------------------- this warp's blocks
    const int RB = a.RB;
    const int NB = (Uc + RB - 1) / RB;
    // with at least as many blocks as warps, warp w takes blocks w, w + W, ... over all the
    // CTA's groups; otherwise warp w takes block w % NB and group split w / NB of GW
    const bool shared_blocks = NB < W;
    const int split = shared_blocks ? warp / NB : 0;
    const bool active = shared_blocks ? (warp < NB * a.GW) : true;
    const int gs0 = shared_blocks ? Gc * split / a.GW : 0, gs1 = shared_blocks ? Gc * (split + 1) / a.GW : Gc;

    // The copies of one slot: group g of the nr units from row n0, 16 rows x 16*b bytes each
    // (16-byte copies, rows past N zero-filled). Which chunks a lane copies does not change
    // between slots, so their row and offsets are computed once.
    constexpr int kChunks = kSmMaxRB * 16 * BITS;              // 16-byte chunks of a full slot
    constexpr int kChunkIters = (kChunks + 31) / 32;
    int c_row[kChunkIters];
    int64_t c_src[kChunkIters];
    uint32_t c_dst[kChunkIters];
#pragma unroll
    for (int i = 0; i < kChunkIters; ++i) {
        const int j = lane + 32 * i;
        const int row = j / BITS, ch = j - row * BITS;        // row of the slot: unit row / 16
        c_row[i] = j < kChunks ? row : 1 << 30;
        c_src[i] = (int64_t)row * a.row_bytes + 16 * ch;
        c_dst[i] = (uint32_t)row * kGB + 16u * ch;
    }
    auto issue = [&](int64_t n0, int nr, int g, uint32_t slot) {
        const uint8_t *base = a.packed + n0 * a.row_bytes + (int64_t)g * kGB;
        const int64_t rows_left = a.N - n0;
#pragma unroll
        for (int i = 0; i < kChunkIters; ++i) {
            if (c_row[i] < 16 * nr) {
                const bool ok = c_row[i] < rows_left;
                cp_async_16(slot + c_dst[i], ok ? base + c_src[i] : a.packed, ok ? 16u : 0u);
            }
        }
        cp_async_commit();
    };
    auto slot_next = [&](uint32_t s) { s += a.slot_bytes; return s == ring + (uint32_t)a.D * a.slot_bytes ? ring : s; };

    // ---------------------------------------------------------------- stage x, steps
    // One commit group of asynchronous copies, issued before the ring prologue so that both
    // are in flight together: the token rows of x for the CTA's groups and the steps of its
    // rows and groups.
    {
        const int chunks = Gc * 16;                            // 16-byte chunks per token row
        const uint32_t xs = smem_u32(smem);
        for (int e = threadIdx.x; e < M * chunks; e += W * 32) {
            const int tok = e / chunks, j = e - tok * chunks;
            cp_async_16(xs + (uint32_t)tok * a.x_stride + 16u * j, a.x + (int64_t)tok * a.K + (int64_t)g0 * 128 + 8 * j, 16u);
        }
        const int rows_v = (int)min((int64_t)rows_c, a.N - n_base);
        const uint32_t ss = smem_u32(st);
        for (int e = threadIdx.x; e < rows_v * Gc; e += W * 32) {
            const int i = e / Gc, gl = e - i * Gc;
            cp_async_4(ss + 4u * (uint32_t)(i * a.gmax + gl), a.scales + (n_base + i) * G + g0 + gl, 4u);
        }
        if (a.l2_staged) {
            // L2 columns [n_base, n_base + rows_c) of every rank row, 8 columns per copy (zeros past N)
            const int per_row = rows_c / 8;
            const uint32_t ls = smem_u32(smem + a.off_l2);
            for (int e = threadIdx.x; e < a.rank * per_row; e += W * 32) {
                const int jr = e / per_row, cj = e - jr * per_row;
                const int64_t n = n_base + 8 * cj;
                const bool ok = n < a.N;
                cp_async_16(ls + 2u * (uint32_t)(jr * a.rows_max + 8 * cj), ok ? a.L2 + (int64_t)jr * a.N + n : a.L2,
                            ok ? 16u : 0u);
            }
        }
        cp_async_commit();
    }

    // the ring's first D - 1 slots, also in flight while the staging copies land
    const int first_ub = shared_blocks ? (warp % NB) * RB : warp * RB;
    uint32_t pf_slot = ring;
    int pf_gl = gs0;
    auto prologue = [&](int ub, int nr) {
        pf_slot = ring;
        pf_gl = gs0;
        for (int i = 0; i < a.D - 1; ++i) {
            if (pf_gl < gs1) {
                issue(n_base + ub * 16, nr, g0 + pf_gl, pf_slot);
                pf_slot = slot_next(pf_slot);
                ++pf_gl;
            } else {
                cp_async_commit();
            }
        }
    };
    if (active && first_ub < Uc) {
        prologue(first_ub, min(RB, Uc - first_ub));
        cp_async_wait_dyn(a.D - 1);                            // the staging group is the oldest
    } else {
        cp_async_wait<0>();
    }
    __syncthreads();
    // sum of each staged token row over each group: 8 lanes per (token, group), 16 values
    // each, then a fixed xor tree over the 8 lanes (deterministic)
    for (int base = warp * 32; base < M * Gc * 8; base += W * 32) {
        const int e = base + lane;
        const bool ok = e < M * Gc * 8;
        const int item = e >> 3, part8 = e & 7;
        const int tok = ok ? item / Gc : 0, gl = ok ? item - tok * Gc : 0;
        float sum = 0.0f;
        if (ok) {
            const uint4 *xp = reinterpret_cast<const uint4 *>(smem + (uint32_t)tok * a.x_stride + (uint32_t)gl * 256u +
                                                              32u * part8);
            const uint4 v0 = xp[0], v1 = xp[1];
            const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            float h[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) h[q] = bf16_bits_to_f32(wv[q] & 0xFFFFu) + bf16_bits_to_f32(wv[q] >> 16);
            sum = ((h[0] + h[1]) + (h[2] + h[3])) + ((h[4] + h[5]) + (h[6] + h[7]));
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 4);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        if (ok && part8 == 0) sx[tok * a.gmax + gl] = sum;
    }
    __syncthreads();

    // ---------------------------------------------------------------- stream and contract
    for (int ub = first_ub; active && ub < Uc; ub += shared_blocks ? Uc : W * RB) {
        const int nr = min(RB, Uc - ub);
        if (ub != first_ub) prologue(ub, nr);
        uint32_t cslot = ring;
        float R[kSmMaxRB][NT][4];
#pragma unroll
        for (int r = 0; r < kSmMaxRB; ++r)
#pragma unroll
            for (int t = 0; t < NT; ++t) R[r][t][0] = R[r][t][1] = R[r][t][2] = R[r][t][3] = 0.0f;
        for (int gl = gs0; gl < gs1; ++gl) {
            if (pf_gl < gs1) {
                issue(n_base + ub * 16, nr, g0 + pf_gl, pf_slot);
                pf_slot = slot_next(pf_slot);
                ++pf_gl;
            } else {
                cp_async_commit();
            }
            cp_async_wait_dyn(a.D - 1);
            __syncwarp();
            // x fragment of the group: token 8t + g, words [16c, 16c + 16) of its 64 (zeros for
            // tokens past M); the correction (128 + 2^(b-1)) sum_k x for the fragment's columns
            uint32_t X[NT][16];
            float corr[NT][4];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const int tok = 8 * t + g_l;
                const uint8_t *xp = smem + (uint32_t)tok * a.x_stride + (uint32_t)gl * 256u + c_l * 64;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = tok < M ? *reinterpret_cast<const uint4 *>(xp + 16 * q) : make_uint4(0, 0, 0, 0);
                    X[t][4 * q] = v.x; X[t][4 * q + 1] = v.y; X[t][4 * q + 2] = v.z; X[t][4 * q + 3] = v.w;
                }
                const int c0 = 8 * t + 2 * c_l;
                const float s0 = c0 < M ? sx[c0 * a.gmax + gl] : 0.0f;
                const float s1 = c0 + 1 < M ? sx[(c0 + 1) * a.gmax + gl] : 0.0f;
                corr[t][0] = corr[t][2] = kBiasF * s0;
                corr[t][1] = corr[t][3] = kBiasF * s1;
            }
            const uint8_t *slot = smem + (cslot - smem_u32(smem));
#pragma unroll
            for (int r = 0; r < kSmMaxRB; ++r) {
                if (r < nr) {
                    uint32_t wa[BITS + 1], wb[BITS + 1];
                    lds_slice<BITS>(slot + (uint32_t)(16 * r + g_l) * kGB + c_l * 4 * BITS, wa);
                    lds_slice<BITS>(slot + (uint32_t)(16 * r + g_l + 8) * kGB + c_l * 4 * BITS, wb);
                    const int row = (ub + r) * 16 + g_l;
                    const float sa = st[row * a.gmax + gl], sb = st[(row + 8) * a.gmax + gl];
                    float acc[NT][CH][4];
#pragma unroll
                    for (int t = 0; t < NT; ++t)
#pragma unroll
                        for (int h = 0; h < CH; ++h) acc[t][h][0] = acc[t][h][1] = acc[t][h][2] = acc[t][h][3] = 0.0f;
                    static_for<4>([&](auto bb) {
                        constexpr int blk = decltype(bb)::value;
                        uint32_t pa[4], pb[4];
                        unpack_pairs_biased<BITS, blk, 1>(wa, pa);
                        unpack_pairs_biased<BITS, blk, 1>(wb, pb);
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
                            float sum = acc[t][0][k] - corr[t][k];
#pragma unroll
                            for (int h = 1; h < CH; ++h) sum += acc[t][h][k];
                            R[r][t][k] = fmaf(k < 2 ? sa : sb, sum, R[r][t][k]);
                        }
                    }
                }
            }
            __syncwarp();              // every lane is done with the slot before it is refilled
            cslot = slot_next(cslot);
        }
        // this block's partial sums -> part[split][token][row of the cluster range]
        float *ps = part + split * part_stride;
#pragma unroll
        for (int r = 0; r < kSmMaxRB; ++r) {
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
    cp_async_wait<0>();
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
    // it, then hold t_hi + t_lo per token and rank column in fp32 where the ring was
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
