/*
 * wq.h -- C ABI of libwq.so: per-group(128) low-bit weight quantization and the fused
 * dequant-GEMM linear layer, for NVIDIA B200 (sm_100a).
 *
 * The operations follow two pages:
 *   [PG]   "Per-group(128) scale + PD mixed precision + multi-bit packed storage for
 *          Wan-Dancer-14B" (mtrt.cn news article 3666).
 *          sec. 3.1  per-group symmetric quantization along the input dimension,
 *          sec. 3.3  multi-bit packed storage (3/4/5/6/7 bits; packing table; pack_int4),
 *          sec. 3.4  GPU-resident dequantize, then the linear layer's matmul (sec. 5.3/5.4).
 *   [SVDQ] "SVDQuant: 4-bit quantization lets diffusion models run efficiently on
 *          consumer GPUs" (kongchang.com), section "Technical principles": a 16-bit
 *          low-rank branch L1*L2 next to the quantized residual.
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers owned by the caller. The library never
 *     allocates, frees or keeps device memory of its own beyond a 4-byte error word.
 *   - bf16 tensors are passed as `const void*` holding IEEE bfloat16 values.
 *   - Layouts are dense row-major. "N" is out_features, "K" in_features, "M" tokens.
 *   - Every tensor pointer must be 16-byte aligned (WQ_ERR_MISALIGNED otherwise).
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream). Argument
 *     checks happen on the host before anything is launched and report a status; no call
 *     traps, asserts or aborts.
 *   - Device-side waits are bounded. A wait that runs out records WQ_ERR_TIMEOUT in the
 *     library's error word, the kernel returns early, and the next wq_device_status()
 *     reports it.
 *   - The current CUDA device must be a compute capability 10.0 GPU (B200); other devices
 *     get WQ_ERR_UNSUPPORTED_DEVICE.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WQ_API __attribute__((visibility("default")))
#else
#define WQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream, so either can be passed. */
typedef struct CUstream_st *wq_stream_t;

typedef enum {
    WQ_OK = 0,
    WQ_ERR_INVALID_ARG = 1,        /* negative size, NULL pointer, K % group != 0, ... */
    WQ_ERR_UNSUPPORTED_BITS = 2,   /* bits not in {3, 4, 5, 6, 7} */
    WQ_ERR_UNSUPPORTED_GROUP = 3,  /* group != 128 */
    WQ_ERR_MISALIGNED = 4,         /* a tensor pointer is not 16-byte aligned */
    WQ_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed; see wq_last_error() */
    WQ_ERR_TIMEOUT = 6,            /* a bounded device-side wait ran out */
    WQ_ERR_WORKSPACE = 7,          /* workspace NULL or smaller than wq_linear_workspace_bytes() */
    WQ_ERR_UNSUPPORTED_DEVICE = 8  /* current device is not sm_100 */
} wq_status;

/* Kernel family used by wq_linear_ex. AUTO picks by M (small-M streaming kernel for few
 * tokens, the tensor-core dequant-GEMM otherwise). */
typedef enum {
    WQ_PATH_AUTO = 0,
    WQ_PATH_SMALL_M = 1,           /* HBM-streaming split-K kernel, any M (re-reads W per 32 tokens) */
    WQ_PATH_TENSOR = 2             /* tcgen05/TMEM dequant-GEMM, any M */
} wq_path;

/* Library version, as 10000*major + 100*minor + patch. */
WQ_API int wq_version(void);

/* Bytes of the packed codes of an N x K weight at `bits` bits with groups of `group`
 * input weights: N * K * bits / 8 ([PG] sec. 3.3 packing table: every 128-weight group
 * takes 16*bits bytes). Returns 0 when the arguments are invalid: bits outside 3..7,
 * group != 128, a negative size, or K not a multiple of the group. */
WQ_API size_t wq_packed_bytes(int64_t N, int64_t K, int bits, int group);

/* Number of fp32 scales of an N x K weight: N * K / group ([PG] sec. 3.1: one step per
 * group of `group` consecutive input weights). Returns -1 when invalid. */
WQ_API int64_t wq_scales_count(int64_t N, int64_t K, int group);

/*
 * Quantize and pack a weight ([PG] sec. 3.1 and 3.3).
 *   W       in : N x K bf16, row-major. Must be finite.
 *   bits       : 3..7.          group : must be 128; K must be a multiple of it.
 *   packed  out: N x (K*bits/8) bytes. Per row, the codes form one bitstream, first code in
 *                the most significant bits; group g of row n is bytes [16*bits*g, 16*bits*(g+1)).
 *   scales  out: N x (K/128) fp32, scales[n][g] = step of that group.
 * For each group: abs_max = fl32(max|w| * 1.01f), step = fl32(2*abs_max / (2^bits - 1)),
 * q = round_half_even(fl32(w / step)) clamped to +-((2^bits - 1) / 2), code = q + 2^(bits-1).
 * A group whose abs_max is 0 gets step 0 and every code 2^(bits-1).
 * Results are bit-identical to the correctly rounded IEEE fp32 evaluation of those formulas.
 * N == 0 is a no-op.
 */
WQ_API wq_status wq_quantize_pack(const void *W, int64_t N, int64_t K, int bits, int group,
                           uint8_t *packed, float *scales, wq_stream_t stream);

/*
 * Dequantize a packed weight to bf16 ([PG] sec. 3.4, dequantize_on_gpu: the step before the
 * page's bf16 matmul):  W_hat[n][k] = bf16(fl32((code - 2^(bits-1)) * step[n][k/128])),
 * rounded to nearest even.
 *   packed, scales in : as wq_quantize_pack writes them (N x K*bits/8 bytes, N x K/128 fp32).
 *   W_hat         out : N x K bf16, row-major.
 * K must be a multiple of group (128). N == 0 is a no-op. wq_linear does not need this: it
 * dequantizes in registers; the call is for callers that want the weight itself.
 */
WQ_API wq_status wq_dequantize(const uint8_t *packed, const float *scales, int64_t N, int64_t K, int bits,
                               int group, void *W_hat, wq_stream_t stream);

/* One tensor of a wq_quantize_pack_many call: the arguments of one wq_quantize_pack. */
typedef struct {
    const void *W;        /* N x K bf16, device */
    int64_t N, K;         /* K a multiple of 128; N == 0 or K == 0: nothing to do */
    int bits;             /* 3..7, per tensor */
    uint8_t *packed;      /* N x (K*bits/8) bytes, device */
    float *scales;        /* N x (K/128) fp32, device */
} wq_pack_job;

/*
 * Quantize and pack many tensors, each at its own width: the whole-model step of [PG]
 * sec. 3.2 (every tensor gets its own bit width, 3..7) followed by sec. 3.1 and 3.3 for each.
 *   jobs    in : host array of n_jobs descriptors (read during the call only; the library
 *                keeps no pointer to it). n_jobs == 0 is a no-op.
 *   group      : must be 128.
 * Each job's outputs are bit-identical to those of wq_quantize_pack on the same arguments.
 * The jobs' output buffers must not overlap one another or any job's W; the order in which
 * the jobs run is unspecified. Tensors of one width are packed together, up to 64 per kernel
 * launch, so a model's ~500 tensors take about a dozen launches instead of ~500.
 * Every job is checked before anything is launched: the first bad job's status is returned
 * (wq_last_error() names it) and nothing runs. A launch failure returns WQ_ERR_CUDA; the
 * launches before it have been queued.
 */
WQ_API wq_status wq_quantize_pack_many(const wq_pack_job *jobs, int n_jobs, int group, wq_stream_t stream);

/*
 * Quantization error table of one weight ([PG] sec. 3.2: the per-tensor error at every
 * candidate width that the PD bit allocation minimizes, its mse_table):
 *   out[b - 3] = sum over all N*K weights of (w - dequant(quantize_b(w)))^2, for b = 3..7,
 *   out[5]     = sum of w^2,
 * where quantize_b / dequant are exactly those of wq_quantize_pack at b bits and wq_linear's
 * dequant(code) = q * step (fp32). So out[b-3] / (N*K) is the tensor's MSE at b bits and
 * 10 log10(out[5] / out[b-3]) its SNR in dB.
 *   W   in : N x K bf16, row-major, finite. K a multiple of group; group must be 128.
 *   out out: device array of 6 doubles (8-byte aligned), overwritten.
 * The squared errors are summed in fp64; the order of the final additions varies between
 * runs, so the last bits of a sum may too. N == 0 writes zeros.
 */
WQ_API wq_status wq_quant_error(const void *W, int64_t N, int64_t K, int group, double *out, wq_stream_t stream);

/* One tensor of a wq_quant_error_many call: the arguments of one wq_quant_error. */
typedef struct {
    const void *W;        /* N x K bf16, device */
    int64_t N, K;         /* K a multiple of 128 */
    double *out;          /* 6 doubles, device */
} wq_error_job;

/* The error table of many tensors (a whole model) in a few launches (up to 64 tensors each).
 * Every job is checked before anything is launched; outputs must not overlap. */
WQ_API wq_status wq_quant_error_many(const wq_error_job *jobs, int n_jobs, int group, wq_stream_t stream);

/*
 * Per-tensor bit-width search ([PG] sec. 3.2, PD-guided mixed precision), on the host: choose
 * one width per tensor from `bits` that minimizes the weight-averaged quantization MSE with
 * a bits-per-weight budget. The relaxation (sigmoid-mapped continuous widths, softmax soft
 * assignment at a temperature annealed from 2 to 0.05, Lagrange term from 0.5 plus a 1e4
 * quadratic penalty, n_iters steps from each of n_restarts starts, rounding to the nearest
 * candidate, best start kept) is described with its readings in the library source.
 *   mse_table  in : n_tensors x n_bits, row-major, host: per-weight MSE of tensor i at
 *                   bits[j] (wq_quant_error's sums divided by N*K).
 *   n_params   in : n_tensors weight counts, host.
 *   bits       in : n_bits candidate widths, strictly increasing (e.g. 3,4,5,6,7), host.
 *   t_init     in : n_restarts x n_tensors starting parameters, host (the page draws them
 *                   as randn * 0.5); the search is deterministic given them.
 *   bits_out  out : n_tensors chosen widths, host.
 *   result    out : 3 doubles, host: the choice's total MSE (weight-averaged), its BPW, and
 *                   the index of the start it came from.
 * Runs synchronously on the calling thread; touches no GPU.
 */
WQ_API wq_status wq_pd_search(const double *mse_table, const int64_t *n_params, int n_tensors, const int *bits,
                              int n_bits, double target_bpw, int n_iters, int n_restarts, const double *t_init,
                              int *bits_out, double *result);

/* Workspace bytes wq_linear / wq_linear_ex need for these sizes on any path
 * (0 if none; the caller then may pass NULL). */
WQ_API size_t wq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int rank);

/*
 * Quantized linear layer ([PG] sec. 3.4 dequantize + matmul; [SVDQ] low-rank branch):
 *   y = x * dequant(packed, scales)^T + (x * L1) * L2 + bias
 * with dequant(code) = (code - 2^(bits-1)) * step of its group, fp32 accumulation, and the
 * result rounded once to bf16.
 *   x       in : M x K bf16.          K a multiple of 128 (pad the weight like the pages' _nin).
 *   packed  in : N x (K*bits/8) bytes, scales in: N x (K/128) fp32, as wq_quantize_pack writes.
 *   L1, L2  in : K x rank and rank x N bf16, or both NULL with rank == 0 (no branch).
 *                rank must be 0..64 and a multiple of 16.
 *   bias    in : N bf16, or NULL.
 *   y       out: M x N bf16.
 *   workspace  : device scratch of at least wq_linear_workspace_bytes(M, N, K, bits, rank)
 *                bytes (16-byte aligned), or NULL when that is 0. Its contents on entry do
 *                not matter. Calls that share a workspace must be ordered on one stream.
 * M == 0 or N == 0 is a no-op.
 */
WQ_API wq_status wq_linear(const void *x, int64_t M, int64_t K,
                    const uint8_t *packed, const float *scales, int bits, int group, int64_t N,
                    const void *L1, const void *L2, int rank, const void *bias,
                    void *y, void *workspace, size_t workspace_bytes, wq_stream_t stream);

/*
 * wq_linear without a caller-provided workspace. There is no counterpart of this call on
 * the pages; it exists for callers that cannot allocate device memory when they run the
 * layer -- for example code that owns no allocator (a plugin handed raw tensors by a host
 * framework), code running under a fixed device-memory budget that has already been handed
 * out, or a real-time loop in which an allocation could block or fail.
 * The low-rank branch needs scratch; this call uses a buffer of WQ_STATIC_SCRATCH_BYTES that
 * is compiled into the library (every GPU that loads libwq.so holds it until the process
 * exits). Sizes whose scratch would exceed it -- wq_linear_workspace_bytes(M, N, K, bits,
 * rank) > WQ_STATIC_SCRATCH_BYTES, e.g. more than 16384 tokens with a low-rank branch --
 * are rejected with WQ_ERR_WORKSPACE before anything is launched; calls without the branch
 * never touch it. The call allocates nothing and frees nothing.
 * The first call on a device looks up the buffer's device address once (with that device
 * current); make that first call before any stream capture. Every call on a device shares
 * the one buffer, and it keeps the last call's contents: calls whose work overlaps on the
 * GPU (different streams, no ordering between them) race on it. Arguments and results are
 * otherwise exactly those of wq_linear.
 */
#define WQ_STATIC_SCRATCH_BYTES ((size_t)4 << 20)
WQ_API wq_status wq_linear_no_workspace(const void *x, int64_t M, int64_t K,
                                        const uint8_t *packed, const float *scales, int bits, int group,
                                        int64_t N, const void *L1, const void *L2, int rank,
                                        const void *bias, void *y, wq_stream_t stream);

/* wq_linear with an explicit kernel family (for tests and benchmarks). */
WQ_API wq_status wq_linear_ex(const void *x, int64_t M, int64_t K,
                       const uint8_t *packed, const float *scales, int bits, int group, int64_t N,
                       const void *L1, const void *L2, int rank, const void *bias,
                       void *y, void *workspace, size_t workspace_bytes, wq_path path,
                       wq_stream_t stream);

/*
 * Synchronize `stream` and report the device-side status recorded since the last clear:
 * WQ_OK, WQ_ERR_TIMEOUT (a bounded wait ran out), or WQ_ERR_CUDA (the stream reported an
 * error). With clear != 0 the recorded status is reset afterwards.
 */
WQ_API wq_status wq_device_status(wq_stream_t stream, int clear);

/*
 * Self-test of the bounded-wait mechanism: launches one tiny kernel that waits on a flag
 * nothing sets, giving up after `timeout_us` microseconds (1..1000000). The kernel then
 * records WQ_ERR_TIMEOUT and returns, so the expected result is WQ_ERR_TIMEOUT and the
 * context stays usable. Synchronizes `stream`.
 */
WQ_API wq_status wq_selftest_bounded_wait(uint32_t timeout_us, wq_stream_t stream);

/* Number of kernels this library has launched in this process (all devices, all threads).
 * A diagnostic for counting device work between two points of a program. */
WQ_API uint64_t wq_launch_count(void);

/* Short static description of a status code. */
WQ_API const char *wq_status_string(wq_status status);

/* Message of the last failure on the calling host thread ("" if none). */
WQ_API const char *wq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */
