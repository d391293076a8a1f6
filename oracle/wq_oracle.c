/*
 * wq_oracle.c -- plain, slow CPU oracle for per-group low-bit weight quantization
 * and the quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. It shares no code with the CUDA path.
 *
 * Sources (cited by page and section):
 *   [PG]   "Per-group(128) scale + PD mixed precision + multi-bit packed storage for
 *          Wan-Dancer-14B" (mtrt.cn news article 3666): sec. 3.1 (per-group symmetric
 *          quantization), sec. 3.3 (multi-bit packed storage, pack_int4/unpack_int4 and
 *          the packing table), sec. 3.4 (GPU-native dequantize: q = q_u - n_half,
 *          w = q * scale).
 *   [SVDQ] "SVDQuant: 4-bit quantization lets diffusion models run efficiently on
 *          consumer GPUs" (kongchang.com article), section "Technical principles":
 *          W = (16-bit low-rank branch) + (4-bit residual), so the layer output is
 *          x * deq(R)^T + x * L1 * L2.
 *
 * Readings taken where the pages leave a step open:
 *   - all quantizer arithmetic is IEEE fp32, round-to-nearest-even, no FMA contraction;
 *     1.01 is rounded to fp32 before the multiply;
 *   - round() is round-half-to-even;
 *   - the stored code is q + 2^(b-1); the clamp bound is (2^b - 1) / 2 (integer division);
 *   - a group whose abs-max is 0 stores step = 0 and q = 0 for every element;
 *   - codes of one row form one bitstream, most significant bit first; byte j of the row
 *     holds stream bits [8j, 8j+8). For 4 bits this is exactly pack_int4 (element 0 in the
 *     high nibble);
 *   - the linear layer is evaluated in fp64 from the same bf16/fp32 values the GPU sees,
 *     t = x * L1 is not rounded.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC (see build.py).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 bits. */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * Per-group symmetric quantization, [PG] sec. 3.1 and sec. 3.3.
 *   W      N x K bf16 bits, row-major (out_features x in_features)
 *   group  group size along the input dimension (128 on the pages; any divisor of K here,
 *          so that per-channel quantization is group = K)
 *   codes  N x K, one unsigned code per byte: q + 2^(bits-1)
 *   scales N x (K/group) fp32: the step of each group
 * Returns 0, or -1 on bad arguments.
 */
int wqo_quantize(const uint16_t *W, int64_t N, int64_t K, int bits, int64_t group,
                 uint8_t *codes, float *scales)
{
    if (N < 0 || K < 0 || bits < 2 || bits > 8 || group <= 0 || K % group != 0)
        return -1;
    const int64_t n_groups = K / group;
    const int levels = (1 << bits) - 1;   /* K - 1 on the page, with K = 2^bits */
    const int q_max = levels / 2;         /* clamp bound (2^b - 1) // 2 */
    const int offset = 1 << (bits - 1);   /* unsigned code offset 2^(b-1) */

#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < n_groups; ++g) {
            const uint16_t *w = W + n * K + g * group;
            uint8_t *c = codes + n * K + g * group;

            /* abs_max over the group, times 1.01 */
            float abs_max = 0.0f;
            for (int64_t k = 0; k < group; ++k) {
                float a = fabsf(bf16_to_f32(w[k]));
                if (a > abs_max)
                    abs_max = a;
            }
            float s = abs_max * 1.01f;
            /* step = 2 * abs_max / (2^b - 1) */
            float step = (2.0f * s) / (float)levels;
            scales[n * n_groups + g] = step;

            /* q = round(w / step).clamp(-q_max, q_max); code = q + offset */
            for (int64_t k = 0; k < group; ++k) {
                int q = 0;
                if (step != 0.0f) {
                    float r = bf16_to_f32(w[k]) / step;
                    q = (int)nearbyintf(r);
                    if (q > q_max) q = q_max;
                    if (q < -q_max) q = -q_max;
                }
                c[k] = (uint8_t)(q + offset);
            }
        }
    }
    return 0;
}

/*
 * Multi-bit packing, [PG] sec. 3.3: per row, the bits-wide codes are written into one
 * bitstream, most significant bit first. Row n occupies packed[n*K*bits/8 ...].
 * Written bit by bit on purpose.
 */
int wqo_pack(const uint8_t *codes, int64_t N, int64_t K, int bits, uint8_t *packed)
{
    if (N < 0 || K < 0 || bits < 2 || bits > 8 || (K * bits) % 8 != 0)
        return -1;
    const int64_t row_bytes = K * bits / 8;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        uint8_t *out = packed + n * row_bytes;
        memset(out, 0, (size_t)row_bytes);
        for (int64_t k = 0; k < K; ++k) {
            unsigned c = codes[n * K + k];
            for (int i = 0; i < bits; ++i) {
                unsigned bit = (c >> (bits - 1 - i)) & 1u;
                int64_t pos = k * bits + i;          /* position in the row's bitstream */
                if (bit)
                    out[pos / 8] |= (uint8_t)(0x80u >> (pos % 8));
            }
        }
    }
    return 0;
}

/* Inverse of wqo_pack ([PG] sec. 3.3 unpack_int4, generalised to every width). */
int wqo_unpack(const uint8_t *packed, int64_t N, int64_t K, int bits, uint8_t *codes)
{
    if (N < 0 || K < 0 || bits < 2 || bits > 8 || (K * bits) % 8 != 0)
        return -1;
    const int64_t row_bytes = K * bits / 8;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *in = packed + n * row_bytes;
        for (int64_t k = 0; k < K; ++k) {
            unsigned c = 0;
            for (int i = 0; i < bits; ++i) {
                int64_t pos = k * bits + i;
                unsigned bit = (in[pos / 8] >> (7 - pos % 8)) & 1u;
                c = (c << 1) | bit;
            }
            codes[n * K + k] = (uint8_t)c;
        }
    }
    return 0;
}

/*
 * Dequantize, [PG] sec. 3.4: w = (q_u - n_half) * scale, in fp32, with n_half = 2^(b-1)
 * (the code offset). deq is N x K fp32.
 */
int wqo_dequant(const uint8_t *codes, const float *scales, int64_t N, int64_t K, int bits,
                int64_t group, float *deq)
{
    if (N < 0 || K < 0 || bits < 2 || bits > 8 || group <= 0 || K % group != 0)
        return -1;
    const int64_t n_groups = K / group;
    const int offset = 1 << (bits - 1);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float q = (float)((int)codes[n * K + k] - offset);
            deq[n * K + k] = q * scales[n * n_groups + k / group];
        }
    return 0;
}

/*
 * Quantized linear layer in fp64, for the token rows listed in `rows`:
 *   y[i][n] = sum_k x[m][k] * deq[n][k]                      ([PG] sec. 3.4 then matmul)
 *           + sum_j t[j] * L2[j][n],  t[j] = sum_k x[m][k] * L1[k][j]   ([SVDQ])
 *           + bias[n]
 * with m = rows[i]. x is M x K bf16, deq N x K fp32, L1 K x r bf16, L2 r x N bf16,
 * bias N bf16; L1/L2 may be NULL when r == 0 and bias may be NULL. y is nrows x N fp64.
 */
int wqo_linear_rows(const uint16_t *x, int64_t M, int64_t K, const float *deq, int64_t N,
                    const uint16_t *L1, const uint16_t *L2, int r, const uint16_t *bias,
                    const int64_t *rows, int64_t nrows, double *y)
{
    if (M < 0 || K < 0 || N < 0 || r < 0 || nrows < 0)
        return -1;
    if (r > 0 && (L1 == NULL || L2 == NULL))
        return -1;
    for (int64_t i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= M)
            return -1;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const uint16_t *xm = x + rows[i] * K;
        double t[256];
        double *yi = y + i * N;
        if (r > 256) {
            /* rank above the fixed buffer is not supported by the oracle */
            for (int64_t n = 0; n < N; ++n) yi[n] = NAN;
            continue;
        }
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)bf16_to_f32(xm[k]) * (double)bf16_to_f32(L1[k * r + j]);
            t[j] = acc;
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            const float *wn = deq + n * K;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)bf16_to_f32(xm[k]) * (double)wn[k];
            for (int j = 0; j < r; ++j)
                acc += t[j] * (double)bf16_to_f32(L2[(int64_t)j * N + n]);
            if (bias != NULL)
                acc += (double)bf16_to_f32(bias[n]);
            yi[n] = acc;
        }
    }
    return 0;
}

/* Number of OpenMP threads the oracle runs with (reported beside its timings). */
int wqo_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
