/*
 * qref.c -- the oracle: a plain, slow, single-threaded CPU statement of
 * symmetric round-to-nearest (RTN) group quantization and of the quantized
 * matmul, used ONLY as test infrastructure.
 *
 * Who may use it: the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg. The CUDA library never links, loads or calls this file,
 * and this file includes nothing from the CUDA library: the two share no code.
 *
 * What it follows (page titles as printed on the pages):
 *  - "量化推理：INT8/INT4 的体积、困惑度与速度为什么不同步", functions pack()
 *    and unpack(): flatten the tensor, cut it into groups of `group`
 *    consecutive values, one fp32 scale per group = max|w| / qmax
 *    (qmax = 2^(bits-1) - 1), a zero scale replaced by 1, codes =
 *    clip(rint(w / scale), -qmax, qmax); int4 codes stored as code + 8, two per
 *    byte, the even element in the low nibble; int8 codes stored as
 *    two's-complement bytes; dequantized weight = float32(code) * scale.
 *  - "Huit bits, puis quatre", section "Arrondir": the same rule (step =
 *    max|w| / 127 or / 7, code = rounded w / step, w' = code x step, error at
 *    most half a step) and the QuantizedMatmul operation (section "Ranger des
 *    entiers dans des f32"), whose result is the plain product with the
 *    dequantized weights up to summation order.
 *
 * Arithmetic: every quotient w / scale and scale = absmax / qmax is one IEEE
 * fp32 division (the pages divide fp32 arrays by fp32 scales / Python ints),
 * rintf() rounds half to even as numpy's rint does, and the matmul
 * accumulates y[m][n] = sum_k w'[n][k] * x[m][k] in fp64 in ascending k.
 * Build flags: -O2 -fno-fast-math -ffp-contract=off (no FMA contraction,
 * no reassociation).
 *
 * Pins (tests under tests/ marked "not gpu"): the eight-weight worked example
 * and its outlier / two-scale variants ("quantization" page, --round,
 * --outlier, --channel), the pack/unpack round trip and payload length checks
 * of pack()'s page, the per-row error figures of the "ai-serving-optimise"
 * page, a brute-force nearest-code search, the half-step bound, and exact
 * rational sums for the matmul. Every function below is pinned.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define QREF_OK 0
#define QREF_ERR_ARG 1
#define QREF_ERR_NONFINITE 4

int qref_qmax(int bits) { return (1 << (bits - 1)) - 1; }

/* pack(): scales for every group, then codes, then the payload bytes.
 * n = number of weights (the flattened size); group must divide n; int4
 * needs n even because bytes pair elements 2t and 2t+1 of the flat array
 * (a byte may straddle two groups when group is odd). */
int qref_pack(const float *w, int64_t n, int bits, int64_t group,
              uint8_t *payload, float *scales, int8_t *codes_out)
{
    if ((bits != 4 && bits != 8) || group < 1 || n < 0 || n % group != 0)
        return QREF_ERR_ARG;
    if (bits == 4 && (n % 2) != 0)
        return QREF_ERR_ARG;
    const int qmax = qref_qmax(bits);
    const int64_t ngroups = n / group;
    int status = QREF_OK;

    for (int64_t j = 0; j < ngroups; ++j) {
        const float *row = w + j * group;
        float absmax = 0.0f;
        for (int64_t i = 0; i < group; ++i) {
            float a = fabsf(row[i]);
            if (!isfinite(a))
                status = QREF_ERR_NONFINITE;
            if (a > absmax)
                absmax = a;
        }
        float s = absmax / (float)qmax;  /* one fp32 IEEE division */
        if (s == 0.0f)
            s = 1.0f;                    /* zero-scale guard of pack() */
        scales[j] = s;
    }

    for (int64_t i = 0; i < n; ++i) {
        const float s = scales[i / group];
        float t = w[i] / s;              /* fp32 quotient */
        float r = rintf(t);              /* round half to even */
        if (r > (float)qmax) r = (float)qmax;
        if (r < (float)-qmax) r = (float)-qmax;
        int8_t c = (int8_t)r;
        if (codes_out)
            codes_out[i] = c;
        if (bits == 8) {
            payload[i] = (uint8_t)c;     /* two's-complement byte */
        } else {
            uint8_t u = (uint8_t)(c + 8);   /* 1..15 */
            if ((i & 1) == 0)
                payload[i >> 1] = u;                      /* even: low nibble */
            else
                payload[i >> 1] = (uint8_t)(payload[i >> 1] | (u << 4)); /* odd: high */
        }
    }
    return status;
}

/* unpack() up to the codes: int4 nibbles b & 15 (even element) and b >> 4
 * (odd element), each minus 8; int8 bytes read as signed. */
int qref_unpack_codes(const uint8_t *payload, int64_t n, int bits, int8_t *codes)
{
    if ((bits != 4 && bits != 8) || n < 0 || (bits == 4 && n % 2))
        return QREF_ERR_ARG;
    if (bits == 8) {
        for (int64_t i = 0; i < n; ++i)
            codes[i] = (int8_t)payload[i];
    } else {
        for (int64_t t = 0; t < n / 2; ++t) {
            codes[2 * t] = (int8_t)((int)(payload[t] & 15) - 8);
            codes[2 * t + 1] = (int8_t)((int)(payload[t] >> 4) - 8);
        }
    }
    return QREF_OK;
}

/* unpack(): w' = float32(code) * scale[group of the element], one fp32
 * multiplication. `payload` may be a slice: base_index is the flat index of
 * its first element within the whole tensor (even for int4), and `scales` is
 * the whole tensor's scale array, so element i uses scales[(base_index+i)/group]. */
int qref_dequant(const uint8_t *payload, const float *scales, int64_t n,
                 int bits, int64_t group, int64_t base_index, float *w_out)
{
    if ((bits != 4 && bits != 8) || group < 1 || n < 0 || base_index < 0 ||
        (bits == 4 && (n % 2 || base_index % 2)))
        return QREF_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        int c;
        if (bits == 8) {
            c = (int8_t)payload[i];
        } else {
            uint8_t b = payload[i >> 1];
            c = (int)((i & 1) ? (b >> 4) : (b & 15)) - 8;
        }
        const float s = scales[(base_index + i) / group];
        w_out[i] = (float)c * s;
    }
    return QREF_OK;
}

/* y[m][n] = sum_k w[n][k] * x[m][k] in fp64, ascending k; bound[m][n] =
 * sum_k |w[n][k] * x[m][k]| (the scale of the tolerance). x is [M][K], w is
 * [N][K], both row-major fp32; y and bound are [M][N]. */
int qref_matmul(const float *x, int64_t M, const float *w, int64_t N, int64_t K,
                double *y, double *bound)
{
    if (M < 0 || N < 0 || K < 0)
        return QREF_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const float *xr = x + m * K;
        for (int64_t nn = 0; nn < N; ++nn) {
            const float *wr = w + nn * K;
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)wr[k] * (double)xr[k];
                acc += p;
                mag += fabs(p);
            }
            y[m * N + nn] = acc;
            if (bound)
                bound[m * N + nn] = mag;
        }
    }
    return QREF_OK;
}
