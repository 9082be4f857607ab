/*
 * PTPC-FP8 oracle: plain, slow, obviously-correct CPU definitions of what the
 * hot path computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark load it.  It shares no code, header, table or constant
 * generator with the CUDA path.
 *
 * Source of the method: "PTPC-FP8: boosting vLLM performance on AMD ROCm"
 * (vLLM blog, 2025-02-24), sections "What is PTPC-FP8" and "Per-Token
 * Activation + Per-Channel Weight Quantization": X is T x Ci, W is Ci x Co,
 * the activation scale is a vector Delta_X[T x 1] (one scale per token) and the
 * weight scale is a vector Delta_W[1 x Co] (one scale per weight column).
 * The page gives no scale formula, no FP8 variant and no rounding rule; the
 * readings used here are:
 *   - FP8 is OCP E4M3 ("e4m3fn"): bias 7, no infinities, S.1111.111 = NaN,
 *     largest finite magnitude 448.
 *   - scale s = amax / 448 in IEEE fp32 round-to-nearest-even; it is the
 *     dequantisation multiplier (x ~= decode(q) * s).
 *   - code q = E4M3_satRNE( fp32_RN(x / s) ): an IEEE fp32 division, then a
 *     saturating round-half-to-even cast to E4M3.
 *   - a group (row of X / column of W) whose amax is 0 gets s = 1.0f and every
 *     code 0x00.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 * Contraction and fast-math are off so that every float operation below is one
 * IEEE-rounded operation in the order written; OpenMP only splits the outer
 * loops over independent rows/columns and does not change any arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define E4M3_MAX 448.0

/* ------------------------------------------------------------------------- */
/* OCP E4M3 codec                                                            */
/* ------------------------------------------------------------------------- */

/* Decode one E4M3 byte.  Exponent field e (4 bits), mantissa m (3 bits):
 * e == 0 -> m * 2^-9 (subnormal); otherwise (8 + m) * 2^(e - 10), i.e.
 * (1 + m/8) * 2^(e - 7).  e == 15 && m == 7 is NaN.  Bit 7 is the sign. */
double oracle_e4m3_decode(uint8_t c)
{
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp((double)(8 + m), e - 10);
    return sign ? -mag : mag;
}

/* Encode one fp32 value to E4M3 with round-half-to-even and saturation to
 * +-448.  Works on the exact value: find the spacing of the E4M3 grid around
 * |v|, round |v| / spacing to an integer (ties to even), and re-encode the
 * rounded magnitude (which may have carried into the next binade). */
uint8_t oracle_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a, step, n, f, rem, q;
    int E;

    if (isnan(v))
        return (uint8_t)(sign | 0x7F); /* outside the contract; defined anyway */
    a = fabs((double)v);
    if (a >= E4M3_MAX)
        return (uint8_t)(sign | 0x7E);

    if (a < ldexp(1.0, -6)) {
        step = ldexp(1.0, -9);             /* subnormal spacing */
    } else {
        frexp(a, &E);                      /* a in [2^(E-1), 2^E) */
        step = ldexp(1.0, (E - 1) - 3);    /* 3 mantissa bits */
    }
    n = a / step;                          /* exact: step is a power of two */
    f = floor(n);
    rem = n - f;
    if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) == 1.0))
        f += 1.0;
    q = f * step;                          /* rounded magnitude, on the grid */

    if (q >= E4M3_MAX)
        return (uint8_t)(sign | 0x7E);
    if (q < ldexp(1.0, -6))                /* zero or subnormal: m = q / 2^-9 */
        return (uint8_t)(sign | (uint8_t)(q / ldexp(1.0, -9)));
    frexp(q, &E);                          /* q in [2^(E-1), 2^E) */
    {
        int e = (E - 1) + 7;
        int m = (int)(q / ldexp(1.0, E - 1) * 8.0) - 8;
        return (uint8_t)(sign | (uint8_t)((e << 3) | m));
    }
}

/* ------------------------------------------------------------------------- */
/* bf16 helpers                                                              */
/* ------------------------------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
float oracle_bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to bf16 (8 significant bits, exponent range of binary32),
 * round-half-to-even, overflow to infinity.  Used to round the fp64 GEMM
 * reference to the output dtype. */
uint16_t oracle_bf16_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    double a, step, n, f, rem, q;
    int E;

    if (isnan(v))
        return 0x7FC0;
    a = fabs(v);
    if (a < ldexp(1.0, -126)) {
        step = ldexp(1.0, -133);           /* subnormal spacing 2^-126 * 2^-7 */
    } else {
        frexp(a, &E);
        step = ldexp(1.0, (E - 1) - 7);    /* 7 stored mantissa bits */
    }
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80);
    n = a / step;
    f = floor(n);
    rem = n - f;
    if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) == 1.0))
        f += 1.0;
    q = f * step;
    if (q >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80);
    if (q < ldexp(1.0, -126))
        return (uint16_t)(sign | (uint16_t)(q / ldexp(1.0, -133)));
    frexp(q, &E);
    {
        int e = (E - 1) + 127;
        int m = (int)(q / ldexp(1.0, E - 1) * 128.0) - 128;
        return (uint16_t)(sign | (uint16_t)((e << 7) | m));
    }
}

/* ------------------------------------------------------------------------- */
/* Quantisation                                                              */
/* ------------------------------------------------------------------------- */

/* Scale of a group whose largest magnitude is amax: amax / 448 in fp32,
 * 1.0f for an all-zero group. */
float oracle_scale_from_amax(float amax)
{
    if (amax == 0.0f)
        return 1.0f;
    return amax / 448.0f;
}

/* Code of one element of a group: saturating RNE E4M3 of fp32_RN(x / s);
 * every code of an all-zero group is 0x00. */
uint8_t oracle_quantize_value(float x, float s, float amax)
{
    float q;
    if (amax == 0.0f)
        return 0x00;
    q = x / s;
    return oracle_e4m3_encode(q);
}

/* Per-token activation quantisation: one scale per row of X (T x Ci, bf16,
 * row-major).  Writes Xq (T x Ci codes, row-major) and x_scale[T]. */
void oracle_quant_act(const uint16_t *X, int64_t T, int64_t Ci,
                      uint8_t *Xq, float *x_scale)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        const uint16_t *row = X + t * Ci;
        float amax = 0.0f, s;
        int64_t k;
        for (k = 0; k < Ci; ++k) {
            float a = fabsf(oracle_bf16_to_float(row[k]));
            if (a > amax)
                amax = a;
        }
        s = oracle_scale_from_amax(amax);
        x_scale[t] = s;
        for (k = 0; k < Ci; ++k)
            Xq[t * Ci + k] = oracle_quantize_value(oracle_bf16_to_float(row[k]), s, amax);
    }
}

/* Per-channel weight quantisation: one scale per output column of W
 * (Ci x Co, bf16, row-major).  Writes the codes transposed, Wq_t (Co x Ci,
 * row-major, i.e. K-major), and w_scale[Co]. */
void oracle_quant_weight(const uint16_t *W, int64_t Ci, int64_t Co,
                         uint8_t *Wq_t, float *w_scale)
{
    int64_t o;
#pragma omp parallel for schedule(static)
    for (o = 0; o < Co; ++o) {
        float amax = 0.0f, s;
        int64_t k;
        for (k = 0; k < Ci; ++k) {
            float a = fabsf(oracle_bf16_to_float(W[k * Co + o]));
            if (a > amax)
                amax = a;
        }
        s = oracle_scale_from_amax(amax);
        w_scale[o] = s;
        for (k = 0; k < Ci; ++k)
            Wq_t[o * Ci + k] = oracle_quantize_value(oracle_bf16_to_float(W[k * Co + o]), s, amax);
    }
}

/* Per-tensor quantisation (the "standard FP8" the page compares against): one
 * scale for the whole tensor of n bf16 values.  Writes q[n] and *scale. */
void oracle_quant_per_tensor(const uint16_t *X, int64_t n, uint8_t *q, float *scale)
{
    float amax = 0.0f, s;
    int64_t i;
    for (i = 0; i < n; ++i) {
        float a = fabsf(oracle_bf16_to_float(X[i]));
        if (a > amax)
            amax = a;
    }
    s = oracle_scale_from_amax(amax);
    *scale = s;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i)
        q[i] = oracle_quantize_value(oracle_bf16_to_float(X[i]), s, amax);
}

/* Per-tensor quantisation of a weight, codes written transposed like
 * oracle_quant_weight (W is Ci x Co, Wq_t is Co x Ci). */
void oracle_quant_weight_per_tensor(const uint16_t *W, int64_t Ci, int64_t Co,
                                    uint8_t *Wq_t, float *scale)
{
    float amax = 0.0f, s;
    int64_t i, o;
    for (i = 0; i < Ci * Co; ++i) {
        float a = fabsf(oracle_bf16_to_float(W[i]));
        if (a > amax)
            amax = a;
    }
    s = oracle_scale_from_amax(amax);
    *scale = s;
#pragma omp parallel for schedule(static)
    for (o = 0; o < Co; ++o) {
        int64_t k;
        for (k = 0; k < Ci; ++k)
            Wq_t[o * Ci + k] = oracle_quantize_value(oracle_bf16_to_float(W[k * Co + o]), s, amax);
    }
}

/* ------------------------------------------------------------------------- */
/* Epilogues (fp32 arithmetic, the order the page writes)                   */
/* ------------------------------------------------------------------------- */

/* Naive step 2 of the page's "two-step" path: read the fp32 GEMM result y
 * (T x Co) and write bf16((y * token_scale[t]) * channel_scale[o]); the two
 * products are separate fp32 roundings, left to right. */
void oracle_apply_scales_f32(const float *y, int64_t T, int64_t Co,
                             const float *x_scale, const float *w_scale,
                             uint16_t *out)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        int64_t o;
        for (o = 0; o < Co; ++o) {
            float v = y[t * Co + o] * x_scale[t];
            v = v * w_scale[o];
            out[t * Co + o] = oracle_bf16_from_double((double)v);
        }
    }
}

/* Fused epilogue with fp32 arithmetic: the same two products applied to the
 * fp32 rounding of each exact fp64 dot product, without an intermediate
 * array.  acc64 is the fp64 accumulator (T x Co). */
void oracle_fused_epilogue_f32(const double *acc64, int64_t T, int64_t Co,
                               const float *x_scale, const float *w_scale,
                               uint16_t *out)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        int64_t o;
        for (o = 0; o < Co; ++o) {
            float acc = (float)acc64[t * Co + o];
            float v = (acc * x_scale[t]) * w_scale[o];
            out[t * Co + o] = oracle_bf16_from_double((double)v);
        }
    }
}

/* fp64 epilogue of the tolerance reference: bf16(x_s[t] * w_s[o] * acc). */
void oracle_reference_epilogue_f64(const double *acc64, int64_t rows, int64_t Co,
                                   const float *x_scale_rows, const float *w_scale,
                                   uint16_t *out)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < rows; ++t) {
        int64_t o;
        for (o = 0; o < Co; ++o) {
            double v = (double)x_scale_rows[t] * (double)w_scale[o] * acc64[t * Co + o];
            out[t * Co + o] = oracle_bf16_from_double(v);
        }
    }
}

/* Array forms of the codec, for the tests. */
void oracle_e4m3_encode_array(const float *v, int64_t n, uint8_t *out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i)
        out[i] = oracle_e4m3_encode(v[i]);
}

void oracle_bf16_from_double_array(const double *v, int64_t n, uint16_t *out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i)
        out[i] = oracle_bf16_from_double(v[i]);
}

/* ------------------------------------------------------------------------- */
/* Sub-byte weight formats: FP6 (E3M2, E2M3) and FP4 (E2M1)                  */
/* ------------------------------------------------------------------------- */
/*
 * Source: the llminfo.tech summary of "Running LLMs at custom floating-points
 * (near-lossless FP6)" (FP6-LLM extended to FP4-FP7 with per-channel
 * quantisation; the exponent/mantissa split is a free choice, and the author
 * names the MX formats as the likely standard), combined with the PTPC page's
 * per-output-channel weight scale.  Readings (the pages give no formula):
 *   - the formats are the OCP MX element types, which the B200 tensor cores
 *     consume natively: E2M1 (bias 1, max 6), E2M3 (bias 1, max 7.5), E3M2
 *     (bias 3, max 28); none has infinities or NaN;
 *   - per output channel o: s = amax_o / max_format (IEEE fp32 division),
 *     1.0f for an all-zero column; code = saturating round-half-to-even of
 *     fp32_RN(w / s) to the format's grid, sign kept (-0 -> sign bit set);
 *   - a code is held in the low bits of a byte: sign at bit (E + M), then E
 *     exponent bits, then M mantissa bits;
 *   - packing along K (the input channels) into the bytes that the weight
 *     occupies in memory: FP4 two codes per byte, the even position in the
 *     low nibble; FP6 sixteen codes per twelve bytes, code j of the group at
 *     bits [6j, 6j + 6) of the group read as a little-endian 96-bit integer.
 * Format ids: 0 E4M3 (the PTPC format, for cross-checks), 1 E2M1, 2 E2M3,
 * 3 E3M2.
 */

typedef struct {
    int ebits, mbits, bias;
    double maxval;
} oracle_fmt;

static oracle_fmt oracle_fmt_of(int f)
{
    oracle_fmt r;
    switch (f) {
    case 1: r.ebits = 2; r.mbits = 1; r.bias = 1; r.maxval = 6.0; break;
    case 2: r.ebits = 2; r.mbits = 3; r.bias = 1; r.maxval = 7.5; break;
    case 3: r.ebits = 3; r.mbits = 2; r.bias = 3; r.maxval = 28.0; break;
    default: r.ebits = 4; r.mbits = 3; r.bias = 7; r.maxval = 448.0; break;
    }
    return r;
}

double oracle_fmt_max(int f)
{
    return oracle_fmt_of(f).maxval;
}

/* Value of a code: exponent field e, mantissa field m.  e == 0 is subnormal,
 * m * 2^(1 - bias - M); otherwise (2^M + m) * 2^(e - bias - M).  E4M3's
 * S.1111.111 is NaN; the sub-byte formats have none. */
double oracle_fmt_decode(uint8_t code, int f)
{
    oracle_fmt t = oracle_fmt_of(f);
    int nb = t.ebits + t.mbits;
    int sign = (code >> nb) & 1;
    int e = (code >> t.mbits) & ((1 << t.ebits) - 1);
    int m = code & ((1 << t.mbits) - 1);
    double mag;
    if (f == 0 && e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, 1 - t.bias - t.mbits);
    else
        mag = ldexp((double)((1 << t.mbits) + m), e - t.bias - t.mbits);
    return sign ? -mag : mag;
}

/* Saturating round-half-to-even of an fp32 value to the format's grid: the
 * same steps as oracle_e4m3_encode, with the format's parameters. */
uint8_t oracle_fmt_encode(float v, int f)
{
    oracle_fmt t = oracle_fmt_of(f);
    int nb = t.ebits + t.mbits;
    uint8_t sign = signbit(v) ? (uint8_t)(1u << nb) : 0;
    double a, step, n, fl, rem, q, min_normal = ldexp(1.0, 1 - t.bias);
    int E;

    if (isnan(v))
        return (uint8_t)(sign | ((1u << nb) - 1u)); /* outside the contract */
    a = fabs((double)v);
    if (a >= t.maxval)
        q = t.maxval;
    else {
        if (a < min_normal) {
            step = ldexp(1.0, 1 - t.bias - t.mbits);
        } else {
            frexp(a, &E);                      /* a in [2^(E-1), 2^E) */
            step = ldexp(1.0, (E - 1) - t.mbits);
        }
        n = a / step;                          /* exact: step is a power of two */
        fl = floor(n);
        rem = n - fl;
        if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) == 1.0))
            fl += 1.0;
        q = fl * step;
        if (q > t.maxval)
            q = t.maxval;
    }
    if (q < min_normal)
        return (uint8_t)(sign | (uint8_t)(q / ldexp(1.0, 1 - t.bias - t.mbits)));
    frexp(q, &E);
    {
        int e = (E - 1) + t.bias;
        int m = (int)(q / ldexp(1.0, E - 1) * (double)(1 << t.mbits)) - (1 << t.mbits);
        return (uint8_t)(sign | (uint8_t)((e << t.mbits) | m));
    }
}

/* Per-output-channel weight quantisation to format f: W is Ci x Co bf16
 * (row-major); writes one code per byte, transposed (codes_t is Co x Ci),
 * and w_scale[Co] = amax / max_format. */
void oracle_quant_weight_fmt(const uint16_t *W, int64_t Ci, int64_t Co, int f,
                             uint8_t *codes_t, float *w_scale)
{
    const float fmax = (float)oracle_fmt_of(f).maxval;
    int64_t o;
#pragma omp parallel for schedule(static)
    for (o = 0; o < Co; ++o) {
        float amax = 0.0f, s;
        int64_t k;
        for (k = 0; k < Ci; ++k) {
            float a = fabsf(oracle_bf16_to_float(W[k * Co + o]));
            if (a > amax)
                amax = a;
        }
        s = amax == 0.0f ? 1.0f : amax / fmax;
        w_scale[o] = s;
        for (k = 0; k < Ci; ++k) {
            float x = oracle_bf16_to_float(W[k * Co + o]);
            codes_t[o * Ci + k] = amax == 0.0f ? 0 : oracle_fmt_encode(x / s, f);
        }
    }
}

/* Bytes a row of K codes of format f occupies once packed. */
int64_t oracle_packed_row_bytes(int64_t K, int f)
{
    if (f == 1)
        return K / 2;
    if (f == 2 || f == 3)
        return K / 16 * 12;
    return K;
}

/* Packs rows x K codes (one per byte) into rows x oracle_packed_row_bytes
 * bytes, bit by bit: code k of a row occupies bits [b*k, b*k + b) of the
 * packed row read as a little-endian bit string (b = 4 for E2M1, 6 for the
 * FP6 formats, 8 for E4M3).  K must be a multiple of 16. */
void oracle_pack_fmt(const uint8_t *codes, int64_t rows, int64_t K, int f, uint8_t *packed)
{
    const int b = f == 1 ? 4 : (f == 2 || f == 3) ? 6 : 8;
    const int64_t rb = oracle_packed_row_bytes(K, f);
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        int64_t k;
        uint8_t *dst = packed + r * rb;
        memset(dst, 0, (size_t)rb);
        for (k = 0; k < K; ++k) {
            int bit;
            uint8_t c = codes[r * K + k];
            for (bit = 0; bit < b; ++bit) {
                int64_t pos = k * b + bit;
                if ((c >> bit) & 1)
                    dst[pos / 8] |= (uint8_t)(1u << (pos % 8));
            }
        }
    }
}

/* Array form of oracle_fmt_encode, for the tests. */
void oracle_fmt_encode_array(const float *v, int64_t n, int f, uint8_t *out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i)
        out[i] = oracle_fmt_encode(v[i], f);
}

/* ------------------------------------------------------------------------- */
/* Per-token quantisation with a given row maximum (tensor parallelism)      */
/* ------------------------------------------------------------------------- */
/*
 * When the input channels of a layer are split over ranks (the row-parallel
 * linear of the PTPC page's TP = 2 evaluation), a rank holds only a slice of
 * every token's row.  The token's scale still comes from the whole row: the
 * ranks combine their slice maxima (a maximum is exact in any order) and each
 * rank quantises its slice with the combined maximum.  These two functions
 * are the two halves of that split: the slice maximum, and the quantisation
 * with a given maximum (s = amax / 448 as for oracle_quant_act; with the row's
 * own maximum it is oracle_quant_act).
 */

/* amax[t] = max_k |X[t, k]| over a T x Ci bf16 slice (fp32, exact). */
void oracle_row_amax(const uint16_t *X, int64_t T, int64_t Ci, float *amax)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        float m = 0.0f;
        int64_t k;
        for (k = 0; k < Ci; ++k) {
            float a = fabsf(oracle_bf16_to_float(X[t * Ci + k]));
            if (a > m)
                m = a;
        }
        amax[t] = m;
    }
}

/* Codes of a T x Ci slice with the given per-row maxima: x_scale[t] =
 * amax[t] / 448 (1.0f and all codes 0x00 when amax[t] == 0). */
void oracle_quant_act_amax(const uint16_t *X, int64_t T, int64_t Ci, const float *amax,
                           uint8_t *Xq, float *x_scale)
{
    int64_t t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        float s = oracle_scale_from_amax(amax[t]);
        int64_t k;
        x_scale[t] = s;
        for (k = 0; k < Ci; ++k)
            Xq[t * Ci + k] = oracle_quantize_value(oracle_bf16_to_float(X[t * Ci + k]), s, amax[t]);
    }
}
