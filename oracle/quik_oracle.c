/*
 * CPU oracle for the hybrid W4A4 + outlier linear layer (QUIK / Atom).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * constant with the CUDA library: it is a second, independent statement of
 * what the layer computes, written to be checked by eye against the pages.
 *
 * What it follows (page title, passage):
 *  - "QUIK: Towards End-to-End 4-Bit Inference on Generative Large Language
 *    Models", abstract: most weights and activations are cast to 4 bits while
 *    a few outlier weights/activations stay in higher precision (FP16).
 *  - "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
 *    Summary: dynamic per-input activation scales and fine-grained group
 *    quantization; Key points: symmetric quantization (no zero points);
 *    Interesting ideas I1: outlier channels are reordered to the end so the
 *    high-precision part is one contiguous block; I3: outliers kept in INT8.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - scale s = max|v| / 7 in fp32 over the INT4 positions only (the outlier
 *    block is excluded); code q = clamp(rintf(v / s), -7, 7) with an IEEE
 *    fp32 division and round-half-to-even; an all-zero row/group gives s = 0
 *    and all codes 0.
 *  - groups are 128 consecutive *reordered* INT4 positions.
 *  - INT8 outliers: s = max|v| / 127, q = clamp(rintf(v / s), -127, 127),
 *    one scale per row (per token for X, per output channel for W).
 *  - 8-bit activations (W4A8): "QQQ: ... Quattuor-bit Quantization", the
 *    abstract on the aggregated "smoothquant" abstracts page, pairs 4-bit
 *    weights with 8-bit activations in per-channel (and per-group) GEMMs but
 *    fixes no quantiser.  Reading: the INT8 rule above (divisor and clamp
 *    127) applied per token to the non-outlier positions, one byte per code
 *    in reordered order.
 *  - 8-bit weights (W8A8, the baseline the same abstracts compare against):
 *    the same INT8 rule per output channel.
 *  - RMS norm fused with the activation quantiser (Atom, Summary and idea
 *    I2: quantisation folded into operators that already run): the norm's
 *    row factor r = 1/sqrt(mean(h^2) + eps) changes no code, so codes and base
 *    scales are taken from h * gamma and r multiplies the stored scales (and
 *    the FP16 outliers, rounded once to fp16).
 *  - 2:4-sparse weights (QUIK abstract: quantisation plus 2:4 sparsity):
 *    aligned groups of four reordered INT4 positions keep their two values
 *    of largest magnitude (lower position on ties), then the usual rule.
 *  - packing: byte i of a row holds code 2i in the low nibble and code 2i+1
 *    in the high nibble, both 4-bit two's complement.
 *  - integer dot products in int64 (checked to fit int32); dequantisation,
 *    outlier products and bias in fp64; the output is NOT rounded to fp16.
 *
 * Every function is plain, row-by-row C; OpenMP only splits independent rows.
 * Return value: 0 on success, negative on a violated precondition.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EBADARG -1
#define ORACLE_EOVERFLOW -2
#define ORACLE_ENOMEM -3

/* IEEE 754 binary16 -> binary64, from the format's definition:
 * normal  : (-1)^s * (1024 + m) * 2^(e - 25)
 * subnorm : (-1)^s * m * 2^-24                                        */
static double half_to_double(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return s ? -v : v;
}

static float half_to_float(uint16_t h) { return (float)half_to_double(h); }

/* Symmetric quantiser of one value: q = clamp(rint(v / s), -qmax, qmax),
 * fp32 division, current (round-to-nearest-even) rounding mode. */
static int quantize_value(float v, float s, int qmax)
{
    if (s == 0.0f)
        return 0;
    float r = rintf(v / s);
    if (r > (float)qmax) r = (float)qmax;
    if (r < (float)-qmax) r = (float)-qmax;
    return (int)r;
}

/* 4-bit two's complement nibble -> signed code. */
static int nibble_to_code(unsigned nib) { return nib >= 8 ? (int)nib - 16 : (int)nib; }

/* Code j of row r of a quantised [*, Ki] operand: packed nibbles (bits 4,
 * Ki / 2 bytes per row, code 2i in the low nibble of byte i) or one signed
 * byte per code (bits 8, Ki bytes per row). */
static int code_at(const uint8_t *Q, int64_t r, int64_t j, int64_t Ki, int bits)
{
    if (bits == 8)
        return (int)(int8_t)Q[r * Ki + j];
    unsigned b = Q[r * (Ki / 2) + j / 2];
    return nibble_to_code(j % 2 ? b >> 4 : b & 0xF);
}

/*
 * oracle_quantize_rows -- reorder, scale, quantise and pack R rows of a
 * [R, K] fp16 matrix.  Used for activations X (one row per token) and for
 * weights W (one row per output channel): the pages apply the same symmetric
 * rule to both.
 *
 *  X      : [R, K] fp16 bit patterns, row-major
 *  perm   : [K]; reordered column j is source column perm[j]; j >= K - k_o
 *           are the outlier channels
 *  group  : 0 (one scale per row) or the group width (e.g. 128)
 *  outlier_int8 : 0 -> O is fp16 [R, k_o] (bit copy); 1 -> O is int8
 *           [R, k_o] with o_scale [R]
 *  bits   : 4 -> Q is [R, (K - k_o) / 2] packed codes, divisor and clamp 7;
 *           8 -> Q is [R, K - k_o] signed bytes, divisor and clamp 127
 *  scale  : [R] (group == 0) or [R, (K - k_o) / group]
 */
int oracle_quantize_rows(int64_t R, int64_t K, int64_t k_o, int64_t group, int outlier_int8,
                         int bits, const uint16_t *X, const int32_t *perm,
                         uint8_t *Q, float *scale, void *O, float *o_scale)
{
    if (R < 0 || K < 0 || k_o < 0 || k_o > K || (bits != 4 && bits != 8)) return ORACLE_EBADARG;
    const int qmax = bits == 8 ? 127 : 7;
    const int64_t Ki = K - k_o;
    if (Ki % 2) return ORACLE_EBADARG;
    if (group < 0 || (group > 0 && Ki % group)) return ORACLE_EBADARG;
    const int64_t gs = group > 0 ? group : Ki;          /* positions per scale */
    const int64_t G = group > 0 ? Ki / group : 1;      /* scales per row      */
    for (int64_t j = 0; j < K; ++j)
        if (perm[j] < 0 || perm[j] >= K) return ORACLE_EBADARG;

    int err = ORACLE_OK;
#pragma omp parallel
    {
        float *xr = (float *)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
        int *codes = (int *)malloc(sizeof(int) * (size_t)(Ki > 0 ? Ki : 1));
        if (!xr || !codes) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        }
        /* every thread reaches the work-sharing loop; one without buffers skips its rows */
#pragma omp for schedule(static)
            for (int64_t r = 0; r < R; ++r) {
                if (!xr || !codes) continue;
                /* step 1: reorder (Atom I1) */
                for (int64_t j = 0; j < K; ++j)
                    xr[j] = half_to_float(X[r * K + perm[j]]);

                /* steps 2-3: per-row (or per-group) scale, then codes */
                for (int64_t g = 0; g < G; ++g) {
                    float amax = 0.0f;
                    for (int64_t j = g * gs; j < (g + 1) * gs; ++j)
                        if (fabsf(xr[j]) > amax) amax = fabsf(xr[j]);
                    float s = amax / (float)qmax;
                    scale[r * G + g] = s;
                    for (int64_t j = g * gs; j < (g + 1) * gs; ++j)
                        codes[j] = quantize_value(xr[j], s, qmax);
                }

                /* step 4: pack, low nibble = even position (or one byte per code) */
                if (bits == 8) {
                    for (int64_t j = 0; j < Ki; ++j)
                        Q[r * Ki + j] = (uint8_t)(int8_t)codes[j];
                } else {
                    for (int64_t i = 0; i < Ki / 2; ++i)
                        Q[r * (Ki / 2) + i] =
                            (uint8_t)((codes[2 * i] & 0xF) | ((codes[2 * i + 1] & 0xF) << 4));
                }

                /* step 6: the outlier block (reordered positions Ki .. K-1) */
                if (k_o > 0) {
                    if (!outlier_int8) {
                        uint16_t *o16 = (uint16_t *)O;
                        for (int64_t i = 0; i < k_o; ++i)
                            o16[r * k_o + i] = X[r * K + perm[Ki + i]];
                    } else {
                        int8_t *o8 = (int8_t *)O;
                        float amax = 0.0f;
                        for (int64_t i = 0; i < k_o; ++i)
                            if (fabsf(xr[Ki + i]) > amax) amax = fabsf(xr[Ki + i]);
                        float s = amax / 127.0f;
                        o_scale[r] = s;
                        for (int64_t i = 0; i < k_o; ++i)
                            o8[r * k_o + i] = (int8_t)quantize_value(xr[Ki + i], s, 127);
                    }
                } else if (outlier_int8 && o_scale) {
                    o_scale[r] = 0.0f;
                }
            }
        free(xr);
        free(codes);
    }
    return err;
}

/* IEEE 754 binary64 -> binary16, round to nearest even, from the format's
 * definition: normal values are m * 2^(e - 10) with m in [1024, 2048) and
 * e in [-14, 15]; below 2^-14 the step is 2^-24 (subnormals); magnitudes
 * that round past 65504 become infinity. */
static uint16_t double_to_half(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return 0x7e00;
    if (a < ldexp(1.0, -14)) {                       /* subnormal (or zero) */
        double q = nearbyint(a / ldexp(1.0, -24));    /* q <= 1024: 1024 is 2^-14 */
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e2;
    frexp(a, &e2);                                    /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                                   /* a in [2^e, 2^(e+1)) */
    double m = nearbyint(a / ldexp(1.0, e - 10));     /* in [1024, 2048] */
    if (m == 2048.0) { m = 1024.0; e += 1; }
    if (e > 15) return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(m - 1024.0));
}

/*
 * oracle_rmsnorm_quantize_rows -- the RMS normalisation that precedes a
 * projection, with the projection's dynamic quantisation and reordering
 * folded into it ("Atom: Low-bit Quantization for Efficient and Accurate LLM
 * Serving", Summary and idea I2: quantisation and reordering are fused into
 * operators that already run).  The normalisation of a row h of K channels
 * with weight gamma [K] (the norm in front of every Llama projection):
 *
 *     r    = 1 / sqrt( (1/K) * sum_{k<K} h[k]^2 + eps )      over ALL K channels
 *     y[k] = h[k] * r * gamma[k]
 *
 * and y is then reordered and quantised by the rule of oracle_quantize_rows.
 * Reading where the pages are silent: r > 0 multiplies every position of the
 * row, so it changes no code (y / s_y = z / s_z for z = h * gamma); the codes
 * and the fp32 base scales are those of z[k] = h[k] * gamma[k] (a product of
 * two fp16 values, exact in fp32), and r moves onto the stored scales:
 *
 *     scale   = fl32(s_z * r),  s_z = fl32(max|z| / 7) per row (or group)
 *     o_scale = fl32(so_z * r), so_z = fl32(max|z_o| / 127)   (INT8 outliers)
 *     O       = fl16(z * r)                                    (FP16 outliers)
 *
 * eps is an fp32 value (the norm's parameter as stored); the sum of
 * squares is taken exactly and rounded once to fp64 (reading: the pages fix
 * no precision; an exact sum makes r independent of summation order), r is
 * taken in fp64, and the stored scales and outliers are one rounding of an
 * fp64 product.  A row with a non-finite value has no norm: the call
 * returns ORACLE_EBADARG.  The unfused pipeline would round y to fp16 before quantising;
 * fusing the two steps removes that intermediate.
 *
 *  X, gamma : [R, K] and [K] fp16 bit patterns (gamma in source channel order)
 *  other arguments as oracle_quantize_rows
 */
int oracle_rmsnorm_quantize_rows(int64_t R, int64_t K, int64_t k_o, int64_t group,
                                 int outlier_int8, int bits, const uint16_t *X,
                                 const uint16_t *gamma, float eps, const int32_t *perm,
                                 uint8_t *Q, float *scale, void *O, float *o_scale)
{
    if (R < 0 || K < 1 || k_o < 0 || k_o > K || (bits != 4 && bits != 8)) return ORACLE_EBADARG;
    if (!(eps >= 0.0f)) return ORACLE_EBADARG;
    const int qmax = bits == 8 ? 127 : 7;
    const int64_t Ki = K - k_o;
    if (Ki % 2) return ORACLE_EBADARG;
    if (group < 0 || (group > 0 && Ki % group)) return ORACLE_EBADARG;
    const int64_t gs = group > 0 ? group : Ki;
    const int64_t G = group > 0 ? Ki / group : 1;
    for (int64_t j = 0; j < K; ++j)
        if (perm[j] < 0 || perm[j] >= K) return ORACLE_EBADARG;

    int err = ORACLE_OK;
#pragma omp parallel
    {
        float *z = (float *)malloc(sizeof(float) * (size_t)K);
        int *codes = (int *)malloc(sizeof(int) * (size_t)(Ki > 0 ? Ki : 1));
        if (!z || !codes) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        }
#pragma omp for schedule(static)
        for (int64_t r = 0; r < R; ++r) {
            if (!z || !codes) continue;
            /* the row's RMS factor, over every channel.  The sum of squares
             * is exact: each fp16 h is a multiple of 2^-24, so h^2 * 2^48 is
             * an integer (below 2^80), summed in 128 bits and rounded once to
             * fp64; the order of the terms cannot matter. */
            unsigned __int128 S = 0;
            int finite = 1;
            for (int64_t k = 0; k < K; ++k) {
                double h = half_to_double(X[r * K + k]);
                if (!isfinite(h)) finite = 0;
                else S += (unsigned __int128)ldexp(h * h, 48);
            }
            if (!finite) {
#pragma omp atomic write
                err = ORACLE_EBADARG;
                continue;
            }
            double ss = ldexp((double)S, -48);
            double rf = 1.0 / sqrt(ss / (double)K + (double)eps);

            /* reorder (Atom I1) the row times its norm weight; exact in fp32 */
            for (int64_t j = 0; j < K; ++j) {
                int64_t c = perm[j];
                z[j] = (float)(half_to_double(X[r * K + c]) * half_to_double(gamma[c]));
            }

            /* scales and codes of z, the stored scales carry r */
            for (int64_t g = 0; g < G; ++g) {
                float amax = 0.0f;
                for (int64_t j = g * gs; j < (g + 1) * gs; ++j)
                    if (fabsf(z[j]) > amax) amax = fabsf(z[j]);
                float s = amax / (float)qmax;
                scale[r * G + g] = (float)((double)s * rf);
                for (int64_t j = g * gs; j < (g + 1) * gs; ++j)
                    codes[j] = quantize_value(z[j], s, qmax);
            }
            if (bits == 8) {
                for (int64_t j = 0; j < Ki; ++j)
                    Q[r * Ki + j] = (uint8_t)(int8_t)codes[j];
            } else {
                for (int64_t i = 0; i < Ki / 2; ++i)
                    Q[r * (Ki / 2) + i] =
                        (uint8_t)((codes[2 * i] & 0xF) | ((codes[2 * i + 1] & 0xF) << 4));
            }

            /* the outlier block: the normalised values in fp16, or INT8 codes of z */
            if (k_o > 0) {
                if (!outlier_int8) {
                    uint16_t *o16 = (uint16_t *)O;
                    for (int64_t i = 0; i < k_o; ++i)
                        o16[r * k_o + i] = double_to_half((double)z[Ki + i] * rf);
                } else {
                    int8_t *o8 = (int8_t *)O;
                    float amax = 0.0f;
                    for (int64_t i = 0; i < k_o; ++i)
                        if (fabsf(z[Ki + i]) > amax) amax = fabsf(z[Ki + i]);
                    float s = amax / 127.0f;
                    o_scale[r] = (float)((double)s * rf);
                    for (int64_t i = 0; i < k_o; ++i)
                        o8[r * k_o + i] = (int8_t)quantize_value(z[Ki + i], s, 127);
                }
            } else if (outlier_int8 && o_scale) {
                o_scale[r] = 0.0f;
            }
        }
        free(z);
        free(codes);
    }
    return err;
}

/*
 * oracle_prune24_quantize_rows -- 2:4-sparse INT4 rows ("QUIK: Towards
 * End-to-End 4-Bit Inference on Generative Large Language Models", abstract:
 * quantisation combined with 2:4 sparsity).  Readings where the page is
 * silent: the pattern applies to the INT4 part of the reordered row, in
 * aligned groups of four positions 4t .. 4t+3 (t < K_i / 4); each group keeps
 * the two values of largest magnitude (on equal magnitudes, the lower
 * position) and the other two become zero; the outlier block stays dense.
 * The per-row scale and codes then follow oracle_quantize_rows (the largest
 * value of every group is kept, so pruning leaves the row's absmax as it is).
 *
 *  Qs    : [R, K_i / 4]; byte t holds the code at the group's lower kept
 *          position in bits 0-3 and the higher one in bits 4-7 (two's
 *          complement nibbles)
 *  meta  : [R, K_i / 8]; group t's four bits i0 | i1 << 2 (the kept
 *          positions within the group, i0 < i1) sit in bits 4 (t % 2) ..
 *          of byte t / 2
 *  scale : [R]; O, o_scale as oracle_quantize_rows
 */
int oracle_prune24_quantize_rows(int64_t R, int64_t K, int64_t k_o, int outlier_int8,
                                 const uint16_t *X, const int32_t *perm, uint8_t *Qs,
                                 uint8_t *meta, float *scale, void *O, float *o_scale)
{
    if (R < 0 || K < 0 || k_o < 0 || k_o > K) return ORACLE_EBADARG;
    const int64_t Ki = K - k_o;
    if (Ki % 8) return ORACLE_EBADARG;
    for (int64_t j = 0; j < K; ++j)
        if (perm[j] < 0 || perm[j] >= K) return ORACLE_EBADARG;

    int err = ORACLE_OK;
#pragma omp parallel
    {
        float *xr = (float *)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
        if (!xr) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        }
#pragma omp for schedule(static)
        for (int64_t r = 0; r < R; ++r) {
            if (!xr) continue;
            for (int64_t j = 0; j < K; ++j)
                xr[j] = half_to_float(X[r * K + perm[j]]);

            /* the scale over the INT4 positions (before pruning: the same value) */
            float amax = 0.0f;
            for (int64_t j = 0; j < Ki; ++j)
                if (fabsf(xr[j]) > amax) amax = fabsf(xr[j]);
            float s = amax / 7.0f;
            scale[r] = s;

            for (int64_t t = 0; t < Ki / 4; ++t) {
                const float *g = xr + 4 * t;
                /* first kept: the largest magnitude, lowest position among equals */
                int a = 0;
                for (int i = 1; i < 4; ++i)
                    if (fabsf(g[i]) > fabsf(g[a])) a = i;
                /* second kept: the largest of the other three, lowest position among equals */
                int b = -1;
                for (int i = 0; i < 4; ++i)
                    if (i != a && (b < 0 || fabsf(g[i]) > fabsf(g[b]))) b = i;
                int i0 = a < b ? a : b, i1 = a < b ? b : a;
                int q0 = quantize_value(g[i0], s, 7), q1 = quantize_value(g[i1], s, 7);
                Qs[r * (Ki / 4) + t] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
                uint8_t nib = (uint8_t)(i0 | (i1 << 2));
                uint8_t *mb = &meta[r * (Ki / 8) + t / 2];
                if (t % 2 == 0)
                    *mb = nib;
                else
                    *mb = (uint8_t)(*mb | (nib << 4));
            }

            if (k_o > 0) {
                if (!outlier_int8) {
                    uint16_t *o16 = (uint16_t *)O;
                    for (int64_t i = 0; i < k_o; ++i)
                        o16[r * k_o + i] = X[r * K + perm[Ki + i]];
                } else {
                    int8_t *o8 = (int8_t *)O;
                    float om = 0.0f;
                    for (int64_t i = 0; i < k_o; ++i)
                        if (fabsf(xr[Ki + i]) > om) om = fabsf(xr[Ki + i]);
                    float so = om / 127.0f;
                    o_scale[r] = so;
                    for (int64_t i = 0; i < k_o; ++i)
                        o8[r * k_o + i] = (int8_t)quantize_value(xr[Ki + i], so, 127);
                }
            } else if (outlier_int8 && o_scale) {
                o_scale[r] = 0.0f;
            }
        }
        free(xr);
    }
    return err;
}

/*
 * oracle_unpack24 -- the dense packed INT4 rows [R, K_i / 2] (the layout of
 * oracle_quantize_rows) that a 2:4 row stands for: the two kept codes at
 * their positions, zero elsewhere.  A metadata nibble that names no valid
 * pair (i0 < i1) is an error.
 */
int oracle_unpack24(int64_t R, int64_t Ki, const uint8_t *Qs, const uint8_t *meta, uint8_t *Q)
{
    if (R < 0 || Ki < 0 || Ki % 8) return ORACLE_EBADARG;
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t i = 0; i < Ki / 2; ++i)
            Q[r * (Ki / 2) + i] = 0;
        for (int64_t t = 0; t < Ki / 4; ++t) {
            unsigned nib = (meta[r * (Ki / 8) + t / 2] >> (4 * (t % 2))) & 0xF;
            int i0 = nib & 3, i1 = nib >> 2;
            if (i0 >= i1) return ORACLE_EBADARG;
            unsigned b = Qs[r * (Ki / 4) + t];
            int pos[2] = {(int)(4 * t + i0), (int)(4 * t + i1)};
            unsigned nibs[2] = {b & 0xF, b >> 4};
            for (int k = 0; k < 2; ++k) {
                uint8_t *q = &Q[r * (Ki / 2) + pos[k] / 2];
                *q = (uint8_t)(pos[k] % 2 ? (*q | (nibs[k] << 4)) : (*q | nibs[k]));
            }
        }
    }
    return ORACLE_OK;
}

/*
 * oracle_int_gemm -- exact integer product of the quantised codes (each of X
 * and W packed INT4, or one byte per code when its bits == 8).
 *  acc[m, n]           = sum_{j < Ki} qx[m, j] * qw[n, j]            (group == 0)
 *  acc[g, m, n]        = sum_{j in group g} qx[m, j] * qw[n, j]      (group > 0)
 * Sums are taken in int64 and must fit int32.
 */
int oracle_int_gemm(int64_t M, int64_t N, int64_t Ki, int64_t group, int x_bits, int w_bits,
                    const uint8_t *Xq, const uint8_t *Wq, int32_t *acc)
{
    if (M < 0 || N < 0 || Ki < 0 || Ki % 2 || (x_bits != 4 && x_bits != 8)) return ORACLE_EBADARG;
    if (w_bits != 4 && w_bits != 8) return ORACLE_EBADARG;
    if (group < 0 || (group > 0 && Ki % group)) return ORACLE_EBADARG;
    const int64_t gs = group > 0 ? group : Ki;
    const int64_t G = group > 0 ? Ki / group : 1;
    int err = ORACLE_OK;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t g = 0; g < G; ++g) {
                int64_t sum = 0;
                for (int64_t j = g * gs; j < (g + 1) * gs; ++j)
                    sum += (int64_t)code_at(Xq, m, j, Ki, x_bits) * (int64_t)code_at(Wq, n, j, Ki, w_bits);
                if (sum > INT32_MAX || sum < INT32_MIN) {
#pragma omp atomic write
                    err = ORACLE_EOVERFLOW;
                }
                acc[(g * M + m) * N + n] = (int32_t)sum;
            }
        }
    }
    return err;
}

/* One output element of the layer, in fp64, from quantised operands.
 * Y = sum_g A_g * sx[m,g] * sw[n,g]  +  O  +  bias[n]                  */
static double linear_element(int64_t m, int64_t n, int64_t M, int64_t N, int64_t K, int64_t k_o,
                             int64_t group, int outlier_int8, int x_bits, int w_bits,
                             const uint8_t *Xq, const float *sx, const void *Xo, const float *sxo,
                             const uint8_t *Wq, const float *sw, const void *Wo, const float *swo,
                             const uint16_t *bias, int32_t *acc_out, int *overflow)
{
    (void)M; (void)N;
    const int64_t Ki = K - k_o;
    const int64_t gs = group > 0 ? group : Ki;
    const int64_t G = group > 0 ? Ki / group : 1;
    double y = 0.0;

    /* steps 5 and 7: exact integer sums, dequantised in fp64 */
    for (int64_t g = 0; g < G; ++g) {
        int64_t sum = 0;
        for (int64_t j = g * gs; j < (g + 1) * gs; ++j)
            sum += (int64_t)code_at(Xq, m, j, Ki, x_bits) * (int64_t)code_at(Wq, n, j, Ki, w_bits);
        if (sum > INT32_MAX || sum < INT32_MIN) *overflow = 1;
        if (acc_out) acc_out[g] = (int32_t)sum;
        if (Ki > 0)
            y += (double)sum * (double)sx[m * G + g] * (double)sw[n * G + g];
    }

    /* step 6: the outlier block */
    if (k_o > 0) {
        if (!outlier_int8) {
            const uint16_t *xo = (const uint16_t *)Xo, *wo = (const uint16_t *)Wo;
            double o = 0.0;
            for (int64_t i = 0; i < k_o; ++i)
                o += half_to_double(xo[m * k_o + i]) * half_to_double(wo[n * k_o + i]);
            y += o;
        } else {
            const int8_t *xo = (const int8_t *)Xo, *wo = (const int8_t *)Wo;
            int64_t sum = 0;
            for (int64_t i = 0; i < k_o; ++i)
                sum += (int64_t)xo[m * k_o + i] * (int64_t)wo[n * k_o + i];
            y += (double)sum * (double)sxo[m] * (double)swo[n];
        }
    }
    if (bias)
        y += half_to_double(bias[n]);
    return y;
}

/*
 * oracle_linear -- the full fp64 output Y [M, N] from quantised operands.
 * Xq and Wq hold packed INT4 (bits 4) or one byte per code (bits 8).  Xo/Wo are fp16 [*, k_o] (outlier_int8 == 0) or int8 [*, k_o] with
 * sxo [M] / swo [N] (outlier_int8 == 1).  bias is fp16 [N] or NULL.
 */
int oracle_linear(int64_t M, int64_t N, int64_t K, int64_t k_o, int64_t group, int outlier_int8,
                  int x_bits, int w_bits,
                  const uint8_t *Xq, const float *sx, const void *Xo, const float *sxo,
                  const uint8_t *Wq, const float *sw, const void *Wo, const float *swo,
                  const uint16_t *bias, double *Y)
{
    if (M < 0 || N < 0 || K < 0 || k_o < 0 || k_o > K || (K - k_o) % 2) return ORACLE_EBADARG;
    if (group < 0 || (group > 0 && (K - k_o) % group)) return ORACLE_EBADARG;
    if ((x_bits != 4 && x_bits != 8) || (w_bits != 4 && w_bits != 8)) return ORACLE_EBADARG;
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            Y[m * N + n] = linear_element(m, n, M, N, K, k_o, group, outlier_int8, x_bits, w_bits,
                                          Xq, sx, Xo,
                                          sxo, Wq, sw, Wo, swo, bias, NULL, &overflow);
    return overflow ? ORACLE_EOVERFLOW : ORACLE_OK;
}

/*
 * oracle_linear_sampled -- the same output at `count` chosen (ms[i], ns[i])
 * positions only; for full-size layers where the whole product would take
 * the CPU too long.  acc (optional) receives the G integer sums per sample
 * ([count, G], G = 1 without groups).
 */
int oracle_linear_sampled(int64_t M, int64_t N, int64_t K, int64_t k_o, int64_t group,
                          int outlier_int8, int x_bits, int w_bits,
                          const uint8_t *Xq, const float *sx, const void *Xo, const float *sxo,
                          const uint8_t *Wq, const float *sw, const void *Wo, const float *swo,
                          const uint16_t *bias, int64_t count, const int64_t *ms,
                          const int64_t *ns, double *Y, int32_t *acc)
{
    if (M < 0 || N < 0 || K < 0 || k_o < 0 || k_o > K || (K - k_o) % 2) return ORACLE_EBADARG;
    if (group < 0 || (group > 0 && (K - k_o) % group)) return ORACLE_EBADARG;
    if ((x_bits != 4 && x_bits != 8) || (w_bits != 4 && w_bits != 8)) return ORACLE_EBADARG;
    const int64_t G = group > 0 ? (K - k_o) / group : 1;
    for (int64_t i = 0; i < count; ++i)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return ORACLE_EBADARG;
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t i = 0; i < count; ++i)
        Y[i] = linear_element(ms[i], ns[i], M, N, K, k_o, group, outlier_int8, x_bits, w_bits,
                              Xq, sx, Xo, sxo,
                              Wq, sw, Wo, swo, bias, acc ? acc + i * G : NULL, &overflow);
    return overflow ? ORACLE_EOVERFLOW : ORACLE_OK;
}

/* Number of OpenMP threads the oracle would use (for reporting). */
int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
