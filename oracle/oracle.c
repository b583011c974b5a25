/*
 * CPU oracle for the quantized linear layer Y = dequant(Xq) . dequant(Wq)^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never
 * calls it.
 *
 * It is deliberately plain and slow: every step is the textbook definition,
 * written out, in exact integer or fp64 arithmetic.
 *
 * Sources (article "Building a High-Performance and Portable vLLM Linear
 * Backend with Helion", as summarised and translated on the pages it was
 * published on):
 *   - formats: "Put algorithm selection inside the search space" (three
 *     formats: FP8_Dynamic per-token activation / per-channel weight scales;
 *     W8A8_INT8 with the same granularity; Block_FP8 with 1x128 activation
 *     and 128x128 weight scales), and the "Alcance" (scope) list of the
 *     Spanish translation, which restates the same three formats.
 *   - every variant (Standard, Split-K, Swap-AB) computes the same product;
 *     only the accumulation path differs ("Put algorithm selection inside
 *     the search space"; the matmul listing under "Codigo").
 *   - scale formula (absmax/448 for e4m3, absmax/127 for int8), round to
 *     nearest even and saturation: the workload definitions this library is
 *     measured on, since the pages only name "dynamic" per-token scaling.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - all-zero row/group/block: amax is clamped to at least 1e-12f before the
 *     division, so the scale is tiny but finite and every code is +-0.
 *   - the scale is the correctly rounded fp32 quotient amax/qmax; a value's
 *     code is taken from the correctly rounded fp32 quotient x/s.
 *   - e4m3 keeps the sign of zero (-0 -> 0x80); NaN -> 0x7F.
 *   - int8 is symmetric: codes are clamped to [-127, 127].
 *
 * Parity pins for every function here live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_E4M3_MAX 448.0
#define ORC_INT8_MAX 127.0
#define ORC_AMAX_FLOOR 1e-12f

enum { ORC_E4M3 = 0, ORC_INT8 = 1 };

/* ------------------------------------------------------------------ */
/* bf16 input                                                          */
/* ------------------------------------------------------------------ */

/* A bf16 value is the upper half of an IEEE binary32. */
static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ */
/* OCP FP8 E4M3 ("fn" variant): 1 sign bit, 4 exponent bits with bias 7,  */
/* 3 mantissa bits, no infinities, NaN = S.1111.111, max finite 448.   */
/* ------------------------------------------------------------------ */

/* Value of a code, straight from the bit fields. */
double orc_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, 1 - 7); /* subnormal: 0.m * 2^(1-bias) */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/*
 * Nearest e4m3 code to v.  Ties go to the code with an even mantissa (its
 * lowest bit clear).  Magnitudes above 448 saturate to 448.  The sign of zero
 * is kept.  The search runs over the ordered positive finite codes 0..0x7E,
 * whose values increase with the code.
 */
uint8_t orc_e4m3_encode(double v)
{
    uint8_t sign, lo, hi, best;
    double a, dlo, dhi;
    if (isnan(v))
        return 0x7F;
    sign = signbit(v) ? 0x80 : 0x00;
    a = fabs(v);
    if (a >= ORC_E4M3_MAX)
        return (uint8_t)(sign | 0x7E);
    /* bisection for the last code whose value is <= a */
    lo = 0;
    hi = 0x7E;
    while (hi - lo > 1) {
        uint8_t mid = (uint8_t)((lo + hi) / 2);
        if (orc_e4m3_decode(mid) <= a)
            lo = mid;
        else
            hi = mid;
    }
    if (orc_e4m3_decode(hi) <= a)
        lo = hi;
    hi = (uint8_t)(lo < 0x7E ? lo + 1 : lo);
    dlo = a - orc_e4m3_decode(lo);
    dhi = orc_e4m3_decode(hi) - a;
    if (dlo < dhi)
        best = lo;
    else if (dhi < dlo)
        best = hi;
    else
        best = (lo & 1) ? hi : lo; /* exact tie: even mantissa */
    return (uint8_t)(sign | best);
}

/* Round half to even to an integer, then clamp to the symmetric int8 range. */
int8_t orc_int8_encode(double v)
{
    double r = floor(v);
    double frac = v - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))
        r += 1.0;
    if (r > ORC_INT8_MAX)
        r = ORC_INT8_MAX;
    if (r < -ORC_INT8_MAX)
        r = -ORC_INT8_MAX;
    return (int8_t)r;
}

/* ------------------------------------------------------------------ */
/* Dynamic quantization of one group of values that share one scale.  */
/* ------------------------------------------------------------------ */

/* Correctly rounded fp32 quotient a/b of two fp32 values: the fp64 quotient
 * carries more than 2*24+2 bits, so rounding it to fp32 is exact rounding. */
static float div_rn_f32(float a, float b)
{
    return (float)((double)a / (double)b);
}

/*
 * Quantize `count` bf16 values read with stride pattern (rows of `len`
 * contiguous values, `nrows` rows, row pitch `pitch`) to one scale.
 * qtype ORC_E4M3 writes uint8 codes; ORC_INT8 writes int8 codes.
 * Returns the scale.
 */
static float quant_group(const uint16_t *x, long nrows, long len, long pitch,
                         int qtype, void *q, long qpitch)
{
    float amax = 0.0f, s;
    double qmax = (qtype == ORC_E4M3) ? ORC_E4M3_MAX : ORC_INT8_MAX;
    long r, k;
    for (r = 0; r < nrows; r++)
        for (k = 0; k < len; k++) {
            float a = fabsf(bf16_to_float(x[r * pitch + k]));
            if (a > amax)
                amax = a;
        }
    if (amax < ORC_AMAX_FLOOR)
        amax = ORC_AMAX_FLOOR;
    s = div_rn_f32(amax, (float)qmax);
    for (r = 0; r < nrows; r++)
        for (k = 0; k < len; k++) {
            float v = div_rn_f32(bf16_to_float(x[r * pitch + k]), s);
            if (qtype == ORC_E4M3)
                ((uint8_t *)q)[r * qpitch + k] = orc_e4m3_encode(v);
            else
                ((int8_t *)q)[r * qpitch + k] = orc_int8_encode(v);
        }
    return s;
}

/* Per-row (per-token activation, or per-output-channel weight) scaling:
 * x [rows, K] bf16 -> q [rows, K], s [rows]. */
void orc_quant_rows(const uint16_t *x, long rows, long K, int qtype, void *q,
                    float *s)
{
    long r;
    for (r = 0; r < rows; r++) {
        void *qrow = (qtype == ORC_E4M3) ? (void *)((uint8_t *)q + r * K)
                                         : (void *)((int8_t *)q + r * K);
        s[r] = quant_group(x + r * K, 1, K, K, qtype, qrow, K);
    }
}

/* 1 x G activation groups: x [M, K] -> e4m3 q [M, K], s [M, K/G]. */
void orc_quant_groups(const uint16_t *x, long M, long K, long G, uint8_t *q,
                      float *s)
{
    long m, g, ng = K / G;
    for (m = 0; m < M; m++)
        for (g = 0; g < ng; g++)
            s[m * ng + g] = quant_group(x + m * K + g * G, 1, G, K, ORC_E4M3,
                                        q + m * K + g * G, K);
}

/* B x B weight blocks: w [N, K] -> e4m3 q [N, K], s [N/B, K/B]. */
void orc_quant_blocks(const uint16_t *w, long N, long K, long B, uint8_t *q,
                      float *s)
{
    long nb, kb, nbs = N / B, kbs = K / B;
    for (nb = 0; nb < nbs; nb++)
        for (kb = 0; kb < kbs; kb++)
            s[nb * kbs + kb] =
                quant_group(w + nb * B * K + kb * B, B, B, K, ORC_E4M3,
                            q + nb * B * K + kb * B, K);
}

/* ------------------------------------------------------------------ */
/* GEMM in exact integer arithmetic                                    */
/* ------------------------------------------------------------------ */

/*
 * Every e4m3 value is an integer multiple of 2^-9 (the smallest subnormal),
 * and 448 * 2^9 = 229376 < 2^18, so code -> value * 2^9 is an exact integer
 * and a product of two codes is an exact integer times 2^-18.  Sums over
 * K <= 2^15 terms stay below 2^51, so int64 holds them exactly.
 */
static int64_t e4m3_as_int(uint8_t code)
{
    return (int64_t)ldexp(orc_e4m3_decode(code), 9);
}

static int64_t code_int(const void *q, long idx, int qtype)
{
    if (qtype == ORC_E4M3)
        return e4m3_as_int(((const uint8_t *)q)[idx]);
    return (int64_t)((const int8_t *)q)[idx];
}

/* Unit of the integer accumulator: 2^-18 for e4m3 x e4m3, 1 for int8. */
static double acc_unit(int qtype)
{
    return qtype == ORC_E4M3 ? ldexp(1.0, -18) : 1.0;
}

/*
 * Exact dot product of row a of A [*, K] with row b of B [*, K] over the
 * index range [k0, k1).  `absacc` (nullable) receives sum |a_k b_k|.
 */
static int64_t dot_range(const void *A, long a, const void *B, long b, long K,
                         long k0, long k1, int qtype, int64_t *absacc)
{
    int64_t acc = 0, aacc = 0;
    long k;
    for (k = k0; k < k1; k++) {
        int64_t p = code_int(A, a * K + k, qtype) * code_int(B, b * K + k, qtype);
        acc += p;
        aacc += p < 0 ? -p : p;
    }
    if (absacc)
        *absacc = aacc;
    return acc;
}

/*
 * Per-row scaled product (FP8_Dynamic and W8A8_INT8):
 *   acc[m,n] = sum_k Xq[m,k] Wq[n,k]              (exact)
 *   y[m,n]   = acc[m,n] * unit * sx[m] * sw[n]    (fp64)
 *   bound[m,n] = sum_k |x^_k| |w^_k|              (fp64, dequantized)
 * A and B are both K-major: Xq [M, K], Wq [N, K].  acc/bound nullable.
 */
void orc_gemm_rowscaled(const void *xq, const float *sx, const void *wq,
                        const float *sw, long M, long N, long K, int qtype,
                        double *y, double *bound, int64_t *acc)
{
    long n;
    double unit = acc_unit(qtype);
#pragma omp parallel for schedule(dynamic, 1)
    for (n = 0; n < N; n++) {
        long m;
        for (m = 0; m < M; m++) {
            int64_t aabs;
            int64_t a = dot_range(xq, m, wq, n, K, 0, K, qtype, &aabs);
            double scale = (double)sx[m] * (double)sw[n];
            y[m * N + n] = (double)a * unit * scale;
            if (bound)
                bound[m * N + n] = (double)aabs * unit * scale;
            if (acc)
                acc[m * N + n] = a;
        }
    }
}

/*
 * Block-scaled product (Block_FP8): one exact partial sum per G-wide K block,
 * each weighted by its own activation-group scale and weight-block scale:
 *   y[m,n] = sum_kb acc_kb[m,n] * 2^-18 * sx[m,kb] * sw[n/G, kb]
 * sx [M, K/G], sw [N/G, K/G].  bound nullable.
 */
void orc_gemm_blockscaled(const uint8_t *xq, const float *sx,
                          const uint8_t *wq, const float *sw, long M, long N,
                          long K, long G, double *y, double *bound)
{
    long n, kbs = K / G;
    double unit = acc_unit(ORC_E4M3);
#pragma omp parallel for schedule(dynamic, 1)
    for (n = 0; n < N; n++) {
        long m, kb;
        for (m = 0; m < M; m++) {
            double s = 0.0, b = 0.0;
            for (kb = 0; kb < kbs; kb++) {
                int64_t aabs;
                int64_t a = dot_range(xq, m, wq, n, K, kb * G, (kb + 1) * G,
                                      ORC_E4M3, &aabs);
                double scale =
                    (double)sx[m * kbs + kb] * (double)sw[(n / G) * kbs + kb];
                s += (double)a * unit * scale;
                b += (double)aabs * unit * scale;
            }
            y[m * N + n] = s;
            if (bound)
                bound[m * N + n] = b;
        }
    }
}

/*
 * Split-K partition of one exact dot product: K is cut into `splits`
 * contiguous chunks of ceil(K/splits) elements (the last may be short or
 * empty) and the chunk sums are added.  In exact arithmetic the result is
 * the same for every split count; the tests pin that.
 */
int64_t orc_dot_split(const void *xq, long m, const void *wq, long n, long K,
                      int qtype, long splits)
{
    long chunk = (K + splits - 1) / splits, s;
    int64_t total = 0;
    for (s = 0; s < splits; s++) {
        long k0 = s * chunk, k1 = k0 + chunk;
        if (k0 >= K)
            break;
        if (k1 > K)
            k1 = K;
        total += dot_range(xq, m, wq, n, K, k0, k1, qtype, NULL);
    }
    return total;
}

/* ------------------------------------------------------------------ */
/* MXFP8: OCP Microscaling Formats (MX) v1.0 block scaling             */
/* ------------------------------------------------------------------ */

/*
 * The fourth format, beside Block_FP8: Blackwell tensor cores scale FP8
 * operands in hardware with MX block scales (the pages list further vLLM
 * formats and name Blackwell as the next target; the format itself is the
 * OCP MX v1.0 specification).  A block of 32 consecutive values along K
 * shares one scale X = 2^e, stored as an E8M0 byte e + 127 (e in -127..127;
 * the byte 255 would be NaN and is never produced).  The elements are E4M3.
 *
 * Conversion of a block (the specification's rule):
 *   e = floor(log2(max |v|)) - 8       (8: exponent of E4M3's largest
 *                                        normal, 448 = 1.75 * 2^8)
 *   clamped to [-127, 127];  code_i = E4M3(v_i / 2^e), round to nearest
 *   even, magnitudes above 448 saturate to 448.
 * Reading where the specification leaves it open: an all-zero block gets
 * the smallest scale, e = -127 (every code +-0).
 */
static int mx_block_exp(double amax)
{
    int ex;
    if (amax == 0.0)
        return -127;
    frexp(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1): floor(log2) = ex - 1 */
    ex = ex - 1 - 8;
    if (ex < -127)
        ex = -127;
    if (ex > 127)
        ex = 127;
    return ex;
}

/* x [rows, K] bf16 (K % 32 == 0) -> e4m3 codes q [rows, K] and E8M0 scale
 * bytes se [rows, K/32]. */
void orc_quant_mx(const uint16_t *x, long rows, long K, uint8_t *q, uint8_t *se)
{
    long r, b, k, nb = K / 32;
    for (r = 0; r < rows; r++)
        for (b = 0; b < nb; b++) {
            double amax = 0.0, unit;
            int e;
            for (k = 0; k < 32; k++) {
                double a = fabs((double)bf16_to_float(x[r * K + b * 32 + k]));
                if (a > amax)
                    amax = a;
            }
            e = mx_block_exp(amax);
            se[r * nb + b] = (uint8_t)(e + 127);
            unit = ldexp(1.0, e);
            for (k = 0; k < 32; k++) /* division by a power of two: exact */
                q[r * K + b * 32 + k] =
                    orc_e4m3_encode((double)bf16_to_float(x[r * K + b * 32 + k]) / unit);
        }
}

/*
 * MXFP8 product: one exact partial sum per 32-wide K block, weighted by the
 * two blocks' scales:
 *   y[m,n] = sum_b acc_b[m,n] * 2^-18 * 2^(sx[m,b]-127) * 2^(sw[n,b]-127)
 * sx [M, K/32], sw [N, K/32] E8M0 bytes.  bound (nullable) = sum |x^||w^|.
 */
void orc_gemm_mx(const uint8_t *xq, const uint8_t *sx, const uint8_t *wq,
                 const uint8_t *sw, long M, long N, long K, double *y,
                 double *bound)
{
    long n, nb = K / 32;
    double unit = acc_unit(ORC_E4M3);
#pragma omp parallel for schedule(dynamic, 1)
    for (n = 0; n < N; n++) {
        long m, b;
        for (m = 0; m < M; m++) {
            double s = 0.0, bb = 0.0;
            for (b = 0; b < nb; b++) {
                int64_t aabs;
                int64_t a = dot_range(xq, m, wq, n, K, b * 32, (b + 1) * 32,
                                      ORC_E4M3, &aabs);
                double scale = ldexp(1.0, (int)sx[m * nb + b] - 127 +
                                              (int)sw[n * nb + b] - 127);
                s += (double)a * unit * scale;
                bb += (double)aabs * unit * scale;
            }
            y[m * N + n] = s;
            if (bound)
                bound[m * N + n] = bb;
        }
    }
}

/* ------------------------------------------------------------------ */
/* NVFP4: E2M1 values, an E4M3 scale per 16 values along K, and an fp32 */
/* second-level scale per row                                           */
/* ------------------------------------------------------------------ */

/*
 * A fifth format, the 4-bit one the pages list among vLLM's formats
 * ("NVFP4").  The pages define no recipe; this oracle follows the format's
 * published definition (4-bit E2M1 elements, one E4M3 scale per 16
 * consecutive values along K, one fp32 scale above those) and the plainest
 * reading for what the format leaves open, listed in the design notes:
 *   - the fp32 scale is per row: per token for the activations (dynamic, as
 *     the pages' FP8_Dynamic) and per output channel for the weights;
 *   - row r with amax_r = max |x| (at least 1e-12f):
 *       g_r  = fp32(amax_r / 2688)              (2688 = 6 * 448: the largest
 *                                                E2M1 value times E4M3's)
 *     block b of 16 with amax_b:
 *       s_b  = E4M3(fp32(amax_b / fp32(6 * g_r)))       (round to nearest
 *                                                even, saturate at 448)
 *       d_b  = fp32(dec(s_b) * g_r)
 *       code = E2M1(fp32(x / d_b))                (nearest even, saturate
 *                                                at 6; +-0 when d_b is 0)
 *   - storage: two codes per byte, element 2i in the low nibble of byte i.
 * E2M1 (OCP Microscaling Formats v1.0, FP4): 1 sign bit, 2 exponent bits
 * with bias 1, 1 mantissa bit, no infinities or NaN: magnitudes 0, 0.5
 * (subnormal), 1, 1.5, 2, 3, 4, 6.  The sign of zero is kept.
 */
double orc_e2m1_decode(uint8_t code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 0x3;
    int m = code & 0x1;
    double v;
    if (e == 0)
        v = ldexp((double)m / 2.0, 1 - 1); /* subnormal: 0.m * 2^(1-bias) */
    else
        v = ldexp(1.0 + (double)m / 2.0, e - 1);
    return sign ? -v : v;
}

/* Nearest E2M1 code to v; ties to the even mantissa; above 6 saturates. */
uint8_t orc_e2m1_encode(double v)
{
    uint8_t sign = signbit(v) ? 0x8 : 0x0, lo = 0, hi, best;
    double a = fabs(v), dlo, dhi;
    if (a >= 6.0)
        return (uint8_t)(sign | 0x7);
    while (lo < 0x7 && orc_e2m1_decode((uint8_t)(lo + 1)) <= a)
        lo++;
    hi = (uint8_t)(lo + 1);
    dlo = a - orc_e2m1_decode(lo);
    dhi = orc_e2m1_decode(hi) - a;
    if (dlo < dhi)
        best = lo;
    else if (dhi < dlo)
        best = hi;
    else
        best = (lo % 2 == 0) ? lo : hi; /* an exact tie goes to the even mantissa */
    return (uint8_t)(sign | best);
}

static float mul_rn_f32(float a, float b)
{
    return (float)((double)a * (double)b); /* exact in fp64, then one rounding */
}

/* x [rows, K] bf16 (K % 16 == 0) -> packed codes q [rows, K/2], E4M3 block
 * scales s [rows, K/16], row scales g [rows]. */
void orc_quant_nv(const uint16_t *x, long rows, long K, uint8_t *q, uint8_t *s, float *g)
{
    long r, b, k, nb = K / 16;
    memset(q, 0, (size_t)(rows * K / 2));
    for (r = 0; r < rows; r++) {
        float amax = 0.0f, gr, six_g;
        for (k = 0; k < K; k++) {
            float a = fabsf(bf16_to_float(x[r * K + k]));
            if (a > amax)
                amax = a;
        }
        if (amax < ORC_AMAX_FLOOR)
            amax = ORC_AMAX_FLOOR;
        gr = div_rn_f32(amax, 2688.0f);
        g[r] = gr;
        six_g = mul_rn_f32(6.0f, gr);
        for (b = 0; b < nb; b++) {
            float bmax = 0.0f, d;
            uint8_t sc;
            for (k = 0; k < 16; k++) {
                float a = fabsf(bf16_to_float(x[r * K + b * 16 + k]));
                if (a > bmax)
                    bmax = a;
            }
            sc = orc_e4m3_encode((double)div_rn_f32(bmax, six_g));
            s[r * nb + b] = sc;
            d = mul_rn_f32((float)orc_e4m3_decode(sc), gr);
            for (k = 0; k < 16; k++) {
                long i = b * 16 + k;
                float xv = bf16_to_float(x[r * K + i]);
                uint8_t c = (d == 0.0f) ? (uint8_t)(signbit(xv) ? 0x8 : 0x0)
                                        : orc_e2m1_encode((double)div_rn_f32(xv, d));
                q[r * (K / 2) + i / 2] |= (uint8_t)((i & 1) ? (c << 4) : c);
            }
        }
    }
}

/* E2M1 code of element k of a packed row, as an integer number of halves. */
static int64_t e2m1_halves(const uint8_t *row, long k)
{
    uint8_t c = (uint8_t)((k & 1) ? (row[k / 2] >> 4) : (row[k / 2] & 0xF));
    return (int64_t)ldexp(orc_e2m1_decode(c), 1);
}

/* E4M3 scale as an integer number of 2^-9 units (every E4M3 value is one). */
static int64_t e4m3_units(uint8_t code)
{
    return (int64_t)(orc_e4m3_decode(code) * 512.0);
}

/*
 * NVFP4 product, exact: with codes in halves and scales in 2^-9 units every
 * term of
 *   y[m,n] = gx[m] gw[n] sum_b dec(sx[m,b]) dec(sw[n,b]) sum_{k in b} c_x c_w
 * is an integer multiple of 2^-20 and the sum fits in int64 (at most
 * 9216 * 229376^2 per block, 2^15 blocks would be 2^63.4; K <= 25600 gives
 * 1600 blocks, under 2^60).  xq [M, K/2], sx [M, K/16], gx [M]; likewise w.
 * bound (nullable) = sum |x^||w^|.
 */
void orc_gemm_nv(const uint8_t *xq, const uint8_t *sx, const float *gx, const uint8_t *wq,
                 const uint8_t *sw, const float *gw, long M, long N, long K, double *y, double *bound)
{
    long n, nb = K / 16;
#pragma omp parallel for schedule(dynamic, 1)
    for (n = 0; n < N; n++) {
        long m, b, k;
        for (m = 0; m < M; m++) {
            int64_t tot = 0, totabs = 0;
            double unit = ldexp((double)gx[m] * (double)gw[n], -20);
            for (b = 0; b < nb; b++) {
                int64_t blk = 0, blkabs = 0, sc;
                for (k = b * 16; k < b * 16 + 16; k++) {
                    int64_t p = e2m1_halves(xq + m * (K / 2), k) * e2m1_halves(wq + n * (K / 2), k);
                    blk += p;
                    blkabs += p < 0 ? -p : p;
                }
                sc = e4m3_units(sx[m * nb + b]) * e4m3_units(sw[n * nb + b]);
                tot += blk * sc;
                totabs += blkabs * sc;
            }
            y[m * N + n] = (double)tot * unit;
            if (bound)
                bound[m * N + n] = (double)totabs * unit;
        }
    }
}

/* Number of OpenMP threads the GEMMs above run on (1 without OpenMP). */
int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Run the GEMMs above on n OpenMP threads from now on (n >= 1); returns the
 * count in force afterwards.  Only the timing of the CPU baseline uses this:
 * the thread count changes no result (every output is one thread's sum). */
int orc_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n >= 1)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
    return orc_num_threads();
}
