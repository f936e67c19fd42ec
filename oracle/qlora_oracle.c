/*
 * qlora_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-file CPU implementation of what the QLoRA NF4 linear
 * layer computes, written from the method's description and used as the
 * parity oracle for the CUDA library.  It shares no code, header, table or
 * constant generator with the CUDA path, and the CUDA path never calls it:
 * only the tests, the graft entry's smoke check and the benchmark's CPU
 * baseline leg may load this library.
 *
 * Sources (web pages about QLoRA, Dettmers et al., arXiv:2305.14314):
 *   [notes]  "QLoRA: Efficient Finetuning of Quantized LLMs" study notes,
 *            gitcode.csdn.net -- sections 3.1 (block-wise k-bit
 *            quantization, eq. 1-2), 3.2 (NF4, eq. 4), 3.3 (double
 *            quantization), 3.5 (QLoRA linear, eq. 5-6) and 4 (LoRA, eq. 3).
 *
 * Where the pages leave a step open the reading taken is stated beside the
 * function.  Every floating-point step is written out unfused (the file is
 * compiled with -ffp-contract=off) so that each rounding is the one named.
 *
 * Parity status: every function here is pinned by CPU tests against facts
 * that the pages or mathematics fix (tests/test_oracle_pins.py).  The 14
 * interior NF4 code values depend on the tail probability delta, which the
 * pages do not print; their agreement with any external NF4 table is
 * "parity unpinned" (the construction itself is pinned by its
 * equal-probability property).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_NONFINITE 5

/* ------------------------------------------------------------------------ */
/* Bit helpers                                                              */
/* ------------------------------------------------------------------------ */

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* bf16 value of a 16-bit pattern, widened exactly to double. */
static double bf16_to_double(uint16_t h) { return (double)u2f(((uint32_t)h) << 16); }

/* Round-to-nearest-even of an fp32 value to bfloat16 (8-bit significand).
 * NaN maps to a quiet NaN; everything else is the IEEE RNE result. */
uint16_t oracle_bf16_rne(float x)
{
    uint32_t u = f2u(x);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return 0x7fc0;
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

void oracle_bf16_rne_array(const float* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_rne(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Inverse standard normal CDF: Wichura, "Algorithm AS 241: The percentage  */
/* points of the normal distribution", Applied Statistics 37 (1988),        */
/* PPND16 (relative accuracy about 1e-16), evaluated in double precision.   */
/* ------------------------------------------------------------------------ */

static double poly8(const double* c, double x)
{
    /* c[0] + c[1] x + ... + c[7] x^7, Horner from the top coefficient. */
    double v = c[7];
    for (int i = 6; i >= 0; --i) v = v * x + c[i];
    return v;
}

double oracle_norm_ppf(double p)
{
    /* central region |p - 1/2| <= 0.425 */
    static const double a[8] = {3.387132872796366608, 133.14166789178437745,
        1971.5909503065514427, 13731.693765509461125, 45921.953931549871457,
        67265.770927008700853, 33430.575583588128105, 2509.0809287301226727};
    static const double b[8] = {1.0, 42.313330701600911252,
        687.1870074920579083, 5394.1960214247511077, 21213.794301586595867,
        39307.89580009271061, 28729.085735721942674, 5226.495278852545925};
    /* intermediate tail, r = sqrt(-log(min(p,1-p))) <= 5 */
    static const double c[8] = {1.42343711074968357734, 4.6303378461565452959,
        5.7694972214606914055, 3.64784832476320460504, 1.27045825245236838258,
        0.24178072517745061177, 0.0227238449892691845833,
        7.7454501427834140764e-4};
    static const double d[8] = {1.0, 2.05319162663775882187,
        1.6763848301838038494, 0.68976733498510000455, 0.14810397642748007459,
        0.0151986665636164571966, 5.475938084995344946e-4,
        1.05075007164441684324e-9};
    /* far tail, r > 5 */
    static const double e[8] = {6.6579046435011037772, 5.4637849111641143699,
        1.7848265399172913358, 0.29656057182850489123, 0.026532189526576123093,
        0.0012426609473880784386, 2.71155556874348757815e-5,
        2.01033439929228813265e-7};
    static const double f[8] = {1.0, 0.59983220655588793769,
        0.13692988092273580531, 0.0148753612908506148525,
        7.868691311456132591e-4, 1.8463183175100546818e-5,
        1.4215117583164458887e-7, 2.04426310338993978564e-15};

    if (!(p > 0.0 && p < 1.0)) {
        if (p == 0.0) return -INFINITY;
        if (p == 1.0) return INFINITY;
        return NAN;
    }
    double q = p - 0.5;
    if (fabs(q) <= 0.425) {
        double r = 0.180625 - q * q;
        return q * poly8(a, r) / poly8(b, r);
    }
    double r = q < 0.0 ? p : 1.0 - p;
    r = sqrt(-log(r));
    double v;
    if (r <= 5.0) {
        r -= 1.6;
        v = poly8(c, r) / poly8(d, r);
    } else {
        r -= 5.0;
        v = poly8(e, r) / poly8(f, r);
    }
    return q < 0.0 ? -v : v;
}

/* ------------------------------------------------------------------------ */
/* a1. NF4 codebook ([notes] 3.2, eq. 4 and the asymmetric construction).   */
/*                                                                          */
/* The type's 2^k values are quantiles of N(0,1).  To hold an exact zero,   */
/* the negative half takes 2^(k-1) quantile points and the positive half    */
/* 2^(k-1)+1, each half including the centre p = 1/2 (value 0), the two     */
/* halves are merged with the duplicate zero removed, and the result is     */
/* normalised into [-1, 1].                                                 */
/*                                                                          */
/* Reading (eq. 4 as printed puts Q(0) = -inf at the end): each half places */
/* its points at evenly spaced probabilities from 1/2 out to a common tail  */
/* probability delta, and delta is eq. 4's "average of two adjacent         */
/* quantile points" applied to the outermost bin of the 15- and 16-bin      */
/* grids: delta = ((1 - 1/30) + (1 - 1/32)) / 2.  Both halves end at        */
/* Q(delta), so dividing by it gives exactly -1 and +1 at the ends.         */
/* ------------------------------------------------------------------------ */

double oracle_nf4_delta(void) { return 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0)); }

void oracle_nf4_codebook(float q[16])
{
    const double delta = oracle_nf4_delta();
    const double qmax = oracle_norm_ppf(delta);
    double v[16];
    int n = 0;
    /* negative half: 8 points from 1/2 to delta, minus the centre -> 7 */
    for (int i = 7; i >= 1; --i) {
        double p = 0.5 + (delta - 0.5) * (double)i / 7.0;
        v[n++] = -oracle_norm_ppf(p);
    }
    v[n++] = 0.0; /* the one shared zero */
    /* positive half: 9 points from 1/2 to delta, minus the centre -> 8 */
    for (int i = 1; i <= 8; ++i) {
        double p = 0.5 + (delta - 0.5) * (double)i / 8.0;
        v[n++] = oracle_norm_ppf(p);
    }
    for (int i = 0; i < 16; ++i) q[i] = (float)(v[i] / qmax);
}

/* ------------------------------------------------------------------------ */
/* a2 + a3. Block-wise absmax and NF4 encoding ([notes] 3.1, 3.2 step 3).   */
/*                                                                          */
/* The tensor is flattened and cut into consecutive blocks of B = 64        */
/* elements; each block keeps its own constant c2 = max |w| (the last block */
/* may be short).  Each element is normalised, n = w / c2 (fp32, RN), and   */
/* mapped to the nearest codebook value: argmin_i |n - q_i| computed in     */
/* fp32, ties to the lower index.  Two codes share a byte, element 2t in    */
/* the high nibble; an odd tail leaves a zero low nibble.  A block whose    */
/* absmax is 0 stores c2 = 0 and the zero code (index 7) everywhere.        */
/* ------------------------------------------------------------------------ */

/* ------------------------------------------------------------------------ */
/* The 4-bit types NF4 is compared with ([notes] 5.1.2, Table 2): FP4 read  */
/* as OCP E2M1 and Int4 as eq. 1 at 4 bits.  Both are 16-entry tables in   */
/* [-1, 1] used exactly like the NF4 table (absmax scaling, nearest value,  */
/* ties to the lower index); a value that repeats is listed twice (the      */
/* second copy is never the nearest).                                       */
/* ------------------------------------------------------------------------ */

/* E2M1 bit pattern -> value: sign bit 3, exponent bits 2..1 (bias 1),      */
/* mantissa bit 0; exponent 0 is subnormal (0 or 0.5).                      */
double oracle_e2m1_decode(int bits)
{
    int sgn = (bits >> 3) & 1, e = (bits >> 1) & 3, m = bits & 1;
    double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sgn ? -mag : mag;
}

/* FP4: the distinct E2M1 values in ascending order, divided by the largest */
/* (6); the top value is repeated to fill 16 entries.                       */
void oracle_fp4_codebook(float q[16])
{
    double v[16];
    int n = 0;
    for (int b = 0; b < 16; ++b) {
        double x = oracle_e2m1_decode(b);
        int dup = 0;
        for (int i = 0; i < n; ++i) if (v[i] == x) dup = 1;   /* -0 == +0 */
        if (!dup) v[n++] = x;
    }
    for (int i = 1; i < n; ++i)                                /* insertion sort */
        for (int j = i; j > 0 && v[j - 1] > v[j]; --j) { double t = v[j]; v[j] = v[j - 1]; v[j - 1] = t; }
    double top = v[n - 1];
    for (int i = 0; i < 16; ++i) q[i] = (float)(v[i < n ? i : n - 1] / top);
}

/* Int4: eq. 1 with 2^(4-1) - 1 = 7 levels per side: k / 7, k = -7..7, the  */
/* top value repeated at index 15.                                          */
void oracle_int4_codebook(float q[16])
{
    for (int i = 0; i < 16; ++i) {
        int k = i < 15 ? i - 7 : 7;
        q[i] = (float)((double)k / 7.0);
    }
}

static int nearest_code(float n, const float q[16])
{
    int best = 0;
    float bd = fabsf(n - q[0]);
    for (int i = 1; i < 16; ++i) {
        float d = fabsf(n - q[i]);
        if (d < bd) { bd = d; best = i; }
    }
    return best;
}

int oracle_quantize_nf4(const float* w, int64_t numel, int block, const float q[16],
                        uint8_t* codes, float* c2)
{
    if (numel < 0 || block <= 0) return OR_ERR_ARG;
    int nonfinite = 0;
    int64_t nb = (numel + block - 1) / block;
    memset(codes, 0, (size_t)((numel + 1) / 2));
    for (int64_t j = 0; j < nb; ++j) {
        int64_t lo = j * block, hi = lo + block < numel ? lo + block : numel;
        float amax = 0.0f;
        for (int64_t i = lo; i < hi; ++i) {
            if (!isfinite(w[i])) nonfinite = 1;
            float a = fabsf(w[i]);
            if (a > amax) amax = a;
        }
        c2[j] = amax;
        for (int64_t i = lo; i < hi; ++i) {
            int code = 7;
            if (amax > 0.0f) {
                float n = w[i] / amax;
                code = nearest_code(n, q);
            }
            if ((i & 1) == 0) codes[i >> 1] |= (uint8_t)(code << 4);
            else codes[i >> 1] |= (uint8_t)code;
        }
    }
    return nonfinite ? OR_ERR_NONFINITE : OR_OK;
}

/* ------------------------------------------------------------------------ */
/* a4. Mean of the first-level constants ([notes] 3.3: c2 is all positive,  */
/* its mean is subtracted before the second quantization).                  */
/*                                                                          */
/* Reading: one mean per tensor (the bits/param count 8/64 + 32/(64*256)    */
/* has no room for per-block means), defined from the exact sum S of all   */
/* c2: mu = RN32( RN64( RN64(S) / nb ) ).  S is accumulated exactly as an  */
/* integer multiple of 2^-149 (every finite fp32 is one) in 64-bit limbs.  */
/* ------------------------------------------------------------------------ */

#define ACC_LIMBS 7

static void acc_add(uint64_t acc[ACC_LIMBS], uint64_t m, int shift)
{
    int limb = shift / 64, off = shift % 64;
    uint64_t lo = m << off;
    uint64_t hi = off ? (m >> (64 - off)) : 0;
    uint64_t old = acc[limb];
    acc[limb] += lo;
    uint64_t carry = acc[limb] < old;
    for (int k = limb + 1; k < ACC_LIMBS && (hi || carry); ++k) {
        uint64_t add = hi + carry;           /* hi < 2^63, no wrap */
        old = acc[k];
        acc[k] += add;
        carry = acc[k] < old;
        hi = 0;
    }
}

/* Round the non-negative integer acc * 2^-149 to the nearest double, ties
 * to even. */
static double acc_to_double(const uint64_t acc[ACC_LIMBS])
{
    int top = -1;
    for (int k = ACC_LIMBS - 1; k >= 0 && top < 0; --k)
        if (acc[k]) top = k * 64 + 63 - __builtin_clzll(acc[k]);
    if (top < 0) return 0.0;
#define BIT(i) ((int)((acc[(i) / 64] >> ((i) % 64)) & 1u))
    uint64_t mant = 0;
    int lo = top - 52 > 0 ? top - 52 : 0;
    for (int i = top; i >= lo; --i) mant = (mant << 1) | (uint64_t)BIT(i);
    int exp = lo; /* value = mant * 2^lo * 2^-149 before rounding */
    if (lo > 0) {
        int rbit = BIT(lo - 1);
        int sticky = 0;
        for (int i = lo - 2; i >= 0 && !sticky; --i) sticky = BIT(i);
        if (rbit && (sticky || (mant & 1u))) mant += 1; /* may reach 2^53: still exact */
    }
#undef BIT
    return ldexp((double)mant, exp - 149);
}

/* Returns OR_OK and writes mu and RN64(S); OR_ERR_NONFINITE if any c2 is not
 * a finite non-negative number. */
int oracle_mean_exact(const float* c2, int64_t nb, float* mu, double* sum_rn64)
{
    uint64_t acc[ACC_LIMBS];
    memset(acc, 0, sizeof acc);
    if (nb <= 0) return OR_ERR_ARG;
    for (int64_t j = 0; j < nb; ++j) {
        uint32_t u = f2u(c2[j]);
        if (u >> 31) { if (u != 0x80000000u) return OR_ERR_NONFINITE; continue; }
        uint32_t ex = u >> 23, fr = u & 0x7fffffu;
        if (ex == 255) return OR_ERR_NONFINITE;
        uint64_t m = ex ? (fr | 0x800000u) : fr;
        int shift = ex ? (int)ex - 1 : 0; /* value = m * 2^(shift-149) */
        acc_add(acc, m, shift);
    }
    double s = acc_to_double(acc);
    if (sum_rn64) *sum_rn64 = s;
    double m64 = s / (double)nb;
    *mu = (float)m64;
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 (OCP "e4m3fn": bias 7, no infinities, 0x7f/0xff = NaN, max     */
/* finite 448, subnormal spacing 2^-9).                                     */
/* ------------------------------------------------------------------------ */

float oracle_e4m3_decode(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* Round-to-nearest-even into E4M3, saturating finite overflow (and
 * infinities) to +-448. */
uint8_t oracle_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7f;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7e;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range (and the rounding up into 2^-6): unit 2^-9 */
        double m = nearbyint(a * 512.0); /* exact scaling, RNE */
        return sign | (uint8_t)m;        /* m == 8 encodes 2^-6 itself */
    }
    int ex;
    double fr = frexp(a, &ex); /* a = fr * 2^ex, fr in [0.5, 1) */
    ex -= 1;                   /* a in [2^ex, 2^(ex+1)) */
    double mant = ldexp(fr, 1) - 1.0;     /* in [0, 1), exact */
    double m = nearbyint(mant * 8.0);     /* RNE */
    if (m == 8.0) { m = 0.0; ex += 1; }
    return sign | (uint8_t)(((ex + 7) << 3) | (int)m);
}

void oracle_e4m3_encode_array(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(x[i]);
}

/* ------------------------------------------------------------------------ */
/* a5. Double quantization ([notes] 3.3): c2 (fp32, one per 64-block) is    */
/* quantized again, to 8-bit floats in blocks of 256, after subtracting     */
/* the mean.  Reading: the 8-bit float is E4M3 and the scaling is the FP8   */
/* analogue of eq. 1's absmax scaling into the type's full range:           */
/*   y = c2 - mu,  c1 = max|y| / 448,  byte = E4M3(y / c1)                  */
/* each operation rounded to fp32 and the byte to nearest even with        */
/* saturation.  A group whose c1 is 0 stores zero bytes.                    */
/* ------------------------------------------------------------------------ */

void oracle_double_quant(const float* c2, int64_t nb, float mu, int block2,
                         uint8_t* c2_fp8, float* c1)
{
    int64_t ng = (nb + block2 - 1) / block2;
    for (int64_t g = 0; g < ng; ++g) {
        int64_t lo = g * block2, hi = lo + block2 < nb ? lo + block2 : nb;
        float amax = 0.0f;
        for (int64_t j = lo; j < hi; ++j) {
            float y = c2[j] - mu;
            float a = fabsf(y);
            if (a > amax) amax = a;
        }
        float c = amax / 448.0f;
        c1[g] = c;
        for (int64_t j = lo; j < hi; ++j) {
            if (c == 0.0f) { c2_fp8[j] = 0; continue; }
            float y = c2[j] - mu;
            float t = y / c;
            c2_fp8[j] = oracle_e4m3_encode(t);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a6 + a7. Double dequantization ([notes] 3.5 eq. 6):                      */
/*   c2'  = RN32( RN32(E4M3(byte) * c1) + mu )                              */
/*   w'   = RN32( q[code] * c2' )                                           */
/* ------------------------------------------------------------------------ */

void oracle_dequant_constants(const uint8_t* c2_fp8, const float* c1, float mu,
                              int64_t nb, int block2, float* c2p)
{
    for (int64_t j = 0; j < nb; ++j) {
        float t = oracle_e4m3_decode(c2_fp8[j]) * c1[j / block2];
        c2p[j] = t + mu;
    }
}

void oracle_dequantize(const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                       float mu, int64_t numel, int block, int block2,
                       const float q[16], float* out)
{
    int64_t nb = (numel + block - 1) / block;
    float* c2p = (float*)malloc(sizeof(float) * (size_t)(nb ? nb : 1));
    oracle_dequant_constants(c2_fp8, c1, mu, nb, block2, c2p);
    for (int64_t i = 0; i < numel; ++i) {
        uint8_t byte = codes[i >> 1];
        int code = (i & 1) ? (byte & 15) : (byte >> 4);
        out[i] = q[code] * c2p[i / block];
    }
    free(c2p);
}

/* ------------------------------------------------------------------------ */
/* a8 - a10. The QLoRA linear ([notes] 3.5 eq. 5, 4 eq. 3), in our row-     */
/* major naming: X (M x K), frozen W (N x K, dequantized and rounded to     */
/* bf16 -- eq. 6 outputs W in BF16), A (r x K) and B (N x r) for the        */
/* pages' L1 = A^T and L2 = B^T, s the LoRA scalar of eq. 3:                */
/*   Y  = X W^T + s (X A^T) B^T                                             */
/*   dX = dY W + s (dY B) A                                                 */
/*   dA = s (dY B)^T X,    dB = s dY^T (X A^T)                              */
/* No gradient for W ([notes] 3.5).  Every sum is accumulated in fp64 and   */
/* the intermediates X A^T and dY B are kept in fp64.  Rows of Y and dX may */
/* be restricted to a sampled list; dA and dB are always full.              */
/* ------------------------------------------------------------------------ */

typedef struct {
    void (*fn)(void* ctx, int64_t lo, int64_t hi);
    void* ctx;
    int64_t lo, hi;
} job_t;

static void* job_run(void* p)
{
    job_t* j = (job_t*)p;
    j->fn(j->ctx, j->lo, j->hi);
    return NULL;
}

static int g_threads = 0;
void oracle_set_threads(int n) { g_threads = n; }
int oracle_get_threads(void)
{
    if (g_threads > 0) return g_threads;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* Run fn over [0, n) split into contiguous ranges, one per thread. */
static void parallel_for(int64_t n, void (*fn)(void*, int64_t, int64_t), void* ctx)
{
    int t = oracle_get_threads();
    if (t > n) t = (int)(n > 0 ? n : 1);
    if (t <= 1) { fn(ctx, 0, n); return; }
    pthread_t th[256];
    job_t jobs[256];
    if (t > 256) t = 256;
    for (int i = 0; i < t; ++i) {
        jobs[i].fn = fn; jobs[i].ctx = ctx;
        jobs[i].lo = n * i / t; jobs[i].hi = n * (i + 1) / t;
        pthread_create(&th[i], NULL, job_run, &jobs[i]);
    }
    for (int i = 0; i < t; ++i) pthread_join(th[i], NULL);
}

/* P (rows x c) = L (rows x k, bf16) * R^T, R (c x k, bf16); fp64 out. */
typedef struct {
    const uint16_t* L; const uint16_t* R; double* P;
    int64_t k, c; const int64_t* rows;
} abt_ctx;

static void abt_body(void* p, int64_t lo, int64_t hi)
{
    abt_ctx* x = (abt_ctx*)p;
    double* lrow = (double*)malloc(sizeof(double) * (size_t)x->k);
    for (int64_t i = lo; i < hi; ++i) {
        int64_t src = x->rows ? x->rows[i] : i;
        for (int64_t t = 0; t < x->k; ++t) lrow[t] = bf16_to_double(x->L[src * x->k + t]);
        for (int64_t j = 0; j < x->c; ++j) {
            const uint16_t* rr = x->R + j * x->k;
            double acc = 0.0;
            for (int64_t t = 0; t < x->k; ++t) acc += lrow[t] * bf16_to_double(rr[t]);
            x->P[i * x->c + j] = acc;
        }
    }
    free(lrow);
}

static void mat_abt(const uint16_t* L, const int64_t* rows, int64_t nrows,
                    const uint16_t* R, int64_t c, int64_t k, double* P)
{
    abt_ctx x = {L, R, P, k, c, rows};
    parallel_for(nrows, abt_body, &x);
}

/* Y rows = X[rows] W^T + s T0[rows] B^T; T0 = X A^T (fp64). */
typedef struct {
    const uint16_t* X; const uint16_t* W; const uint16_t* A; const uint16_t* B;
    int64_t N, K, r; double s; const int64_t* rows; double* Y; double* T0;
} fwd_ctx;

static void fwd_body(void* p, int64_t lo, int64_t hi)
{
    fwd_ctx* c = (fwd_ctx*)p;
    double* x = (double*)malloc(sizeof(double) * (size_t)c->K);
    double* t0 = (double*)malloc(sizeof(double) * (size_t)(c->r ? c->r : 1));
    for (int64_t i = lo; i < hi; ++i) {
        int64_t m = c->rows ? c->rows[i] : i;
        for (int64_t k = 0; k < c->K; ++k) x[k] = bf16_to_double(c->X[m * c->K + k]);
        for (int64_t j = 0; j < c->r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < c->K; ++k) acc += x[k] * bf16_to_double(c->A[j * c->K + k]);
            t0[j] = acc;
            if (c->T0) c->T0[i * c->r + j] = acc;
        }
        for (int64_t n = 0; n < c->N; ++n) {
            const uint16_t* wr = c->W + n * c->K;
            double acc = 0.0;
            for (int64_t k = 0; k < c->K; ++k) acc += x[k] * bf16_to_double(wr[k]);
            double lora = 0.0;
            for (int64_t j = 0; j < c->r; ++j) lora += t0[j] * bf16_to_double(c->B[n * c->r + j]);
            c->Y[i * c->N + n] = acc + c->s * lora;
        }
    }
    free(x); free(t0);
}

/* X: M x K bf16, W: N x K bf16 (the dequantized frozen weight), A: r x K,
 * B: N x r.  rows (nullable) selects which rows of Y to compute; Y is
 * nrows x N, T0 (nullable) nrows x r holds X A^T. */
int oracle_linear_fwd(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                      const uint16_t* W, const uint16_t* A, const uint16_t* B,
                      int64_t r, double s, const int64_t* rows, int64_t nrows,
                      double* Y, double* T0)
{
    if (M < 0 || N < 0 || K < 0 || r < 0) return OR_ERR_ARG;
    if (!rows) nrows = M;
    fwd_ctx c = {X, W, A, B, N, K, r, s, rows, Y, T0};
    parallel_for(nrows, fwd_body, &c);
    return OR_OK;
}

/* dX rows = dY[rows] W + s U0[rows] A, with U0 = dY B. */
typedef struct {
    const uint16_t* dY; const uint16_t* W; const uint16_t* A; const double* U0;
    int64_t N, K, r; double s; const int64_t* rows; double* dX;
} dx_ctx;

static void dx_body(void* p, int64_t lo, int64_t hi)
{
    dx_ctx* c = (dx_ctx*)p;
    double* acc = (double*)malloc(sizeof(double) * (size_t)(c->K ? c->K : 1));
    for (int64_t i = lo; i < hi; ++i) {
        int64_t m = c->rows ? c->rows[i] : i;
        for (int64_t k = 0; k < c->K; ++k) acc[k] = 0.0;
        for (int64_t n = 0; n < c->N; ++n) {
            double g = bf16_to_double(c->dY[m * c->N + n]);
            const uint16_t* wr = c->W + n * c->K;
            for (int64_t k = 0; k < c->K; ++k) acc[k] += g * bf16_to_double(wr[k]);
        }
        for (int64_t k = 0; k < c->K; ++k) {
            double lora = 0.0;
            for (int64_t j = 0; j < c->r; ++j)
                lora += c->U0[m * c->r + j] * bf16_to_double(c->A[j * c->K + k]);
            c->dX[i * c->K + k] = acc[k] + c->s * lora;
        }
    }
    free(acc);
}

/* dA (r x K) = s U0^T X, parallel over k columns. */
typedef struct {
    const uint16_t* X; const double* U0; int64_t M, K, r; double s; double* dA;
} da_ctx;

static void da_body(void* p, int64_t lo, int64_t hi)
{
    da_ctx* c = (da_ctx*)p;
    for (int64_t j = 0; j < c->r; ++j)
        for (int64_t k = lo; k < hi; ++k) c->dA[j * c->K + k] = 0.0;
    for (int64_t m = 0; m < c->M; ++m) {
        const uint16_t* xr = c->X + m * c->K;
        for (int64_t j = 0; j < c->r; ++j) {
            double u = c->U0[m * c->r + j];
            double* row = c->dA + j * c->K;
            for (int64_t k = lo; k < hi; ++k) row[k] += u * bf16_to_double(xr[k]);
        }
    }
    for (int64_t j = 0; j < c->r; ++j)
        for (int64_t k = lo; k < hi; ++k) c->dA[j * c->K + k] *= c->s;
}

/* dB (N x r) = s dY^T T0, parallel over n rows. */
typedef struct {
    const uint16_t* dY; const double* T0; int64_t M, N, r; double s; double* dB;
} db_ctx;

static void db_body(void* p, int64_t lo, int64_t hi)
{
    db_ctx* c = (db_ctx*)p;
    for (int64_t n = lo; n < hi; ++n)
        for (int64_t j = 0; j < c->r; ++j) c->dB[n * c->r + j] = 0.0;
    for (int64_t m = 0; m < c->M; ++m) {
        const double* t = c->T0 + m * c->r;
        const uint16_t* gr = c->dY + m * c->N;
        for (int64_t n = lo; n < hi; ++n) {
            double g = bf16_to_double(gr[n]);
            double* row = c->dB + n * c->r;
            for (int64_t j = 0; j < c->r; ++j) row[j] += g * t[j];
        }
    }
    for (int64_t n = lo; n < hi; ++n)
        for (int64_t j = 0; j < c->r; ++j) c->dB[n * c->r + j] *= c->s;
}

/* dY: M x N bf16.  dX (nullable) is nrows x K for the selected rows (all
 * rows when rows is NULL); dA r x K and dB N x r are always full. */
int oracle_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, int64_t N,
                      int64_t K, const uint16_t* W, const uint16_t* A, const uint16_t* B,
                      int64_t r, double s, const int64_t* rows, int64_t nrows,
                      double* dX, double* dA, double* dB)
{
    if (M < 0 || N < 0 || K < 0 || r < 0) return OR_ERR_ARG;
    if (!rows) nrows = M;
    size_t mr = (size_t)(M * r ? M * r : 1);
    double* U0 = (double*)malloc(sizeof(double) * mr);  /* dY B^T-free: dY (MxN) * B (Nxr) */
    double* T0 = (double*)malloc(sizeof(double) * mr);  /* X A^T */
    /* U0[m][j] = sum_n dY[m][n] B[n][j]  -- B is N x r, so use its transpose view */
    {
        uint16_t* Bt = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(N * r ? N * r : 1));
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < r; ++j) Bt[j * N + n] = B[n * r + j];
        mat_abt(dY, NULL, M, Bt, r, N, U0);
        free(Bt);
    }
    mat_abt(X, NULL, M, A, r, K, T0);
    if (dX) {
        dx_ctx c = {dY, W, A, U0, N, K, r, s, rows, dX};
        parallel_for(nrows, dx_body, &c);
    }
    if (dA) {
        da_ctx c = {X, U0, M, K, r, s, dA};
        parallel_for(K, da_body, &c);
    }
    if (dB) {
        db_ctx c = {dY, T0, M, N, r, s, dB};
        parallel_for(N, db_body, &c);
    }
    free(U0); free(T0);
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Block-wise Int8 absmax quantization, [notes] 3.1 eq. 1 and eq. 2 (the    */
/* 8-bit baseline the NF4 type is compared with).                           */
/*   c = 127 / absmax(X),  X_int8 = round(c X),  dequant = X_int8 / c       */
/* round() is the pages' "round half away from zero" (C's round()).  The    */
/* arithmetic is fp32 throughout.  A block whose absmax is 0 stores c = 0   */
/* and codes 0 and dequantizes to 0 (eq. 2 would divide by 0; the pages do  */
/* not treat that case).                                                     */
/* ------------------------------------------------------------------------ */

void oracle_int8_quant(const float* x, int64_t n, int8_t* out, float* c)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) { float a = fabsf(x[i]); if (a > amax) amax = a; }
    float cc = amax > 0.0f ? 127.0f / amax : 0.0f;
    *c = cc;
    for (int64_t i = 0; i < n; ++i) {
        float t = cc * x[i];
        out[i] = (int8_t)roundf(t);
    }
}

void oracle_int8_dequant(const int8_t* xq, int64_t n, float c, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = c != 0.0f ? (float)xq[i] / c : 0.0f;
}

/* The same over consecutive blocks of `block` elements of a flattened    */
/* tensor (the last block may be partial): one constant c per block.      */
void oracle_int8_quant_blocks(const float* x, int64_t n, int64_t block, int8_t* out, float* c)
{
    for (int64_t b0 = 0, j = 0; b0 < n; b0 += block, ++j) {
        int64_t len = n - b0 < block ? n - b0 : block;
        oracle_int8_quant(x + b0, len, out + b0, c + j);
    }
}

void oracle_int8_dequant_blocks(const int8_t* xq, int64_t n, int64_t block, const float* c, float* out)
{
    for (int64_t b0 = 0, j = 0; b0 < n; b0 += block, ++j) {
        int64_t len = n - b0 < block ? n - b0 : block;
        oracle_int8_dequant(xq + b0, len, c[j], out + b0);
    }
}
