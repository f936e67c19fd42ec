// codebook.cu -- host construction of the 4-bit data types (NF4, and FP4 and
// Int4 for comparison) and of their encoder tables.
//
// The NF4 values follow the QLoRA study notes (gitcode.csdn.net), section 3.2:
// quantiles of N(0,1), 2^(k-1) for the negative half and 2^(k-1)+1 for the
// positive half, both halves including p = 1/2 (value 0) and sharing it,
// normalised into [-1, 1].  Eq. (4) as printed reaches Q(0) = -inf at the
// end of its grid; the reading taken is that each half spaces its
// probabilities evenly from 1/2 to delta, where delta averages the
// outermost quantile points of the 15- and 16-bin grids:
// delta = ((1 - 1/30) + (1 - 1/32)) / 2.
//
// The standard normal quantile here is computed by root finding on the
// complementary error function of the C library (bisection to the last
// bit, then Newton polishing), in double precision.
#include <math.h>
#include <mutex>
#include <stdint.h>
#include <string.h>

#include "common.cuh"

namespace qlora {
namespace {

// Upper-tail probability P(Z > x) = erfc(x / sqrt 2) / 2, accurate relative
// to the tail itself.
double upper_tail(double x) { return 0.5 * erfc(x * 0.70710678118654752440); }

// Q(p) for p in (0, 1).  Works on the smaller tail t = min(p, 1 - p) (exact
// for p >= 1/2 by Sterbenz), solves upper_tail(x) = t for x >= 0 and
// restores the sign.
double normal_quantile(double p) {
    if (p == 0.5) return 0.0;
    const double t = p < 0.5 ? p : 1.0 - p;
    double lo = 0.0, hi = 40.0;  // upper_tail is decreasing on [0, 40]
    for (int it = 0; it < 2000; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (upper_tail(mid) > t) lo = mid; else hi = mid;
    }
    double x = 0.5 * (lo + hi);
    for (int it = 0; it < 2; ++it) {  // Newton on upper_tail(x) - t
        const double dens = exp(-0.5 * x * x) * 0.39894228040143267794;
        x += (upper_tail(x) - t) / dens;
    }
    return p < 0.5 ? -x : x;
}

void build_nf4(float q[16]) {
    const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
    const double top = normal_quantile(delta);
    double v[16];
    // negative half: probabilities 1/2 + (delta - 1/2) * i / 7, i = 7..1
    for (int i = 7; i >= 1; --i) v[7 - i] = -normal_quantile(0.5 + (delta - 0.5) * i / 7.0);
    v[7] = 0.0;
    // positive half: probabilities 1/2 + (delta - 1/2) * i / 8, i = 1..8
    for (int i = 1; i <= 8; ++i) v[7 + i] = normal_quantile(0.5 + (delta - 0.5) * i / 8.0);
    for (int i = 0; i < 16; ++i) q[i] = static_cast<float>(v[i] / top);
}

// FP4 as OCP E2M1 (1 sign, 2 exponent, 1 mantissa bit): magnitudes 0, 0.5,
// 1, 1.5, 2, 3, 4, 6, normalised by the largest so that absmax maps to +-1.
// The 15 distinct signed values in ascending order (the two zeros of the
// format are one value), the top one repeated at index 15.
void build_fp4(float q[16]) {
    const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    for (int i = 7; i >= 1; --i) q[7 - i] = static_cast<float>(-mag[i] / 6.0);
    q[7] = 0.0f;
    for (int i = 1; i <= 7; ++i) q[7 + i] = static_cast<float>(mag[i] / 6.0);
    q[15] = q[14];
}

// Int4 as the 4-bit case of the absmax integer quantization of eq. (1): the
// symmetric levels k / 7, k = -7 .. 7, the top one repeated at index 15.
void build_int4(float q[16]) {
    for (int k = -7; k <= 7; ++k) q[k + 7] = static_cast<float>(static_cast<double>(k) / 7.0);
    q[15] = q[14];
}

// fp32 total order on bit patterns (for bisection over representable values)
int64_t fkey(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return (u & 0x80000000u) ? -static_cast<int64_t>(u & 0x7fffffffu) : static_cast<int64_t>(u);
}
float from_key(int64_t k) {
    uint32_t u = k < 0 ? (static_cast<uint32_t>(-k) | 0x80000000u) : static_cast<uint32_t>(k);
    float f;
    memcpy(&f, &u, 4);
    return f;
}

// Nearest-code rule in fp32 between neighbours j and j+1: the upper code
// wins iff RN(n - q_j) > RN(q_{j+1} - n) (a tie keeps the lower index).
// The predicate is monotone in n; the threshold is the smallest fp32 n in
// [q_j, q_{j+1}] where it holds.
bool upper_wins(float n, float qj, float qj1) {
    volatile float a = n - qj;    // volatile: one fp32 rounding each, no reassociation
    volatile float b = qj1 - n;
    return a > b;
}

float threshold(float qj, float qj1) {
    int64_t lo = fkey(qj), hi = fkey(qj1);  // predicate false at lo, true at hi
    while (hi - lo > 1) {
        int64_t mid = lo + (hi - lo) / 2;
        if (upper_wins(from_key(mid), qj, qj1)) hi = mid; else lo = mid;
    }
    return from_key(hi);
}

// Bin of n on the device: b = (bits(RN(n + 3)) >> 18) - 0x1000, i.e. 32
// equal bins of width 1/16 over [-1, 1) plus bin 32 for n = 1.
int bin_of(float n) {
    volatile float v = n + 3.0f;
    float vv = v;
    uint32_t u;
    memcpy(&u, &vv, 4);
    return static_cast<int>(u >> 18) - 0x1000;
}

Nf4Tables build_tables(int qtype) {
    Nf4Tables t;
    if (qtype == QLORA_TYPE_FP4)
        build_fp4(t.q);
    else if (qtype == QLORA_TYPE_INT4)
        build_int4(t.q);
    else
        build_nf4(t.q);
    // a repeated value never wins (ties go to the lower index): its threshold
    // lies beyond the range of n
    float thr[15];
    for (int j = 0; j < 15; ++j) thr[j] = t.q[j] == t.q[j + 1] ? 2.0f : threshold(t.q[j], t.q[j + 1]);
    auto code_of = [&](float n) {
        int c = 0;
        for (int j = 0; j < 15; ++j) c += (n >= thr[j]);
        return c;
    };
    // For every bin, the smallest n in [-1, 1] that maps to it; the bins'
    // preimages are consecutive intervals because n -> bin is monotone.
    int64_t lo_key[34];
    for (int b = 0; b <= 32; ++b) {
        int64_t lo = fkey(-1.0f), hi = fkey(1.0f);
        if (bin_of(from_key(lo)) >= b) { lo_key[b] = lo; continue; }
        while (hi - lo > 1) {  // bin_of(lo) < b <= bin_of(hi)
            int64_t mid = lo + (hi - lo) / 2;
            if (bin_of(from_key(mid)) >= b) hi = mid; else lo = mid;
        }
        lo_key[b] = hi;
    }
    lo_key[33] = fkey(1.0f) + 1;
    for (int b = 0; b <= 32; ++b) {
        const float first = from_key(lo_key[b]);
        const float last = from_key(lo_key[b + 1] - 1);
        t.base[b] = code_of(first);
        t.thr[b] = 2.0f;  // no threshold inside: never reached for |n| <= 1
        int inside = 0;
        for (int j = 0; j < 15; ++j)
            if (thr[j] > first && thr[j] <= last) { t.thr[b] = thr[j]; ++inside; }
        if (inside > 1 || code_of(last) != t.base[b] + inside) {
            // cannot happen for the three types (their thresholds are at
            // least 0.08 apart, the bins 1/16 wide); keep the failure loud
            t.base[b] = -1000;
        }
    }
    return t;
}

std::once_flag g_once[3];
Nf4Tables g_tables[3];

}  // namespace

const Nf4Tables& tables(int qtype) {
    const int t = (qtype == QLORA_TYPE_FP4 || qtype == QLORA_TYPE_INT4) ? qtype : QLORA_TYPE_NF4;
    std::call_once(g_once[t], [t] { g_tables[t] = build_tables(t); });
    return g_tables[t];
}

bool valid_qtype(int qtype) {
    return qtype == QLORA_TYPE_NF4 || qtype == QLORA_TYPE_FP4 || qtype == QLORA_TYPE_INT4;
}

}  // namespace qlora

extern "C" int qlora_codebook(int qtype, float out_host[16]) {
    if (!out_host || !qlora::valid_qtype(qtype)) return QLORA_ERR_INVALID_ARG;
    memcpy(out_host, qlora::tables(qtype).q, sizeof(float) * 16);
    return QLORA_OK;
}

extern "C" int qlora_nf4_codebook(float out_host[16]) { return qlora_codebook(QLORA_TYPE_NF4, out_host); }
