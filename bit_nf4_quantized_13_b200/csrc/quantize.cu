// quantize.cu -- NF4 block-wise quantization fused with the exact-sum pass of
// the double quantization, and the FP8 double-quantization pass itself.
//
// QLoRA study notes (gitcode.csdn.net): section 3.1 (block-wise absmax
// quantization, blocks of 64 consecutive elements of the flattened tensor),
// section 3.2 step 3 (normalise by absmax, then quantize to the nearest NF4
// value), section 3.3 (double quantization: the fp32 constants c2 minus
// their mean, quantized to 8-bit floats in blocks of 256).
//
// Kernel 1 (k_nf4_quantize) streams W once: HBM-bound at 4 B read + 0.5 B
// written per weight.  A warp takes 512 consecutive weights per step: in
// load i (0..3) lane l holds weights 4(32i + l) .. +3, so every load is one
// fully coalesced 512-byte row and lanes 0-15 / 16-31 hold the two 64-blocks
// of that row.  The block absmax is a 16-lane shuffle reduction.  Each
// constant c2 is also added, exactly, into 256 integer bins (one per fp32
// exponent) so that the mean of all c2 is exact and independent of the
// order in which blocks finish.
//
// Kernel 2 (k_double_quant) turns the bins into the mean, then per group of
// 256 constants computes c1 = max|c2 - mean| / 448 and the E4M3 bytes.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

struct EncTab {
    float thr;
    int base;
};

// rcp.approx: within 2^-22 relative of 1/a for normal a (the PTX ISA
// bounds its error by 1 ulp)
__device__ __forceinline__ float rcp_approx(float a) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(a));
    return y;
}

__device__ __forceinline__ float4 ld_stream(const float* p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// max that propagates NaN, so one test per block catches NaN and Inf
__device__ __forceinline__ float max_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

constexpr int kQuantThreads = 256;
constexpr int kChunk = 512;  // weights per warp step

// Absmax of the two 64-blocks a warp holds in one load (lanes 0-15: the
// first, lanes 16-31: the second), as fp32 bit patterns with the sign
// cleared: two whole-warp integer max reductions.  |NaN| (max.NaN gives the
// canonical NaN) and Inf compare above every finite value.
__device__ __forceinline__ void block_absmax_bits(const float4& v, int lane, uint32_t& lo, uint32_t& hi) {
    const float a = max_nan(max_nan(fabsf(v.x), fabsf(v.y)), max_nan(fabsf(v.z), fabsf(v.w)));
    const uint32_t u = __float_as_uint(a);
    const bool upper = lane >= 16;
    lo = __reduce_max_sync(0xffffffffu, upper ? 0u : u);
    hi = __reduce_max_sync(0xffffffffu, upper ? u : 0u);
}

// The lane's 4 codes (two bytes, little-endian) for block absmax m (finite,
// non-zero).
//
// Codes without dividing in the common case: with y ~ 1/m (relative error
// <= 2^-22), n~ = RN(w y) lies within 2^-21 of n = RN(w / m) for |n| <= 1.
// The code is a step function of n whose steps (thresholds) lie at least
// 1.6e-3 from the table's bin edges, so the bin of n~ serves n as well, and
// the one threshold comparison agrees for n~ and n whenever n~ is more than
// 2^-20 from the threshold (d = RN(n~ - thr) gives both: d >= 0 iff
// n~ >= thr).  A lane whose four quotients are all clear of their
// thresholds is done; otherwise (rarely) it divides exactly.  The table has
// one extra entry below -1 (index 0) because n~ may undershoot -1 by a
// rounding, so finite inputs never need clamping.  Every lane reads its own
// copy of the table (entry i of lane l at 8 (32 i + l) bytes, so a warp's
// lookups never share a bank): `tabl` is the lane's copy shifted by the
// 0xFFF bin-index bias, addressed by (bits(n + 3) >> 18) * 256 bytes.
__device__ __forceinline__ const EncTab& lane_entry(const uint8_t* tabl, float n) {
    return *reinterpret_cast<const EncTab*>(tabl + ((__float_as_uint(n) >> 10) & ~0xFFu));
}

__device__ __forceinline__ uint32_t encode4(const float4& v, float m, const EncTab* tab, const uint8_t* tabl) {
    const float w[4] = {v.x, v.y, v.z, v.w};
    uint32_t q[4];
    bool exact = !(m >= 0x1p-120f && m <= 0x1p120f);  // extreme scales: always divide
    if (!exact) {
        const float y = rcp_approx(m);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float na = __fmul_rn(w[i], y);
            const EncTab e = lane_entry(tabl, __fadd_rn(na, 3.0f));
            const float d = __fsub_rn(na, e.thr);
            q[i] = static_cast<uint32_t>(e.base) + (d >= 0.0f ? 1u : 0u);
            exact |= fabsf(d) <= 0x1p-20f;
        }
    }
    if (exact) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float n = __fdiv_rn(w[i], m);
            const unsigned b = (__float_as_uint(__fadd_rn(n, 3.0f)) >> 18) - 0xFFFu;
            const EncTab e = tab[b > 33u ? 33u : b];
            q[i] = static_cast<uint32_t>(e.base) + (n >= e.thr ? 1u : 0u);
        }
    }
    // byte e/2 = (code e << 4) | code e+1, little-endian in the returned pair
    return (q[0] << 4) | q[1] | (q[2] << 12) | (q[3] << 8);
}

__global__ void __launch_bounds__(kQuantThreads, 3)
k_nf4_quantize(const float* __restrict__ W, int64_t numel, uint8_t* __restrict__ codes,
               float* __restrict__ c2, unsigned long long* __restrict__ bins,
               int* __restrict__ flag, Nf4Tables tabs) {
    __shared__ EncTab tab[34];       // [0]: below -1; [1 + b]: bin b of the host table
    __shared__ EncTab tabr[34 * 32];  // the same, one copy per lane: [i][lane]
    // exact-sum bins of this CTA, as 32-bit words plus carry counts (native
    // 32-bit shared atomics; a carry out of the low word is counted apart)
    __shared__ uint32_t sbin_lo[256], sbin_hi[256];
    __shared__ int sbad;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sbin_lo[i] = sbin_hi[i] = 0u;
    for (int i = threadIdx.x; i < 34 * 32; i += blockDim.x) {
        const int e = i >> 5;
        tabr[i] = e == 0 ? EncTab{2.0f, 0} : EncTab{tabs.thr[e - 1], tabs.base[e - 1]};
    }
    if (threadIdx.x < 33) tab[1 + threadIdx.x] = EncTab{tabs.thr[threadIdx.x], tabs.base[threadIdx.x]};
    if (threadIdx.x == 33) tab[0] = EncTab{2.0f, 0};
    if (threadIdx.x == 0) sbad = 0;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    // this lane's copy, biased so that byte offset (bits >> 18) * 256 finds entry (bits >> 18) - 0xFFF
    const uint8_t* tabl = reinterpret_cast<const uint8_t*>(tabr) + 8 * lane - 0xFFF * 256;
    const int64_t nb = ceil_div(numel, kBlock);
    const int64_t nfull = numel / kChunk;  // whole 512-weight chunks
    const int64_t nchunks = ceil_div(numel, kChunk);
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    bool bad = false;

    auto load_full = [&](int64_t c, float4 (&v)[4]) {
        const float* src = W + c * kChunk + 4 * lane;
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = ld_stream(src + 128 * i);
    };
    // Lanes 0-7 finish the chunk's 8 blocks: the constant c2 (coalesced) and
    // its exact addition into the exponent bins.
    auto finish_chunk = [&](int64_t base, float mb) {
        if (lane < 8) {
            const int64_t blk = (base >> 6) + lane;
            if (blk < nb) {
                c2[blk] = mb;
                const uint32_t u = __float_as_uint(mb);
                const uint32_t ex = u >> 23;
                const uint32_t mant = ex ? ((u & 0x7fffffu) | 0x800000u) : (u & 0x7fffffu);
                if (mant) {
                    const uint32_t old = atomicAdd(&sbin_lo[ex & 255u], mant);
                    if (old + mant < old) atomicAdd(&sbin_hi[ex & 255u], 1u);
                }
            }
        }
    };
    // One chunk: 4 loads of 512 bytes, each holding two 64-blocks.
    auto encode_chunk = [&](int64_t c, const float4 (&v)[4]) {
        const int64_t base = c * kChunk;
        uint16_t* dst = reinterpret_cast<uint16_t*>(codes + (base >> 1)) + lane;
        float mb = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t lo, hi;
            block_absmax_bits(v[i], lane, lo, hi);
            const uint32_t mine = lane >= 16 ? hi : lo;
            if ((lane >> 1) == i) mb = __uint_as_float((lane & 1) ? hi : lo);
            // NaN or Inf in the block: flagged, codes unspecified; an all-zero
            // block gets the zero code
            bad |= mine >= 0x7f800000u;
            const bool ok = mine - 1u < 0x7f7fffffu;  // finite and non-zero
            // otherwise encode zeros: the table index stays in range only for |w| <= m
            const float4 vi = ok ? v[i] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            const uint32_t b01 = encode4(vi, ok ? __uint_as_float(mine) : 1.0f, tab, tabl);
            dst[32 * i] = static_cast<uint16_t>(ok ? b01 : 0x7777u);  // bytes (base + 128 i + 4 lane) / 2
        }
        finish_chunk(base, mb);
    };

    // whole chunks, the next chunk's loads in flight while one encodes
    int64_t c = warp0;
    float4 va[4], vb[4];
    if (c < nfull) load_full(c, va);
    while (c < nfull) {
        if (c + nwarps < nfull) load_full(c + nwarps, vb);
        encode_chunk(c, va);
        c += nwarps;
        if (c >= nfull) break;
        if (c + nwarps < nfull) load_full(c + nwarps, va);
        encode_chunk(c, vb);
        c += nwarps;
    }
    // the ragged last chunk (at most one), by the warp whose turn it is
    if (nfull < nchunks && (nfull % nwarps) == warp0) {
        const int64_t base = nfull * kChunk;
        float mb = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t e = base + 4 * (32 * i + lane);
            float4 v;
            v.x = e + 0 < numel ? W[e + 0] : 0.0f;
            v.y = e + 1 < numel ? W[e + 1] : 0.0f;
            v.z = e + 2 < numel ? W[e + 2] : 0.0f;
            v.w = e + 3 < numel ? W[e + 3] : 0.0f;
            uint32_t lo, hi;
            block_absmax_bits(v, lane, lo, hi);
            const uint32_t mine = lane >= 16 ? hi : lo;
            if ((lane >> 1) == i) mb = __uint_as_float((lane & 1) ? hi : lo);
            uint32_t b01 = 0x7777u;
            if (mine >= 0x7f800000u)
                bad = true;
            else if (mine != 0u)
                b01 = encode4(v, __uint_as_float(mine), tab, tabl);
            if (e < numel) codes[e >> 1] = static_cast<uint8_t>(e + 1 < numel ? (b01 & 0xff) : (b01 & 0xf0));
            if (e + 2 < numel) codes[(e >> 1) + 1] = static_cast<uint8_t>(e + 3 < numel ? (b01 >> 8) : ((b01 >> 8) & 0xf0));
        }
        finish_chunk(base, mb);
    }
    // the double-quant kernel may now be scheduled onto SMs this grid frees
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (bad) sbad = 1;
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
        const unsigned long long t = (static_cast<unsigned long long>(sbin_hi[i]) << 32) | sbin_lo[i];
        if (t) atomicAdd(&bins[i], t);
    }
    if (threadIdx.x == 0 && sbad) atomicOr(flag, 1);
}

// ------------------------------------------------------------------------
// Exact mean from the exponent bins.  Bin E holds the integer sum of the
// 24-bit significands of all c2 with exponent field E; its value is
// bins[E] * 2^(max(E,1) - 150).  As an integer multiple of 2^-149 the total
// is sum_E bins[E] << (max(E,1) - 1).  Lane l folds its eight bins
// E = 8l .. 8l+7 into one 128-bit value relative to 2^(max(8l,1) - 1)
// (each term < 2^64 shifted by at most 7: the sum stays below 2^75).  The
// non-zero lane values (one or two for real weights, whose constants share
// a few exponents) are then added, by every lane alike, into 32-bit digits
// held in registers (only compile-time indices, so nothing goes to local
// memory); the total is rounded once to the nearest double (round bit and
// sticky bit, from the leading 64 bits), divided by nb in double and
// rounded to fp32.  Called by one whole warp; every lane returns the mean.
constexpr int kDigits = 12;

__device__ float mean_from_bins(const unsigned long long* __restrict__ bins, int64_t nb) {
    const int lane = threadIdx.x & 31;
    unsigned long long lo = 0, hi = 0;
    const int e0 = 8 * lane, base = e0 ? e0 : 1;  // exponent field whose bin shift is the lane's origin
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int e = e0 + k;
        const unsigned long long v = bins[e];
        const int sh = (e ? e : 1) - base;  // 0..7
        const unsigned long long vlo = v << sh, vhi = sh ? (v >> (64 - sh)) : 0ull;
        lo += vlo;
        hi += vhi + (lo < vlo ? 1ull : 0ull);
    }
    uint32_t d[kDigits + 1];
#pragma unroll
    for (int i = 0; i <= kDigits; ++i) d[i] = 0u;
    // the same mask in every lane, so the loop is warp-uniform
    unsigned rest = __ballot_sync(0xffffffffu, (lo | hi) != 0ull);
    while (rest) {
        const int l = __ffs(rest) - 1;
        rest &= rest - 1u;
        const unsigned long long vlo = __shfl_sync(0xffffffffu, lo, l), vhi = __shfl_sync(0xffffffffu, hi, l);
        const int sh = (l ? 8 * l : 1) - 1;  // bit position of the lane value's origin, <= 247
        const int d0 = sh >> 5, off = sh & 31;
        // the value (< 2^75) as 32-bit words, shifted by off into 4 words at digits d0 .. d0+3
        const uint32_t w0 = static_cast<uint32_t>(vlo), w1 = static_cast<uint32_t>(vlo >> 32),
                       w2 = static_cast<uint32_t>(vhi);
        const uint32_t p0 = w0 << off;
        const uint32_t p1 = off ? (w1 << off) | (w0 >> (32 - off)) : w1;
        const uint32_t p2 = off ? (w2 << off) | (w1 >> (32 - off)) : w2;
        const uint32_t p3 = off ? (w2 >> (32 - off)) : 0u;
        unsigned long long carry = 0;
#pragma unroll
        for (int i = 0; i <= kDigits; ++i) {
            const int k = i - d0;
            const uint32_t add = k == 0 ? p0 : k == 1 ? p1 : k == 2 ? p2 : k == 3 ? p3 : 0u;
            const unsigned long long t = static_cast<unsigned long long>(d[i]) + add + carry;
            d[i] = static_cast<uint32_t>(t);
            carry = t >> 32;
        }
    }
    // highest non-zero digit, the two under it, and whether any lower digit is non-zero
    int top = -1;
#pragma unroll
    for (int i = 0; i <= kDigits; ++i)
        if (d[i]) top = i;
    if (top < 0) return 0.0f;
    uint32_t dt = 0u, dt1 = 0u, dt2 = 0u;
    bool sticky = false;
#pragma unroll
    for (int i = 0; i <= kDigits; ++i) {
        dt = i == top ? d[i] : dt;
        dt1 = i == top - 1 ? d[i] : dt1;
        dt2 = i == top - 2 ? d[i] : dt2;
        sticky |= i < top - 2 && d[i] != 0u;
    }
    // the leading 64 bits of the total (digits top, top-1, top-2), left aligned
    const unsigned long long t0 = (static_cast<unsigned long long>(dt) << 32) | dt1;
    const int lz = __clzll(t0);  // < 32: dt != 0
    const unsigned long long lead = lz ? (t0 << lz) | (static_cast<unsigned long long>(dt2) >> (32 - lz)) : t0;
    // bit position (over the whole total) of the lead's lowest bit
    const int lead_lsb = 32 * top + 32 - lz - 64;  // = msb - 63, may be negative
    unsigned long long m = lead >> 11;              // 53 bits
    const bool rnd = (lead >> 10) & 1ull;
    sticky |= (lead & 0x3ffull) != 0;
    // dt2's bits under the lead
    sticky |= (lz ? (dt2 & ((1u << (32 - lz)) - 1u)) : dt2) != 0u;
    if (rnd && (sticky || (m & 1ull))) m += 1ull;  // 2^53 stays exact
    const double sum = ldexp(static_cast<double>(m), lead_lsb + 11 - 149);
    return __double2float_rn(__ddiv_rn(sum, static_cast<double>(nb)));
}

constexpr int kDqThreads = 256;  // 8 warps, one 256-group per warp at a time

__global__ void __launch_bounds__(kDqThreads)
k_double_quant(const float* __restrict__ c2, int64_t nb, const unsigned long long* __restrict__ bins,
               const int* __restrict__ flag, uint8_t* __restrict__ c2_fp8, float* __restrict__ c1,
               float* __restrict__ mean_out, int32_t* __restrict__ status) {
    __shared__ float smu;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ng = ceil_div(nb, kBlock2);
    const int64_t wpb = kDqThreads / 32;
    const int64_t g0 = static_cast<int64_t>(blockIdx.x) * wpb + warp;
    float y[kBlock2 / 32];  // the constants of this warp's current group
    auto load_group = [&](int64_t g) {
#pragma unroll
        for (int i = 0; i < kBlock2 / 32; ++i) {
            const int64_t j = g * kBlock2 + 32 * i + lane;
            y[i] = j < nb ? c2[j] : 0.0f;
        }
    };
    // launched as a programmatic dependent of k_nf4_quantize: wait for that
    // grid's completion (and its bins, c2 and flag) before reading anything
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (g0 < ng) load_group(g0);  // in flight while warp 0 finds the mean
    if (warp == 0) {
        const float mu = mean_from_bins(bins, nb);
        if (lane == 0) smu = mu;
    }
    __syncthreads();
    const float mu = smu;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *mean_out = mu;
        if (status) *status = (*flag) ? QLORA_ERR_NONFINITE : QLORA_OK;
    }
    for (int64_t g = g0; g < ng; g += static_cast<int64_t>(gridDim.x) * wpb) {
        if (g != g0) load_group(g);
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < kBlock2 / 32; ++i) {
            const int64_t j = g * kBlock2 + 32 * i + lane;
            y[i] = j < nb ? __fsub_rn(y[i], mu) : 0.0f;
            a = fmaxf(a, fabsf(y[i]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const float c = __fdiv_rn(a, 448.0f);
        if (lane == 0) c1[g] = c;
#pragma unroll
        for (int i = 0; i < kBlock2 / 32; ++i) {
            const int64_t j = g * kBlock2 + 32 * i + lane;
            if (j < nb) c2_fp8[j] = (c == 0.0f) ? static_cast<uint8_t>(0) : f32_to_e4m3(__fdiv_rn(y[i], c));
        }
    }
}

__global__ void k_e4m3_encode(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t n) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        out[i] = f32_to_e4m3(x[i]);
}

}  // namespace

cudaError_t launch_quantize_nf4_dq(const float* W, int64_t numel, uint8_t* codes, uint8_t* c2_fp8,
                                   float* c1, float* mean, void* ws, int32_t* status,
                                   cudaStream_t stream, int qtype) {
    const int64_t nb = ceil_div(numel, kBlock);
    auto* bins = reinterpret_cast<unsigned long long*>(ws);
    int* flag = reinterpret_cast<int*>(reinterpret_cast<char*>(ws) + kBinBytes);
    float* c2 = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kBinBytes + kFlagBytes);
    cudaError_t err = cudaMemsetAsync(ws, 0, kBinBytes + kFlagBytes, stream);
    if (err != cudaSuccess) return err;
    const int64_t nchunks = ceil_div(numel, kChunk);
    const int64_t want = ceil_div(nchunks, kQuantThreads / 32);
    // CTAs of k_nf4_quantize per SM, asked once per context
    static ContextMemo<int> resident_memo;
    int resident = 2;
    uint64_t ctx = 0;
    if (current_context_id(&ctx))
        resident_memo.get(ctx, &resident, [](int* v) {
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, k_nf4_quantize, kQuantThreads, 0) != cudaSuccess ||
                *v < 1) {
                cudaGetLastError();
                *v = 2;
            }
            return true;
        });
    const int64_t cap = static_cast<int64_t>(num_sms()) * resident;
    const int grid1 = static_cast<int>(want < cap ? want : cap);
    k_nf4_quantize<<<grid1, kQuantThreads, 0, stream>>>(W, numel, codes, c2, bins, flag, tables(qtype));
    note_launches(1);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const int64_t ng = ceil_div(nb, kBlock2);
    const int64_t want2 = ceil_div(ng, kDqThreads / 32);
    const int grid2 = static_cast<int>(want2 < num_sms() * 4LL ? want2 : num_sms() * 4LL);
    // programmatic stream serialization: its launch overlaps the quantize
    // kernel's tail; griddepcontrol.wait inside orders every read after it
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid2));
    cfg.blockDim = dim3(kDqThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, k_double_quant, static_cast<const float*>(c2), nb,
                             static_cast<const unsigned long long*>(bins), static_cast<const int*>(flag), c2_fp8, c1,
                             mean, status);
    note_launches(1);
    return err;
}

cudaError_t launch_e4m3_encode(const float* x, uint8_t* out, int64_t n, cudaStream_t stream) {
    const int64_t want = ceil_div(n, 256);
    const int grid = static_cast<int>(want < num_sms() * 16LL ? want : num_sms() * 16LL);
    k_e4m3_encode<<<grid, 256, 0, stream>>>(x, out, n);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace qlora
