// dequant.cu -- double dequantization of an NF4 weight (QLoRA study notes,
// gitcode.csdn.net, section 3.5 eq. 6): the FP8 constants are expanded with
// their second-level scale and the mean, then every code is looked up in
// the NF4 type and scaled by its block constant.
//
// HBM-bound: 0.5 + 1/64 + 1/16384 bytes read and 4 (fp32) or 2 (bf16) bytes
// written per weight, the writes dominating.  A warp expands 1024 weights
// per step, and every store instruction writes one contiguous 512-byte run
// (whole sectors): for bf16 output lane l takes the four 8-weight groups at
// 8 l + 256 i, for fp32 output the eight 4-weight groups at 4 l + 128 i.
// The 16 codebook values live one per lane (lanes i and i + 16 hold q[i]),
// and a warp shuffle indexed by the 4-bit code fetches each weight's value:
// no shared memory, so the launch needs no carve-out change and no table
// set-up, which is most of the fixed cost at the sizes of one linear.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 1024;  // weights per warp per step
constexpr int kDepthBf16 = 3;  // chunks whose codes and constants a warp has in flight
constexpr int kDepthF32 = 2;   // (fewer for fp32 output: twice the parts per chunk)

// (q[high nibble], q[low nibble]) of byte `byte` of `word`; qv is q[lane % 16]
__device__ __forceinline__ float2 q_pair(float qv, uint32_t word, int byte) {
    const uint32_t b = (word >> (8 * byte)) & 0xFFu;
    return make_float2(__shfl_sync(0xffffffffu, qv, static_cast<int>(b >> 4)),
                       __shfl_sync(0xffffffffu, qv, static_cast<int>(b & 15u)));
}

__device__ __forceinline__ uint32_t ld_nc_u32(const uint8_t* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_nc_u16(const uint8_t* p) {
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// 8 weights of one group (4 code bytes, element 2t the high nibble of byte
// t) scaled by the block constant: w[i] = RN32(q[code_i] * c2').  All 32
// lanes must take part (warp shuffles).
__device__ __forceinline__ void expand8(uint32_t cw, float cp, float qv, float (&w)[8]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 q2 = q_pair(qv, cw, j);
        w[2 * j] = __fmul_rn(q2.x, cp);
        w[2 * j + 1] = __fmul_rn(q2.y, cp);
    }
}

template <bool OUT_BF16>
__device__ __forceinline__ void store8(void* out, int64_t e, const float (&w)[8]) {
    if (OUT_BF16) {
        __stcs(reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + e),
               make_uint4(pack_bf16x2(w[0], w[1]), pack_bf16x2(w[2], w[3]), pack_bf16x2(w[4], w[5]),
                          pack_bf16x2(w[6], w[7])));
    } else {
        float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + e);
        __stcs(o, make_float4(w[0], w[1], w[2], w[3]));
        __stcs(o + 1, make_float4(w[4], w[5], w[6], w[7]));
    }
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(kThreads)
k_dequant(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ c2_fp8,
          const float* __restrict__ c1, const float* __restrict__ mean, int64_t numel,
          void* __restrict__ out, Nf4Tables tabs) {
    const int lane = threadIdx.x & 31;
    const float qv = tabs.q[lane & 15];
    const float mu = *mean;
    const int64_t nfull = numel / kChunk;  // whole 1024-weight chunks
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    int64_t c = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;

    // The lane's parts of a chunk.  bf16 output: part p is the 8 weights at
    // 256 p + 8 lane (4 code bytes; one 16-byte store, 512 contiguous bytes
    // per warp).  fp32 output: part p is the 4 weights at 128 p + 4 lane
    // (2 code bytes; one 16-byte store, again 512 contiguous bytes per warp,
    // so every store instruction writes whole sectors).  kDepth chunks of
    // codes and constants are in flight per warp (a register ring).
    constexpr int kParts = OUT_BF16 ? 4 : 8;
    constexpr int kDepth = OUT_BF16 ? kDepthBf16 : kDepthF32;
    struct Chunk {
        uint32_t cw[kParts], fb[kParts];
        float s1[kParts];
    };
    auto first = [&](int64_t ch, int p) -> int64_t {
        return ch * kChunk + (OUT_BF16 ? 256 * p + 8 * lane : 128 * p + 4 * lane);
    };
    auto load = [&](int64_t ch, Chunk& k) {
#pragma unroll
        for (int p = 0; p < kParts; ++p) {
            const int64_t e = first(ch, p);
            k.cw[p] = OUT_BF16 ? ld_nc_u32(codes + (e >> 1)) : ld_nc_u16(codes + (e >> 1));
            k.fb[p] = __ldg(c2_fp8 + (e >> 6));
            k.s1[p] = __ldg(c1 + (e >> 14));
        }
    };
    Chunk ring[kDepth];
#pragma unroll
    for (int k = 0; k < kDepth; ++k)
        if (c + k * nwarps < nfull) load(c + k * nwarps, ring[k]);
    for (int64_t base = c; base < nfull; base += kDepth * nwarps) {
#pragma unroll
        for (int k = 0; k < kDepth; ++k) {
            const int64_t ch = base + k * nwarps;
            if (ch >= nfull) break;
#pragma unroll
            for (int p = 0; p < kParts; ++p) {
                const float cp = dq_constant(static_cast<uint8_t>(ring[k].fb[p]), ring[k].s1[p], mu);
                const int64_t e = first(ch, p);
                if (OUT_BF16) {
                    float w[8];
                    expand8(ring[k].cw[p], cp, qv, w);
                    store8<true>(out, e, w);
                } else {
                    const float2 a = q_pair(qv, ring[k].cw[p], 0);
                    const float2 b = q_pair(qv, ring[k].cw[p], 1);
                    __stcs(reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + e),
                           make_float4(__fmul_rn(a.x, cp), __fmul_rn(a.y, cp), __fmul_rn(b.x, cp),
                                       __fmul_rn(b.y, cp)));
                }
            }
            if (ch + kDepth * nwarps < nfull) load(ch + kDepth * nwarps, ring[k]);
        }
    }
    // the ragged last chunk (< 1024 weights), by one warp, lanes diverging:
    // direct table reads, whole 8-weight groups stored as vectors, the last
    // partial group element by element
    const int64_t wid = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    if (nfull * kChunk < numel && wid == nfull % nwarps) {
#pragma unroll 1
        for (int i = 0; i < 4; ++i) {
            const int64_t e = nfull * kChunk + 8 * lane + 256 * i;
            if (e >= numel) continue;
            const float cp = dq_constant(c2_fp8[e >> 6], c1[e >> 14], mu);
            if (e + 8 <= numel) {
                const uint32_t w4 = static_cast<uint32_t>(codes[e >> 1]) | (static_cast<uint32_t>(codes[(e >> 1) + 1]) << 8) |
                                    (static_cast<uint32_t>(codes[(e >> 1) + 2]) << 16) |
                                    (static_cast<uint32_t>(codes[(e >> 1) + 3]) << 24);
                float w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t b = (w4 >> (8 * (j >> 1))) & 0xFFu;
                    w[j] = __fmul_rn(tabs.q[(j & 1) ? (b & 15u) : (b >> 4)], cp);
                }
                store8<OUT_BF16>(out, e, w);
            } else {
                for (int64_t k = e; k < numel; ++k) {
                    const uint8_t byte = codes[k >> 1];
                    const int code = (k & 1) ? (byte & 15) : (byte >> 4);
                    const float v = __fmul_rn(tabs.q[code], cp);
                    if (OUT_BF16)
                        reinterpret_cast<uint16_t*>(out)[k] = f32_to_bf16_bits(v);
                    else
                        reinterpret_cast<float*>(out)[k] = v;
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                              const float* mean, int64_t numel, void* out, int out_dtype,
                              cudaStream_t stream, int qtype) {
    const int64_t chunks = ceil_div(numel, kChunk);
    const int64_t want = ceil_div(chunks, kThreads / 32);
    const int grid = static_cast<int>(want < num_sms() * 3LL ? (want > 0 ? want : 1) : num_sms() * 3LL);
    if (out_dtype == 1)
        k_dequant<true><<<grid, kThreads, 0, stream>>>(codes, c2_fp8, c1, mean, numel, out, tables(qtype));
    else
        k_dequant<false><<<grid, kThreads, 0, stream>>>(codes, c2_fp8, c1, mean, numel, out, tables(qtype));
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace qlora
