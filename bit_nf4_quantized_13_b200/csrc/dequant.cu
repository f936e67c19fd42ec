// dequant.cu -- double dequantization of an NF4 weight (QLoRA study notes,
// gitcode.csdn.net, section 3.5 eq. 6): the FP8 constants are expanded with
// their second-level scale and the mean, then every code is looked up in
// the NF4 type and scaled by its block constant.
//
// HBM-bound: 0.5 + 1/64 + 1/16384 bytes read and 4 (fp32) or 2 (bf16) bytes
// written per weight.  Each lane expands 32 consecutive weights per step
// from one 16-byte load of codes and one block constant; code nibbles become
// table byte offsets with shift/mask and byte_perm, and pairs of weights are
// scaled with one f32x2 multiply.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;
constexpr int kRun = 32;  // weights per lane per step: 16 code bytes, one block constant

__device__ __forceinline__ uint4 ld_nc_v4(const uint8_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// q[code] from the 16-entry table by byte offset (code * 4)
__device__ __forceinline__ float lut_at(const float* lut, uint32_t byte_off) {
    return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(lut) + byte_off);
}

// 32 weights of one block from 16 code bytes: element 2t is the high nibble
// of byte t.  out[i] = RN32(q[code_i] * c2').
__device__ __forceinline__ void expand32(const uint4& cw, float cp, const float* lut, float (&w)[kRun]) {
    const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const uint32_t hi4 = (w4[h] >> 2) & 0x3C3C3C3Cu;
        const uint32_t lo4 = (w4[h] << 2) & 0x3C3C3C3Cu;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 x = __fmul2_rn(make_float2(lut_at(lut, __byte_perm(hi4, 0u, 0x4440u | j)),
                                                    lut_at(lut, __byte_perm(lo4, 0u, 0x4440u | j))),
                                        make_float2(cp, cp));
            w[8 * h + 2 * j] = x.x;
            w[8 * h + 2 * j + 1] = x.y;
        }
    }
}

// Each lane owns 32 consecutive weights per step (one 16-byte load of
// codes, one block constant), grid-stride with the next step's loads in
// flight.  OUT_BF16 selects bf16 (64-byte) or fp32 (128-byte) output runs.
template <bool OUT_BF16>
__global__ void __launch_bounds__(kThreads)
k_dequant(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ c2_fp8,
          const float* __restrict__ c1, const float* __restrict__ mean, int64_t numel,
          void* __restrict__ out, Nf4Tables tabs) {
    __shared__ float s_lut[16];
    if (threadIdx.x < 16) s_lut[threadIdx.x] = tabs.q[threadIdx.x];
    __syncthreads();
    const float mu = *mean;
    const int64_t nfull = numel / kRun;  // whole 32-weight runs
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;

    uint4 cw = make_uint4(0u, 0u, 0u, 0u);
    uint32_t sb = 0u;
    float sc1 = 0.0f;
    auto load = [&](int64_t run, uint4& c, uint32_t& b, float& s1) {
        const int64_t e = run * kRun;
        c = ld_nc_v4(codes + (e >> 1));
        b = __ldg(c2_fp8 + (e >> 6));
        s1 = __ldg(c1 + (e >> 14));
    };
    if (t < nfull) load(t, cw, sb, sc1);
    for (; t < nfull; t += stride) {
        uint4 ncw = cw;
        uint32_t nsb = sb;
        float ns1 = sc1;
        if (t + stride < nfull) load(t + stride, ncw, nsb, ns1);
        float w[kRun];
        expand32(cw, dq_constant(static_cast<uint8_t>(sb), sc1, mu), s_lut, w);
        const int64_t e = t * kRun;
        if (OUT_BF16) {
            uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + e);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                __stcs(o + c, make_uint4(pack_bf16x2(w[8 * c + 0], w[8 * c + 1]), pack_bf16x2(w[8 * c + 2], w[8 * c + 3]),
                                         pack_bf16x2(w[8 * c + 4], w[8 * c + 5]), pack_bf16x2(w[8 * c + 6], w[8 * c + 7])));
        } else {
            float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + e);
#pragma unroll
            for (int c = 0; c < 8; ++c)
                __stcs(o + c, make_float4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]));
        }
        cw = ncw;
        sb = nsb;
        sc1 = ns1;
    }
    // ragged tail (< 32 weights), one thread
    if (blockIdx.x == 0 && threadIdx.x == 0 && nfull * kRun < numel) {
        for (int64_t e = nfull * kRun; e < numel; ++e) {
            const uint8_t byte = codes[e >> 1];
            const int code = (e & 1) ? (byte & 15) : (byte >> 4);
            const float cp = dq_constant(c2_fp8[e >> 6], c1[e >> 14], mu);
            const float v = __fmul_rn(s_lut[code], cp);
            if (OUT_BF16)
                reinterpret_cast<uint16_t*>(out)[e] = f32_to_bf16_bits(v);
            else
                reinterpret_cast<float*>(out)[e] = v;
        }
    }
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                              const float* mean, int64_t numel, void* out, int out_dtype,
                              cudaStream_t stream) {
    const int64_t runs = ceil_div(numel, kRun);
    const int64_t want = ceil_div(runs, kThreads);
    const int grid = static_cast<int>(want < num_sms() * 8LL ? (want > 0 ? want : 1) : num_sms() * 8LL);
    if (out_dtype == 1)
        k_dequant<true><<<grid, kThreads, 0, stream>>>(codes, c2_fp8, c1, mean, numel, out, tables());
    else
        k_dequant<false><<<grid, kThreads, 0, stream>>>(codes, c2_fp8, c1, mean, numel, out, tables());
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace qlora
