// dequant.cu -- double dequantization of an NF4 weight (QLoRA study notes,
// gitcode.csdn.net, section 3.5 eq. 6): the FP8 constants are expanded with
// their second-level scale and the mean, then every code is looked up in
// the NF4 type and scaled by its block constant.
//
// HBM-bound: 0.5 + 1/64 + 1/16384 bytes read and 4 (fp32) or 2 (bf16) bytes
// written per weight.  A warp owns 1024 consecutive weights (16 blocks):
// lanes 0-15 first expand the 16 block constants, then in store step i
// lane l writes the i-th 16-byte row slot of the warp's output, so every
// store instruction is one contiguous run across the warp.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpElems = 1024;

__device__ __forceinline__ uint32_t ld_nc_u32(const uint8_t* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_nc_u16(const uint8_t* p) {
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// OUT_BF16 = false: fp32 output, 4 weights (2 code bytes) per lane per step.
// OUT_BF16 = true : bf16 output, 8 weights (4 code bytes) per lane per step.
template <bool OUT_BF16>
__global__ void __launch_bounds__(kThreads)
k_dequant(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ c2_fp8,
          const float* __restrict__ c1, const float* __restrict__ mean, int64_t numel,
          void* __restrict__ out, Nf4Tables tabs) {
    __shared__ float sq[16];
    if (threadIdx.x < 16) sq[threadIdx.x] = tabs.q[threadIdx.x];
    __syncthreads();
    const float mu = *mean;
    const int lane = threadIdx.x & 31;
    const int64_t nb = ceil_div(numel, kBlock);
    const int64_t nwc = ceil_div(numel, kWarpElems);
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    constexpr int kPer = OUT_BF16 ? 8 : 4;           // weights per lane per step
    constexpr int kSteps = kWarpElems / (32 * kPer);  // 8 (fp32) or 4 (bf16)

    for (int64_t c = warp0; c < nwc; c += nwarps) {
        const int64_t base = c * kWarpElems;
        // block constants of the warp's 16 blocks, one per lane 0..15
        float cp = 0.0f;
        {
            const int64_t blk = (base >> 6) + (lane & 15);
            if (blk < nb) cp = dq_constant(c2_fp8[blk], c1[blk >> 8], mu);
        }
        const bool full = base + kWarpElems <= numel;
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            const int64_t e = base + static_cast<int64_t>(kPer) * (32 * i + lane);
            // weights e .. e+kPer-1 share one block: kPer divides 64
            const float scale = __shfl_sync(0xffffffffu, cp, static_cast<int>(((e - base) >> 6) & 15));
            uint32_t cw;
            if (full) {
                cw = OUT_BF16 ? ld_nc_u32(codes + (e >> 1)) : ld_nc_u16(codes + (e >> 1));
            } else {
                cw = 0;
                for (int b = 0; b < kPer / 2; ++b)
                    if (e + 2 * b < numel) cw |= static_cast<uint32_t>(codes[(e >> 1) + b]) << (8 * b);
            }
            float w[kPer];
#pragma unroll
            for (int b = 0; b < kPer / 2; ++b) {
                const uint32_t byte = (cw >> (8 * b)) & 0xffu;
                w[2 * b] = __fmul_rn(sq[byte >> 4], scale);
                w[2 * b + 1] = __fmul_rn(sq[byte & 15u], scale);
            }
            if (OUT_BF16) {
                uint16_t* o = reinterpret_cast<uint16_t*>(out) + e;
                if (full) {
                    uint4 v;
                    v.x = pack_bf16x2(w[0], w[1]);
                    v.y = pack_bf16x2(w[2], w[3]);
                    v.z = pack_bf16x2(w[4], w[5]);
                    v.w = pack_bf16x2(w[6], w[7]);
                    __stcs(reinterpret_cast<uint4*>(o), v);
                } else {
                    for (int t = 0; t < kPer; ++t)
                        if (e + t < numel) o[t] = f32_to_bf16_bits(w[t]);
                }
            } else {
                float* o = reinterpret_cast<float*>(out) + e;
                if (full) {
                    __stcs(reinterpret_cast<float4*>(o), make_float4(w[0], w[1], w[2], w[3]));
                } else {
                    for (int t = 0; t < kPer; ++t)
                        if (e + t < numel) o[t] = w[t];
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                              const float* mean, int64_t numel, void* out, int out_dtype,
                              cudaStream_t stream) {
    const int64_t nwc = ceil_div(numel, kWarpElems);
    const int64_t want = ceil_div(nwc, kThreads / 32);
    const int grid = static_cast<int>(want < num_sms() * 8LL ? want : num_sms() * 8LL);
    if (out_dtype == 1)
        k_dequant<true><<<grid, kThreads, 0, stream>>>(codes, c2_fp8, c1, mean, numel, out, tables());
    else
        k_dequant<false><<<grid, kThreads, 0, stream>>>(codes, c2_fp8, c1, mean, numel, out, tables());
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace qlora
