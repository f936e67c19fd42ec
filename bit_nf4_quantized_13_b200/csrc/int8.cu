// int8.cu -- block-wise Int8 absmax quantization and dequantization, the
// 8-bit baseline the QLoRA study notes (gitcode.csdn.net) set out in
// section 3.1, eq. (1) and eq. (2):
//
//   c = RN32(127 / absmax(block)),  code = round_half_away(RN32(c * x)),
//   x' = RN32(code / c)             (a block with absmax 0: c = 0, x' = 0)
//
// HBM-bound: 4 bytes read and 1 + 4/block written per element to quantize,
// 1 + 4/block read and 4 written to dequantize.  A warp takes blocks of
// `kB` consecutive elements, two to four at a time (all their loads issued
// before any is used); lane l holds elements kB/32 * l ... of a block
// (contiguous), so loads and stores are vector accesses per lane and whole
// warps read and write contiguous runs.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;

template <int kPer>
struct Vec;  // kPer fp32 values / kPer int8 codes held by one lane
template <>
struct Vec<1> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[1]) { v[0] = __ldcs(p); }
};
template <>
struct Vec<2> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[2]) {
        const float2 a = __ldcs(reinterpret_cast<const float2*>(p));
        v[0] = a.x;
        v[1] = a.y;
    }
};
template <>
struct Vec<4> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
        const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
        v[0] = a.x;
        v[1] = a.y;
        v[2] = a.z;
        v[3] = a.w;
    }
};
template <>
struct Vec<8> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
        const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
        const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
        v[0] = a.x;
        v[1] = a.y;
        v[2] = a.z;
        v[3] = a.w;
        v[4] = b.x;
        v[5] = b.y;
        v[6] = b.z;
        v[7] = b.w;
    }
};

template <int kPer>
__device__ __forceinline__ void store_codes(int8_t* p, const int (&q)[kPer]) {
    if (kPer == 1) {
        p[0] = static_cast<int8_t>(q[0]);
    } else if (kPer == 2) {
        *reinterpret_cast<uint16_t*>(p) = static_cast<uint16_t>((q[0] & 0xff) | ((q[1 % kPer] & 0xff) << 8));
    } else {
#pragma unroll
        for (int w = 0; w < kPer / 4; ++w) {
            const uint32_t v = (q[4 * w] & 0xff) | ((q[4 * w + 1] & 0xff) << 8) | ((q[4 * w + 2] & 0xff) << 16) |
                               (static_cast<uint32_t>(q[4 * w + 3] & 0xff) << 24);
            reinterpret_cast<uint32_t*>(p)[w] = v;
        }
    }
}

// Whole blocks: warp per block, grid-stride.  The ragged last block (if
// any) is done by the host-selected tail kernel.
template <int kB>
__global__ void __launch_bounds__(kThreads)
k_int8_quantize(const float* __restrict__ x, int64_t nfull, int8_t* __restrict__ codes, float* __restrict__ c,
                int* __restrict__ bad_flag) {
    constexpr int kPer = kB / 32;
    constexpr int kU = kPer >= 8 ? 2 : 4;  // blocks a warp has in flight
    const int lane = threadIdx.x & 31;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    bool bad = false;
    for (int64_t b0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5; b0 < nfull; b0 += nw * kU) {
        float v[kU][kPer];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t b = b0 + u * nw;
            if (b < nfull) Vec<kPer>::load(x + b * kB + static_cast<int64_t>(lane) * kPer, v[u]);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t b = b0 + u * nw;
            if (b >= nfull) break;
            const int64_t e = b * kB + static_cast<int64_t>(lane) * kPer;
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < kPer; ++i) a = fmaxf(a, fabsf(v[u][i]));
            bool nonfinite = false;
#pragma unroll
            for (int i = 0; i < kPer; ++i) nonfinite |= !isfinite(v[u][i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            const float cc = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
            nonfinite |= !isfinite(cc);
            bad |= nonfinite;
            int q[kPer];
#pragma unroll
            for (int i = 0; i < kPer; ++i) q[i] = isfinite(cc) ? static_cast<int>(roundf(__fmul_rn(cc, v[u][i]))) : 0;
            store_codes<kPer>(codes + e, q);
            if (lane == 0) c[b] = cc;
        }
    }
    if (bad && bad_flag) atomicExch(bad_flag, QLORA_ERR_NONFINITE);
}

// The ragged last block (len < kB elements), by one warp.
__global__ void k_int8_quantize_tail(const float* __restrict__ x, int64_t start, int len, int8_t* __restrict__ codes,
                                     float* __restrict__ c_out, int* __restrict__ bad_flag) {
    const int lane = threadIdx.x & 31;
    float a = 0.0f;
    bool bad = false;
    for (int i = lane; i < len; i += 32) {
        const float v = x[start + i];
        a = fmaxf(a, fabsf(v));
        bad |= !isfinite(v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const float cc = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
    bad |= !isfinite(cc);
    for (int i = lane; i < len; i += 32)
        codes[start + i] = static_cast<int8_t>(isfinite(cc) ? static_cast<int>(roundf(__fmul_rn(cc, x[start + i]))) : 0);
    if (lane == 0) *c_out = cc;
    if (__any_sync(0xffffffffu, bad) && lane == 0 && bad_flag) atomicExch(bad_flag, QLORA_ERR_NONFINITE);
}

template <int kPer>
__device__ __forceinline__ void load_codes(const int8_t* p, int (&q)[kPer]) {
    if (kPer == 1) {
        q[0] = p[0];
    } else if (kPer == 2) {
        const uint16_t v = __ldcs(reinterpret_cast<const unsigned short*>(p));
        q[0] = static_cast<int8_t>(v & 0xff);
        q[1 % kPer] = static_cast<int8_t>(v >> 8);
    } else {
#pragma unroll
        for (int w = 0; w < kPer / 4; ++w) {
            const uint32_t v = __ldcs(reinterpret_cast<const unsigned int*>(p) + w);
#pragma unroll
            for (int j = 0; j < 4; ++j) q[4 * w + j] = static_cast<int8_t>((v >> (8 * j)) & 0xff);
        }
    }
}

template <int kB>
__global__ void __launch_bounds__(kThreads)
k_int8_dequantize(const int8_t* __restrict__ codes, const float* __restrict__ c, int64_t numel,
                  float* __restrict__ out) {
    constexpr int kPer = kB / 32;
    constexpr int kU = kPer >= 8 ? 2 : 4;  // blocks a warp has in flight
    const int lane = threadIdx.x & 31;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    const int64_t nfull = numel / kB;
    for (int64_t b0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5; b0 < nfull; b0 += nw * kU) {
        int q[kU][kPer];
        float cc[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t b = b0 + u * nw;
            if (b < nfull) {
                load_codes<kPer>(codes + b * kB + static_cast<int64_t>(lane) * kPer, q[u]);
                cc[u] = __ldg(c + b);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t b = b0 + u * nw;
            if (b >= nfull) break;
            const int64_t e = b * kB + static_cast<int64_t>(lane) * kPer;
            float v[kPer];
#pragma unroll
            for (int i = 0; i < kPer; ++i)
                v[i] = cc[u] != 0.0f ? __fdiv_rn(static_cast<float>(q[u][i]), cc[u]) : 0.0f;
#pragma unroll
            for (int i = 0; i < kPer; i += (kPer >= 4 ? 4 : kPer)) {
                if (kPer >= 4)
                    __stcs(reinterpret_cast<float4*>(out + e + i), make_float4(v[i], v[(i + 1) % kPer], v[(i + 2) % kPer],
                                                                               v[(i + 3) % kPer]));
                else if (kPer == 2)
                    __stcs(reinterpret_cast<float2*>(out + e), make_float2(v[0], v[1 % kPer]));
                else
                    __stcs(out + e, v[0]);
            }
        }
    }
    // the ragged last block, by the warp whose turn it is
    const int64_t tail = numel - nfull * kB;
    if (tail > 0 && ((static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5) == nfull % nw) {
        const float ct = c[nfull];
        for (int64_t i = nfull * kB + lane; i < numel; i += 32)
            out[i] = ct != 0.0f ? __fdiv_rn(static_cast<float>(codes[i]), ct) : 0.0f;
    }
}

int grid_for(int64_t blocks) {
    const int64_t want = ceil_div(blocks, kThreads / 32);
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    return static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
}

template <int kB>
cudaError_t quantize_b(const float* x, int64_t numel, int8_t* codes, float* c, int* flag, cudaStream_t st) {
    const int64_t nfull = numel / kB;
    if (nfull > 0) {
        k_int8_quantize<kB><<<grid_for(nfull), kThreads, 0, st>>>(x, nfull, codes, c, flag);
        note_launches(1);
    }
    const int64_t tail = numel - nfull * kB;
    if (tail > 0) {
        k_int8_quantize_tail<<<1, 32, 0, st>>>(x, nfull * kB, static_cast<int>(tail), codes, c + nfull, flag);
        note_launches(1);
    }
    return cudaGetLastError();
}

template <int kB>
cudaError_t dequantize_b(const int8_t* codes, const float* c, int64_t numel, float* out, cudaStream_t st) {
    k_int8_dequantize<kB><<<grid_for(ceil_div(numel, kB)), kThreads, 0, st>>>(codes, c, numel, out);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace

bool int8_block_supported(int block) { return block == 32 || block == 64 || block == 128 || block == 256; }

// status (nullable): cleared to QLORA_OK in stream order, then set to
// QLORA_ERR_NONFINITE by any block holding a NaN or Inf (or whose constant
// overflows).
cudaError_t launch_int8_quantize(const float* x, int64_t numel, int block, int8_t* codes, float* c,
                                 int32_t* status, cudaStream_t st) {
    int* flag = reinterpret_cast<int*>(status);
    if (flag) {
        const cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(int), st);
        if (e != cudaSuccess) return e;
    }
    switch (block) {
        case 32: return quantize_b<32>(x, numel, codes, c, flag, st);
        case 64: return quantize_b<64>(x, numel, codes, c, flag, st);
        case 128: return quantize_b<128>(x, numel, codes, c, flag, st);
        default: return quantize_b<256>(x, numel, codes, c, flag, st);
    }
}

cudaError_t launch_int8_dequantize(const int8_t* codes, const float* c, int64_t numel, int block, float* out,
                                   cudaStream_t st) {
    switch (block) {
        case 32: return dequantize_b<32>(codes, c, numel, out, st);
        case 64: return dequantize_b<64>(codes, c, numel, out, st);
        case 128: return dequantize_b<128>(codes, c, numel, out, st);
        default: return dequantize_b<256>(codes, c, numel, out, st);
    }
}

}  // namespace qlora
