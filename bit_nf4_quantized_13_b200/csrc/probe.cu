// probe.cu -- plain kernels that measure the DRAM ceilings the HBM-bound
// kernels are compared with: a write-only fill (one pass of CTAs over the
// buffer, plain 16-byte stores) and a read-only pass (a grid of resident
// CTAs, streaming 16-byte loads, four in flight per thread), both in whole
// 512-byte warp runs.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

constexpr int kProbeThreads = 512;
constexpr int kUnroll = 4;

// One CTA per 512 x 4 runs of 16 bytes (the grid covers the buffer once):
// thread t of CTA b stores runs 2048 b + t + 512 u, u < 4 (whole 512-byte
// warp runs).
__global__ void __launch_bounds__(kProbeThreads) k_probe_fill(uint4* __restrict__ dst, int64_t n16, uint32_t v) {
    const uint4 val = make_uint4(v, v, v, v);
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * (kProbeThreads * kUnroll) + threadIdx.x;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = i0 + u * kProbeThreads;
        if (i < n16) dst[i] = val;
    }
}

// The loaded words are folded into one value per thread, which is written
// only if it equals `never` (so the loads cannot be dropped and, in
// practice, nothing is written).
__global__ void __launch_bounds__(kProbeThreads)
k_probe_read(const uint4* __restrict__ src, int64_t n16, uint32_t never, uint32_t* __restrict__ sink) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kProbeThreads;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kProbeThreads + threadIdx.x;
    uint32_t acc = 0;
    for (; i + (kUnroll - 1) * stride < n16; i += kUnroll * stride) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) v[u] = __ldcs(src + i + u * stride);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n16; i += stride) {
        const uint4 v = __ldcs(src + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
    if (acc == never) sink[0] = acc;
}

int probe_grid(int64_t n16) {
    const int64_t cap = static_cast<int64_t>(num_sms()) * (2048 / kProbeThreads);
    const int64_t want = ceil_div(n16, kProbeThreads);
    return static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_probe_fill(uint32_t* dst, int64_t n_words, uint32_t value, cudaStream_t st) {
    const int64_t n16 = n_words / 4;
    if (n16 == 0) return cudaSuccess;
    const int64_t blocks = ceil_div(n16, kProbeThreads * kUnroll);
    if (blocks >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    k_probe_fill<<<static_cast<unsigned>(blocks), kProbeThreads, 0, st>>>(reinterpret_cast<uint4*>(dst), n16, value);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_probe_read(const uint32_t* src, int64_t n_words, uint32_t never, uint32_t* sink, cudaStream_t st) {
    const int64_t n16 = n_words / 4;
    if (n16 == 0) return cudaSuccess;
    k_probe_read<<<probe_grid(n16), kProbeThreads, 0, st>>>(reinterpret_cast<const uint4*>(src), n16, never, sink);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace qlora
