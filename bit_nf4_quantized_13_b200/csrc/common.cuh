// common.cuh -- shared device/host helpers of the QLoRA NF4 CUDA library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/qlora.h"
#include "ctx_memo.h"

namespace qlora {

constexpr int kBlock = QLORA_BLOCK;    // 64 weights per absmax constant
constexpr int kBlock2 = QLORA_BLOCK2;  // 256 constants per FP8 scale
constexpr int kBinBytes = 256 * 8;     // exact-sum bins, one u64 per fp32 exponent
constexpr int kFlagBytes = 16;         // workspace flag words

// The 16-value NF4 type plus the tables the encoder derives from it; built
// once on the host (codebook.cu) and passed to kernels by value.
struct Nf4Tables {
    float q[16];        // codebook, ascending
    // Encoder: n in [-1, 1] falls into bin b = bits(RN(n + 3)) >> 18 minus
    // 0x1000 (33 bins).  code(n) = base[b] + (n >= thr[b]).
    float thr[33];
    int base[33];
};

// host: lazily built per data type (QLORA_TYPE_*), immutable
const Nf4Tables& tables(int qtype = QLORA_TYPE_NF4);
bool valid_qtype(int qtype);

// ---------------------------------------------------------------- bf16 bits
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    // cvt.rn.bf16x2.f32 packs (hi, lo): the first source lands in the upper half
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------- FP8 E4M3
// Hardware conversions (PTX cvt): fp32 -> e4m3 with RNE and saturation to
// +-448, and e4m3 -> f16 (exact) -> f32.
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return static_cast<uint8_t>(r & 0xff);
}
__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
    uint32_t h2;
    uint16_t in = b;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xffff)));
}

// Double-dequantized constant of one 64-block: RN(RN(e4m3 * c1) + mean).
__device__ __forceinline__ float dq_constant(uint8_t b, float c1, float mean) {
    return __fadd_rn(__fmul_rn(e4m3_to_f32(b), c1), mean);
}

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms();  // cached SM count of the current device

// Raises `kernel`'s dynamic shared-memory limit to `bytes` once per CUDA
// context (function attributes belong to the loaded module, which a device
// reset unloads); `memo` is the launcher's own, one per kernel instance.
template <typename Kernel>
cudaError_t ensure_smem_limit(ContextMemo<int>& memo, Kernel kernel, int bytes) {
    uint64_t ctx = 0;
    if (!current_context_id(&ctx)) return cudaErrorDeviceUninitialized;
    cudaError_t err = cudaSuccess;
    int have = 0;
    const bool ok = memo.get(ctx, &have, [&](int* v) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        *v = bytes;
        return err == cudaSuccess;
    });
    if (!ok) return err != cudaSuccess ? err : cudaErrorUnknown;
    if (have < bytes) {  // a larger request than the one made in this context
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

// Counts kernel launches for qlora_kernel_launch_count (host side).
void note_launches(int n);

}  // namespace qlora
