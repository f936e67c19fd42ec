// quantize_noalloc.cu -- qlora_quantize_nf4_dq_noalloc: the NF4 + double
// quantization of qlora_quantize_nf4_dq for callers that have no way to
// hand the library a workspace.
//
// Some callers cannot allocate device memory at the point where they need
// a weight quantized: a plugin inside a host program that owns the whole
// device-memory budget and exposes no allocator to it, or a loop that must
// not pay cudaMalloc's implicit device-wide synchronisation.  For them the
// scratch this operation needs (exact-sum bins, flags and the fp32 block
// maxima passed between the two kernels) lives in one file-scope device
// array of fixed size, reserved on every GPU that loads this library until
// the process exits.
//
// Host code must not hand the array's symbol to a kernel: on the host that
// name is only a stand-in, not a device address.  The first call in each
// CUDA context (with that context's device current) looks up the real
// address with cudaGetSymbolAddress and memoizes it under the context's
// process-unique id; later calls in the same context reuse it.  A context
// made again after a device reset has a new id, so its first call looks the
// address up afresh (the reloaded module's array may sit elsewhere).
#include "common.cuh"
#include "ctx_memo.h"
#include "kernels.h"

namespace qlora {
namespace {

constexpr int64_t kNoAllocMaxNumel = QLORA_NOALLOC_MAX_NUMEL;
constexpr size_t kNoAllocScratchBytes =
    static_cast<size_t>(kBinBytes + kFlagBytes) + static_cast<size_t>(kNoAllocMaxNumel / kBlock) * 4;

static __device__ __align__(256) unsigned char g_quant_scratch[kNoAllocScratchBytes];

ContextMemo<void*> g_addr;

// Device address of g_quant_scratch in the current context (looked up once
// per context).
cudaError_t scratch_address(void** out) {
    uint64_t ctx = 0;
    if (!current_context_id(&ctx)) return cudaErrorDeviceUninitialized;
    cudaError_t err = cudaSuccess;
    const bool ok = g_addr.get(ctx, out, [&](void** p) {
        err = cudaGetSymbolAddress(p, g_quant_scratch);
        return err == cudaSuccess && *p != nullptr;
    });
    if (!ok) return err != cudaSuccess ? err : cudaErrorInvalidSymbol;
    return cudaSuccess;
}

}  // namespace
}  // namespace qlora

extern "C" int qlora_quantize_nf4_dq_noalloc(const float* W, int64_t numel, int block, int block2,
                                             uint8_t* codes, uint8_t* c2_fp8, float* c1, float* mean,
                                             int32_t* status, void* stream) {
    using namespace qlora;
    if (numel < 0) return QLORA_ERR_INVALID_ARG;
    if (block != QLORA_BLOCK || block2 != QLORA_BLOCK2) return QLORA_ERR_UNSUPPORTED;
    if (numel > kNoAllocMaxNumel) return QLORA_ERR_WORKSPACE;  // beyond the built-in scratch
    if (numel == 0) return QLORA_OK;
    auto ok = [](const void* p) { return p != nullptr && aligned16(p); };
    if (!ok(W) || !ok(codes) || !ok(c2_fp8) || !ok(c1) || !ok(mean)) return QLORA_ERR_INVALID_ARG;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return QLORA_ERR_INVALID_ARG;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return QLORA_ERR_CUDA;
    // The launch clears the bins and flags at the start of the scratch in
    // stream order before the kernels use them; the staged block maxima are
    // fully rewritten by every call.
    cudaError_t e = launch_quantize_nf4_dq(W, numel, codes, c2_fp8, c1, mean, ws, status,
                                           reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}
