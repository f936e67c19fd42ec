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
// name is only a stand-in, not a device address.  The first call on each
// device (with that device current) looks up the real address once with
// cudaGetSymbolAddress and caches it; later calls reuse it.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

constexpr int64_t kNoAllocMaxNumel = QLORA_NOALLOC_MAX_NUMEL;
constexpr size_t kNoAllocScratchBytes =
    static_cast<size_t>(kBinBytes + kFlagBytes) + static_cast<size_t>(kNoAllocMaxNumel / kBlock) * 4;

static __device__ __align__(256) unsigned char g_quant_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_quant_scratch on the current device (looked up once).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_addr_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_quant_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
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
