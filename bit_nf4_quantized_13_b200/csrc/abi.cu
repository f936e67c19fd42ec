// abi.cu -- the extern "C" entry points declared in include/qlora.h:
// argument validation on the host, then kernel launches on the caller's
// stream.  Nothing here allocates device memory or synchronizes.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {
std::atomic<uint64_t> g_launches{0};
}

void note_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

cudaError_t launch_fwd_gemm(const uint16_t* X, const Nf4Weight& w, const uint16_t* T,
                            const uint16_t* B, int64_t M, int r, uint16_t* Y, void* ws, size_t ws_bytes,
                            cudaStream_t st) {
    if (pair_gemm_supported(M, w, r, false)) {
        const cudaError_t e = launch_fwd_gemm_pair(X, w, T, B, M, r, Y, ws, ws_bytes, st);
        if (e != cudaErrorNotSupported) return e;
    }
    return launch_fwd_gemm_simt(X, w, T, B, M, r, Y, st);
}

cudaError_t launch_bwd_dx_gemm(const uint16_t* dY, const Nf4Weight& w, const uint16_t* U,
                               const uint16_t* A, int64_t M, int r, uint16_t* dX, void* ws, size_t ws_bytes,
                               cudaStream_t st) {
    if (pair_gemm_supported(M, w, r, true)) {
        const cudaError_t e = launch_bwd_dx_gemm_pair(dY, w, U, A, M, r, dX, ws, ws_bytes, st);
        if (e != cudaErrorNotSupported) return e;
    }
    return launch_bwd_dx_gemm_simt(dY, w, U, A, M, r, dX, st);
}

// The rank-r products: tensor cores where the shapes allow TMA (r % 8 == 0,
// N % 8 == 0), CUDA cores otherwise.
cudaError_t lora_xat(const uint16_t* X, const uint16_t* A, int64_t M, int64_t N, int64_t K, int r, float s,
                     uint16_t* T, cudaStream_t st) {
    if (lora_tc_supported(M, N, K, r)) return launch_lora_xat_tc(X, A, M, K, r, s, T, st);
    return launch_lora_xat_simt(X, A, M, K, r, s, T, st);
}

cudaError_t lora_dyb(const uint16_t* dY, const uint16_t* B, int64_t M, int64_t N, int64_t K, int r, float s,
                     uint16_t* U, cudaStream_t st) {
    if (lora_tc_supported(M, N, K, r)) return launch_lora_dyb_tc(dY, B, M, N, r, s, U, st);
    return launch_lora_dyb_simt(dY, B, M, N, r, s, U, st);
}

cudaError_t lora_grads(const uint16_t* dY, const uint16_t* X, const uint16_t* T, const uint16_t* U, int64_t M,
                       int64_t N, int64_t K, int r, uint16_t* dA, uint16_t* dB, cudaStream_t st) {
    if (!lora_tc_supported(M, N, K, r)) return launch_lora_grads_simt(dY, X, T, U, M, N, K, r, dA, dB, st);
    return launch_lora_grads_tc(X, U, dY, T, M, N, K, r, dA, dB, st);
}

}  // namespace qlora

using namespace qlora;

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

inline bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }

constexpr int64_t kMaxNumel = int64_t(1) << 46;
constexpr uint64_t kMaxSelftestWaitNs = 1000000000ull;  // the self-test waits at most 1 s

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_weight(const uint8_t* codes, const uint8_t* c2_fp8, const float* c1, const float* mean) {
    if (!ok_ptr(codes) || !ok_ptr(c2_fp8) || !ok_ptr(c1) || !ok_ptr(mean)) return QLORA_ERR_INVALID_ARG;
    return QLORA_OK;
}

int check_linear(int64_t M, int64_t N, int64_t K, int r) {
    if (M < 0 || N < 1 || K < 1 || r < 1) return QLORA_ERR_INVALID_ARG;
    if (K % QLORA_BLOCK != 0 || r > QLORA_MAX_RANK) return QLORA_ERR_UNSUPPORTED;
    if (N * K >= kMaxNumel || M > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
    return QLORA_OK;
}

}  // namespace

extern "C" {

size_t qlora_quantize_workspace_size(int64_t numel) {
    if (numel < 0) return 0;
    const int64_t nb = ceil_div(numel, QLORA_BLOCK);
    return static_cast<size_t>(kBinBytes + kFlagBytes + round_up(nb * 4, 16));
}

int qlora_quantize_4bit_dq(int qtype, const float* W, int64_t numel, int block, int block2, uint8_t* codes,
                           uint8_t* c2_fp8, float* c1, float* mean, void* ws, size_t ws_bytes,
                           int32_t* status, void* stream) {
    if (numel < 0 || !valid_qtype(qtype)) return QLORA_ERR_INVALID_ARG;
    if (block != QLORA_BLOCK || block2 != QLORA_BLOCK2) return QLORA_ERR_UNSUPPORTED;
    if (numel >= kMaxNumel) return QLORA_ERR_UNSUPPORTED;
    if (numel == 0) return QLORA_OK;
    if (!ok_ptr(W) || !ok_ptr(codes) || !ok_ptr(c2_fp8) || !ok_ptr(c1) || !ok_ptr(mean))
        return QLORA_ERR_INVALID_ARG;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return QLORA_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < qlora_quantize_workspace_size(numel)) return QLORA_ERR_WORKSPACE;
    return cuda_status(
        launch_quantize_nf4_dq(W, numel, codes, c2_fp8, c1, mean, ws, status, as_stream(stream), qtype));
}

int qlora_quantize_nf4_dq(const float* W, int64_t numel, int block, int block2, uint8_t* codes,
                          uint8_t* c2_fp8, float* c1, float* mean, void* ws, size_t ws_bytes,
                          int32_t* status, void* stream) {
    return qlora_quantize_4bit_dq(QLORA_TYPE_NF4, W, numel, block, block2, codes, c2_fp8, c1, mean, ws, ws_bytes,
                                  status, stream);
}

int qlora_dequantize_4bit(int qtype, const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                          const float* mean, int64_t numel, int block, int block2, void* out, int out_dtype,
                          void* stream) {
    if (numel < 0 || (out_dtype != 0 && out_dtype != 1) || !valid_qtype(qtype)) return QLORA_ERR_INVALID_ARG;
    if (block != QLORA_BLOCK || block2 != QLORA_BLOCK2) return QLORA_ERR_UNSUPPORTED;
    if (numel >= kMaxNumel) return QLORA_ERR_UNSUPPORTED;
    if (numel == 0) return QLORA_OK;
    if (check_weight(codes, c2_fp8, c1, mean) != QLORA_OK || !ok_ptr(out)) return QLORA_ERR_INVALID_ARG;
    return cuda_status(launch_dequantize(codes, c2_fp8, c1, mean, numel, out, out_dtype, as_stream(stream), qtype));
}

int qlora_dequantize(const uint8_t* codes, const uint8_t* c2_fp8, const float* c1, const float* mean,
                     int64_t numel, int block, int block2, void* out, int out_dtype, void* stream) {
    return qlora_dequantize_4bit(QLORA_TYPE_NF4, codes, c2_fp8, c1, mean, numel, block, block2, out, out_dtype,
                                 stream);
}

size_t qlora_linear_fwd_workspace_size(int64_t M, int64_t N, int64_t K, int r) {
    if (check_linear(M, N, K, r) != QLORA_OK) return 0;
    // T (used when T_save is NULL), then the GEMM's split-tile scratch
    return align256(static_cast<size_t>(M) * r * 2) + pair_gemm_workspace();
}

size_t qlora_linear_bwd_workspace_size(int64_t M, int64_t N, int64_t K, int r) {
    if (check_linear(M, N, K, r) != QLORA_OK) return 0;
    const size_t mr = align256(static_cast<size_t>(M) * r * 2);
    // U, T (when T is NULL), then the dX GEMM's split-tile scratch
    return 2 * mr + pair_gemm_workspace();
}

int qlora_linear_fwd_4bit(int qtype, const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint8_t* codes,
                          const uint8_t* c2_fp8, const float* c1, const float* mean, const uint16_t* A,
                          const uint16_t* B, int r, float s, uint16_t* Y, uint16_t* T_save, void* ws,
                          size_t ws_bytes, void* stream) {
    if (!valid_qtype(qtype)) return QLORA_ERR_INVALID_ARG;
    int st = check_linear(M, N, K, r);
    if (st != QLORA_OK) return st;
    if (check_weight(codes, c2_fp8, c1, mean) != QLORA_OK) return QLORA_ERR_INVALID_ARG;
    if (!ok_ptr(A) || !ok_ptr(B) || (M > 0 && (!ok_ptr(X) || !ok_ptr(Y)))) return QLORA_ERR_INVALID_ARG;
    if (T_save && !aligned16(T_save)) return QLORA_ERR_INVALID_ARG;
    if (M == 0) return QLORA_OK;
    if (!ws || !aligned16(ws) || ws_bytes < qlora_linear_fwd_workspace_size(M, N, K, r))
        return QLORA_ERR_WORKSPACE;
    uint16_t* T = T_save ? T_save : reinterpret_cast<uint16_t*>(ws);
    const size_t t_bytes = align256(static_cast<size_t>(M) * r * 2);
    void* gws = reinterpret_cast<char*>(ws) + t_bytes;
    const size_t gws_bytes = ws_bytes - t_bytes;
    cudaStream_t cs = as_stream(stream);
    Nf4Weight w{codes, c2_fp8, c1, mean, N, K, qtype};
    if (gemv_supported(M, N, K, r)) {  // a few tokens: one stream over the weight
        const cudaError_t g = launch_fwd_gemv(X, w, A, B, M, r, s, Y, T_save, cs);
        if (g != cudaErrorNotSupported) return cuda_status(g);  // else: no cluster shape fits
    }
    cudaError_t e = lora_xat(X, A, M, N, K, r, s, T, cs);
    if (e == cudaSuccess) e = launch_fwd_gemm(X, w, T, B, M, r, Y, gws, gws_bytes, cs);
    return cuda_status(e);
}

int qlora_linear_fwd(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint8_t* codes,
                     const uint8_t* c2_fp8, const float* c1, const float* mean, const uint16_t* A,
                     const uint16_t* B, int r, float s, uint16_t* Y, uint16_t* T_save, void* ws,
                     size_t ws_bytes, void* stream) {
    return qlora_linear_fwd_4bit(QLORA_TYPE_NF4, X, M, N, K, codes, c2_fp8, c1, mean, A, B, r, s, Y, T_save, ws,
                                 ws_bytes, stream);
}

int qlora_linear_bwd_4bit(int qtype, const uint16_t* dY, const uint16_t* X, int64_t M, int64_t N, int64_t K,
                          const uint8_t* codes, const uint8_t* c2_fp8, const float* c1, const float* mean,
                          const uint16_t* A, const uint16_t* B, int r, float s, const uint16_t* T,
                          uint16_t* dX, uint16_t* dA, uint16_t* dB, void* ws, size_t ws_bytes,
                          void* stream) {
    if (!valid_qtype(qtype)) return QLORA_ERR_INVALID_ARG;
    int st = check_linear(M, N, K, r);
    if (st != QLORA_OK) return st;
    if (check_weight(codes, c2_fp8, c1, mean) != QLORA_OK) return QLORA_ERR_INVALID_ARG;
    if (!ok_ptr(A) || !ok_ptr(B) || !ok_ptr(dA) || !ok_ptr(dB)) return QLORA_ERR_INVALID_ARG;
    if (M > 0 && (!ok_ptr(dY) || !ok_ptr(X))) return QLORA_ERR_INVALID_ARG;
    if ((T && !aligned16(T)) || (dX && !aligned16(dX))) return QLORA_ERR_INVALID_ARG;
    cudaStream_t cs = as_stream(stream);
    if (M == 0) {  // empty batch: the adapter gradients are zero
        cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * K * 2, cs);
        if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * r * 2, cs);
        return cuda_status(e);
    }
    if (!ws || !aligned16(ws) || ws_bytes < qlora_linear_bwd_workspace_size(M, N, K, r))
        return QLORA_ERR_WORKSPACE;
    const size_t mr = align256(static_cast<size_t>(M) * r * 2);
    uint16_t* U = reinterpret_cast<uint16_t*>(ws);
    uint16_t* Tw = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(ws) + mr);
    Nf4Weight w{codes, c2_fp8, c1, mean, N, K, qtype};
    void* dxws = reinterpret_cast<char*>(ws) + 2 * mr;
    const size_t dxws_bytes = ws_bytes - 2 * mr;
    cudaError_t e = cudaSuccess;
    if (!T) {
        e = lora_xat(X, A, M, N, K, r, s, Tw, cs);
        T = Tw;
    }
    if (e == cudaSuccess) e = lora_dyb(dY, B, M, N, K, r, s, U, cs);
    if (e == cudaSuccess && dX) e = launch_bwd_dx_gemm(dY, w, U, A, M, r, dX, dxws, dxws_bytes, cs);
    if (e == cudaSuccess) e = lora_grads(dY, X, T, U, M, N, K, r, dA, dB, cs);
    return cuda_status(e);
}

int qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, int64_t N, int64_t K,
                     const uint8_t* codes, const uint8_t* c2_fp8, const float* c1, const float* mean,
                     const uint16_t* A, const uint16_t* B, int r, float s, const uint16_t* T,
                     uint16_t* dX, uint16_t* dA, uint16_t* dB, void* ws, size_t ws_bytes,
                     void* stream) {
    return qlora_linear_bwd_4bit(QLORA_TYPE_NF4, dY, X, M, N, K, codes, c2_fp8, c1, mean, A, B, r, s, T, dX, dA, dB,
                                 ws, ws_bytes, stream);
}

size_t qlora_linear_group_fwd_workspace_size(int64_t M, int G, int r) {
    if (M < 0 || G < 1 || G > kMaxGroupLinears || r < 1 || static_cast<int64_t>(G) * r > QLORA_MAX_RANK) return 0;
    return align256(static_cast<size_t>(M) * G * r * 2) + pair_gemm_workspace();
}

size_t qlora_linear_group_bwd_workspace_size(int64_t M, int G, int r) {
    if (M < 0 || G < 1 || G > kMaxGroupLinears || r < 1 || static_cast<int64_t>(G) * r > QLORA_MAX_RANK) return 0;
    return 2 * align256(static_cast<size_t>(M) * G * r * 2) + pair_gemm_workspace();
}

}  // extern "C"

namespace {

// Validates a group's descriptors and fills `g`; QLORA_OK or the error.
int check_group(int qtype, int64_t M, int64_t K, const qlora_weight_4bit* W, int G, int r, Nf4Group* g) {
    if (!valid_qtype(qtype) || !W || M < 0 || K < 1 || r < 1 || G < 1) return QLORA_ERR_INVALID_ARG;
    if (G > kMaxGroupLinears || static_cast<int64_t>(G) * r > QLORA_MAX_RANK || K % QLORA_BLOCK != 0 || r % 8 != 0)
        return QLORA_ERR_UNSUPPORTED;
    g->G = G;
    for (int i = 0; i < G; ++i) {
        if (check_weight(W[i].codes, W[i].c2_fp8, W[i].c1, W[i].mean) != QLORA_OK || W[i].N < 1)
            return QLORA_ERR_INVALID_ARG;
        if (check_linear(M, W[i].N, K, r) != QLORA_OK) return QLORA_ERR_UNSUPPORTED;
        g->w[i] = Nf4Weight{W[i].codes, W[i].c2_fp8, W[i].c1, W[i].mean, W[i].N, K, qtype};
    }
    int64_t n_all = 0;
    for (int i = 0; i < G; ++i) n_all += W[i].N;
    if (M > 0 && (!pair_group_supported(M, *g, r) || !lora_tc_supported(M, n_all, K, G * r)))
        return QLORA_ERR_UNSUPPORTED;
    return QLORA_OK;
}

int64_t group_n(const Nf4Group& g) {
    int64_t n = 0;
    for (int i = 0; i < g.G; ++i) n += g.w[i].N;
    return n;
}

int pair_status(cudaError_t e) { return e == cudaErrorNotSupported ? QLORA_ERR_UNSUPPORTED : cuda_status(e); }

}  // namespace

extern "C" {

int qlora_linear_group_fwd(int qtype, const uint16_t* X, int64_t M, int64_t K, const qlora_weight_4bit* W, int G,
                           const uint16_t* A_cat, const uint16_t* B_cat, int r, float s, uint16_t* Y,
                           uint16_t* T_save, void* ws, size_t ws_bytes, void* stream) {
    Nf4Group g{};
    const int st = check_group(qtype, M, K, W, G, r, &g);
    if (st != QLORA_OK) return st;
    if (!ok_ptr(A_cat) || !ok_ptr(B_cat) || (M > 0 && (!ok_ptr(X) || !ok_ptr(Y)))) return QLORA_ERR_INVALID_ARG;
    if (T_save && !aligned16(T_save)) return QLORA_ERR_INVALID_ARG;
    if (M == 0) return QLORA_OK;
    if (!ws || !aligned16(ws) || ws_bytes < qlora_linear_group_fwd_workspace_size(M, G, r)) return QLORA_ERR_WORKSPACE;
    const int rc = G * r;
    const size_t t_bytes = align256(static_cast<size_t>(M) * rc * 2);
    uint16_t* T = T_save ? T_save : reinterpret_cast<uint16_t*>(ws);
    cudaStream_t cs = as_stream(stream);
    // every adapter's T in one rank-(G r) product: column g r + j is s X A_g[j]^T
    cudaError_t e = lora_xat(X, A_cat, M, group_n(g), K, rc, s, T, cs);
    if (e != cudaSuccess) return cuda_status(e);
    return pair_status(launch_fwd_gemm_pair_group(X, g, T, B_cat, M, r, Y, reinterpret_cast<char*>(ws) + t_bytes,
                                                  ws_bytes - t_bytes, cs));
}

int qlora_linear_group_bwd(int qtype, const uint16_t* dY, const uint16_t* X, int64_t M, int64_t K,
                           const qlora_weight_4bit* W, int G, const uint16_t* A_cat, const uint16_t* B_cat, int r,
                           float s, const uint16_t* T, uint16_t* dX, uint16_t* dA_cat, uint16_t* dB_cat, void* ws,
                           size_t ws_bytes, void* stream) {
    Nf4Group g{};
    const int st = check_group(qtype, M, K, W, G, r, &g);
    if (st != QLORA_OK) return st;
    if (!ok_ptr(A_cat) || !ok_ptr(B_cat) || !ok_ptr(dA_cat) || !ok_ptr(dB_cat)) return QLORA_ERR_INVALID_ARG;
    if (M > 0 && (!ok_ptr(dY) || !ok_ptr(X))) return QLORA_ERR_INVALID_ARG;
    if ((T && !aligned16(T)) || (dX && !aligned16(dX))) return QLORA_ERR_INVALID_ARG;
    const int rc = G * r;
    const int64_t n_all = group_n(g);
    cudaStream_t cs = as_stream(stream);
    if (M == 0) {  // empty batch: the adapter gradients are zero
        cudaError_t e = cudaMemsetAsync(dA_cat, 0, static_cast<size_t>(rc) * K * 2, cs);
        if (e == cudaSuccess) e = cudaMemsetAsync(dB_cat, 0, static_cast<size_t>(n_all) * r * 2, cs);
        return cuda_status(e);
    }
    if (!ws || !aligned16(ws) || ws_bytes < qlora_linear_group_bwd_workspace_size(M, G, r)) return QLORA_ERR_WORKSPACE;
    const size_t mr = align256(static_cast<size_t>(M) * rc * 2);
    uint16_t* U = reinterpret_cast<uint16_t*>(ws);
    uint16_t* Tw = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(ws) + mr);
    cudaError_t e = cudaSuccess;
    if (!T) {
        e = lora_xat(X, A_cat, M, n_all, K, rc, s, Tw, cs);
        T = Tw;
    }
    // U_g = s dY_g B_g into columns g r .. of U (dY_g a column block of dY), one launch
    int64_t Ns[kMaxGroupLinears];
    for (int i = 0; i < G; ++i) Ns[i] = g.w[i].N;
    if (e == cudaSuccess) e = launch_lora_dyb_group(dY, B_cat, M, Ns, G, r, s, U, cs);
    if (e == cudaSuccess && dX) {
        e = launch_bwd_dx_gemm_pair_group(dY, g, U, A_cat, M, r, dX, reinterpret_cast<char*>(ws) + 2 * mr,
                                          ws_bytes - 2 * mr, cs);
        if (e == cudaErrorNotSupported) return QLORA_ERR_UNSUPPORTED;
    }
    // dA_g = U_g^T X for all g at once (rows of dA_cat); dB_g = dY_g^T T_g, one launch
    if (e == cudaSuccess) e = launch_lora_da_tc(X, U, M, K, rc, dA_cat, cs);
    if (e == cudaSuccess) e = launch_lora_db_group(dY, T, M, Ns, G, r, dB_cat, cs);
    return cuda_status(e);
}

int qlora_device_error(int reset) {
    const int a = pair_device_error(reset);
    const int b = lora_device_error(reset);
    const int c = gemv_device_error(reset);
    return a != QLORA_OK ? a : b != QLORA_OK ? b : c;
}

int qlora_int8_quantize(const float* x, int64_t numel, int block, int8_t* codes, float* c, int32_t* status,
                        void* stream) {
    if (numel < 0) return QLORA_ERR_INVALID_ARG;
    if (!int8_block_supported(block)) return QLORA_ERR_UNSUPPORTED;
    if (numel >= kMaxNumel) return QLORA_ERR_UNSUPPORTED;
    if (numel == 0) return QLORA_OK;
    if (!ok_ptr(x) || !ok_ptr(codes) || !ok_ptr(c)) return QLORA_ERR_INVALID_ARG;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return QLORA_ERR_INVALID_ARG;
    return cuda_status(launch_int8_quantize(x, numel, block, codes, c, status, as_stream(stream)));
}

int qlora_int8_dequantize(const int8_t* codes, const float* c, int64_t numel, int block, float* out, void* stream) {
    if (numel < 0) return QLORA_ERR_INVALID_ARG;
    if (!int8_block_supported(block)) return QLORA_ERR_UNSUPPORTED;
    if (numel >= kMaxNumel) return QLORA_ERR_UNSUPPORTED;
    if (numel == 0) return QLORA_OK;
    if (!ok_ptr(codes) || !ok_ptr(c) || !ok_ptr(out)) return QLORA_ERR_INVALID_ARG;
    return cuda_status(launch_int8_dequantize(codes, c, numel, block, out, as_stream(stream)));
}

int qlora_debug_wait_timeout(uint64_t limit_ns, void* stream) {
    if (limit_ns == 0 || limit_ns > kMaxSelftestWaitNs) return QLORA_ERR_INVALID_ARG;
    return cuda_status(launch_wait_selftest(limit_ns, as_stream(stream)));
}

int qlora_debug_fill(uint32_t* dst, int64_t n_words, uint32_t value, void* stream) {
    if (n_words < 0 || n_words % 4 != 0 || (n_words > 0 && !ok_ptr(dst))) return QLORA_ERR_INVALID_ARG;
    return cuda_status(launch_probe_fill(dst, n_words, value, as_stream(stream)));
}

int qlora_debug_read(const uint32_t* src, int64_t n_words, uint32_t never, uint32_t* sink, void* stream) {
    if (n_words < 0 || n_words % 4 != 0 || (n_words > 0 && (!ok_ptr(src) || !sink))) return QLORA_ERR_INVALID_ARG;
    return cuda_status(launch_probe_read(src, n_words, never, sink, as_stream(stream)));
}

uint64_t qlora_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int qlora_fp8_e4m3_encode(const float* x, uint8_t* out, int64_t n, void* stream) {
    if (n < 0) return QLORA_ERR_INVALID_ARG;
    if (n == 0) return QLORA_OK;
    if (!ok_ptr(x) || !ok_ptr(out)) return QLORA_ERR_INVALID_ARG;
    return cuda_status(launch_e4m3_encode(x, out, n, as_stream(stream)));
}

}  // extern "C"
