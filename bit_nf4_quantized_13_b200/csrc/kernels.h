// kernels.h -- internal launch interface between the C ABI (abi.cu) and the
// kernel files.  All launches are asynchronous on `stream` and return the
// CUDA error of the launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qlora.h"

namespace qlora {

// quantize.cu
cudaError_t launch_quantize_nf4_dq(const float* W, int64_t numel, uint8_t* codes, uint8_t* c2_fp8,
                                   float* c1, float* mean, void* ws, int32_t* status,
                                   cudaStream_t stream, int qtype = QLORA_TYPE_NF4);
cudaError_t launch_e4m3_encode(const float* x, uint8_t* out, int64_t n, cudaStream_t stream);

// dequant.cu
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                              const float* mean, int64_t numel, void* out, int out_dtype,
                              cudaStream_t stream, int qtype = QLORA_TYPE_NF4);

// probe.cu -- the DRAM ceilings: a write-only fill and a read-only pass
// (16-byte accesses; n_words a multiple of 4, pointers 16-byte aligned)
cudaError_t launch_probe_fill(uint32_t* dst, int64_t n_words, uint32_t value, cudaStream_t stream);
cudaError_t launch_probe_read(const uint32_t* src, int64_t n_words, uint32_t never, uint32_t* sink,
                              cudaStream_t stream);

// int8.cu -- block-wise Int8 absmax quantization (eq. 1) and dequantization
// (eq. 2), block in {32, 64, 128, 256}
bool int8_block_supported(int block);
cudaError_t launch_int8_quantize(const float* x, int64_t numel, int block, int8_t* codes, float* c,
                                 int32_t* status, cudaStream_t stream);
cudaError_t launch_int8_dequantize(const int8_t* codes, const float* c, int64_t numel, int block, float* out,
                                   cudaStream_t stream);

// The frozen NF4 weight W (N x K row-major) as the GEMM kernels see it.
struct Nf4Weight {
    const uint8_t* codes;   // N*K/2 bytes
    const uint8_t* c2_fp8;  // N*K/64 bytes
    const float* c1;        // N*K/16384 floats (rounded up)
    const float* mean;      // 1 float
    int64_t N, K;
    int qtype = QLORA_TYPE_NF4;  // the 4-bit data type the codes index
};

// The skinny rank-r products of the LoRA path
//   T  = bf16(s * X A^T)   (M x r)
//   U  = bf16(s * dY B)    (M x r)
//   dA = bf16(U^T X)       (r x K)
//   dB = bf16(dY^T T)      (N x r)
// lora_sm100.cu: tensor-core versions (split-K over a thread-block cluster,
// reduced in distributed shared memory: no workspace)
bool lora_tc_supported(int64_t M, int64_t N, int64_t K, int r);
cudaError_t launch_lora_xat_tc(const uint16_t* X, const uint16_t* A, int64_t M, int64_t K, int r, float s,
                               uint16_t* T, cudaStream_t stream);
cudaError_t launch_lora_dyb_tc(const uint16_t* dY, const uint16_t* B, int64_t M, int64_t N, int r, float s,
                               uint16_t* U, cudaStream_t stream, int64_t ld_dy = 0, int ld_u = 0);
cudaError_t launch_lora_da_tc(const uint16_t* X, const uint16_t* U, int64_t M, int64_t K, int r, uint16_t* dA,
                              cudaStream_t stream);
cudaError_t launch_lora_db_tc(const uint16_t* dY, const uint16_t* T, int64_t M, int64_t N, int r, uint16_t* dB,
                              cudaStream_t stream, int64_t ld_dy = 0, int64_t ld_t = 0);
// the G linears of a group in one launch each: U_g (columns g r .. of U,
// row pitch G r) and dB_g (rows n_g .. of dB_cat); dY is M x sum(Ns)
cudaError_t launch_lora_dyb_group(const uint16_t* dY, const uint16_t* B_cat, int64_t M, const int64_t* Ns, int G,
                                  int r, float s, uint16_t* U, cudaStream_t stream);
cudaError_t launch_lora_db_group(const uint16_t* dY, const uint16_t* T, int64_t M, const int64_t* Ns, int G, int r,
                                 uint16_t* dB_cat, cudaStream_t stream);
// dA and dB in one launch
cudaError_t launch_lora_grads_tc(const uint16_t* X, const uint16_t* U, const uint16_t* dY, const uint16_t* T,
                                 int64_t M, int64_t N, int64_t K, int r, uint16_t* dA, uint16_t* dB,
                                 cudaStream_t stream);
int lora_device_error(int reset);
// gemm_pair_sm100.cu: a kernel whose one bounded wait is never satisfied
// (records QLORA_ERR_TIMEOUT after limit_ns)
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream);
// gemm_simt.cu: CUDA-core versions (any shape)
cudaError_t launch_lora_xat_simt(const uint16_t* X, const uint16_t* A, int64_t M, int64_t K, int r, float s,
                                 uint16_t* T, cudaStream_t stream);
cudaError_t launch_lora_dyb_simt(const uint16_t* dY, const uint16_t* B, int64_t M, int64_t N, int r, float s,
                                 uint16_t* U, cudaStream_t stream);
cudaError_t launch_lora_grads_simt(const uint16_t* dY, const uint16_t* X, const uint16_t* T, const uint16_t* U,
                                   int64_t M, int64_t N, int64_t K, int r, uint16_t* dA, uint16_t* dB,
                                   cudaStream_t stream);

// gemm_simt.cu -- CUDA-core versions of the frozen-weight GEMMs below
cudaError_t launch_fwd_gemm_simt(const uint16_t* X, const Nf4Weight& w, const uint16_t* T,
                                 const uint16_t* B, int64_t M, int r, uint16_t* Y, cudaStream_t stream);
cudaError_t launch_bwd_dx_gemm_simt(const uint16_t* dY, const Nf4Weight& w, const uint16_t* U,
                                    const uint16_t* A, int64_t M, int r, uint16_t* dX,
                                    cudaStream_t stream);

// gemm_pair_sm100.cu -- the frozen-weight GEMMs on the tensor cores, on
// pairs of SMs (cta_group::2, 256 weight rows x 512 tokens per tile, the
// converted weight staged in shared memory; the backward reads the
// row-major codes).  The tiles' contraction stages are shared out evenly
// over the pairs; a tile split between pairs is finished through the
// workspace (pair_gemm_workspace bytes, 256-byte aligned).  Returns
// cudaErrorNotSupported (nothing launched) when no pair of CTAs fits the
// device.
bool pair_gemm_supported(int64_t M, const Nf4Weight& w, int r, bool bwd);
size_t pair_gemm_workspace();
cudaError_t launch_fwd_gemm_pair(const uint16_t* X, const Nf4Weight& w, const uint16_t* T, const uint16_t* B,
                                 int64_t M, int r, uint16_t* Y, void* ws, size_t ws_bytes, cudaStream_t stream);
cudaError_t launch_bwd_dx_gemm_pair(const uint16_t* dY, const Nf4Weight& w, const uint16_t* U, const uint16_t* A,
                                    int64_t M, int r, uint16_t* dX, void* ws, size_t ws_bytes,
                                    cudaStream_t stream);
int pair_device_error(int reset);

// Linears that read the same input (q/k/v, gate/up), stacked along N: the
// forward and the dX GEMM of the whole group in one launch each.  Every
// N_g a multiple of 256, at most 4 linears, G * r <= 256.
//   forward:  Y[:, n_g ..] = X W_g'^T + T[:, g r ..] B_g^T     (T: M x G r)
//   backward: dX = sum_g dY[:, n_g ..] W_g' + U A_cat          (U: M x G r)
constexpr int kMaxGroupLinears = 4;
struct Nf4Group {
    Nf4Weight w[kMaxGroupLinears];
    int G;
};
bool pair_group_supported(int64_t M, const Nf4Group& g, int r);
cudaError_t launch_fwd_gemm_pair_group(const uint16_t* X, const Nf4Group& g, const uint16_t* T, const uint16_t* B_cat,
                                       int64_t M, int r, uint16_t* Y, void* ws, size_t ws_bytes, cudaStream_t stream);
cudaError_t launch_bwd_dx_gemm_pair_group(const uint16_t* dY, const Nf4Group& g, const uint16_t* U,
                                          const uint16_t* A_cat, int64_t M, int r, uint16_t* dX, void* ws,
                                          size_t ws_bytes, cudaStream_t stream);

// gemv_sm100.cu -- the small-batch forward (1 <= M <= 16): T and Y in one
// kernel that streams the weight once; T is written to T_save when it is not
// null.  Returns cudaErrorNotSupported (nothing launched) when no cluster
// shape fits the device.
bool gemv_supported(int64_t M, int64_t N, int64_t K, int r);
cudaError_t launch_fwd_gemv(const uint16_t* X, const Nf4Weight& w, const uint16_t* A, const uint16_t* B, int64_t M,
                            int r, float s, uint16_t* Y, uint16_t* T_save, cudaStream_t stream);
int gemv_device_error(int reset);

// abi.cu -- the frozen-weight GEMMs with the LoRA slab fused in, on the
// tensor cores where the shapes allow, else on the CUDA cores
//   Y  = bf16(X W'^T + T B^T)      (M x N)
//   dX = bf16(dY W' + U A)         (M x K)
cudaError_t launch_fwd_gemm(const uint16_t* X, const Nf4Weight& w, const uint16_t* T,
                            const uint16_t* B, int64_t M, int r, uint16_t* Y, void* ws, size_t ws_bytes,
                            cudaStream_t stream);
cudaError_t launch_bwd_dx_gemm(const uint16_t* dY, const Nf4Weight& w, const uint16_t* U,
                               const uint16_t* A, int64_t M, int r, uint16_t* dX, void* ws, size_t ws_bytes,
                               cudaStream_t stream);

}  // namespace qlora
