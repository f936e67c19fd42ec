// gemm_simt.cu -- straightforward CUDA-core GEMMs for every product of the
// QLoRA linear (QLoRA study notes, gitcode.csdn.net, section 3.5 eq. 5 and
// section 4 eq. 3):
//   C[i][j] = bf16( alpha * ( sum_k a1(i,k) b1(j,k) + sum_k a2(i,k) b2(j,k) ) )
// with fp32 accumulation.  Each operand is either a strided bf16 matrix or
// the frozen NF4 weight, double-dequantized on the fly (eq. 6) to
// bf16(RN32(q[code] * c2')), read row-wise (W') or transposed (W'^T).  The
// second sum is the rank-r LoRA slab.
//
// These kernels are the portable correctness path of the library: the
// LoRA-side products (T, U, dA, dB) run here, and so do the frozen-weight
// GEMMs for shapes the tensor-core kernels do not take.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

struct Opnd {
    int kind;  // 0 bf16 strided, 1 W'[i][k], 2 W'[k][i]
    const uint16_t* p;
    int64_t si, sk;
    Nf4Weight w;
};

constexpr int BM = 64, BN = 64, BK = 16, kThreads = 256;

__device__ __forceinline__ float w_elem(const Nf4Weight& w, int64_t e, const float* sq, float mu) {
    const uint8_t byte = w.codes[e >> 1];
    const int code = (e & 1) ? (byte & 15) : (byte >> 4);
    const float cp = dq_constant(w.c2_fp8[e >> 6], w.c1[e >> 14], mu);
    return bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(sq[code], cp)));
}

__device__ __forceinline__ float fetch(const Opnd& o, int64_t i, int64_t k, const float* sq, float mu) {
    if (o.kind == 0) return bf16_bits_to_f32(o.p[i * o.si + k * o.sk]);
    if (o.kind == 1) return w_elem(o.w, i * o.w.K + k, sq, mu);
    return w_elem(o.w, k * o.w.K + i, sq, mu);
}

__global__ void __launch_bounds__(kThreads)
k_gemm_simt(int64_t Mo, int64_t No, Opnd a1, Opnd b1, int64_t K1, Opnd a2, Opnd b2, int64_t K2,
            float alpha, uint16_t* __restrict__ C, int64_t ldc, Nf4Tables tabs) {
    __shared__ float As[BK][BM];
    __shared__ float Bs[BK][BN];
    __shared__ float sq[16];
    if (threadIdx.x < 16) sq[threadIdx.x] = tabs.q[threadIdx.x];
    __syncthreads();
    float mu = 0.0f;
    if (a1.kind != 0) mu = *a1.w.mean;
    if (b1.kind != 0) mu = *b1.w.mean;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int64_t i0 = static_cast<int64_t>(blockIdx.y) * BM, j0 = static_cast<int64_t>(blockIdx.x) * BN;
    float acc[4][4] = {};
    for (int seg = 0; seg < 2; ++seg) {
        const Opnd& A = seg ? a2 : a1;
        const Opnd& B = seg ? b2 : b1;
        const int64_t Kc = seg ? K2 : K1;
        for (int64_t k0 = 0; k0 < Kc; k0 += BK) {
#pragma unroll
            for (int t = 0; t < (BM * BK) / kThreads; ++t) {
                const int idx = tid + kThreads * t;
                const int kk = idx / BM, ii = idx % BM;
                const int64_t gi = i0 + ii, gk = k0 + kk;
                As[kk][ii] = (gi < Mo && gk < Kc) ? fetch(A, gi, gk, sq, mu) : 0.0f;
                const int64_t gj = j0 + ii;
                Bs[kk][ii] = (gj < No && gk < Kc) ? fetch(B, gj, gk, sq, mu) : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < BK; ++kk) {
                float av[4], bv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) { av[u] = As[kk][ty * 4 + u]; bv[u] = Bs[kk][tx * 4 + u]; }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
            }
            __syncthreads();
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int64_t gi = i0 + ty * 4 + u, gj = j0 + tx * 4 + v;
            if (gi < Mo && gj < No) C[gi * ldc + gj] = f32_to_bf16_bits(alpha * acc[u][v]);
        }
}

Opnd bf16_op(const uint16_t* p, int64_t si, int64_t sk) {
    Opnd o{};
    o.kind = 0; o.p = p; o.si = si; o.sk = sk;
    return o;
}
Opnd nf4_op(const Nf4Weight& w, bool transposed) {
    Opnd o{};
    o.kind = transposed ? 2 : 1; o.w = w;
    return o;
}

cudaError_t gemm(int64_t Mo, int64_t No, const Opnd& a1, const Opnd& b1, int64_t K1, const Opnd& a2,
                 const Opnd& b2, int64_t K2, float alpha, uint16_t* C, int64_t ldc, cudaStream_t st) {
    if (Mo == 0 || No == 0) return cudaSuccess;
    dim3 grid(static_cast<unsigned>(ceil_div(No, BN)), static_cast<unsigned>(ceil_div(Mo, BM)));
    const int qtype = a1.kind != 0 ? a1.w.qtype : (b1.kind != 0 ? b1.w.qtype : QLORA_TYPE_NF4);
    k_gemm_simt<<<grid, kThreads, 0, st>>>(Mo, No, a1, b1, K1, a2, b2, K2, alpha, C, ldc, tables(qtype));
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_lora_xat_simt(const uint16_t* X, const uint16_t* A, int64_t M, int64_t K, int r,
                            float s, uint16_t* T, cudaStream_t st) {
    // T(m, j) = s * sum_k X[m][k] A[j][k]
    return gemm(M, r, bf16_op(X, K, 1), bf16_op(A, K, 1), K, Opnd{}, Opnd{}, 0, s, T, r, st);
}

cudaError_t launch_lora_dyb_simt(const uint16_t* dY, const uint16_t* B, int64_t M, int64_t N, int r,
                            float s, uint16_t* U, cudaStream_t st) {
    // U(m, j) = s * sum_n dY[m][n] B[n][j]
    return gemm(M, r, bf16_op(dY, N, 1), bf16_op(B, 1, r), N, Opnd{}, Opnd{}, 0, s, U, r, st);
}

cudaError_t launch_lora_grads_simt(const uint16_t* dY, const uint16_t* X, const uint16_t* T,
                              const uint16_t* U, int64_t M, int64_t N, int64_t K, int r,
                              uint16_t* dA, uint16_t* dB, cudaStream_t st) {
    // dA(j, k) = sum_m U[m][j] X[m][k];  dB(n, j) = sum_m dY[m][n] T[m][j]
    cudaError_t e = gemm(r, K, bf16_op(U, 1, r), bf16_op(X, 1, K), M, Opnd{}, Opnd{}, 0, 1.0f, dA, K, st);
    if (e != cudaSuccess) return e;
    return gemm(N, r, bf16_op(dY, 1, N), bf16_op(T, 1, r), M, Opnd{}, Opnd{}, 0, 1.0f, dB, r, st);
}

cudaError_t launch_fwd_gemm_simt(const uint16_t* X, const Nf4Weight& w, const uint16_t* T,
                                 const uint16_t* B, int64_t M, int r, uint16_t* Y, cudaStream_t st) {
    // Y(m, n) = sum_k X[m][k] W'[n][k] + sum_j T[m][j] B[n][j]
    return gemm(M, w.N, bf16_op(X, w.K, 1), nf4_op(w, false), w.K, bf16_op(T, r, 1), bf16_op(B, r, 1),
                r, 1.0f, Y, w.N, st);
}

cudaError_t launch_bwd_dx_gemm_simt(const uint16_t* dY, const Nf4Weight& w, const uint16_t* U,
                                    const uint16_t* A, int64_t M, int r, uint16_t* dX,
                                    cudaStream_t st) {
    // dX(m, k) = sum_n dY[m][n] W'[n][k] + sum_j U[m][j] A[j][k]
    return gemm(M, w.K, bf16_op(dY, w.N, 1), nf4_op(w, true), w.N, bf16_op(U, r, 1), bf16_op(A, 1, w.K),
                r, 1.0f, dX, w.K, st);
}

}  // namespace qlora
