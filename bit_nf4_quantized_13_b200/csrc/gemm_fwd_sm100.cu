// gemm_fwd_sm100.cu -- the fused QLoRA forward on the 5th-generation tensor
// cores (QLoRA study notes, gitcode.csdn.net, section 3.5 eq. 5 and 6,
// section 4 eq. 3):
//
//   Y = X W'^T + T B^T,   W' = bf16(q[code] * c2'),   T = bf16(s X A^T)
//
// The NF4 weight is double-dequantized on the fly and never written to
// memory.  The kernel computes Y^T tile by tile with the frozen weight as
// the MMA's A operand held in tensor memory:
//
//   D[n][m] (TMEM, fp32) += W'[n][k] (TMEM, bf16) * X[m][k] (smem)
//
// so the dequantized tile goes from registers straight into tensor memory
// (tcgen05.st) and costs no shared-memory bandwidth; only X is staged in
// shared memory, by TMA in the 128-byte swizzled K-major layout.  The rank-r
// LoRA product is the same GEMM continued over ceil(r/64) extra 64-wide
// slabs: A = B[n][j] (copied to TMEM like the weight), B operand = T[m][j]
// (TMA).  Tile: 128 weight rows x 256 tokens x 64; fp32 accumulator in
// 256 TMEM columns; 6 pipeline stages.
//
// Warp roles (320 threads, persistent over tiles, one CTA per SM):
//   warp 0       TMA producer for the X / T tiles
//   warp 1       MMA issuer (one thread)
//   warps 2..9   dequant producers (each a TMEM lane quarter and a 32-wide
//                half of every 64-wide stage), then the epilogue of the
//                same tile: tcgen05.ld, bf16, coalesced stores of Y
// Every wait is bounded; a timeout records QLORA_ERR_TIMEOUT and ends the
// kernel.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qlora {

// Sticky device-side error word of the tensor-core kernels (0 = none).
__device__ int g_tc_error = 0;

namespace {

using namespace sm100;

constexpr int kTileW = 128;   // weight rows per tile (MMA M)
constexpr int kTileT = 256;   // tokens per tile (MMA N)
constexpr int kBK = 64;       // contraction per stage
constexpr int kStages = 6;
constexpr int kXStageBytes = kTileT * kBK * 2;  // 32 KiB
constexpr int kAccCols = kTileT;                // fp32 accumulator columns
constexpr int kAStageCols = kBK / 2;            // bf16 pairs per TMEM column
constexpr uint32_t kTmemCols = 512;
constexpr int kDqWarps = 8;
constexpr int kThreads = 32 * (2 + kDqWarps);
constexpr int kSmemBytes = kStages * kXStageBytes + 1024 /* align */ + 1024 /* barriers etc. */;
static_assert(kAccCols + kStages * kAStageCols <= static_cast<int>(kTmemCols), "TMEM budget");

struct FwdParams {
    const uint8_t* codes;
    const uint8_t* c2_fp8;
    const float* c1;
    const float* mean;
    const uint16_t* Bm;  // N x r
    uint16_t* Y;         // M x N
    int M, N, K, r;
    float q[16];
};

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

struct Pipe {
    uint8_t* sX;       // kStages x 32 KiB of X (or T) tiles
    uint32_t bar0;     // full_b[S], full_a[S], empty[S], acc_full, acc_empty
    uint32_t tmem;     // accumulator at columns [0, 256), A stages after it
    int num_t, num_tiles, kb_w, kb_total;
    __device__ uint32_t full_b(int s) const { return bar0 + 8u * s; }
    __device__ uint32_t full_a(int s) const { return bar0 + 8u * (kStages + s); }
    __device__ uint32_t empty(int s) const { return bar0 + 8u * (2 * kStages + s); }
    __device__ uint32_t acc_full() const { return bar0 + 8u * (3 * kStages); }
    __device__ uint32_t acc_empty() const { return bar0 + 8u * (3 * kStages + 1); }
};

// warp 0, one thread: X tiles, then the T slabs, into the stage ring.
__device__ void role_tma(const Pipe& P, const CUtensorMap* tmap_x, const CUtensorMap* tmap_t, int* err) {
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < P.num_tiles; tile += gridDim.x) {
        const int t0 = (tile % P.num_t) * kTileT;
        for (int kb = 0; kb < P.kb_total; ++kb, ++it) {
            const int s = static_cast<int>(it % kStages);
            const uint32_t ph = (it / kStages) & 1u;
            if (!mbar_wait(P.empty(s), ph ^ 1u, err)) return;
            mbar_arrive_expect_tx(P.full_b(s), kXStageBytes);
            const uint32_t dst = smem_u32(P.sX + s * kXStageBytes);
            if (kb < P.kb_w)
                tma_load_2d(dst, tmap_x, P.full_b(s), kb * kBK, t0);
            else
                tma_load_2d(dst, tmap_t, P.full_b(s), (kb - P.kb_w) * kBK, t0);
        }
    }
}

// warp 1, one thread: four 128x256x16 MMAs per stage into the accumulator.
__device__ void role_mma(const Pipe& P, int* err) {
    constexpr uint32_t idesc = idesc_bf16(kTileW, kTileT);
    uint32_t it = 0, tcount = 0;
    for (int tile = blockIdx.x; tile < P.num_tiles; tile += gridDim.x, ++tcount) {
        if (!mbar_wait(P.acc_empty(), (tcount & 1u) ^ 1u, err)) return;
        tc_fence_after();
        for (int kb = 0; kb < P.kb_total; ++kb, ++it) {
            const int s = static_cast<int>(it % kStages);
            const uint32_t ph = (it / kStages) & 1u;
            if (!mbar_wait(P.full_b(s), ph, err)) return;
            if (!mbar_wait(P.full_a(s), ph, err)) return;
            tc_fence_after();
            const uint32_t a_col = P.tmem + kAccCols + s * kAStageCols;
            const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(P.sX + s * kXStageBytes));
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
                mma_bf16_ts(P.tmem, a_col + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc, (kb | kk) != 0);
            tc_commit(P.empty(s));
        }
        tc_commit(P.acc_full());
    }
}

// All lanes of the calling warp wait; the warp gives up together.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int* err) {
    const bool ok = mbar_wait(bar, parity, err);
    return __all_sync(0xffffffffu, ok);
}

// warps 2..9: dequantize the weight tile into TMEM stage by stage, then
// write this tile's outputs.
__device__ void role_dequant_epilogue(const Pipe& P, const FwdParams& p, const float* lut, int warp, int lane,
                                      int* err) {
    const int dq = warp - 2;
    const int quarter = warp & 3;  // the TMEM lanes this warp may touch
    const int half = dq >> 2;      // 32-wide half of each 64-wide stage
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float mu = *p.mean;
    const int64_t kblocks_per_row = p.K / kBK;
    uint32_t it = 0, tcount = 0;
    for (int tile = blockIdx.x; tile < P.num_tiles; tile += gridDim.x, ++tcount) {
        const int t0 = (tile % P.num_t) * kTileT;
        const int n = (tile / P.num_t) * kTileW + row;
        const bool row_ok = n < p.N;
        const uint8_t* crow = p.codes + static_cast<int64_t>(n) * (p.K / 2) + half * 16;
        const int64_t blk0 = static_cast<int64_t>(n) * kblocks_per_row;
        for (int kb = 0; kb < P.kb_total; ++kb, ++it) {
            uint32_t v[16];
            if (!row_ok) {
#pragma unroll
                for (int t = 0; t < 16; ++t) v[t] = 0u;
            } else if (kb < P.kb_w) {
                const uint4 cw = ldg_nc_v4(crow + kb * (kBK / 2));
                const int64_t blk = blk0 + kb;
                const float sc = dq_constant(p.c2_fp8[blk], __ldg(p.c1 + (blk >> 8)), mu);
                const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const uint32_t byte = (w4[t >> 2] >> (8 * (t & 3))) & 0xffu;
                    // element 2t (high nibble) -> low half, 2t+1 -> high half
                    v[t] = pack_bf16x2(__fmul_rn(lut[byte >> 4], sc), __fmul_rn(lut[byte & 15u], sc));
                }
            } else {
                const int j0 = (kb - P.kb_w) * kBK + half * 32;
                const uint16_t* brow = p.Bm + static_cast<int64_t>(n) * p.r + j0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 u = make_uint4(0u, 0u, 0u, 0u);
                    if (j0 + 8 * c < p.r) u = *reinterpret_cast<const uint4*>(brow + 8 * c);
                    v[4 * c + 0] = u.x;
                    v[4 * c + 1] = u.y;
                    v[4 * c + 2] = u.z;
                    v[4 * c + 3] = u.w;
                }
            }
            const int s = static_cast<int>(it % kStages);
            const uint32_t ph = (it / kStages) & 1u;
            if (!warp_wait(P.empty(s), ph ^ 1u, err)) return;
            tmem_st_32x32b_x16(P.tmem + lane_base + kAccCols + s * kAStageCols + half * 16, v);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(P.full_a(s));
        }
        // epilogue: this warp's lane quarter, columns [128 half, 128 half + 128)
        if (!warp_wait(P.acc_full(), tcount & 1u, err)) return;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            const int col = half * 128 + c * 32;
            uint32_t acc[32];
            tmem_ld_32x32b_x32(P.tmem + lane_base + col, acc);
            tmem_wait_ld();
            if (c == 3) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(P.acc_empty());
            }
            if (row_ok) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int m = t0 + col + j;
                    if (m < p.M) p.Y[static_cast<int64_t>(m) * p.N + n] = f32_to_bf16_bits(__uint_as_float(acc[j]));
                }
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
k_fwd_nf4_tc(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_t,
             const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kXStageBytes);
    float* lut = reinterpret_cast<float*>(bars + 3 * kStages + 2);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lut + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    Pipe P;
    P.sX = smem;
    P.bar0 = smem_u32(bars);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(P.full_b(s), 1);
            mbar_init(P.full_a(s), kDqWarps);
            mbar_init(P.empty(s), 1);
        }
        mbar_init(P.acc_full(), 1);
        mbar_init(P.acc_empty(), kDqWarps);
        fence_barrier_init();
    }
    if (threadIdx.x < 16) lut[threadIdx.x] = p.q[threadIdx.x];
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_t);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    P.tmem = *tmem_slot;
    P.num_t = (p.M + kTileT - 1) / kTileT;
    P.num_tiles = P.num_t * ((p.N + kTileW - 1) / kTileW);
    P.kb_w = p.K / kBK;
    P.kb_total = P.kb_w + (p.r + kBK - 1) / kBK;
    int* err = &g_tc_error;

    if (warp == 0) {
        if (lane == 0) role_tma(P, &tmap_x, &tmap_t, err);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) role_mma(P, err);
        __syncwarp();
    } else {
        role_dequant_epilogue(P, p, lut, warp, lane, err);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(P.tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Row-major bf16 matrix (outer x inner), 128-byte swizzled boxes of
// box_inner (<= 64) x box_outer elements.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                   uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fwd_tc_supported(int64_t M, const Nf4Weight& w, int r) {
    return M >= 1 && w.K >= kBK && w.K % kBK == 0 && r % 8 == 0 && r >= 8 && M < (int64_t(1) << 31) &&
           w.N < (int64_t(1) << 31) && w.K < (int64_t(1) << 31) && encode_fn() != nullptr;
}

cudaError_t launch_fwd_gemm_tc(const uint16_t* X, const Nf4Weight& w, const uint16_t* T, const uint16_t* B,
                               int64_t M, int r, uint16_t* Y, cudaStream_t st) {
    CUtensorMap mx, mt;
    if (!make_map_bf16(&mx, X, static_cast<uint64_t>(w.K), static_cast<uint64_t>(M), kBK, kTileT) ||
        !make_map_bf16(&mt, T, static_cast<uint64_t>(r), static_cast<uint64_t>(M), kBK, kTileT))
        return cudaErrorInvalidValue;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(k_fwd_nf4_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    FwdParams p;
    p.codes = w.codes;
    p.c2_fp8 = w.c2_fp8;
    p.c1 = w.c1;
    p.mean = w.mean;
    p.Bm = B;
    p.Y = Y;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.r = r;
    for (int i = 0; i < 16; ++i) p.q[i] = tables().q[i];
    const int64_t tiles = ceil_div(M, kTileT) * ceil_div(w.N, kTileW);
    const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
    k_fwd_nf4_tc<<<grid, kThreads, kSmemBytes, st>>>(mx, mt, p);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace qlora

extern "C" int qlora_device_error(int reset) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, qlora::g_tc_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    if (reset && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(qlora::g_tc_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return v;
}
