// lora_sm100.cu -- the rank-r products of the LoRA path (QLoRA study notes,
// gitcode.csdn.net, section 4 eq. 3 and the adapter gradients of section
// 3.5) on the 5th-generation tensor cores:
//
//   T  = bf16(s X A^T)      (M x r)   contraction over K
//   U  = bf16(s dY B)       (M x r)   contraction over N
//   dA = bf16(U^T X)        (r x K)   contraction over the M tokens
//   dB = bf16(dY^T T)       (N x r)   contraction over the M tokens
//
// Each is a skinny GEMM C[rows x r] = sum_k Aop[row][k] Bop[j][k] whose
// operands are row-major bf16 matrices read either along their contiguous
// dimension (K-major) or across it (MN-major); TMA loads both in the
// 128-byte swizzled layout and tcgen05.mma takes either major-ness.  The
// outputs have only r columns, so the contraction is split across the S
// CTAs (S = 1..8, a power of two) of a thread-block cluster to fill the GPU.
//
// One CTA = one 128-row tile x one contraction split: warp 0 issues TMA,
// warp 1 the MMAs (M = 128, N = r rounded up to 16) into two accumulators
// in turn (even and odd 16-wide k steps), then all four warps add the two
// and copy the fp32 sum from tensor memory into the CTA's shared memory.  After a cluster barrier, rank c sums rows [c 128/S, (c+1) 128/S)
// of the tile over the S CTAs in rank order (distributed shared memory;
// deterministic), scales, rounds to bf16 and stores them: no partials in
// HBM and no second kernel.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace qlora {

__device__ int g_lora_error = 0;  // sticky: QLORA_ERR_TIMEOUT if a wait gave up

namespace {

using namespace sm100;

constexpr int kRows = 128;   // output rows per tile (MMA M)
constexpr int kBK = 64;      // contraction per stage
constexpr int kThreads = 128;
constexpr int kABytes = kRows * kBK * 2;  // 16 KiB
constexpr int kMaxSmem = 200 * 1024;

// One product of a launch: its output, rows x r bf16 (row pitch ldo), or
// r x rows when transposed, scaled by `scale` before the rounding; its
// contraction length; its first row tile in the grid.
struct SkinnyOut {
    uint16_t* out;
    int ldo;
    float scale;
    int transposed;
    int rows;      // output rows
    int kb_total;  // 64-wide contraction blocks
    int tile0;     // grid x of its first row tile
};

// A launch computes up to kMaxProducts products of one kind (the same
// operand majorness and rank: dA with dB, or the U or dB of the linears of a
// group), CTA column blockIdx.x belonging to the last product whose tile0
// it has reached.
constexpr int kMaxProducts = 4;
struct SkinnyParams {
    SkinnyOut o[kMaxProducts];
    int nprod;
    int r;
    int nt;        // r rounded up to 16 (MMA N)
    int splits;    // CTAs per cluster, a power of two
    int stages;
    int b_bytes;   // bytes of one B stage
    uint32_t tmem_cols;
};

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads)
k_lora_tc(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap tb0,
          const __grid_constant__ CUtensorMap ta1, const __grid_constant__ CUtensorMap tb1,
          const __grid_constant__ CUtensorMap ta2, const __grid_constant__ CUtensorMap tb2,
          const __grid_constant__ CUtensorMap ta3, const __grid_constant__ CUtensorMap tb3, const SkinnyParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stage_bytes = kABytes + p.b_bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.stages * stage_bytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * p.stages + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (p.stages + s); };
    const uint32_t done = bar0 + 8u * (2 * p.stages);

    const int bx = static_cast<int>(blockIdx.x);
    const int prod = (p.nprod > 1 && bx >= p.o[1].tile0 ? 1 : 0) + (p.nprod > 2 && bx >= p.o[2].tile0 ? 1 : 0) +
                     (p.nprod > 3 && bx >= p.o[3].tile0 ? 1 : 0);
    const SkinnyOut o = prod == 0 ? p.o[0] : prod == 1 ? p.o[1] : prod == 2 ? p.o[2] : p.o[3];
    const CUtensorMap* mapa = prod == 0 ? &ta0 : prod == 1 ? &ta1 : prod == 2 ? &ta2 : &ta3;
    const CUtensorMap* mapb = prod == 0 ? &tb0 : prod == 1 ? &tb1 : prod == 2 ? &tb2 : &tb3;
    const int row0 = (bx - o.tile0) * kRows;
    const int split = static_cast<int>(cluster_ctarank());  // == blockIdx.y: the cluster spans the splits
    const int kb_begin = static_cast<int>(static_cast<int64_t>(split) * o.kb_total / p.splits);
    const int kb_end = static_cast<int>(static_cast<int64_t>(split + 1) * o.kb_total / p.splits);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(done, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int* err = &g_lora_error;
    bool ok = true;

    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(mapa);
        tma_prefetch_desc(mapb);
        for (int kb = kb_begin, it = 0; kb < kb_end; ++kb, ++it) {
            const int s = it % p.stages;
            const uint32_t ph = (it / p.stages) & 1u;
            if (!mbar_wait(empty(s), ph ^ 1u, err)) break;
            mbar_arrive_expect_tx(full(s), kABytes + p.b_bytes);
            const uint32_t sa = smem_u32(smem + s * stage_bytes);
            const uint32_t sb = sa + kABytes;
            if (A_MN) {  // 128 MN-contiguous rows as two 64-wide boxes, 64 contraction rows each
                tma_load_2d(sa, mapa, full(s), row0, kb * kBK);
                tma_load_2d(sa + 8192, mapa, full(s), row0 + 64, kb * kBK);
            } else {
                tma_load_2d(sa, mapa, full(s), kb * kBK, row0);
            }
            if (B_MN) {
                for (int b = 0; b * 64 < p.nt; ++b) tma_load_2d(sb + b * 8192, mapb, full(s), b * 64, kb * kBK);
            } else {
                tma_load_2d(sb, mapb, full(s), kb * kBK, 0);
            }
        }
    } else if (warp == 1 && lane == 0) {
        const uint32_t idesc = idesc_bf16(kRows, p.nt, A_MN ? 1 : 0, B_MN ? 1 : 0);
        for (int kb = kb_begin, it = 0; kb < kb_end; ++kb, ++it) {
            const int s = it % p.stages;
            const uint32_t ph = (it / p.stages) & 1u;
            if (!mbar_wait(full(s), ph, err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * stage_bytes);
            const uint32_t sb = sa + kABytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                // 16 contraction steps: +32 bytes along a K-major row, +16 rows of 128 bytes MN-major
                const uint64_t ad = A_MN ? sdesc_mnmajor_sw128(sa + kk * 2048, 8192)
                                         : sdesc_kmajor_sw128(sa) + static_cast<uint64_t>(kk * 2);
                const uint64_t bd = B_MN ? sdesc_mnmajor_sw128(sb + kk * 2048, 8192)
                                         : sdesc_kmajor_sw128(sb) + static_cast<uint64_t>(kk * 2);
                // two accumulators in turn (even and odd k steps): consecutive
                // MMAs are independent, which nearly halves their issue time
                mma_bf16_ss(tmem + (kk & 1) * (p.tmem_cols / 2), ad, bd, idesc, (kb > kb_begin || kk >= 2) ? 1u : 0u);
            }
            tc_commit(empty(s));
        }
        if (ok) tc_commit(done);
    }
    __syncwarp();
    // the split's accumulator -> this CTA's shared memory [128][nt + 4] fp32
    // (the pipeline stages are free once `done` has fired)
    const int ld = p.nt + 4;
    float* acc = reinterpret_cast<float*>(smem);
    const bool fin = __all_sync(0xffffffffu, mbar_wait(done, 0, err));
    if (fin) {
        tc_fence_after();
        const int lr = warp * 32 + lane;
        for (int c0 = 0; c0 < p.nt; c0 += 16) {
            uint32_t v[16], w[16];
            tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
            tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + p.tmem_cols / 2 + c0, w);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 16; t += 4)  // even k steps + odd k steps
                *reinterpret_cast<float4*>(acc + lr * ld + c0 + t) = make_float4(
                    __uint_as_float(v[t]) + __uint_as_float(w[t]), __uint_as_float(v[t + 1]) + __uint_as_float(w[t + 1]),
                    __uint_as_float(v[t + 2]) + __uint_as_float(w[t + 2]),
                    __uint_as_float(v[t + 3]) + __uint_as_float(w[t + 3]));
        }
    } else {
        for (int i = threadIdx.x; i < kRows * ld; i += kThreads) acc[i] = 0.0f;
    }
    tc_fence_before();
    cluster_arrive();  // every split's accumulator is in its CTA's shared memory
    cluster_wait();
    {
        const int rows_per = kRows / p.splits;
        const int q4 = p.nt / 4;
        const uint32_t acc_s = smem_u32(acc);
        for (int idx = threadIdx.x; idx < rows_per * q4; idx += kThreads) {
            // consecutive threads take consecutive columns of one row, or (a
            // transposed output, whose rows are the columns in memory)
            // consecutive rows of one column group: coalesced stores either way
            const int lr = split * rows_per + (o.transposed ? idx % rows_per : idx / q4);
            const int c = (o.transposed ? idx / rows_per : idx % q4) * 4;
            const uint32_t off = static_cast<uint32_t>((lr * ld + c) * 4);
            // all ranks' values in flight together, then summed in rank order
            float4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (q < p.splits) v[q] = ld_cluster_f4(cluster_map(acc_s + off, static_cast<uint32_t>(q)));
            float4 sum = v[0];
#pragma unroll
            for (int q = 1; q < 8; ++q) {
                if (q < p.splits) {
                    sum.x += v[q].x; sum.y += v[q].y; sum.z += v[q].z; sum.w += v[q].w;
                }
            }
            const int row = row0 + lr;
            if (row < o.rows && c < p.r) {
                const uint32_t lo = pack_bf16x2(sum.x * o.scale, sum.y * o.scale);
                const uint32_t hi = pack_bf16x2(sum.z * o.scale, sum.w * o.scale);
                if (o.transposed) {
                    uint16_t* dst = o.out + static_cast<int64_t>(c) * o.rows + row;
                    dst[0] = static_cast<uint16_t>(lo & 0xffffu);
                    dst[o.rows] = static_cast<uint16_t>(lo >> 16);
                    dst[2 * static_cast<int64_t>(o.rows)] = static_cast<uint16_t>(hi & 0xffffu);
                    dst[3 * static_cast<int64_t>(o.rows)] = static_cast<uint16_t>(hi >> 16);
                } else {
                    *reinterpret_cast<uint2*>(o.out + static_cast<int64_t>(row) * o.ldo + c) = make_uint2(lo, hi);
                }
            }
        }
    }
    cluster_arrive();  // no CTA leaves while its shared memory may still be read
    cluster_wait();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() { return tensor_map_encoder(); }

// Row-major bf16 matrix (outer x inner, rows `pitch` elements apart; 0 =
// inner), 128-byte swizzled boxes of box_inner x box_outer.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer, uint64_t pitch = 0) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {(pitch ? pitch : inner) * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Plan {
    int nt, kb_total, splits, stages, b_bytes, smem;
    uint32_t tmem_cols;
    int64_t tiles;
};

// Splits: the smallest power of two (<= 8, <= the contraction blocks) that
// gives about two CTAs per SM.
Plan plan(int64_t rows, int64_t ctr, int r, bool b_mn) {
    Plan pl;
    pl.nt = static_cast<int>(round_up(r, 16));
    pl.kb_total = static_cast<int>(ceil_div(ctr > 0 ? ctr : 1, kBK));
    pl.tiles = ceil_div(rows > 0 ? rows : 1, kRows);
    const int64_t want = ceil_div(2LL * num_sms(), pl.tiles);
    int splits = 1;
    while (splits < want && splits * 2 <= 8 && splits * 2 <= pl.kb_total) splits *= 2;
    pl.splits = splits;
    pl.b_bytes = b_mn ? static_cast<int>(ceil_div(pl.nt, 64)) * 8192 : pl.nt * kBK * 2;
    const int stage = kABytes + pl.b_bytes;
    pl.stages = (kMaxSmem - 2048) / stage;
    pl.stages = pl.stages > 4 ? 4 : pl.stages;  // keeps two CTAs per SM for r <= 64
    const int staging = kRows * (pl.nt + 4) * 4;  // the accumulator, reusing the stages
    pl.smem = (pl.stages * stage > staging ? pl.stages * stage : staging) + 1024 + 1024;
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(pl.nt)) c <<= 1;
    pl.tmem_cols = 2 * c;  // two accumulators of c columns; at most 512 per SM for every r <= 256
                           // (r > 64 leaves room for one CTA per SM, r <= 64 for two)
    return pl;
}

SkinnyOut out_desc(uint16_t* out, int64_t rows, int r, float scale, bool transposed, int ldo, int kb_total) {
    SkinnyOut o;
    o.out = out;
    o.ldo = ldo ? ldo : r;
    o.scale = scale;
    o.transposed = transposed ? 1 : 0;
    o.rows = static_cast<int>(rows);
    o.kb_total = kb_total;
    o.tile0 = 0;
    return o;
}

// Launches n (1 .. kMaxProducts) products of one kind in one grid: product
// i's ceil(rows / 128) row tiles after those of the products before it.
// pl supplies the shared shape (rank, stages, shared memory, splits).
template <bool A_MN, bool B_MN>
cudaError_t launch_skinny(const Plan& pl, int n, const CUtensorMap* ma, const CUtensorMap* mb, const SkinnyOut* o,
                          int r, cudaStream_t st) {
    static ContextMemo<int> attr_memo;
    const cudaError_t attr = ensure_smem_limit(attr_memo, k_lora_tc<A_MN, B_MN>, kMaxSmem + 2048);
    if (attr != cudaSuccess) return attr;
    if (n < 1 || n > kMaxProducts) return cudaErrorInvalidValue;
    SkinnyParams p{};
    int64_t tiles = 0;
    for (int i = 0; i < kMaxProducts; ++i) {
        p.o[i] = o[i < n ? i : 0];
        p.o[i].tile0 = static_cast<int>(tiles);
        if (i < n) tiles += ceil_div(o[i].rows > 0 ? o[i].rows : 1, kRows);
    }
    p.nprod = n;
    p.r = r;
    p.nt = pl.nt;
    p.splits = pl.splits;
    p.stages = pl.stages;
    p.b_bytes = pl.b_bytes;
    p.tmem_cols = pl.tmem_cols;
    if (tiles >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr_c[1];
    attr_c[0].id = cudaLaunchAttributeClusterDimension;
    attr_c[0].val.clusterDim.x = 1;
    attr_c[0].val.clusterDim.y = static_cast<unsigned>(pl.splits);
    attr_c[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(pl.splits));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(pl.smem);
    cfg.stream = st;
    cfg.attrs = attr_c;
    cfg.numAttrs = 1;
    auto m = [&](const CUtensorMap* v, int i) -> const CUtensorMap& { return v[i < n ? i : 0]; };
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k_lora_tc<A_MN, B_MN>, m(ma, 0), m(mb, 0), m(ma, 1), m(mb, 1),
                                             m(ma, 2), m(mb, 2), m(ma, 3), m(mb, 3), p);
    note_launches(1);
    return e;
}

template <bool A_MN, bool B_MN>
cudaError_t run(const Plan& pl, const CUtensorMap& ma, const CUtensorMap& mb, int64_t rows, int r, float scale,
                uint16_t* out, bool transposed, cudaStream_t st, int ldo = 0) {
    const SkinnyOut o = out_desc(out, rows, r, scale, transposed, ldo, pl.kb_total);
    return launch_skinny<A_MN, B_MN>(pl, 1, &ma, &mb, &o, r, st);
}

}  // namespace

bool lora_tc_supported(int64_t M, int64_t N, int64_t K, int r) {
    return r % 8 == 0 && r >= 8 && r <= 256 && N % 8 == 0 && K % 64 == 0 && M >= 1 && M < (int64_t(1) << 31) &&
           N < (int64_t(1) << 31) && encode_fn() != nullptr;
}

// T = bf16(s X A^T): A operand X (K-major), B operand A (K-major).
cudaError_t launch_lora_xat_tc(const uint16_t* X, const uint16_t* A, int64_t M, int64_t K, int r, float s,
                               uint16_t* T, cudaStream_t st) {
    const Plan pl = plan(M, K, r, false);
    CUtensorMap ma, mb;
    if (!make_map(&ma, X, K, M, kBK, kRows) || !make_map(&mb, A, K, r, kBK, pl.nt)) return cudaErrorInvalidValue;
    return run<false, false>(pl, ma, mb, M, r, s, T, false, st);
}

// U = bf16(s dY B): A operand dY (K-major over n), B operand B^T (MN-major).
// dY and U may be column blocks of wider matrices (row pitches ld_dy, ld_u).
cudaError_t launch_lora_dyb_tc(const uint16_t* dY, const uint16_t* B, int64_t M, int64_t N, int r, float s,
                               uint16_t* U, cudaStream_t st, int64_t ld_dy, int ld_u) {
    const Plan pl = plan(M, N, r, true);
    CUtensorMap ma, mb;
    if (!make_map(&ma, dY, N, M, kBK, kRows, static_cast<uint64_t>(ld_dy)) || !make_map(&mb, B, r, N, 64, kBK))
        return cudaErrorInvalidValue;
    return run<false, true>(pl, ma, mb, M, r, s, U, false, st, ld_u);
}

// dA = bf16(U^T X) computed as dA^T[k][j] = sum_m X[m][k] U[m][j]: both MN-major.
cudaError_t launch_lora_da_tc(const uint16_t* X, const uint16_t* U, int64_t M, int64_t K, int r, uint16_t* dA,
                              cudaStream_t st) {
    const Plan pl = plan(K, M, r, true);
    CUtensorMap ma, mb;
    if (!make_map(&ma, X, K, M, 64, kBK) || !make_map(&mb, U, r, M, 64, kBK)) return cudaErrorInvalidValue;
    return run<true, true>(pl, ma, mb, K, r, 1.0f, dA, true, st);
}

// dB = bf16(dY^T T), dB[n][j] = sum_m dY[m][n] T[m][j]: both MN-major.
// dY and T may be column blocks of wider matrices (row pitches ld_dy, ld_t).
cudaError_t launch_lora_db_tc(const uint16_t* dY, const uint16_t* T, int64_t M, int64_t N, int r, uint16_t* dB,
                              cudaStream_t st, int64_t ld_dy, int64_t ld_t) {
    const Plan pl = plan(N, M, r, true);
    CUtensorMap ma, mb;
    if (!make_map(&ma, dY, N, M, 64, kBK, static_cast<uint64_t>(ld_dy)) ||
        !make_map(&mb, T, r, M, 64, kBK, static_cast<uint64_t>(ld_t)))
        return cudaErrorInvalidValue;
    return run<true, true>(pl, ma, mb, N, r, 1.0f, dB, false, st);
}

// dA and dB of one linear in one launch: both read their operands across
// the contraction (MN-major) over the same M tokens.  The split count is
// the largest (<= 8) that keeps both products' row tiles x splits within
// two CTAs per SM: measured on the 7B and 65B shapes, more splits only add
// waves of clusters (and their fixed cost), fewer leave SMs idle.
cudaError_t launch_lora_grads_tc(const uint16_t* X, const uint16_t* U, const uint16_t* dY, const uint16_t* T,
                                 int64_t M, int64_t N, int64_t K, int r, uint16_t* dA, uint16_t* dB,
                                 cudaStream_t st) {
    Plan pl = plan(K + N, M, r, true);
    const int64_t tiles_a = ceil_div(K, kRows), tiles_b = ceil_div(N, kRows);
    int splits = 1;
    while (splits * 2 <= 8 && splits * 2 <= pl.kb_total && (tiles_a + tiles_b) * splits * 2 <= 2LL * num_sms())
        splits *= 2;
    pl.splits = splits;
    CUtensorMap ma[2], mb[2];
    if (!make_map(&ma[0], X, K, M, 64, kBK) || !make_map(&mb[0], U, r, M, 64, kBK) ||
        !make_map(&ma[1], dY, N, M, 64, kBK) || !make_map(&mb[1], T, r, M, 64, kBK))
        return cudaErrorInvalidValue;
    const SkinnyOut o[2] = {out_desc(dA, K, r, 1.0f, true, 0, pl.kb_total), out_desc(dB, N, r, 1.0f, false, 0, pl.kb_total)};
    return launch_skinny<true, true>(pl, 2, ma, mb, o, r, st);
}

namespace {

// Largest split count (<= 8, <= kb) whose CTAs (tiles x splits) stay within
// two per SM.
int group_splits(int64_t tiles, int kb) {
    int splits = 1;
    while (splits * 2 <= 8 && splits * 2 <= kb && tiles * splits * 2 <= 2LL * num_sms()) splits *= 2;
    return splits;
}

}  // namespace

// U_g = bf16(s dY_g B_g) for the G linears of a group in one launch: dY_g is
// the column block n_g .. of dY (row pitch n_all), B_g the rows n_g .. of
// B_cat, U_g the columns g r .. of U (row pitch G r).
cudaError_t launch_lora_dyb_group(const uint16_t* dY, const uint16_t* B_cat, int64_t M, const int64_t* Ns, int G,
                                  int r, float s, uint16_t* U, cudaStream_t st) {
    if (G < 1 || G > kMaxProducts) return cudaErrorInvalidValue;
    int64_t n_all = 0, n_max = 0, n_min = -1;
    for (int g = 0; g < G; ++g) {
        n_all += Ns[g];
        n_max = Ns[g] > n_max ? Ns[g] : n_max;
        n_min = (n_min < 0 || Ns[g] < n_min) ? Ns[g] : n_min;
    }
    Plan pl = plan(M * G, n_max, r, true);
    pl.splits = group_splits(G * ceil_div(M, kRows), static_cast<int>(ceil_div(n_min, kBK)));
    CUtensorMap ma[kMaxProducts], mb[kMaxProducts];
    SkinnyOut o[kMaxProducts];
    int64_t n0 = 0;
    for (int g = 0; g < G; ++g) {
        if (!make_map(&ma[g], dY + n0, Ns[g], M, kBK, kRows, static_cast<uint64_t>(n_all)) ||
            !make_map(&mb[g], B_cat + n0 * r, r, Ns[g], 64, kBK))
            return cudaErrorInvalidValue;
        o[g] = out_desc(U + static_cast<int64_t>(g) * r, M, r, s, false, G * r, static_cast<int>(ceil_div(Ns[g], kBK)));
        n0 += Ns[g];
    }
    return launch_skinny<false, true>(pl, G, ma, mb, o, r, st);
}

// dB_g = bf16(dY_g^T T_g) for the G linears of a group in one launch (dB_g
// the rows n_g .. of dB_cat; T_g the columns g r .. of T, row pitch G r).
cudaError_t launch_lora_db_group(const uint16_t* dY, const uint16_t* T, int64_t M, const int64_t* Ns, int G, int r,
                                 uint16_t* dB_cat, cudaStream_t st) {
    if (G < 1 || G > kMaxProducts) return cudaErrorInvalidValue;
    int64_t n_all = 0;
    for (int g = 0; g < G; ++g) n_all += Ns[g];
    Plan pl = plan(n_all, M, r, true);
    int64_t tiles = 0;
    for (int g = 0; g < G; ++g) tiles += ceil_div(Ns[g], kRows);
    pl.splits = group_splits(tiles, pl.kb_total);
    CUtensorMap ma[kMaxProducts], mb[kMaxProducts];
    SkinnyOut o[kMaxProducts];
    int64_t n0 = 0;
    for (int g = 0; g < G; ++g) {
        if (!make_map(&ma[g], dY + n0, Ns[g], M, 64, kBK, static_cast<uint64_t>(n_all)) ||
            !make_map(&mb[g], T + static_cast<int64_t>(g) * r, r, M, 64, kBK, static_cast<uint64_t>(G) * r))
            return cudaErrorInvalidValue;
        o[g] = out_desc(dB_cat + n0 * r, Ns[g], r, 1.0f, false, 0, pl.kb_total);
        n0 += Ns[g];
    }
    return launch_skinny<true, true>(pl, G, ma, mb, o, r, st);
}

int lora_device_error(int reset) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_lora_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    if (reset && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_lora_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return v;
}

}  // namespace qlora
