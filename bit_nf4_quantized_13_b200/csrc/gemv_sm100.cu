// gemv_sm100.cu -- the small-batch QLoRA forward (1 <= M <= 16 tokens):
//
//   T = bf16(s * X A^T)          (M x r)
//   Y = bf16(X W'^T + T B^T)     (M x N)
//
// QLoRA study notes (gitcode.csdn.net), section 3.5, eq. (5) with the LoRA
// scalar of section 4, eq. (3).  With a handful of tokens the product is a
// stream over the NF4 weight (0.516 bytes per parameter), so the design
// targets HBM bandwidth, not tensor throughput:
//
//  * Work unit: 16 consecutive weight rows over all of K.  Each CTA of a
//    cluster of C CTAs copies its K-slice of the 16 rows' codes (one
//    tensor-map box) into a stage of a shared-memory ring (3 to 6 deep);
//    the rows' FP8 block constants and c1 are plain loads, a unit ahead, by
//    the lanes that form c2'.  Few, large copies matter: issuing a copy
//    costs the producer thread hundreds of cycles under load.
//  * Decode: a 256-entry table maps one code byte (two 4-bit codes) to the
//    two bf16 codebook values as one 32-bit MMA operand register.  Each
//    table entry is replicated across the 32 banks (lane l reads word l of
//    a 256-byte row), so the lookups of a warp never conflict; the byte and
//    the lane offset form the address in one byte permute.
//  * Math: mma.m16n8k16 with the 16 weight rows as the A operand and up to
//    8 tokens per B tile.  K inside each 64-block is permuted consistently
//    in both operands so a lane's codes are 8 contiguous bytes per row.  The
//    block constant c2' multiplies each block's 64-term partial product
//    (the weight enters as bf16(q[code]) * c2' instead of
//    bf16(RN(q[code] * c2')); both are one bf16 rounding from w').
//  * X fragments stay in registers for the whole kernel: a warp always owns
//    the same K-blocks of its CTA's slice.
//  * Split-K across the cluster, reduced once: every unit's partials go
//    from the compute warps into one of two reduction slots; the producer
//    warp sums a slot's warps in warp order into this CTA's own per-unit
//    sums (kept in its shared memory for the whole kernel) and frees the
//    slot.  No warp waits on another's per-unit work unless it runs two
//    units ahead of the reduction.  At the end, after one cluster barrier,
//    CTA rank c finishes the units c, c + C, ...: it adds the C CTAs' sums
//    in rank order (distributed shared memory; deterministic), adds T B^T
//    with one more MMA per 16 ranks and stores Y.
//  * T = bf16(s X A^T) is formed in the same kernel from the register
//    resident X fragments (the rows of A take the MMA's A operand in the
//    permuted k order), reduced like the unit partials; every CTA forms the
//    same T from the cluster's sums.
//  * 14 compute warps stream the units; a 15th issues the copies and
//    reduces the slots; a 16th pulls the constants and the rows of B into
//    L2 early; all 16 finish the units at the end.
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace qlora {
namespace {

using namespace sm100;

__device__ int g_gemv_error;

constexpr int kRows = 16;                    // weight rows per unit
constexpr int kWarps = 14;                   // decode + MMA warps
constexpr int kCompute = kWarps * 32;
constexpr int kBarThreads = kCompute + 32;   // named-barrier hand-off: compute warps + producer warp
constexpr int kThreads = kBarThreads + 32;   // + the epilogue warp (16 warps: 128 registers a thread)
constexpr int kMaxBw = 3;                    // 64-blocks per warp per unit
constexpr int kMaxCtaBlocks = kWarps * kMaxBw;
constexpr int kMaxCl = 8;                    // CTAs per cluster
constexpr int kStages = 6;                   // most stages a launch uses
constexpr int kLutBytes = 256 * 256;         // 256 entries x 64 words (32 used)
constexpr int kMaxRankTiles = 4;             // r <= 64
constexpr int kTStride = 16 * kMaxRankTiles; // T staging row (ranks), bf16
constexpr int kRedSlots = 2;                 // reduction slots (units in flight between compute and reduce)

struct GemvParams {
    const uint8_t* codes;
    const uint8_t* c2_fp8;
    const float* c1;
    const float* mean;
    const uint16_t* X;      // M x K
    const uint16_t* A;      // r x K
    const uint16_t* B;      // N x r
    uint16_t* Y;            // M x N
    uint16_t* T_save;       // M x r or null
    int M, N, K, r;
    float s;
    int KB;                 // K / 64
    int units;              // N / 16
    int cl;                 // CTAs per cluster
    int row_stride;         // bytes between rows of a stage
    int stage_bytes;
    int nstages;            // ring depth, <= kStages
    int nmax;               // most units a cluster owns (the per-unit sums kept in shared memory)
    float q[16];
};

struct GemvSmem {
    size_t red_off, part_off, tpart_off, tbuf_off, bar_off, total;
};

// LUT | stages | reduction slots [2][kWarps][NT][32] | this CTA's unit sums
// [nmax][NT][32] | its T sums [rt][NT][32] | T (bf16) | barriers
__host__ __device__ constexpr GemvSmem gemv_smem(int NT, int stage_bytes, int nstages, int nmax, int rt) {
    GemvSmem m{};
    m.red_off = kLutBytes + static_cast<size_t>(nstages) * stage_bytes;
    m.part_off = m.red_off + static_cast<size_t>(kRedSlots) * kWarps * NT * 32 * 16;
    m.tpart_off = m.part_off + static_cast<size_t>(nmax) * NT * 32 * 16;
    m.tbuf_off = m.tpart_off + static_cast<size_t>(rt) * NT * 32 * 16;
    m.bar_off = m.tbuf_off + 16 * kTStride * 2;
    m.total = m.bar_off + (2 * kStages + 2 * kRedSlots) * 8;
    return m;
}

// Two bf16 codebook values for one code byte: the lower half holds the even
// element (high nibble), the upper half the odd one.
__device__ __forceinline__ uint32_t lut_pair(const uint8_t* lut, uint32_t word, uint32_t lane_off, int byte) {
    const uint32_t addr = __byte_perm(word, lane_off, 0x5504u | (static_cast<uint32_t>(byte) << 4));
    return *reinterpret_cast<const uint32_t*>(lut + addr);
}

// Issues the copy of unit `u` into `stage`, completing on `bar`: one
// tensor-map box of the codes (16 rows x row_stride bytes from block b0 on;
// this CTA's blocks plus a few of the next slice, or zeros past the row,
// which also pads the rows to a bank-friendly pitch).
__device__ __forceinline__ void issue_unit(const CUtensorMap* map, const GemvParams& p, int u, uint8_t* stage,
                                           uint64_t* bar, int b0) {
    const uint32_t b = smem_u32(bar);
    mbar_arrive_expect_tx(b, kRows * p.row_stride);
    tma_load_2d(smem_u32(stage), map, b, b0 * 4, u * kRows);
}

// Rows 16u + g and 16u + g + 8 of B as the A operand of the LoRA MMA
// (ranks 16 st ..), plain loads issued a unit ahead of their use.
__device__ __forceinline__ void load_b_rows(const GemvParams& p, int u, int g, int qd,
                                            uint32_t (&a)[kMaxRankTiles][4]) {
#pragma unroll
    for (int st = 0; st < kMaxRankTiles; ++st) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int64_t row = static_cast<int64_t>(u) * kRows + g + 8 * (h & 1);
            const int j = 16 * st + 2 * qd + 8 * (h >> 1);
            a[st][h] = j < p.r ? __ldg(reinterpret_cast<const uint32_t*>(p.B + row * p.r + j)) : 0u;
        }
    }
}

// The barriers: full[s] (TMA bytes of stage s), empty[s] (every compute
// lane has read stage s), red_full[b] (every compute lane has written slot
// b), red_empty[b] (the reducer has read slot b).
struct GemvBars {
    uint64_t* full;
    uint64_t* empty;
    uint64_t* red_full;
    uint64_t* red_empty;
};

// The producer warp of every CTA: issues and refills the stages and reduces
// the compute warps' partials, slot after slot (the units, then T's rank
// tiles), into this CTA's own sums in shared memory.
template <int NT>
__device__ __forceinline__ void producer_warp(const CUtensorMap* map, const GemvParams& p, uint8_t* smem,
                                              const GemvSmem& L, const GemvBars& B, int cid, int ncl, int n_local,
                                              int b0, int lane) {
    const int RT = (p.r + 15) >> 4;
    const int nst = p.nstages;
    uint8_t* stages = smem + kLutBytes;
    const float4* red = reinterpret_cast<const float4*>(smem + L.red_off);
    float4* part = reinterpret_cast<float4*>(smem + L.part_off);
    float4* tpart = reinterpret_cast<float4*>(smem + L.tpart_off);
    if (lane == 0) {
        const int pre = n_local < nst ? n_local : nst;
        for (int i = 0; i < pre; ++i) issue_unit(map, p, cid + i * ncl, stages + i * p.stage_bytes, &B.full[i], b0);
    }

    const int nq = n_local + RT;
#pragma unroll 1
    for (int q = 0; q < nq; ++q) {
        const int b = q % kRedSlots;
        const int i = q < n_local ? q : -1;  // unit, or one of T's rank tiles after the units
        if (i >= 0 && lane == 0 && i + nst < n_local) {
            // unit i has been read from its stage: refill the stage with unit i + nst
            const int s = i % nst;
            if (mbar_wait(smem_u32(&B.empty[s]), (i / nst) & 1, &g_gemv_error))
                issue_unit(map, p, cid + (i + nst) * ncl, stages + s * p.stage_bytes, &B.full[s], b0);
        }
        mbar_wait(smem_u32(&B.red_full[b]), (q / kRedSlots) & 1, &g_gemv_error);
        float4* dst = i >= 0 ? part + static_cast<size_t>(i) * NT * 32
                             : tpart + static_cast<size_t>(q - n_local) * NT * 32;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float4 sum = red[((b * kWarps + 0) * NT + nt) * 32 + lane];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) {  // warp order: deterministic
                const float4 x = red[((b * kWarps + w) * NT + nt) * 32 + lane];
                sum.x += x.x; sum.y += x.y; sum.z += x.z; sum.w += x.w;
            }
            dst[nt * 32 + lane] = sum;
        }
        mbar_arrive(smem_u32(&B.red_empty[b]));
    }
}

// Every warp of every CTA, after the cluster barrier: T = bf16(s * the
// cluster's T sums in rank order) into tbuf (warp 0; rank 0 of cluster 0
// also stores T_save), then the units c, c + C, ... of this CTA (rank c):
// the C CTAs' sums in rank order, plus T B^T, stored as Y.
template <int NT>
__device__ __forceinline__ void final_epilogue(const GemvParams& p, uint8_t* smem, const GemvSmem& L, uint32_t crank,
                                               int cid, int ncl, int n_local, int warp, int lane) {
    const int g = lane >> 2, qd = lane & 3;
    const int RT = (p.r + 15) >> 4;
    uint16_t* tbuf = reinterpret_cast<uint16_t*>(smem + L.tbuf_off);  // [16 tokens][kTStride]
    const uint32_t part0 = smem_u32(smem + L.part_off);
    const uint32_t tpart0 = smem_u32(smem + L.tpart_off);
    if (warp == 0) {
        for (int rt = 0; rt < RT; ++rt) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint32_t off = static_cast<uint32_t>(((rt * NT + nt) * 32 + lane) * 16);
                float4 v = ld_cluster_f4(cluster_map(tpart0 + off, 0));
                for (int rk = 1; rk < p.cl; ++rk) {
                    const float4 w = ld_cluster_f4(cluster_map(tpart0 + off, static_cast<uint32_t>(rk)));
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                }
                const float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 16 * rt + g + 8 * (e >> 1);
                    const int tok = 8 * nt + 2 * qd + (e & 1);
                    const uint16_t tb = f32_to_bf16_bits(e4[e] * p.s);
                    tbuf[tok * kTStride + j] = tb;
                    if (p.T_save && cid == 0 && crank == 0 && tok < p.M && j < p.r)
                        p.T_save[static_cast<int64_t>(tok) * p.r + j] = tb;
                }
            }
        }
    }
    __syncthreads();
    uint32_t tf[NT][kMaxRankTiles][2];  // T as the B operand of the LoRA MMA: (k = rank, n = token)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int st = 0; st < kMaxRankTiles; ++st)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
                tf[nt][st][hf] = (16 * st < p.r)
                                     ? *reinterpret_cast<const uint32_t*>(&tbuf[(8 * nt + g) * kTStride + 16 * st + 2 * qd + 8 * hf])
                                     : 0u;
    const int nw = kThreads / 32;
#pragma unroll 1
    for (int i = static_cast<int>(crank) + p.cl * warp; i < n_local; i += p.cl * nw) {
        const int n0 = (cid + i * ncl) * kRows;
        uint32_t ba[kMaxRankTiles][4];
        load_b_rows(p, cid + i * ncl, g, qd, ba);
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t off = static_cast<uint32_t>(((i * NT + nt) * 32 + lane) * 16);
            float4 sum = ld_cluster_f4(cluster_map(part0 + off, 0));
            for (int rk = 1; rk < p.cl; ++rk) {
                const float4 v = ld_cluster_f4(cluster_map(part0 + off, static_cast<uint32_t>(rk)));
                sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
            }
            acc[nt][0] = sum.x; acc[nt][1] = sum.y; acc[nt][2] = sum.z; acc[nt][3] = sum.w;
        }
#pragma unroll
        for (int st = 0; st < kMaxRankTiles; ++st) {
            if (16 * st >= p.r) break;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)  // A: a0a1 row g, a2a3 row g+8, a4..a7 the same 8 ranks further
                mma_16816(acc[nt], ba[st][0], ba[st][1], ba[st][2], ba[st][3], tf[nt][st][0], tf[nt][st][1]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = nt * 8 + 2 * qd + (e & 1);
                const int row = n0 + g + 8 * (e >> 1);
                if (tok < p.M) p.Y[static_cast<int64_t>(tok) * p.N + row] = f32_to_bf16_bits(acc[nt][e]);
            }
        }
    }
}

// X fragments of warp `warp`'s blocks: block jloc = warp + kWarps * jj.
// Lane (g, qd) of token tile nt holds X[nt*8 + g][64*kb + 16*qd .. +16);
// inside a block, k is permuted alike in both MMA operands so that MMA t of
// the block takes the elements 4t .. 4t+3 of every lane's run.
template <int NT>
__device__ __forceinline__ void load_x_frags(const GemvParams& p, int b0, int nblk, int warp, int lane,
                                             uint32_t (&xf)[kMaxBw][NT][8]) {
    const int g = lane >> 2, qd = lane & 3;
#pragma unroll
    for (int jj = 0; jj < kMaxBw; ++jj) {
        const int jloc = warp + kWarps * jj;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int tok = nt * 8 + g;
            uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
            if (jloc < nblk && tok < p.M) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    p.X + static_cast<int64_t>(tok) * p.K + static_cast<int64_t>(b0 + jloc) * 64 + 16 * qd);
                lo = __ldg(src);
                hi = __ldg(src + 1);
            }
            xf[jj][nt][0] = lo.x; xf[jj][nt][1] = lo.y; xf[jj][nt][2] = lo.z; xf[jj][nt][3] = lo.w;
            xf[jj][nt][4] = hi.x; xf[jj][nt][5] = hi.y; xf[jj][nt][6] = hi.z; xf[jj][nt][7] = hi.w;
        }
    }
}

// The 16th warp of every CTA pulls into L2 what the other warps will load
// later: the units' FP8 constants and c1, the rows of B the epilogue needs
// and the rows of A over this CTA's K-slice.
__device__ __forceinline__ void prefetch_warp(const GemvParams& p, int cid, int ncl, int n_local, int b0, int nblk,
                                              int lane) {
    for (int i = 0; i < n_local; ++i) {
        const int64_t row0 = static_cast<int64_t>(cid + i * ncl) * kRows;
        if (lane < kRows) {  // row lane of the unit: its FP8 bytes of this slice, and its c1 words
            const int64_t blk0 = (row0 + lane) * p.KB + b0;
            for (int j = 0; j < nblk; j += 128)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.c2_fp8 + blk0 + j));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.c1 + (blk0 >> 8)));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.B + (row0 + lane) * p.r));
        }
    }
    // the rows of A over this CTA's K-slice (for X A^T after the units)
    const int64_t k0 = static_cast<int64_t>(b0) * 64, kn = static_cast<int64_t>(nblk) * 64;
    for (int j = 0; j < p.r; ++j)
        for (int64_t k = 64 * lane; k < kn; k += 64 * 32)  // one 128-byte line per lane
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.A + j * static_cast<int64_t>(p.K) + k0 + k));
}

// Writes this warp's partial of slot sequence number q into reduction slot
// q % 2 (after the reducer has freed it) and arrives on the slot.
template <int NT>
__device__ __forceinline__ void put_partial(uint8_t* smem, const GemvSmem& L, const GemvBars& B, int q, int warp,
                                            int lane, const float (&v)[NT][4]) {
    const int b = q % kRedSlots;
    if (q >= kRedSlots) mbar_wait(smem_u32(&B.red_empty[b]), ((q / kRedSlots) - 1) & 1, &g_gemv_error);
    float4* red = reinterpret_cast<float4*>(smem + L.red_off) + (b * kWarps + warp) * NT * 32;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) red[nt * 32 + lane] = make_float4(v[nt][0], v[nt][1], v[nt][2], v[nt][3]);
    mbar_arrive(smem_u32(&B.red_full[b]));
}

template <int NT>
__device__ __forceinline__ void compute_warp(const GemvParams& p, uint8_t* smem, const GemvSmem& L, const GemvBars& B,
                                             int cid, int ncl, int n_local, int b0, int nblk, int warp, int lane,
                                             const uint32_t (&xf)[kMaxBw][NT][8]) {
    const int g = lane >> 2, qd = lane & 3;
    const int RT = (p.r + 15) >> 4;
    const int nst = p.nstages;
    const uint8_t* lut = smem;
    const uint8_t* stages = smem + kLutBytes;

    const float mean = __ldg(p.mean);
    const uint32_t lane_off = static_cast<uint32_t>(lane) * 4;
    // inputs of the block constant of (row = lane, block jloc) of unit i, for
    // lanes < 16: the FP8 byte and c1, loaded a unit ahead of their use
    auto load_consts = [&](int i, float (&c1v)[kMaxBw], uint32_t (&fb)[kMaxBw]) {
#pragma unroll
        for (int jj = 0; jj < kMaxBw; ++jj) {
            const int jloc = warp + kWarps * jj;
            c1v[jj] = 0.0f;
            fb[jj] = 0u;
            if (lane < kRows && jloc < nblk && i < n_local) {
                const int64_t blk = (static_cast<int64_t>(cid + i * ncl) * kRows + lane) * p.KB + b0 + jloc;
                c1v[jj] = __ldg(p.c1 + (blk >> 8));
                fb[jj] = __ldg(p.c2_fp8 + blk);
            }
        }
    };
    float c1c[kMaxBw], c1n[kMaxBw];
    uint32_t fbc[kMaxBw], fbn[kMaxBw];
    load_consts(0, c1c, fbc);

#pragma unroll 1
    for (int i = 0; i < n_local; ++i) {
        const int s = i % nst;
        load_consts(i + 1, c1n, fbn);  // the next unit's: the loads overlap this unit
        mbar_wait(smem_u32(&B.full[s]), (i / nst) & 1, &g_gemv_error);
        const uint8_t* stg = stages + s * p.stage_bytes;

        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
        for (int jj = 0; jj < kMaxBw; ++jj) {
            const int jloc = warp + kWarps * jj;
            if (jloc < nblk) {
                const uint2 cg = *reinterpret_cast<const uint2*>(stg + g * p.row_stride + jloc * 32 + qd * 8);
                const uint2 ch = *reinterpret_cast<const uint2*>(stg + (g + 8) * p.row_stride + jloc * 32 + qd * 8);
                // block constants c2' of the 16 rows: lane r < 16 forms row r's, then shuffles
                float c2v = 0.0f;
                if (lane < kRows) c2v = dq_constant(static_cast<uint8_t>(fbc[jj]), c1c[jj], mean);
                const float sg = __shfl_sync(0xffffffffu, c2v, g);
                const float sh = __shfl_sync(0xffffffffu, c2v, g + 8);
                float bacc[NT][4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint32_t wg = t < 2 ? cg.x : cg.y, wh = t < 2 ? ch.x : ch.y;
                    const int by = (t & 1) * 2;
                    const uint32_t a0 = lut_pair(lut, wg, lane_off, by);
                    const uint32_t a1 = lut_pair(lut, wh, lane_off, by);
                    const uint32_t a2 = lut_pair(lut, wg, lane_off, by + 1);
                    const uint32_t a3 = lut_pair(lut, wh, lane_off, by + 1);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (t == 0)
                            mma_16816_zc(bacc[nt], a0, a1, a2, a3, xf[jj][nt][0], xf[jj][nt][1]);
                        else
                            mma_16816(bacc[nt], a0, a1, a2, a3, xf[jj][nt][2 * t], xf[jj][nt][2 * t + 1]);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    acc[nt][0] = fmaf(bacc[nt][0], sg, acc[nt][0]);
                    acc[nt][1] = fmaf(bacc[nt][1], sg, acc[nt][1]);
                    acc[nt][2] = fmaf(bacc[nt][2], sh, acc[nt][2]);
                    acc[nt][3] = fmaf(bacc[nt][3], sh, acc[nt][3]);
                }
            }
        }
        mbar_arrive(smem_u32(&B.empty[s]));  // this lane has read the stage
#pragma unroll
        for (int jj = 0; jj < kMaxBw; ++jj) {
            c1c[jj] = c1n[jj];
            fbc[jj] = fbn[jj];
        }
        put_partial<NT>(smem, L, B, i, warp, lane, acc);
    }
    // This CTA's part of X A^T, one 16-rank tile at a time, after the units
    // (the rows of A were pulled into L2 meanwhile): the rows of A are the
    // MMA's A operand in the same permuted k order as the codes.
    for (int rt = 0; rt < RT; ++rt) {
        float ta[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) ta[nt][0] = ta[nt][1] = ta[nt][2] = ta[nt][3] = 0.0f;
#pragma unroll
        for (int jj = 0; jj < kMaxBw; ++jj) {
            const int jloc = warp + kWarps * jj;
            if (jloc < nblk) {
                uint4 ra[2][2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = 16 * rt + g + 8 * h;
                    ra[h][0] = ra[h][1] = make_uint4(0, 0, 0, 0);
                    if (j < p.r) {
                        const uint4* src = reinterpret_cast<const uint4*>(
                            p.A + static_cast<int64_t>(j) * p.K + static_cast<int64_t>(b0 + jloc) * 64 + 16 * qd);
                        ra[h][0] = __ldg(src);
                        ra[h][1] = __ldg(src + 1);
                    }
                }
                const uint32_t wg[8] = {ra[0][0].x, ra[0][0].y, ra[0][0].z, ra[0][0].w,
                                        ra[0][1].x, ra[0][1].y, ra[0][1].z, ra[0][1].w};
                const uint32_t wh[8] = {ra[1][0].x, ra[1][0].y, ra[1][0].z, ra[1][0].w,
                                        ra[1][1].x, ra[1][1].y, ra[1][1].z, ra[1][1].w};
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816(ta[nt], wg[2 * t], wh[2 * t], wg[2 * t + 1], wh[2 * t + 1], xf[jj][nt][2 * t],
                                  xf[jj][nt][2 * t + 1]);
            }
        }
        put_partial<NT>(smem, L, B, n_local + rt, warp, lane, ta);
    }

}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) k_gemv_nf4(const __grid_constant__ CUtensorMap map_codes,
                                                           const __grid_constant__ GemvParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int RT = (p.r + 15) >> 4;
    const GemvSmem L = gemv_smem(NT, p.stage_bytes, p.nstages, p.nmax, RT);
    GemvBars B;
    B.full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
    B.empty = B.full + kStages;
    B.red_full = B.empty + kStages;
    B.red_empty = B.red_full + kRedSlots;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = cluster_ctarank();
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(num_clusters_x());
    const int b0 = static_cast<int>(static_cast<int64_t>(crank) * p.KB / p.cl);
    const int nblk = static_cast<int>(static_cast<int64_t>(crank + 1) * p.KB / p.cl) - b0;
    const int n_local = cid < p.units ? (p.units - 1 - cid) / ncl + 1 : 0;

    // the producer arms the barriers and sends off the first copies at once;
    // the compute warps' X fragment loads fly during the rest of the set-up
    if (warp == kWarps && lane == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(smem_u32(&B.full[i]), 1);
            mbar_init(smem_u32(&B.empty[i]), kCompute);   // every compute lane
        }
        for (int i = 0; i < kRedSlots; ++i) {
            mbar_init(smem_u32(&B.red_full[i]), kCompute);
            mbar_init(smem_u32(&B.red_empty[i]), 32);     // every reducer lane
        }
        fence_barrier_init();
        tma_prefetch_desc(&map_codes);
    }
    uint32_t xf[kMaxBw][NT][8];
    if (warp < kWarps) load_x_frags<NT>(p, b0, nblk, warp, lane, xf);
    if (tid < 256) {  // the decode table: entry v replicated into words 0..31 of row v
        const uint32_t e = pack_bf16x2(p.q[tid >> 4], p.q[tid & 15]);
        uint4* row = reinterpret_cast<uint4*>(smem + tid * 256);
#pragma unroll
        for (int i = 0; i < 8; ++i) row[i] = make_uint4(e, e, e, e);
    }
    __syncthreads();

    if (warp == kWarps)
        producer_warp<NT>(&map_codes, p, smem, L, B, cid, ncl, n_local, b0, lane);
    else if (warp < kWarps)
        compute_warp<NT>(p, smem, L, B, cid, ncl, n_local, b0, nblk, warp, lane, xf);
    else
        prefetch_warp(p, cid, ncl, n_local, b0, nblk, lane);
    __syncthreads();   // this CTA's sums are complete
    cluster_arrive();  // ... and every CTA's
    cluster_wait();
    final_epilogue<NT>(p, smem, L, crank, cid, ncl, n_local, warp, lane);
    cluster_arrive();  // no CTA leaves while cluster peers may still read its shared memory
    cluster_wait();
}

struct Plan {
    int cl, clusters, row_stride, stage_bytes, nstages, nmax;
    size_t smem;
};

// Largest number of co-resident clusters of `cl` CTAs with `smem` bytes of
// shared memory each, cached per (CUDA context, cluster size, smem).
template <int NT>
int max_clusters(int cl, size_t smem) {
    static std::mutex mu;
    static std::map<std::tuple<uint64_t, int, size_t>, int> cache;
    uint64_t ctx = 0;
    if (!current_context_id(&ctx)) return 0;
    const auto key = std::make_tuple(ctx, cl, smem);
    std::lock_guard<std::mutex> lk(mu);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    if (cudaFuncSetAttribute(k_gemv_nf4<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(cl * num_sms());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_gemv_nf4<NT>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    cache[key] = n;
    return n;
}

template <int NT>
bool make_plan(int64_t N, int64_t K, int r, Plan& best) {
    const int KB = static_cast<int>(K / 64);
    const int units = static_cast<int>(N / kRows);
    const int RT = (r + 15) / 16;
    double best_eff = -1.0;
    const int sms = num_sms();
    for (int cl : {1, 2, 4, 8}) {
        const int maxblk = static_cast<int>(ceil_div(KB, cl));
        if (maxblk > kMaxCtaBlocks || KB < cl) continue;
        Plan pl{};
        pl.cl = cl;
        pl.row_stride = static_cast<int>(round_up(maxblk * 32, 128) + 32);  // = 32 mod 128: no bank conflicts
        if (pl.row_stride / 8 > 256) continue;                                 // tensor-map box width
        pl.stage_bytes = static_cast<int>(round_up(kRows * pl.row_stride, 128));
        // the units of a cluster, for the largest cluster count this size allows
        const int cl_max = sms / cl;
        const int nmax_est = static_cast<int>(ceil_div(units, units < cl_max ? units : cl_max));
        pl.nstages = 0;
        for (int ns = kStages; ns >= 3 && !pl.nstages; --ns)
            if (gemv_smem(NT, pl.stage_bytes, ns, nmax_est, RT).total <= 227 * 1024) pl.nstages = ns;
        if (!pl.nstages) continue;
        pl.nmax = nmax_est;
        pl.smem = gemv_smem(NT, pl.stage_bytes, pl.nstages, pl.nmax, RT).total;
        const int maxc = max_clusters<NT>(cl, pl.smem);
        if (maxc <= 0) continue;
        pl.clusters = units < maxc ? units : maxc;
        // fewer clusters fit than assumed: more units each, fewer stages if need be
        pl.nmax = static_cast<int>(ceil_div(units, pl.clusters));
        while (pl.nstages >= 3 && gemv_smem(NT, pl.stage_bytes, pl.nstages, pl.nmax, RT).total > 227 * 1024)
            --pl.nstages;
        if (pl.nstages < 3) continue;
        pl.smem = gemv_smem(NT, pl.stage_bytes, pl.nstages, pl.nmax, RT).total;
        const int per = static_cast<int>(ceil_div(units, pl.clusters));
        const double eff = static_cast<double>(units) / (static_cast<double>(pl.clusters) * per) *
                           (static_cast<double>(pl.clusters) * cl / sms);
        if (eff > best_eff + 0.01) {
            best_eff = eff;
            best = pl;
        }
    }
    return best_eff > 0.0;
}

// The codes as a row-major [N][K/16] array of 64-bit words; boxes of
// row_stride / 8 words x 16 rows, zero fill past the end of a row.
bool make_codes_map(CUtensorMap* m, const GemvParams& p) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.K / 16), static_cast<cuuint64_t>(p.N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.K / 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(p.row_stride / 8), static_cast<cuuint32_t>(kRows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(p.codes), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT>
cudaError_t launch_gemv(const GemvParams& p, const Plan& pl, cudaStream_t st) {
    CUtensorMap map;
    if (!make_codes_map(&map, p)) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(k_gemv_nf4<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(pl.smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(pl.cl * pl.clusters);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_gemv_nf4<NT>, map, p);
    note_launches(1);
    return e;
}

}  // namespace

bool gemv_supported(int64_t M, int64_t N, int64_t K, int r) {
    return M >= 1 && M <= 16 && N >= kRows && N % kRows == 0 && K >= 64 && K % 64 == 0 &&
           K / 64 <= kMaxCl * kMaxCtaBlocks && N / kRows < (int64_t(1) << 30) && r >= 8 && r % 8 == 0 &&
           r <= 16 * kMaxRankTiles;
}

cudaError_t launch_fwd_gemv(const uint16_t* X, const Nf4Weight& w, const uint16_t* A, const uint16_t* B, int64_t M,
                            int r, float s, uint16_t* Y, uint16_t* T_save, cudaStream_t st) {
    const bool two = M > 8;
    Plan pl{};
    if (!(two ? make_plan<2>(w.N, w.K, r, pl) : make_plan<1>(w.N, w.K, r, pl))) return cudaErrorNotSupported;
    GemvParams p{};
    p.codes = w.codes;
    p.c2_fp8 = w.c2_fp8;
    p.c1 = w.c1;
    p.mean = w.mean;
    p.X = X;
    p.A = A;
    p.B = B;
    p.Y = Y;
    p.T_save = T_save;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.r = r;
    p.s = s;
    p.KB = static_cast<int>(w.K / 64);
    p.units = static_cast<int>(w.N / kRows);
    p.cl = pl.cl;
    p.row_stride = pl.row_stride;
    p.stage_bytes = pl.stage_bytes;
    p.nstages = pl.nstages;
    p.nmax = pl.nmax;
    const float* q = tables(w.qtype).q;
    for (int i = 0; i < 16; ++i) p.q[i] = q[i];
    return two ? launch_gemv<2>(p, pl, st) : launch_gemv<1>(p, pl, st);
}

int gemv_device_error(int reset) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemv_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    if (reset && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_gemv_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return v;
}

}  // namespace qlora
