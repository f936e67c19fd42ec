// gemm_nf4_sm100.cu -- the two frozen-weight GEMMs of the QLoRA linear on
// the 5th-generation tensor cores (QLoRA study notes, gitcode.csdn.net,
// section 3.5 eq. 5 and 6, section 4 eq. 3, and the gradient through the
// bf16 weight of section 3.5):
//
//   forward:  Y  = X  W'^T + T B^T     T = bf16(s X A^T)      (M x N)
//   backward: dX = dY W'   + U A       U = bf16(s dY B)       (M x K)
//   W' = bf16(q[code] * c2'), double-dequantized on the fly, never stored.
//
// Both compute the transposed product tile by tile with the weight as the
// MMA's A operand held in tensor memory:
//
//   forward:  D[n][m]     += W'[n][k]     * X[m][k]     (contract over k)
//   backward: D[k][m]     += W'[n][k]     * dY[m][n]    (contract over n)
//
// so a dequantized tile goes from registers straight into tensor memory
// (tcgen05.st) and costs no shared-memory bandwidth; only the activation
// operand (X or dY) is staged in shared memory, by TMA in the 128-byte
// swizzled K-major layout.  The rank-r LoRA product is the same GEMM
// continued over ceil(r/64) extra 64-wide slabs whose A operand is B (or
// A^T) copied into tensor memory and whose B operand is T (or U) by TMA.
//
// Tile: 128 weight rows (n forward, k backward) x 256 tokens x 64; fp32
// accumulator in 256 TMEM columns; 6 pipeline stages.  Warp roles (320
// threads, persistent over tiles, one CTA per SM):
//   warp 0       TMA producer for the activation tiles
//   warp 1       MMA issuer (one thread)
//   warps 2..9   dequant producers (each a TMEM lane quarter and a 32-wide
//                half of every 64-wide stage), then the epilogue of the
//                same tile: tcgen05.ld, bf16, stores coalesced along the
//                weight-row index
// Every wait is bounded; a timeout records QLORA_ERR_TIMEOUT in a sticky
// device word (qlora_device_error) and ends the kernel.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

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
constexpr int kDqWarps = 16;                    // four per TMEM lane quarter
constexpr int kParts = kDqWarps / 4;            // stage kb is converted by the warps with part == kb % 4
template <bool kBwd>
struct Prefetch {  // own stages of codes in flight per dequant thread
    static constexpr int value = kBwd ? 1 : 2;
};
constexpr int kThreads = 32 * (2 + kDqWarps);   // 576
constexpr int kStageWords = 4 * 68 + 64;        // backward transpose staging per warp (64 rows)
constexpr uint32_t kNoRow = 0x100u;             // prefetch slot holds no weights
constexpr int kSmemBytes = kStages * kXStageBytes + 1024 /* align */ + 1024 /* barriers etc. */ +
                           kDqWarps * kStageWords * 4;
static_assert(kAccCols + kStages * kAStageCols <= static_cast<int>(kTmemCols), "TMEM budget");

struct GemmParams {
    const uint8_t* codes;
    const uint8_t* c2_fp8;
    const float* c1;
    const float* mean;
    const uint16_t* lora;  // forward: B (N x r); backward: A (r x K)
    uint16_t* out;         // forward: Y (M x N); backward: dX (M x K)
    int M;                 // tokens
    int rows;              // weight rows of the product: N forward, K backward
    int ctr;               // contraction over the weight: K forward, N backward
    int N, K, r;
    float q[16];
};

__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

struct Pipe {
    uint8_t* sA;       // kStages x 32 KiB of activation tiles
    uint32_t bar0;     // full_b[S], full_a[S], empty[S], acc_full, acc_empty
    uint32_t tmem;     // accumulator at columns [0, 256), A stages after it
    int num_t, num_tiles, kb_w, kb_total;
    __device__ uint32_t full_b(int s) const { return bar0 + 8u * s; }
    __device__ uint32_t full_a(int s) const { return bar0 + 8u * (kStages + s); }
    __device__ uint32_t empty(int s) const { return bar0 + 8u * (2 * kStages + s); }
    __device__ uint32_t acc_full() const { return bar0 + 8u * (3 * kStages); }
    __device__ uint32_t acc_empty() const { return bar0 + 8u * (3 * kStages + 1); }
};

// warp 0, one thread: activation tiles, then the LoRA slabs, into the ring.
__device__ void role_tma(const Pipe& P, const CUtensorMap* tmap_act, const CUtensorMap* tmap_lora, int* err) {
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < P.num_tiles; tile += gridDim.x) {
        const int t0 = (tile % P.num_t) * kTileT;
        for (int kb = 0; kb < P.kb_total; ++kb, ++it) {
            const int s = static_cast<int>(it % kStages);
            const uint32_t ph = (it / kStages) & 1u;
            if (!mbar_wait(P.empty(s), ph ^ 1u, err)) return;
            mbar_arrive_expect_tx(P.full_b(s), kXStageBytes);
            const uint32_t dst = smem_u32(P.sA + s * kXStageBytes);
            if (kb < P.kb_w)
                tma_load_2d(dst, tmap_act, P.full_b(s), kb * kBK, t0);
            else
                tma_load_2d(dst, tmap_lora, P.full_b(s), (kb - P.kb_w) * kBK, t0);
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
            const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(P.sA + s * kXStageBytes));
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
                mma_bf16_ts(P.tmem, a_col + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc, (kb | kk) != 0);
            tc_commit(P.empty(s));
        }
        tc_commit(P.acc_full());
    }
}

// Lane 0 of the calling warp waits; the result is broadcast so the warp
// proceeds (or gives up) together.  __syncwarp orders the other lanes
// after the observed phase.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int* err, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, err) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// q[code] read from the 16-entry table by a byte offset (code * 4).
__device__ __forceinline__ float lut_at(const float* lut, uint32_t byte_off) {
    return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(lut) + byte_off);
}

__device__ __forceinline__ uint32_t scale_pack(float a, float b, float sc) {
    const float2 x = __fmul2_rn(make_float2(a, b), make_float2(sc, sc));
    return pack_bf16x2(x.x, x.y);
}

// Per-lane, per-stage inputs of the dequantization, loaded kPrefetch
// stages ahead.  Forward: the lane's weight row, 64 consecutive codes (32
// bytes, one sector) under one block constant.  Backward: weight rows
// n0 + lane and n0 + 32 + lane, the 32 columns of this warp (16 bytes
// each), each row with its own block constant.
struct StageIn {
    uint4 c0, c1v;      // forward: codes bytes 0..15, 16..31; backward: row lane, row 32+lane
    uint32_t b0, b1;    // FP8 constant byte(s) (kNoRow: no weights)
    float s0, s1;       // c1 of the block(s)
};

// Forward: 32 TMEM columns = 64 contraction values of one row.  In each
// code byte the high nibble is the even element, which lands in the low
// half of its column.
__device__ __forceinline__ void convert_row(const StageIn& in, float mu, const float* lut, uint32_t (&v)[32]) {
    const float sc = in.b0 == kNoRow ? 0.0f : dq_constant(static_cast<uint8_t>(in.b0), in.s0, mu);
    const uint32_t w8[8] = {in.c0.x, in.c0.y, in.c0.z, in.c0.w, in.c1v.x, in.c1v.y, in.c1v.z, in.c1v.w};
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        const uint32_t hi4 = (w8[h] >> 2) & 0x3C3C3C3Cu;  // even-element code * 4, per byte
        const uint32_t lo4 = (w8[h] << 2) & 0x3C3C3C3Cu;  // odd-element code * 4, per byte
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a = lut_at(lut, __byte_perm(hi4, 0u, 0x4440u | j));
            const float b = lut_at(lut, __byte_perm(lo4, 0u, 0x4440u | j));
            v[4 * h + j] = scale_pack(a, b, sc);
        }
    }
}

// Backward: lane = weight column k; its 64 contraction values are 64 weight
// rows n.  The warp exchanges the rows' code words and constants through a
// small shared buffer; each lane rotates its own nibble out of each word.
__device__ __forceinline__ void convert_cols(const StageIn& in, float mu, const float* lut, uint32_t* wsm,
                                             int lane, uint32_t (&v)[32]) {
    float* ssm = reinterpret_cast<float*>(wsm + 4 * 68);
    const float sc0 = in.b0 == kNoRow ? 0.0f : dq_constant(static_cast<uint8_t>(in.b0), in.s0, mu);
    const float sc1 = in.b1 == kNoRow ? 0.0f : dq_constant(static_cast<uint8_t>(in.b1), in.s1, mu);
    wsm[0 * 68 + lane] = in.c0.x;
    wsm[1 * 68 + lane] = in.c0.y;
    wsm[2 * 68 + lane] = in.c0.z;
    wsm[3 * 68 + lane] = in.c0.w;
    wsm[0 * 68 + 32 + lane] = in.c1v.x;
    wsm[1 * 68 + 32 + lane] = in.c1v.y;
    wsm[2 * 68 + 32 + lane] = in.c1v.z;
    wsm[3 * 68 + 32 + lane] = in.c1v.w;
    ssm[lane] = sc0;
    ssm[32 + lane] = sc1;
    __syncwarp();
    const int wi = lane >> 3;  // the 32-bit word holding this column's nibbles
    const int shift = ((lane & 7) >> 1) * 8 + ((lane & 1) ? 0 : 4);
    const uint32_t rot = static_cast<uint32_t>(shift + 30) & 31u;  // nibble -> bits [2, 6)
#pragma unroll
    for (int g = 0; g < 16; ++g) {
        const uint4 c4 = *reinterpret_cast<const uint4*>(wsm + wi * 68 + 4 * g);
        const float4 s4 = *reinterpret_cast<const float4*>(ssm + 4 * g);
        const float x0 = lut_at(lut, __funnelshift_r(c4.x, c4.x, rot) & 0x3Cu);
        const float x1 = lut_at(lut, __funnelshift_r(c4.y, c4.y, rot) & 0x3Cu);
        const float x2 = lut_at(lut, __funnelshift_r(c4.z, c4.z, rot) & 0x3Cu);
        const float x3 = lut_at(lut, __funnelshift_r(c4.w, c4.w, rot) & 0x3Cu);
        const float2 y01 = __fmul2_rn(make_float2(x0, x1), make_float2(s4.x, s4.y));
        const float2 y23 = __fmul2_rn(make_float2(x2, x3), make_float2(s4.z, s4.w));
        v[2 * g] = pack_bf16x2(y01.x, y01.y);
        v[2 * g + 1] = pack_bf16x2(y23.x, y23.y);
    }
    __syncwarp();
}

// warps 2..17: each converts every fourth stage of the weight tile into
// TMEM (quarter = its TMEM lanes, part = which stages), then writes a
// quarter of this tile's outputs.
template <bool kBwd>
__device__ __forceinline__ void role_dequant_epilogue(const Pipe& P, const GemmParams& p, const float* lut,
                                                      uint32_t* wsm, int warp, int lane, int* err) {
    const int dq = warp - 2;
    const int quarter = warp & 3;  // the TMEM lanes this warp may touch
    const int part = dq >> 2;      // converts the stages kb with kb % 4 == part
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float mu = *p.mean;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < P.num_tiles; tile += gridDim.x, ++tcount) {
        const int t0 = (tile % P.num_t) * kTileT;
        const int row0 = (tile / P.num_t) * kTileW;
        const int grow = row0 + row;             // this lane's weight row of the product
        const bool lane_ok = grow < p.rows;
        const int wcol0 = row0 + quarter * 32;   // backward: first weight column of this warp
        const bool warp_cols_ok = wcol0 < p.rows;
        const uint32_t g0 = tcount * static_cast<uint32_t>(P.kb_total);  // ring index of stage 0

        constexpr int kPrefetch = Prefetch<kBwd>::value;
        StageIn buf[kPrefetch];
        auto issue = [&](int kb, StageIn& in) {
            in.c0 = make_uint4(0u, 0u, 0u, 0u);
            in.c1v = make_uint4(0u, 0u, 0u, 0u);
            in.b0 = kNoRow;
            in.b1 = kNoRow;
            in.s0 = in.s1 = 0.0f;
            if (kb >= P.kb_w) return;
            if (kBwd) {
                if (!warp_cols_ok) return;
                const int n0 = kb * kBK + lane;
                if (n0 < p.N) {
                    const int64_t e = static_cast<int64_t>(n0) * p.K + wcol0;
                    in.c0 = ldg_nc_v4(p.codes + (e >> 1));
                    in.b0 = __ldg(p.c2_fp8 + (e >> 6));
                    in.s0 = __ldg(p.c1 + (e >> 14));
                }
                if (n0 + 32 < p.N) {
                    const int64_t e = static_cast<int64_t>(n0 + 32) * p.K + wcol0;
                    in.c1v = ldg_nc_v4(p.codes + (e >> 1));
                    in.b1 = __ldg(p.c2_fp8 + (e >> 6));
                    in.s1 = __ldg(p.c1 + (e >> 14));
                }
            } else {
                if (!lane_ok) return;
                const int64_t e = static_cast<int64_t>(grow) * p.K + kb * kBK;
                in.c0 = ldg_nc_v4(p.codes + (e >> 1));
                in.c1v = ldg_nc_v4(p.codes + (e >> 1) + 16);
                in.b0 = __ldg(p.c2_fp8 + (e >> 6));
                in.s0 = __ldg(p.c1 + (e >> 14));
            }
        };
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u) issue(part + kParts * u, buf[u]);
        for (int i0 = 0; part + kParts * i0 < P.kb_total; i0 += kPrefetch) {
#pragma unroll
            for (int u = 0; u < kPrefetch; ++u) {
                const int kb = part + kParts * (i0 + u);
                if (kb >= P.kb_total) break;
                uint32_t v[32];
                if (kb < P.kb_w) {
                    if (kBwd)
                        convert_cols(buf[u], mu, lut, wsm, lane, v);
                    else
                        convert_row(buf[u], mu, lut, v);
                } else {
                    const int j0 = (kb - P.kb_w) * kBK;
                    if (kBwd) {  // A^T: lane = column k of A (r x K), in groups of 16 loads
#pragma unroll
                        for (int t = 0; t < 32; ++t) {
                            const int j = j0 + 2 * t;
                            const uint32_t a = (lane_ok && j < p.r) ? p.lora[static_cast<int64_t>(j) * p.K + grow] : 0u;
                            const uint32_t b =
                                (lane_ok && j + 1 < p.r) ? p.lora[static_cast<int64_t>(j + 1) * p.K + grow] : 0u;
                            v[t] = a | (b << 16);
                            if ((t & 7) == 7) asm volatile("" ::: "memory");  // bound loads in flight
                        }
                    } else {  // B: lane = row n of B (N x r)
                        const uint16_t* brow = p.lora + static_cast<int64_t>(grow) * p.r + j0;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            uint4 w = make_uint4(0u, 0u, 0u, 0u);
                            if (lane_ok && j0 + 8 * c < p.r) w = *reinterpret_cast<const uint4*>(brow + 8 * c);
                            v[4 * c + 0] = w.x;
                            v[4 * c + 1] = w.y;
                            v[4 * c + 2] = w.z;
                            v[4 * c + 3] = w.w;
                        }
                    }
                }
                if (!kBwd && !lane_ok) {
#pragma unroll
                    for (int t = 0; t < 32; ++t) v[t] = 0u;
                }
                issue(kb + kParts * kPrefetch, buf[u]);
                const uint32_t g = g0 + static_cast<uint32_t>(kb);
                const int s = static_cast<int>(g % kStages);
                const uint32_t ph = (g / kStages) & 1u;
                if (!warp_wait(P.empty(s), ph ^ 1u, err, lane)) return;
                tmem_st_32x32b_x32(P.tmem + lane_base + kAccCols + s * kAStageCols, v);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(P.full_a(s));
            }
        }
        // epilogue: this warp's lane quarter, columns [64 part, 64 part + 64)
        if (!warp_wait(P.acc_full(), tcount & 1u, err, lane)) return;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            const int col = part * 64 + c * 16;
            uint32_t acc[16];
            tmem_ld_32x32b_x16(P.tmem + lane_base + col, acc);
            tmem_wait_ld();
            if (c == 3) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(P.acc_empty());
            }
            if (lane_ok) {
                uint16_t* o = p.out + static_cast<int64_t>(t0 + col) * p.rows + grow;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (t0 + col + j < p.M) o[static_cast<int64_t>(j) * p.rows] = f32_to_bf16_bits(__uint_as_float(acc[j]));
            }
        }
    }
}

template <bool kBwd>
__global__ void __launch_bounds__(kThreads, 1)
k_nf4_gemm_tc(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_lora,
              const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ float s_lut[16];  // static, so table reads use an immediate address
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kXStageBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 2);
    uint32_t* stage_words = reinterpret_cast<uint32_t*>(smem + kStages * kXStageBytes + 1024);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    Pipe P;
    P.sA = smem;
    P.bar0 = smem_u32(bars);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(P.full_b(s), 1);
            mbar_init(P.full_a(s), 4);  // one converting warp per TMEM lane quarter
            mbar_init(P.empty(s), 1);
        }
        mbar_init(P.acc_full(), 1);
        mbar_init(P.acc_empty(), kDqWarps);
        fence_barrier_init();
    }
    if (threadIdx.x < 16) s_lut[threadIdx.x] = p.q[threadIdx.x];
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&tmap_act);
        tma_prefetch_desc(&tmap_lora);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    P.tmem = *tmem_slot;
    P.num_t = (p.M + kTileT - 1) / kTileT;
    P.num_tiles = P.num_t * ((p.rows + kTileW - 1) / kTileW);
    P.kb_w = (p.ctr + kBK - 1) / kBK;
    P.kb_total = P.kb_w + (p.r + kBK - 1) / kBK;
    int* err = &g_tc_error;

    if (warp == 0) {
        if (lane == 0) role_tma(P, &tmap_act, &tmap_lora, err);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) role_mma(P, err);
        __syncwarp();
    } else {
        role_dequant_epilogue<kBwd>(P, p, s_lut, stage_words + (warp - 2) * kStageWords, warp, lane, err);
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

template <bool kBwd>
cudaError_t launch_tc(const uint16_t* act, const Nf4Weight& w, const uint16_t* lora_act,
                      const uint16_t* lora_w, int64_t M, int r, uint16_t* out, cudaStream_t st) {
    const int64_t ctr = kBwd ? w.N : w.K;
    const int64_t rows = kBwd ? w.K : w.N;
    CUtensorMap ma, ml;
    if (!make_map_bf16(&ma, act, static_cast<uint64_t>(ctr), static_cast<uint64_t>(M), kBK, kTileT) ||
        !make_map_bf16(&ml, lora_act, static_cast<uint64_t>(r), static_cast<uint64_t>(M), kBK, kTileT))
        return cudaErrorInvalidValue;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(k_nf4_gemm_tc<kBwd>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    GemmParams p;
    p.codes = w.codes;
    p.c2_fp8 = w.c2_fp8;
    p.c1 = w.c1;
    p.mean = w.mean;
    p.lora = lora_w;
    p.out = out;
    p.M = static_cast<int>(M);
    p.rows = static_cast<int>(rows);
    p.ctr = static_cast<int>(ctr);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.r = r;
    for (int i = 0; i < 16; ++i) p.q[i] = tables().q[i];
    const int64_t tiles = ceil_div(M, kTileT) * ceil_div(rows, kTileW);
    const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
    k_nf4_gemm_tc<kBwd><<<grid, kThreads, kSmemBytes, st>>>(ma, ml, p);
    note_launches(1);
    return cudaGetLastError();
}

bool tc_common_ok(int64_t M, const Nf4Weight& w, int r) {
    return M >= 1 && w.K >= kBK && w.K % kBK == 0 && r % 8 == 0 && r >= 8 && M < (int64_t(1) << 31) &&
           w.N < (int64_t(1) << 31) && w.K < (int64_t(1) << 31) && encode_fn() != nullptr;
}

}  // namespace

bool fwd_tc_supported(int64_t M, const Nf4Weight& w, int r) { return tc_common_ok(M, w, r); }

// The dY tensor map needs a row stride that is a multiple of 16 bytes.
bool dx_tc_supported(int64_t M, const Nf4Weight& w, int r) { return tc_common_ok(M, w, r) && w.N % 8 == 0; }

cudaError_t launch_fwd_gemm_tc(const uint16_t* X, const Nf4Weight& w, const uint16_t* T, const uint16_t* B,
                               int64_t M, int r, uint16_t* Y, cudaStream_t st) {
    return launch_tc<false>(X, w, T, B, M, r, Y, st);
}

cudaError_t launch_bwd_dx_gemm_tc(const uint16_t* dY, const Nf4Weight& w, const uint16_t* U, const uint16_t* A,
                                  int64_t M, int r, uint16_t* dX, cudaStream_t st) {
    return launch_tc<true>(dY, w, U, A, M, r, dX, st);
}

}  // namespace qlora

namespace qlora {

int gemm_device_error(int reset) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    if (reset && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return v;
}

}  // namespace qlora
