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
//   forward:  D[n][m] += W'[n][k]   * X[m][k]     (contract over k)
//   backward: D[k][m] += W'^T[k][n] * dY[m][n]    (contract over n)
//
// so a dequantized tile goes from registers straight into tensor memory
// (tcgen05.st) and costs no shared-memory bandwidth; only the activation
// operand (X or dY) is staged in shared memory, by TMA in the 128-byte
// swizzled K-major layout.  The rank-r LoRA product is the same GEMM
// continued over ceil(r/64) extra 64-wide slabs whose A operand is B (or
// A^T) copied into tensor memory and whose B operand is T (or U) by TMA.
//
// The backward reads the weight through a transposed copy made per call by
// k_prep_bwd: codes of W^T (two consecutive n per byte), the block
// constants c2' in fp32 laid out [k/64][n], and A^T.  A lane then owns one
// weight column k and converts 64 consecutive contraction values from one
// 32-byte run of codes, exactly like the forward owns a row n.  The 64
// constants of a stage (one per row n, shared by the warp's 32 columns) are
// loaded two per lane with the codes and exchanged through a small
// warp-private shared buffer.
//
// Tile: 128 weight rows (n forward, k backward) x 2w tokens x 64, w = 128,
// 160, 176, 192 or 208 chosen per problem so the tiles fill the CTAs' rounds
// evenly: each dequantized weight stage feeds two 128 x w MMAs (two fp32
// accumulators, 2w TMEM columns), so the conversion work per FLOP is that
// of a 2w-token tile; 3 pipeline stages (A stages in TMEM after the
// accumulators).  The
// codes are expanded through a 64 KiB table that maps a code byte to both
// of its fp32 codebook values (one 8-byte copy per lane: no bank
// conflicts), so a pair of weights costs one byte permute, one shared load,
// two multiplies and one pack.  Warp
// roles (448
// threads, persistent over tiles, one CTA per SM):
//   warp 0        TMA producer for the activation tiles (and constants)
//   warp 1        MMA issuer (one thread)
//   warps 2..13   dequant producers: warp w converts the stages kb with
//                 kb % 3 == (w - 2) / 4 (always ring slot kb % 3) for the
//                 TMEM lane quarter w % 4, then
//                 the epilogue of the tile: tcgen05.ld, bf16, stores
//                 coalesced along the weight-row index
// Every wait is bounded; a timeout records QLORA_ERR_TIMEOUT in a sticky
// device word (qlora_device_error) and ends the kernel.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace qlora {

// Sticky device-side error word of the tensor-core kernels (0 = none).
__device__ int g_tc_error = 0;

namespace {

using namespace sm100;

constexpr int kTileW = 128;   // weight rows per tile (MMA M)
constexpr int kSubs = 2;      // MMAs per stage sharing one dequantized weight stage
constexpr int kBK = 64;       // contraction per stage
constexpr int kStages = 3;
constexpr int kAStageCols = kBK / 2;            // bf16 pairs per TMEM column
constexpr uint32_t kTmemCols = 512;
constexpr int kDqWarps = 12;                    // three per TMEM lane quarter
constexpr int kParts = kDqWarps / 4;            // stage kb is converted by the warps with part == kb % 3
static_assert(kParts == kStages, "a part's stages must always use the same ring slot");
constexpr int kPrefetchFwd = 2;                 // own stages of codes in flight per dequant thread
constexpr int kPrefetchBwd = 2;                 // (the backward also holds its constants)
constexpr int kThreads = 32 * (2 + kDqWarps);   // 448: 128 registers a thread
constexpr int kLutBytes = 256 * 256;             // code byte -> fp32 pair, one 8-byte copy per lane

// Token-tile geometry: a tile is kSubs MMAs of kSubT tokens that share every
// dequantized weight stage.  The launcher picks kSubT per problem so that
// the tiles fill the persistent CTAs' rounds evenly (a 384-token tile leaves
// a 4096-token, 4096-row product at 77% of its last round's slots).
template <int kSubT>
struct Geo {
    static constexpr int kTileT = kSubT * kSubs;          // tokens per tile
    static constexpr int kSubBytes = kSubT * kBK * 2;     // one MMA's activation tile
    static constexpr int kXStageBytes = kTileT * kBK * 2;
    static constexpr int kAccCols = kTileT;               // fp32 accumulator columns
    static constexpr int kChunks = kTileT / 16;           // epilogue chunks of 16 columns
    static constexpr int kLutOff = kStages * kXStageBytes + 1024 + kDqWarps * kBK * 4;
    static constexpr int kSmemBytes = 1024 /* align */ + kLutOff + kLutBytes;
    static_assert(kSubT % 16 == 0 && kSubT >= 64 && kSubT <= 256, "MMA N for M = 128");
    static_assert(kSubBytes % 1024 == 0, "128-byte swizzle atoms stay aligned");
    static_assert(kAccCols + kStages * kAStageCols <= static_cast<int>(kTmemCols), "TMEM budget");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(kChunks >= kDqWarps / 4, "every part stores at least one chunk");
};

struct GemmParams {
    const uint8_t* codes;  // forward: W codes (N x K/2); backward: W^T codes (K x ldT)
    const uint8_t* c2_fp8; // forward only
    const float* c1;       // forward only
    const float* mean;     // forward only
    const float* scalesT;  // backward only: c2' laid out [k/64][n], row stride ld_scales
    int64_t ld_scales;
    const uint16_t* lora;  // forward: B (N x r); backward: A^T (K x r)
    uint16_t* out;         // forward: Y (M x N); backward: dX (M x K)
    int64_t ld_codes;      // bytes per weight row of `codes`
    int M;                 // tokens
    int rows;              // weight rows of the product: N forward, K backward
    int ctr;               // contraction over the weight: K forward, N backward
    int K, r;
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
    uint8_t* sA;       // kStages activation stages of 2w tokens x 64 (two w-token halves)
    float* sS;         // backward: per dequant warp, 64 block constants
    uint32_t bar0;     // full_b[S], full_a[S], empty[S], acc_full, acc_empty
    uint32_t tmem;     // accumulators at columns [0, 2w), A stages after them
    int num_t, num_tiles, kb_w, kb_total;
    __device__ uint32_t full_b(int s) const { return bar0 + 8u * s; }
    __device__ uint32_t full_a(int s) const { return bar0 + 8u * (kStages + s); }
    __device__ uint32_t empty(int s) const { return bar0 + 8u * (2 * kStages + s); }
    __device__ uint32_t acc_full() const { return bar0 + 8u * (3 * kStages); }
    __device__ uint32_t acc_empty() const { return bar0 + 8u * (3 * kStages + 1); }
};

// Ring slot of contraction stage kb: slot kb % kStages, always, so the
// dequant warps of part p (the stages kb % kStages == p) own slot p for the
// whole kernel and no two parts ever wait on the same slot's barriers.
// Returns the slot's use count before this stage (tile tcount): its parity
// is the phase every role waits on.
__device__ __forceinline__ uint32_t slot_use(int kb, uint32_t tcount, int kb_total) {
    const int s = kb % kStages;
    const uint32_t uses_per_tile = static_cast<uint32_t>((kb_total - s + kStages - 1) / kStages);
    return tcount * uses_per_tile + static_cast<uint32_t>(kb / kStages);
}

// Token tile and weight-row tile of persistent tile index `tile`.  The
// forward walks the token tiles fastest (its activation X is shared by all
// weight tiles and stays in L2); the backward walks the weight tiles
// fastest, so the CTAs working at the same time share a few token tiles of
// dY (whose full size can exceed L2) while the small transposed weight is
// reused from L2.
template <bool kBwd, int kSubT>
__device__ __forceinline__ void tile_coords(const Pipe& P, int tile, int& t0, int& row0) {
    constexpr int kTileT = Geo<kSubT>::kTileT;
    if (kBwd) {
        const int num_w = P.num_tiles / P.num_t;
        t0 = (tile / num_w) * kTileT;
        row0 = (tile % num_w) * kTileW;
    } else {
        t0 = (tile % P.num_t) * kTileT;
        row0 = (tile / P.num_t) * kTileW;
    }
}

// warp 0, one thread: activation tiles, then the LoRA slabs, into the ring.
template <bool kBwd, int kSubT>
__device__ void role_tma(const Pipe& P, const CUtensorMap* tmap_act, const CUtensorMap* tmap_lora, int* err) {
    using G = Geo<kSubT>;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < P.num_tiles; tile += gridDim.x, ++tcount) {
        int t0, row0;
        tile_coords<kBwd, kSubT>(P, tile, t0, row0);
        for (int kb = 0; kb < P.kb_total; ++kb) {
            const int s = kb % kStages;
            const uint32_t ph = slot_use(kb, tcount, P.kb_total) & 1u;
            if (!mbar_wait(P.empty(s), ph ^ 1u, err)) return;
            const uint32_t dst = smem_u32(P.sA + s * G::kXStageBytes);
            if (kb < P.kb_w) {
                mbar_arrive_expect_tx(P.full_b(s), G::kXStageBytes);
                for (int sub = 0; sub < kSubs; ++sub)
                    tma_load_2d(dst + sub * G::kSubBytes, tmap_act, P.full_b(s), kb * kBK, t0 + sub * kSubT);
            } else {
                mbar_arrive_expect_tx(P.full_b(s), G::kXStageBytes);
                for (int sub = 0; sub < kSubs; ++sub)
                    tma_load_2d(dst + sub * G::kSubBytes, tmap_lora, P.full_b(s), (kb - P.kb_w) * kBK,
                                t0 + sub * kSubT);
            }
        }
    }
}

// warp 1, one thread: per stage, four 128 x w x 16 MMAs into each of the two
// accumulators, all reading the same weight stage in TMEM.
template <int kSubT>
__device__ void role_mma(const Pipe& P, int* err) {
    using G = Geo<kSubT>;
    constexpr uint32_t idesc = idesc_bf16(kTileW, kSubT);
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < P.num_tiles; tile += gridDim.x, ++tcount) {
        if (!mbar_wait(P.acc_empty(), (tcount & 1u) ^ 1u, err)) return;
        tc_fence_after();
        for (int kb = 0; kb < P.kb_total; ++kb) {
            const int s = kb % kStages;
            const uint32_t ph = slot_use(kb, tcount, P.kb_total) & 1u;
            if (!mbar_wait(P.full_b(s), ph, err)) return;
            if (!mbar_wait(P.full_a(s), ph, err)) return;
            tc_fence_after();
            const uint32_t a_col = P.tmem + G::kAccCols + s * kAStageCols;
#pragma unroll
            for (int sub = 0; sub < kSubs; ++sub) {
                const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(P.sA + s * G::kXStageBytes + sub * G::kSubBytes));
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    mma_bf16_ts(P.tmem + sub * kSubT, a_col + kk * 8, bdesc + static_cast<uint64_t>(kk * 2), idesc,
                                (kb | kk) != 0);
            }
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

// The two codebook values of one code byte, (q[high nibble], q[low nibble]),
// from the lane's own copy of the 256-entry table: entry b, lane l at byte
// 256 b + 8 l, so a warp's reads never share a bank; the byte and the lane
// offset form the address in one byte permute.
__device__ __forceinline__ float2 lut_pair(const uint8_t* lut, uint32_t word, uint32_t lane_off, int byte) {
    const uint32_t addr = __byte_perm(word, lane_off, 0x5504u | (static_cast<uint32_t>(byte) << 4));
    return *reinterpret_cast<const float2*>(lut + addr);
}

// 64 contraction values of one weight row (forward) or column (backward):
// 32 code bytes, the high nibble of each byte the even element, which lands
// in the low half of its TMEM column.  The block constant is one value for
// the whole run (forward) or one per contraction value (backward, read from
// shared memory).
template <bool kPerElem>
__device__ __forceinline__ void convert_run(const uint4& c0, const uint4& c1, float sc, const float* sp,
                                            const uint8_t* lut, uint32_t lane_off, uint32_t (&v)[32]) {
    const uint32_t w8[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int h = 0; h < 8; ++h) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 q2 = lut_pair(lut, w8[h], lane_off, j);
            // backward: the constants of contraction values 8h + 2j, 8h + 2j + 1
            const float2 s2 = kPerElem ? *reinterpret_cast<const float2*>(sp + 8 * h + 2 * j) : make_float2(sc, sc);
            v[4 * h + j] = pack_bf16x2(__fmul_rn(q2.x, s2.x), __fmul_rn(q2.y, s2.y));
        }
    }
}

// A position in one part's sequence of stages over all of this CTA's
// tiles: the stages kb == part (mod 3) of tile 0, then of tile 1, ...
struct Cursor {
    int tile;         // persistent tile index (>= num_tiles: past the end)
    uint32_t tcount;  // tiles of this CTA before it
    int kb;           // contraction stage
    int t0, row0;     // the tile's first token and first weight row
};

template <bool kBwd, int kSubT>
__device__ __forceinline__ void cursor_start(Cursor& c, const Pipe& P, int part) {
    c.tile = blockIdx.x;
    c.tcount = 0;
    c.kb = part;
    tile_coords<kBwd, kSubT>(P, c.tile, c.t0, c.row0);
}

template <bool kBwd, int kSubT>
__device__ __forceinline__ void cursor_next(Cursor& c, const Pipe& P, int part) {
    c.kb += kParts;
    if (c.kb >= P.kb_total) {
        c.kb = part;
        c.tile += gridDim.x;
        ++c.tcount;
        if (c.tile < P.num_tiles) tile_coords<kBwd, kSubT>(P, c.tile, c.t0, c.row0);
    }
}

// Epilogue of this CTA's tile number tcount (first token t0, first weight
// row row0): this warp's lane quarter, the 16-column chunks part, part + 3,
// part + 6, ...; the accumulator is released after the warp's last load.
template <int kSubT>
__device__ __forceinline__ void tile_epilogue(const Pipe& P, const GemmParams& p, uint32_t tcount, int t0,
                                              int row0, int part, int row, uint32_t lane_base, int lane,
                                              int* err, bool& ok) {
    using G = Geo<kSubT>;
    if (!warp_wait(P.acc_full(), tcount & 1u, err, lane)) {
        ok = false;
        return;
    }
    tc_fence_after();
    const int grow = row0 + row;
    const bool lane_ok = grow < p.rows;
#pragma unroll 1
    for (int c = part; c < G::kChunks; c += kParts) {
        const int col = c * 16;
        uint32_t acc[16];
        tmem_ld_32x32b_x16(P.tmem + lane_base + col, acc);
        tmem_wait_ld();
        if (c + kParts >= G::kChunks) {  // this warp's last chunk
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

// warps 2..13: each converts every third stage of the weight tiles into
// TMEM (quarter = its TMEM lanes, part = which stages) and writes a third
// of each tile's outputs for its lane quarter.  The stages form one stream
// over all of the CTA's tiles (the codes of the next tile are loaded while
// the current one ends), and a tile's epilogue runs after the warp has
// stored its first stage of the next tile, so the MMAs of the next tile
// find their first stages ready once the accumulator is free.
template <bool kBwd, int kSubT>
__device__ __forceinline__ void role_dequant_epilogue(const Pipe& P, const GemmParams& p, const uint8_t* lut,
                                                      float* wsc, int warp, int lane, int* err) {
    const uint32_t lane_off = static_cast<uint32_t>(lane) * 8;
    const int dq = warp - 2;
    const int quarter = warp & 3;  // the TMEM lanes this warp may touch
    const int part = dq >> 2;      // converts the stages kb with kb % 3 == part
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float mu = kBwd ? 0.0f : *p.mean;
    bool ok = true;

    if (part >= P.kb_total) {  // no stages for this part: epilogues only
        uint32_t tcount = 0;
        for (int tile = blockIdx.x; tile < P.num_tiles && ok; tile += gridDim.x, ++tcount) {
            int t0, row0;
            tile_coords<kBwd, kSubT>(P, tile, t0, row0);
            tile_epilogue<kSubT>(P, p, tcount, t0, row0, part, row, lane_base, lane, err, ok);
        }
        return;
    }

    // codes (and, forward, the block constant's inputs) of the next
    // kPrefetch own stages; the constant itself is formed at use so the
    // loads stay in flight
    constexpr int kPrefetch = kBwd ? kPrefetchBwd : kPrefetchFwd;
    uint4 cb0[kPrefetch], cb1[kPrefetch];
    uint32_t sbyte[kPrefetch];
    float sc1[kPrefetch];
    float2 s2[kPrefetch];  // backward: constants of rows 2 lane, 2 lane + 1 of the stage
    auto issue = [&](const Cursor& c, int u) {
        cb0[u] = make_uint4(0u, 0u, 0u, 0u);
        cb1[u] = cb0[u];
        sbyte[u] = 0u;
        sc1[u] = 0.0f;
        s2[u] = make_float2(0.0f, 0.0f);
        if (c.tile >= P.num_tiles || c.kb >= P.kb_w) return;
        const int grow = c.row0 + row;
        if (kBwd && (c.row0 + quarter * 32) < p.rows) {
            // this warp's 32 columns lie in one 64-wide block group
            const float* srow = p.scalesT + static_cast<int64_t>((c.row0 + quarter * 32) / kBK) * p.ld_scales;
            s2[u] = __ldg(reinterpret_cast<const float2*>(srow + c.kb * kBK) + lane);
        }
        if (grow >= p.rows) return;
        const uint8_t* crow = p.codes + static_cast<int64_t>(grow) * p.ld_codes;
        cb0[u] = ldg_nc_v4(crow + c.kb * (kBK / 2));
        cb1[u] = ldg_nc_v4(crow + c.kb * (kBK / 2) + 16);
        if (!kBwd) {
            const int64_t blk = static_cast<int64_t>(grow) * (p.K / kBK) + c.kb;
            sbyte[u] = __ldg(p.c2_fp8 + blk);
            sc1[u] = __ldg(p.c1 + (blk >> 8));
        }
    };

    Cursor ci, cc;  // the next stage to load, the next stage to convert
    cursor_start<kBwd, kSubT>(ci, P, part);
    cursor_start<kBwd, kSubT>(cc, P, part);
#pragma unroll
    for (int u = 0; u < kPrefetch; ++u) {
        issue(ci, u);
        cursor_next<kBwd, kSubT>(ci, P, part);
    }
    int prev_t0 = 0, prev_row0 = 0;  // the tile whose epilogue is pending
    while (cc.tile < P.num_tiles) {
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u) {
            if (cc.tile >= P.num_tiles) break;
            const int kb = cc.kb;
            const int s = part;  // == kb % kStages
            const uint32_t ph = slot_use(kb, cc.tcount, P.kb_total) & 1u;
            const int grow = cc.row0 + row;  // this lane's weight row of the product
            uint32_t v[32];
            if (kb < P.kb_w) {
                if (kBwd) {
                    reinterpret_cast<float2*>(wsc)[lane] = s2[u];
                    __syncwarp();
                }
                const float sc = kBwd ? 0.0f : dq_constant(static_cast<uint8_t>(sbyte[u]), sc1[u], mu);
                // rows beyond the weight hold finite garbage (zero codes times
                // the constant of empty inputs): their outputs are never
                // stored and rows do not mix in this product
                convert_run<kBwd>(cb0[u], cb1[u], sc, wsc, lut, lane_off, v);
                if (kBwd) __syncwarp();  // wsc is rewritten by the warp's next stage
            } else {  // LoRA slab: lane = row of B (forward) or of A^T (backward), r contiguous
                const int j0 = (kb - P.kb_w) * kBK;
                const uint16_t* lrow = p.lora + static_cast<int64_t>(grow) * p.r + j0;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 w = make_uint4(0u, 0u, 0u, 0u);
                    if (grow < p.rows && j0 + 8 * c < p.r) w = *reinterpret_cast<const uint4*>(lrow + 8 * c);
                    v[4 * c + 0] = w.x;
                    v[4 * c + 1] = w.y;
                    v[4 * c + 2] = w.z;
                    v[4 * c + 3] = w.w;
                }
            }
            issue(ci, u);
            cursor_next<kBwd, kSubT>(ci, P, part);
            if (!warp_wait(P.empty(s), ph ^ 1u, err, lane)) return;
            tmem_st_32x32b_x32(P.tmem + lane_base + Geo<kSubT>::kAccCols + s * kAStageCols, v);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(P.full_a(s));
            if (kb == part && cc.tcount > 0) {  // first own stage of a tile: end the previous one
                tile_epilogue<kSubT>(P, p, cc.tcount - 1, prev_t0, prev_row0, part, row, lane_base, lane, err, ok);
                if (!ok) return;
            }
            prev_t0 = cc.t0;
            prev_row0 = cc.row0;
            cursor_next<kBwd, kSubT>(cc, P, part);
        }
    }
    // the CTA's last tile
    tile_epilogue<kSubT>(P, p, cc.tcount - 1, prev_t0, prev_row0, part, row, lane_base, lane, err, ok);
}

template <bool kBwd, int kSubT>
__global__ void __launch_bounds__(kThreads, 1)
k_nf4_gemm_tc(const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_lora,
              const __grid_constant__ GemmParams p) {
    using G = Geo<kSubT>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, derived by pointer arithmetic so that every
    // access below stays a (32-bit) shared-memory access
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * G::kXStageBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    Pipe P;
    P.sA = smem;
    P.sS = reinterpret_cast<float*>(smem + kStages * G::kXStageBytes + 1024);
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
    uint8_t* lut = smem + G::kLutOff;
    for (int i = threadIdx.x; i < 256 * 32; i += kThreads)
        reinterpret_cast<float2*>(lut)[i] = make_float2(p.q[i >> 9], p.q[(i >> 5) & 15]);
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
    P.num_t = (p.M + G::kTileT - 1) / G::kTileT;
    P.num_tiles = P.num_t * ((p.rows + kTileW - 1) / kTileW);
    P.kb_w = (p.ctr + kBK - 1) / kBK;
    P.kb_total = P.kb_w + (p.r + kBK - 1) / kBK;
    int* err = &g_tc_error;

    if (warp == 0) {
        if (lane == 0) role_tma<kBwd, kSubT>(P, &tmap_act, &tmap_lora, err);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) role_mma<kSubT>(P, err);
        __syncwarp();
    } else {
        role_dequant_epilogue<kBwd, kSubT>(P, p, lut, P.sS + (warp - 2) * kBK, warp, lane, err);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(P.tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------
// k_prep_bwd: the transposed weight the backward reads.
//   codesT[k][j]  = (code(W[2j][k]) << 4) | code(W[2j+1][k])   (K x ldT bytes)
//   scalesT[g][n] = c2' of the block holding W[n][64g .. 64g+63] (K/64 x ldS)
//   AT[k][j]      = A[j][k]                                     (K x r)
// One CTA per 64 x 256 weight tile (64 rows n, up to 256 columns k; plus
// CTAs for A^T); padding is zero.  A thread loads 32 bytes of one row n
// (two 16-byte loads), then builds the 32 bytes of one row k of W^T from
// shared memory and stores them as two 16-byte stores.
constexpr int kPrepThreads = 256;
constexpr int kPrepK = 256;  // weight columns per CTA

__global__ void __launch_bounds__(kPrepThreads)
k_prep_bwd(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ c2_fp8, const float* __restrict__ c1,
           const float* __restrict__ mean, const uint16_t* __restrict__ A, int N, int K, int r, int64_t ldT,
           int64_t ldS, uint8_t* __restrict__ codesT, float* __restrict__ scalesT, uint16_t* __restrict__ AT,
           int weight_tiles) {
    __shared__ __align__(16) uint8_t tile[64][kPrepK / 2];
    __shared__ uint16_t at[64][65];
    const int t = threadIdx.x;
    const int npad_tiles = static_cast<int>(ldS / 64);
    if (static_cast<int>(blockIdx.x) < weight_tiles) {
        const int nt = blockIdx.x % npad_tiles, kq = blockIdx.x / npad_tiles;
        const int n0 = nt * 64, k0 = kq * kPrepK;
        const int kspan = min(kPrepK, K - k0);  // a multiple of 64
        {   // rows n0 .. n0 + 63, bytes k0/2 .. (k0 + kspan)/2 of the codes (zero beyond N)
            const int rr = t >> 2, cc = (t & 3) * 32;
            uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
            if (n0 + rr < N && 2 * cc < kspan) {
                const uint8_t* src = codes + static_cast<int64_t>(n0 + rr) * (K / 2) + k0 / 2 + cc;
                v0 = *reinterpret_cast<const uint4*>(src);
                v1 = *reinterpret_cast<const uint4*>(src + 16);
            }
            *reinterpret_cast<uint4*>(&tile[rr][cc]) = v0;
            *reinterpret_cast<uint4*>(&tile[rr][cc + 16]) = v1;
        }
        {   // the constants of the (up to) four 64-blocks of each row
            const int n = n0 + (t & 63), g = t >> 6;
            if (64 * g < kspan) {
                const int kt = k0 / 64 + g;
                float c = 0.0f;
                if (n < N) {
                    const int64_t blk = static_cast<int64_t>(n) * (K / 64) + kt;
                    c = dq_constant(c2_fp8[blk], c1[blk >> 8], *mean);
                }
                scalesT[static_cast<int64_t>(kt) * ldS + n] = c;
            }
        }
        __syncthreads();
        if (t < kspan) {  // row k0 + t of W^T: 32 bytes, each two consecutive n
            const int col = t >> 1;
            const int shift = (t & 1) ? 0 : 4;  // even k: the high nibble
            uint32_t out[8];
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                uint32_t acc = 0u;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int j = 4 * w + b;
                    const uint32_t ne = (tile[2 * j][col] >> shift) & 15u;
                    const uint32_t no = (tile[2 * j + 1][col] >> shift) & 15u;
                    acc |= ((ne << 4) | no) << (8 * b);
                }
                out[w] = acc;
            }
            uint8_t* dst = codesT + static_cast<int64_t>(k0 + t) * ldT + n0 / 2;
            *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
            *reinterpret_cast<uint4*>(dst + 16) = make_uint4(out[4], out[5], out[6], out[7]);
        }
    } else {
        const int kt = blockIdx.x - weight_tiles;  // 64 columns of A
        const int k0 = kt * 64;
        for (int j0 = 0; j0 < r; j0 += 64) {
            for (int i = t; i < 64 * 64; i += kPrepThreads) {
                const int jj = i >> 6, kk = i & 63;
                at[jj][kk] = (j0 + jj < r && k0 + kk < K) ? A[static_cast<int64_t>(j0 + jj) * K + k0 + kk] : 0;
            }
            __syncthreads();
            for (int i = t; i < 64 * 64; i += kPrepThreads) {
                const int kk = i >> 6, jj = i & 63;
                if (j0 + jj < r && k0 + kk < K) AT[static_cast<int64_t>(k0 + kk) * r + j0 + jj] = at[jj][kk];
            }
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() { return tensor_map_encoder(); }

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

template <bool kBwd, int kSubT>
cudaError_t launch_tc_geo(const uint16_t* act, const uint16_t* lora_act, const GemmParams& p0, int grid,
                          cudaStream_t st) {
    using G = Geo<kSubT>;
    CUtensorMap ma, ml;
    if (!make_map_bf16(&ma, act, static_cast<uint64_t>(p0.ctr), static_cast<uint64_t>(p0.M), kBK, kSubT) ||
        !make_map_bf16(&ml, lora_act, static_cast<uint64_t>(p0.r), static_cast<uint64_t>(p0.M), kBK, kSubT))
        return cudaErrorInvalidValue;
    static ContextMemo<int> attr_memo;
    const cudaError_t attr_err = ensure_smem_limit(attr_memo, k_nf4_gemm_tc<kBwd, kSubT>, G::kSmemBytes);
    if (attr_err != cudaSuccess) return attr_err;
    GemmParams p = p0;
    for (int i = 0; i < 16; ++i) p.q[i] = tables().q[i];
    k_nf4_gemm_tc<kBwd, kSubT><<<grid, kThreads, G::kSmemBytes, st>>>(ma, ml, p);
    note_launches(1);
    return cudaGetLastError();
}

// MMA widths the launcher chooses from (tokens per tile = 2 x width).
constexpr int kSubChoices[] = {128, 160, 176, 192, 208};

// The width whose tiles finish soonest on `sms` persistent CTAs: rounds
// (tiles per CTA, rounded up) times the time of one tile.  A 128-row MMA
// instruction costs about the same issue time whatever its width up to 256
// (measured on B200: 187 cycles per instruction with two accumulators in
// turn, for widths 64 to 256), so a tile's time is mostly a fixed cost per
// 64-wide stage: measured, about 790 tokens' worth of width-proportional
// time.  Ties go to the wider tile.
int pick_sub(int64_t M, int64_t rows, int64_t sms) {
    int best = kSubChoices[0];
    int64_t best_cost = -1;
    for (int sub : kSubChoices) {
        const int64_t tiles = ceil_div(M, 2 * sub) * ceil_div(rows, kTileW);
        const int64_t rounds = ceil_div(tiles, sms);
        const int64_t cost = rounds * (2 * sub + 790);
        if (best_cost < 0 || cost <= best_cost) {
            best = sub;
            best_cost = cost;
        }
    }
    return best;
}

template <bool kBwd>
cudaError_t launch_tc(const uint16_t* act, const uint16_t* lora_act, const GemmParams& p0, cudaStream_t st) {
    const int64_t sms = num_sms();
    const int sub = pick_sub(p0.M, p0.rows, sms);
    const int64_t tiles = ceil_div(static_cast<int64_t>(p0.M), 2 * sub) * ceil_div(static_cast<int64_t>(p0.rows), kTileW);
    const int grid = static_cast<int>(tiles < sms ? tiles : sms);
    switch (sub) {
        case 128: return launch_tc_geo<kBwd, 128>(act, lora_act, p0, grid, st);
        case 160: return launch_tc_geo<kBwd, 160>(act, lora_act, p0, grid, st);
        case 176: return launch_tc_geo<kBwd, 176>(act, lora_act, p0, grid, st);
        case 192: return launch_tc_geo<kBwd, 192>(act, lora_act, p0, grid, st);
        default: return launch_tc_geo<kBwd, 208>(act, lora_act, p0, grid, st);
    }
}

bool tc_common_ok(int64_t M, const Nf4Weight& w, int r) {
    return M >= 1 && w.K >= kBK && w.K % kBK == 0 && r % 8 == 0 && r >= 8 && M < (int64_t(1) << 31) &&
           w.N < (int64_t(1) << 31) && w.K < (int64_t(1) << 31) && encode_fn() != nullptr;
}

int64_t ld_codesT(const Nf4Weight& w) { return round_up(w.N, 64) / 2; }
int64_t ld_scalesT(const Nf4Weight& w) { return round_up(w.N, 64); }

}  // namespace

bool fwd_tc_supported(int64_t M, const Nf4Weight& w, int r) { return tc_common_ok(M, w, r); }

// The dY tensor map needs a row stride that is a multiple of 16 bytes.
bool dx_tc_supported(int64_t M, const Nf4Weight& w, int r) { return tc_common_ok(M, w, r) && w.N % 8 == 0; }

size_t dx_tc_workspace(const Nf4Weight& w, int r) {
    const size_t a = static_cast<size_t>(w.K) * ld_codesT(w);
    const size_t b = static_cast<size_t>(w.K / kBK) * ld_scalesT(w) * 4;
    const size_t c = static_cast<size_t>(w.K) * r * 2;
    return round_up(a, 256) + round_up(b, 256) + round_up(c, 256);
}

cudaError_t launch_fwd_gemm_tc(const uint16_t* X, const Nf4Weight& w, const uint16_t* T, const uint16_t* B,
                               int64_t M, int r, uint16_t* Y, cudaStream_t st) {
    GemmParams p{};
    p.codes = w.codes;
    p.c2_fp8 = w.c2_fp8;
    p.c1 = w.c1;
    p.mean = w.mean;
    p.lora = B;
    p.out = Y;
    p.ld_codes = w.K / 2;
    p.M = static_cast<int>(M);
    p.rows = static_cast<int>(w.N);
    p.ctr = static_cast<int>(w.K);
    p.K = static_cast<int>(w.K);
    p.r = r;
    return launch_tc<false>(X, T, p, st);
}

cudaError_t launch_bwd_dx_gemm_tc(const uint16_t* dY, const Nf4Weight& w, const uint16_t* U, const uint16_t* A,
                                  int64_t M, int r, uint16_t* dX, void* ws, cudaStream_t st) {
    const int64_t ldT = ld_codesT(w), ldS = ld_scalesT(w);
    uint8_t* codesT = reinterpret_cast<uint8_t*>(ws);
    float* scalesT = reinterpret_cast<float*>(codesT + round_up(static_cast<size_t>(w.K) * ldT, 256));
    uint16_t* AT = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(scalesT) +
                                               round_up(static_cast<size_t>(w.K / kBK) * ldS * 4, 256));
    const int weight_tiles = static_cast<int>((ldS / 64) * ceil_div(w.K, kPrepK));
    const int a_tiles = static_cast<int>(ceil_div(w.K, 64));
    k_prep_bwd<<<weight_tiles + a_tiles, kPrepThreads, 0, st>>>(w.codes, w.c2_fp8, w.c1, w.mean, A,
                                                                static_cast<int>(w.N), static_cast<int>(w.K), r,
                                                                ldT, ldS, codesT, scalesT, AT, weight_tiles);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    GemmParams p{};
    p.codes = codesT;
    p.scalesT = scalesT;
    p.ld_scales = ldS;
    p.lora = AT;
    p.out = dX;
    p.ld_codes = ldT;
    p.M = static_cast<int>(M);
    p.rows = static_cast<int>(w.K);
    p.ctr = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.r = r;
    return launch_tc<true>(dY, U, p, st);
}

// The failure-detection self-test: one thread waits, with the given limit,
// for a phase of an mbarrier that nothing ever arrives on.  No copy or MMA
// is in flight, so when the limit passes the wait records QLORA_ERR_TIMEOUT
// in the sticky word and the kernel simply returns.
__global__ void k_wait_selftest(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(sm100::smem_u32(&bar), 1);
        sm100::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) sm100::mbar_wait(sm100::smem_u32(&bar), 0u, &g_tc_error, limit_ns);
    __syncthreads();
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st) {
    k_wait_selftest<<<1, 32, 0, st>>>(limit_ns);
    note_launches(1);
    return cudaGetLastError();
}

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
