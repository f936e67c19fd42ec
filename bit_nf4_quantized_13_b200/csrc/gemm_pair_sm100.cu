// gemm_pair_sm100.cu -- the two frozen-weight GEMMs of the QLoRA linear on
// pairs of SMs (QLoRA study notes, gitcode.csdn.net, section 3.5 eq. 5 and
// 6, section 4 eq. 3, and the gradient through the bf16 weight of 3.5):
//
//   forward:  Y  = X  W'^T + T B^T     T = bf16(s X A^T)      (M x N)
//   backward: dX = dY W'   + U A       U = bf16(s dY B)       (M x K)
//   W' = bf16(q[code] * c2'), double-dequantized on the fly, never stored.
//
// Both compute the transposed product tile by tile with the weight as the
// MMA's A operand:
//
//   forward:  D[n][m] += W'[n][k]   * X[m][k]     (contract over k)
//   backward: D[k][m] += W'^T[k][n] * dY[m][n]    (contract over n)
//
// A tile is 256 weight rows x 512 tokens, computed by a pair of CTAs on two
// SMs with tcgen05.mma.cta_group::2 (M = 256, N = 256): each CTA holds 128
// of the weight rows (its half of A, converted from NF4 by its own warps
// into its shared memory) and two fp32 accumulators of 128 rows x 256 tokens
// in tensor memory (all 512 columns); each accumulator's 256 tokens are
// staged half in each CTA (B, by TMA in the 128-byte swizzled K-major
// layout), so every MMA instruction is the full 128 x 256 x 16 per SM.
//
// The converted weight is written into shared memory in the 128-byte
// swizzled layout the tensor cores read: K-major in the forward (a row n
// holds 64 consecutive k), MN-major in the backward (a row holds 64
// consecutive k of one contraction index n, two 64-wide blocks per CTA).
// Both read the NF4 codes in their natural row-major layout (a 64-weight
// run of one row shares one block constant), so the backward needs no
// transposed copy of the weight.  The rank-r LoRA term continues the same
// contraction over ceil(r/64) extra 64-wide slabs whose A operand (B
// forward, A^T backward) and B operand (T forward, U backward) both come
// by TMA.
//
// Codes are expanded without a table in memory: each 64-weight run forms
// its block's 16 possible bf16 values in registers and picks four weights
// at a time with byte permutes (convert_run), so the conversion adds no
// shared-memory traffic beside the converted tile itself.
//
// Warp roles (576 threads per CTA, persistent over the pair's tiles):
//   warp 0      TMA producer (both CTAs, into their own shared memory; the
//               completion bytes count on the even CTA's barrier)
//   warp 1      MMA issuer (one thread of the even CTA only)
//   warps 2-17  converters: warp w handles the stages kb with kb % 4 ==
//               (w - 2) / 4 (always ring slot kb % 4), 32 of the stage's 128
//               64-weight runs; then the epilogue of its TMEM lane quarter
//               w % 4: tcgen05.ld, bf16, stores coalesced along the
//               weight-row index.
// Every wait is bounded; a timeout records QLORA_ERR_TIMEOUT in a sticky
// device word and ends the role.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace qlora {

__device__ int g_pair_error = 0;  // sticky: QLORA_ERR_TIMEOUT if a wait gave up

namespace {

using namespace sm100;

constexpr int kRowsCta = 128;                       // weight rows per CTA
constexpr int kRowsPair = 2 * kRowsCta;             // MMA M
constexpr int kSubTok = 256;                        // MMA N: tokens per accumulator
constexpr int kSubs = 2;                            // accumulators
constexpr int kTileTok = kSubs * kSubTok;           // tokens per tile
constexpr int kHalfTok = kSubTok / 2;               // one accumulator's tokens staged by one CTA
constexpr int kBK = 64;                             // contraction per stage
constexpr int kStages = 4;
constexpr int kABytes = kRowsCta * kBK * 2;         // 16 KiB
constexpr int kBHalfBytes = kHalfTok * kBK * 2;     // 16 KiB
constexpr int kStageBytes = kABytes + kSubs * kBHalfBytes;
constexpr int kDqWarps = 16;
constexpr int kParts = kDqWarps / 4;
static_assert(kParts == kStages, "a part's stages must always use the same ring slot");
constexpr int kThreads = 32 * (2 + kDqWarps);       // 576: 112 registers a thread
constexpr uint32_t kTmemCols = 512;
constexpr int kChunks = kSubs * kSubTok / 16;       // epilogue chunks of 16 columns
constexpr int kBarOff = kStages * kStageBytes;
constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOff + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
constexpr uint16_t kPairMask = 0x3;                 // both CTAs of the cluster
// completion bytes of one stage over the pair: B halves of both CTAs, plus
// (LoRA slabs) the A operand of both CTAs
constexpr uint32_t kTxWeight = 2u * kSubs * kBHalfBytes;
constexpr uint32_t kTxLora = kTxWeight + 2u * kABytes;
// a split tile's partial sums: fp32, [CTA][chunk][row][16 columns], so each
// lane stores and loads 64 contiguous bytes per chunk
constexpr int kSlotFloats = kRowsPair * kTileTok;
constexpr int kFlagCount = 2 * kDqWarps;            // warps of both CTAs that store a slot
constexpr int kMinStagesPerPair = 8;

constexpr int kMaxGroups = 4;  // linears sharing one input, stacked along N

struct PairParams {
    // the frozen weights: G linears stacked along N (rows gstart[g] ..
    // gstart[g+1] - 1 of the product belong to linear g), each its own four
    // NF4 buffers (codes N_g x K/2 row-major, two k per byte; N_g x K/64
    // FP8 constants; c1; mean)
    const uint8_t* codes[kMaxGroups];
    const uint8_t* c2_fp8[kMaxGroups];
    const float* c1[kMaxGroups];
    const float* mean[kMaxGroups];
    int gstart[kMaxGroups + 1];
    int G;
    int r_lora_off;         // forward: T columns of linear g start at g * r_lora_off
    uint16_t* out;          // forward: Y (M x N); backward: dX (M x K)
    int M;                  // tokens
    int rows;               // output rows of the product: N forward, K backward
    int ctr;                // contraction over the weight: K forward, N backward
    int N, K, r;
    int kb_w;               // weight stages: ceil(ctr / 64)
    int kb_total;           // + LoRA slabs
    int num_t;              // token tiles
    int num_tiles;          // tiles (pair units)
    int64_t iters;          // num_tiles * kb_total
    int split_tail;         // share the last round's stages over all pairs (else whole tiles only)
    float* partial;         // split tiles: one slot of kSlotFloats per pair
    int* flags;             // per pair: warps that have stored its slot
    float q[16];
};

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// The linear holding row n of the stacked weights.
__device__ __forceinline__ int group_of(const PairParams& p, int64_t n) {
    int g = 0;
#pragma unroll
    for (int i = 1; i < kMaxGroups; ++i)
        if (i < p.G && n >= p.gstart[i]) g = i;
    return g;
}

struct Pipe {
    uint32_t smem;      // shared address of stage 0; stage s at + s * kStageBytes: A (16 KiB), then the B halves
    uint32_t bar0;      // full_b[S], full_a[S], empty[S], acc_full, acc_empty, drain (this CTA)
    uint32_t tmem;
    uint32_t rank;      // 0: the even CTA (issues the MMAs), 1: its peer
    int pair, num_pairs;
    __device__ uint32_t full_b(int s) const { return bar0 + 8u * s; }
    __device__ uint32_t full_a(int s) const { return bar0 + 8u * (kStages + s); }
    __device__ uint32_t empty(int s) const { return bar0 + 8u * (2 * kStages + s); }
    __device__ uint32_t acc_full() const { return bar0 + 8u * (3 * kStages); }
    __device__ uint32_t acc_empty() const { return bar0 + 8u * (3 * kStages + 1); }
    __device__ uint32_t drain() const { return bar0 + 8u * (3 * kStages + 2); }
    __device__ uint32_t sA(int s) const { return smem + static_cast<uint32_t>(s * kStageBytes); }
    __device__ uint32_t sB(int s, int sub) const { return sA(s) + kABytes + sub * kBHalfBytes; }
};

// First token and first weight row (of the pair) of tile `tile`.  The
// forward takes the weight rows in bands of kBand row tiles and, inside a
// band, the token tiles slowest: the pairs working at the same time then
// cover a compact block of a few token tiles of X and a few weight row
// tiles, which stays in L2 even when X does not.  The backward walks the
// weight tiles fastest, so the pairs working at the same time share a few
// token tiles of dY while the weight's codes are reused from L2.
constexpr int kBand = 8;

template <bool kBwd>
__device__ __forceinline__ void tile_coords(const PairParams& p, int tile, int& t0, int& row0) {
    const int num_w = p.num_tiles / p.num_t;
    if (kBwd) {
        t0 = (tile / num_w) * kTileTok;
        row0 = (tile % num_w) * kRowsPair;
    } else {
        const int band_tiles = kBand * p.num_t;  // tiles in a full band
        const int band = tile / band_tiles, in = tile % band_tiles;
        const int rows_in_band = min(kBand, num_w - band * kBand);
        t0 = (in / rows_in_band) * kTileTok;
        row0 = (band * kBand + in % rows_in_band) * kRowsPair;
    }
}

// The pair's share of the work.  Whole tiles go round-robin to the pairs
// (tile pair + round * num_pairs), so the tiles in flight at any time are
// neighbours in the tile order (and share their X / dY and W in L2).  When
// the launcher asks for it (split_tail), only the full rounds go so and the
// stages of the remaining tiles, the tail, are shared out evenly: pair j takes the contiguous range
// [j It / P, (j+1) It / P) of the tail's iterations tile * kb_total + kb
// (It = tail tiles * kb_total), which may start or end inside a tile.  A
// segment is one tile's part of the pair's work; stage `local` of the
// pair's sequence uses ring slot local % kStages for the
// (local / kStages)-th time.  Iteration counts stay below 2^31.
struct Range {
    int rounds;           // whole tiles: pair + r * num_pairs, r < rounds
    int tail_tile0;       // first tile of the tail: rounds * num_pairs
    int tail_it;          // the tail's iterations
    int lo, hi;           // this pair's share of them
    int t_first;          // its first tail tile, relative to tail_tile0
    int nseg;             // segments: rounds, then the tail's
};

__device__ __forceinline__ Range pair_range(const PairParams& p, int pair, int num_pairs) {
    Range r;
    if (p.split_tail) {
        r.rounds = p.num_tiles / num_pairs;
        r.tail_tile0 = r.rounds * num_pairs;
        r.tail_it = (p.num_tiles - r.tail_tile0) * p.kb_total;
    } else {  // whole tiles only: the last round leaves some pairs idle
        r.rounds = (p.num_tiles - pair + num_pairs - 1) / num_pairs;
        r.tail_tile0 = p.num_tiles;
        r.tail_it = 0;
    }
    r.lo = static_cast<int>(static_cast<int64_t>(pair) * r.tail_it / num_pairs);
    r.hi = static_cast<int>(static_cast<int64_t>(pair + 1) * r.tail_it / num_pairs);
    r.t_first = r.lo / p.kb_total;
    r.nseg = r.rounds + (r.hi > r.lo ? (r.hi - 1) / p.kb_total - r.t_first + 1 : 0);
    return r;
}

// The pair whose tail share holds tail iteration g.
__device__ __forceinline__ int pair_of(const Range& R, int g, int num_pairs) {
    return static_cast<int>((static_cast<int64_t>(g + 1) * num_pairs - 1) / R.tail_it);
}

struct Seg {
    int tile, kb_begin, kb_end;  // stages [kb_begin, kb_end) of tile `tile`
    int t0, row0;
    int tail_tile;               // tail tiles: index relative to tail_tile0, else -1
};

template <bool kBwd>
__device__ __forceinline__ void seg_of(const PairParams& p, const Range& R, int pair, int num_pairs, int i,
                                       Seg& sg) {
    if (i < R.rounds) {
        sg.tile = pair + i * num_pairs;
        sg.kb_begin = 0;
        sg.kb_end = p.kb_total;
        sg.tail_tile = -1;
    } else {
        sg.tail_tile = R.t_first + (i - R.rounds);
        sg.tile = R.tail_tile0 + sg.tail_tile;
        const int base = sg.tail_tile * p.kb_total;
        sg.kb_begin = R.lo > base ? R.lo - base : 0;
        sg.kb_end = R.hi - base < p.kb_total ? R.hi - base : p.kb_total;
    }
    tile_coords<kBwd>(p, sg.tile, sg.t0, sg.row0);
}

// Segment and contraction step of stage `local` of the pair's sequence.
__device__ __forceinline__ int stage_seg(const PairParams& p, const Range& R, int local, int& kb) {
    const int kbt = p.kb_total;
    const int full = R.rounds * kbt;
    if (local < full) {
        const int seg = local / kbt;
        kb = local - seg * kbt;
        return seg;
    }
    const int g = R.lo + (local - full);
    const int t = g / kbt;
    kb = g - t * kbt;
    return R.rounds + (t - R.t_first);
}

// Stages in the pair's sequence.
__device__ __forceinline__ int pair_stages(const PairParams& p, const Range& R) {
    return R.rounds * p.kb_total + (R.hi - R.lo);
}

// warp 0, one thread, both CTAs: the activation halves of every stage (and
// the LoRA slabs' A operand) into this CTA's ring; the even CTA also arms
// the stage's completion byte count for the pair.
template <bool kBwd>
__device__ void role_tma(const Pipe& P, const PairParams& p, const Range& R, const CUtensorMap* tm_act,
                         const CUtensorMap* tm_lact, const CUtensorMap* tm_lw) {
    int local = 0;  // stage index within the pair's range
    for (int i = 0; i < R.nseg; ++i) {
        Seg sg;
        seg_of<kBwd>(p, R, P.pair, P.num_pairs, i, sg);
        const int my_row0 = sg.row0 + static_cast<int>(P.rank) * kRowsCta;
        for (int kb = sg.kb_begin; kb < sg.kb_end; ++kb, ++local) {
            const int s = local % kStages;
            const uint32_t ph = static_cast<uint32_t>(local / kStages) & 1u;
            if (!mbar_wait(P.empty(s), ph ^ 1u, &g_pair_error)) return;
            const uint32_t bar = cluster_map(P.full_b(s), 0);
            const bool lora = kb >= p.kb_w;
            if (P.rank == 0) mbar_arrive_expect_tx(P.full_b(s), lora ? kTxLora : kTxWeight);
            const CUtensorMap* act = lora ? tm_lact : tm_act;
            // forward: the tile's linear picks its own columns of T
            const int t_off = (!kBwd && lora) ? group_of(p, sg.row0) * p.r_lora_off : 0;
            const int x = lora ? t_off + (kb - p.kb_w) * kBK : kb * kBK;
            for (int sub = 0; sub < kSubs; ++sub)
                tma_load_2d_pair(P.sB(s, sub), act, bar, x,
                                 sg.t0 + sub * kSubTok + static_cast<int>(P.rank) * kHalfTok);
            if (lora) {
                const int j0 = (kb - p.kb_w) * kBK;
                if (kBwd) {  // A^T rows k (MN-major): two 64-wide k blocks of A[j0 .. j0+63][k]
                    tma_load_2d_pair(P.sA(s), tm_lw, bar, my_row0, j0);
                    tma_load_2d_pair(P.sA(s) + 8192, tm_lw, bar, my_row0 + 64, j0);
                } else {     // B rows n (K-major): B[n][j0 .. j0+63]
                    tma_load_2d_pair(P.sA(s), tm_lw, bar, j0, my_row0);
                }
            }
        }
    }
}

// warp 1, one thread of the even CTA: per stage, for each 16-wide
// contraction step, one pair MMA into each accumulator in turn; one
// accumulation per segment.
template <bool kBwd>
__device__ void role_mma(const Pipe& P, const PairParams& p, const Range& R) {
    constexpr uint32_t idesc = idesc_bf16(kRowsPair, kSubTok, kBwd ? 1 : 0, 0);
    int local = 0;
    for (int i = 0; i < R.nseg; ++i) {
        Seg sg;
        seg_of<kBwd>(p, R, P.pair, P.num_pairs, i, sg);
        if (!mbar_wait(P.acc_empty(), (static_cast<uint32_t>(i) & 1u) ^ 1u, &g_pair_error)) return;
        tc_fence_after();
        for (int kb = sg.kb_begin; kb < sg.kb_end; ++kb, ++local) {
            const int s = local % kStages;
            const uint32_t ph = static_cast<uint32_t>(local / kStages) & 1u;
            if (!mbar_wait(P.full_b(s), ph, &g_pair_error)) return;
            if (!mbar_wait(P.full_a(s), ph, &g_pair_error)) return;
            tc_fence_after();
            const uint32_t sa = P.sA(s);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                // 16 contraction steps: +32 bytes along a K-major row, +16 rows of 128 bytes MN-major
                const uint64_t ad = kBwd ? sdesc_mnmajor_sw128(sa + kk * 2048, 8192)
                                         : sdesc_kmajor_sw128(sa) + static_cast<uint64_t>(kk * 2);
#pragma unroll
                for (int sub = 0; sub < kSubs; ++sub) {
                    const uint64_t bd = sdesc_kmajor_sw128(P.sB(s, sub)) + static_cast<uint64_t>(kk * 2);
                    mma_bf16_ss_pair(P.tmem + sub * kSubTok, ad, bd, idesc, (kb > sg.kb_begin || kk > 0) ? 1u : 0u);
                }
            }
            tc_commit_pair_mc(P.empty(s), kPairMask);
        }
        tc_commit_pair_mc(P.acc_full(), kPairMask);
    }
}

// Lane 0 of the calling warp waits; the result is broadcast so the warp
// proceeds (or gives up) together.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, &g_pair_error) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// One 64-weight run (32 code bytes, element 2t in the high nibble of byte
// t) times its block constant, as 32 bf16 pairs (the even element in the
// low half, i.e. at the lower address), without any table in memory.
//
// The run's 16 possible values p_i = bf16(RN32(q_i * c2')) are formed once
// (16 multiplies, 8 packs) and split into a low-byte plane L and a
// high-byte plane H of 16 bytes each (4 registers each).  For four weights
// (two code bytes w, nibbles n0..n3 from the least significant end, i.e.
// weights 1, 0, 3, 2) one byte permute per plane and half of the table
// picks byte (n_j & 7) for result byte j from entries 0-7 and another from
// entries 8-15; bit 3 of each nibble, spread to a byte mask by a
// sign-replicating permute, chooses between them; two more permutes
// interleave the planes into the two bf16 pairs.  Every value is exactly
// bf16(RN32(q[code] * c2')).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}
__device__ __forceinline__ uint32_t lop_select(uint32_t a, uint32_t b, uint32_t m) {
    return (a & ~m) | (b & m);  // one LOP3
}


// The same conversion into registers (32 bf16 pairs, even element in the
// low half), for a store after the ring slot is free.
__device__ __forceinline__ void convert_run(const uint4& c0, const uint4& c1, float sc, const float (&q)[16],
                                            uint32_t (&v)[32]) {
    uint32_t L[4], H[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t t0 = pack_bf16x2(__fmul_rn(q[4 * k], sc), __fmul_rn(q[4 * k + 1], sc));
        const uint32_t t1 = pack_bf16x2(__fmul_rn(q[4 * k + 2], sc), __fmul_rn(q[4 * k + 3], sc));
        L[k] = prmt(t0, t1, 0x6420u);
        H[k] = prmt(t0, t1, 0x7531u);
    }
    const uint32_t w8[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int h = 0; h < 8; ++h) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t w = (w8[h] >> (16 * half)) & 0xffffu;
            const uint32_t sel = w & 0x7777u;
            const uint32_t m = prmt(w << 4, w, 0xD9C8u);
            const uint32_t lo = lop_select(prmt(L[0], L[1], sel), prmt(L[2], L[3], sel), m);
            const uint32_t hi = lop_select(prmt(H[0], H[1], sel), prmt(H[2], H[3], sel), m);
            v[4 * h + 2 * half] = prmt(lo, hi, 0x4051u);
            v[4 * h + 2 * half + 1] = prmt(lo, hi, 0x6273u);
        }
    }
}

// Writes one converted run as row `row` (128 bytes at shared address
// `row_base`) in the 128-byte swizzled layout.
__device__ __forceinline__ void store_swizzled_row(uint32_t row_base, int row, const uint32_t (&v)[32]) {
#pragma unroll
    for (int h = 0; h < 8; ++h)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_base + ((h ^ (row & 7)) << 4)),
                     "r"(v[4 * h]), "r"(v[4 * h + 1]), "r"(v[4 * h + 2]), "r"(v[4 * h + 3])
                     : "memory");
}


// The 64-weight run that lane task `t` (0..127) of a weight stage converts:
// its weight row n and first column kcol in W (valid = inside W), and where
// it goes in this CTA's A tile (row `arow` of 128 bytes at byte offset
// `aoff`).  Forward: task t is weight row row0 + t, columns 64 kb ...
// Backward: task t is contraction index n = 64 kb + (t & 63) and the k block
// (t >> 6) of this CTA's 128 output rows.
template <bool kBwd>
__device__ __forceinline__ bool task_of(const PairParams& p, int kb, int my_row0, int t, int64_t& n, int64_t& kcol,
                                        int& arow, int& aoff) {
    if (kBwd) {
        const int i = t & 63, b = t >> 6;
        n = static_cast<int64_t>(kb) * kBK + i;
        kcol = my_row0 + 64 * b;
        arow = i;
        aoff = b * 8192 + i * 128;
    } else {
        n = my_row0 + t;
        kcol = static_cast<int64_t>(kb) * kBK;
        arow = t;
        aoff = t * 128;
    }
    return n < p.N && kcol < p.K;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
    float4 v;
    asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// Epilogue of the pair's segment i, by one converter warp: its TMEM lane
// quarter (this CTA's weight rows my_row0 + 32 quarter ...), the 16-column
// chunks part, part + 4, ...; the accumulators are released on the even
// CTA's barrier after the warp's last load.  A whole tile is rounded to
// bf16 and stored.  A segment that does not start the tile stores its fp32
// sums into this pair's slot and counts the warp in the pair's flag.  A
// segment that starts the tile but does not end it adds, in pair order, the
// slots of the pairs that hold the rest of the tile once their flags are
// complete, then stores bf16.
// kLast: the pair's last segment, the only one that can finish a split
// tile (the other instance leaves that path out, to spare registers in the
// conversion loop).
template <bool kBwd, bool kLast>
__device__ __forceinline__ void seg_epilogue(const Pipe& P, const PairParams& p, const Range& R, int i, int part,
                                             int quarter, int lane, bool& ok) {
    Seg sg;
    seg_of<kBwd>(p, R, P.pair, P.num_pairs, i, sg);
    if (!warp_wait(P.acc_full(), static_cast<uint32_t>(i) & 1u, lane)) {
        ok = false;
        return;
    }
    tc_fence_after();
    const bool first = sg.kb_begin == 0, last = sg.kb_end == p.kb_total;
    int jlo = 1, jhi = 0;  // pairs whose slots this segment adds
    if (kLast && first && !last) {
        jlo = P.pair + 1;
        jhi = pair_of(R, sg.tail_tile * p.kb_total + p.kb_total - 1, P.num_pairs);
        int good = 1;
        if (lane == 0) {
            for (int j = jlo; j <= jhi && good; ++j) {
                if (ld_acquire_gpu(p.flags + j) >= kFlagCount) continue;
                const uint64_t t_start = globaltimer_ns();
                while (ld_acquire_gpu(p.flags + j) < kFlagCount) {
                    if (globaltimer_ns() - t_start > 2000000000ull) {
                        atomicExch(&g_pair_error, 6 /* QLORA_ERR_TIMEOUT */);
                        good = 0;
                        break;
                    }
                }
            }
        }
        good = __shfl_sync(0xffffffffu, good, 0);
        __syncwarp();
        if (!good) jhi = jlo - 1;  // give up on the fix-up (the outputs are invalid; the error is recorded)
    }
    const int my_row0 = sg.row0 + static_cast<int>(P.rank) * kRowsCta;
    const int lrow = quarter * 32 + lane;
    const int grow = my_row0 + lrow;
    const bool lane_ok = grow < p.rows;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const size_t cta_off = static_cast<size_t>(P.rank) * (kSlotFloats / 2);
    auto slot_at = [&](int j, int c) {  // this lane's 16 values of chunk c in pair j's slot
        return p.partial + static_cast<size_t>(j) * kSlotFloats + cta_off + (static_cast<size_t>(c) * kRowsCta + lrow) * 16;
    };
    // the first partner's values of the next chunk are loaded one chunk
    // ahead, so their latency overlaps the current chunk
    float4 pre[4];
    if (kLast && jhi >= jlo) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) pre[q4] = ld_cg_f4(slot_at(jlo, part) + 4 * q4);
    }
#pragma unroll 1
    for (int c = part; c < kChunks; c += kParts) {
        const int col = c * 16;  // accumulator c / 16, its columns 16 (c % 16) ..: tokens t0 + col ..
        uint32_t acc[16];
        tmem_ld_32x32b_x16(P.tmem + lane_base + col, acc);
        tmem_wait_ld();
        if (c + kParts >= kChunks) {  // this warp's last chunk
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(cluster_map(P.acc_empty(), 0));
        }
        if (!first) {
            float4* dst = reinterpret_cast<float4*>(slot_at(P.pair, c));
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                dst[q4] = make_float4(__uint_as_float(acc[4 * q4]), __uint_as_float(acc[4 * q4 + 1]),
                                      __uint_as_float(acc[4 * q4 + 2]), __uint_as_float(acc[4 * q4 + 3]));
            continue;
        }
        if (kLast && jhi >= jlo) {  // the slots in pair order: deterministic
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                acc[4 * q4] = __float_as_uint(__uint_as_float(acc[4 * q4]) + pre[q4].x);
                acc[4 * q4 + 1] = __float_as_uint(__uint_as_float(acc[4 * q4 + 1]) + pre[q4].y);
                acc[4 * q4 + 2] = __float_as_uint(__uint_as_float(acc[4 * q4 + 2]) + pre[q4].z);
                acc[4 * q4 + 3] = __float_as_uint(__uint_as_float(acc[4 * q4 + 3]) + pre[q4].w);
            }
            if (c + kParts < kChunks) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) pre[q4] = ld_cg_f4(slot_at(jlo, c + kParts) + 4 * q4);
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {  // further partners (a tile split over three or more pairs)
                float a0 = __uint_as_float(acc[4 * q4]), a1 = __uint_as_float(acc[4 * q4 + 1]);
                float a2 = __uint_as_float(acc[4 * q4 + 2]), a3 = __uint_as_float(acc[4 * q4 + 3]);
#pragma unroll 1
                for (int j = jlo + 1; j <= jhi; ++j) {
                    const float4 x = ld_cg_f4(slot_at(j, c) + 4 * q4);
                    a0 += x.x;
                    a1 += x.y;
                    a2 += x.z;
                    a3 += x.w;
                }
                acc[4 * q4] = __float_as_uint(a0);
                acc[4 * q4 + 1] = __float_as_uint(a1);
                acc[4 * q4 + 2] = __float_as_uint(a2);
                acc[4 * q4 + 3] = __float_as_uint(a3);
            }
        }
        if (lane_ok) {
            uint16_t* o = p.out + static_cast<int64_t>(sg.t0 + col) * p.rows + grow;
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (sg.t0 + col + j < p.M) o[static_cast<int64_t>(j) * p.rows] = f32_to_bf16_bits(__uint_as_float(acc[j]));
        }
    }
    if (!first) {  // the slot is complete once all warps of both CTAs have counted themselves
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.flags + P.pair, 1);
    }
}

// warps 2..17 of both CTAs: each converts every fourth stage of the pair's
// range (the stages i with i % 4 == part, always ring slot part), 32 of
// the stage's 128 weight runs, into this CTA's A tile, then arrives on the
// even CTA's full_a barrier; for LoRA slabs (loaded by TMA) it only
// arrives.  After storing a stage of segment i it writes its share of the
// outputs of every earlier segment not yet done, so the MMAs of the next
// segment find the first stages ready once the accumulators are free.
template <bool kBwd>
__device__ __forceinline__ void role_convert(const Pipe& P, const PairParams& p, const Range& R, int warp,
                                             int lane) {
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    const int t = quarter * 32 + lane;  // this lane's run within a stage
    const uint32_t full_a_leader0 = cluster_map(P.full_a(0), 0);
    const int n_local = pair_stages(p, R);
    bool ok = true;
    int next_epi = 0;  // the next segment whose outputs this warp writes

    // The segment of a stage, cached: stages only move forward, and the
    // segment changes once per tile.
    struct SegCache {
        int seg = -1;
        int my_row0 = 0;
    };
    auto seg_for = [&](SegCache& c, int local, int& kb) {
        const int seg = stage_seg(p, R, local, kb);
        if (seg != c.seg) {
            Seg sg;
            seg_of<kBwd>(p, R, P.pair, P.num_pairs, seg, sg);
            c.seg = seg;
            c.my_row0 = sg.row0 + static_cast<int>(P.rank) * kRowsCta;
        }
        return seg;
    };

    SegCache cload, cconv;
    uint4 cb0 = make_uint4(0u, 0u, 0u, 0u), cb1 = cb0;
    uint32_t sbyte = 0u;
    float sc1 = 0.0f, smu = 0.0f;
    auto issue = [&](int local) {
        cb0 = make_uint4(0u, 0u, 0u, 0u);
        cb1 = cb0;
        sbyte = 0u;
        sc1 = 0.0f;
        smu = 0.0f;
        if (local >= n_local) return;
        int kb;
        seg_for(cload, local, kb);
        if (kb >= p.kb_w) return;
        int64_t n, kcol;
        int arow, aoff;
        if (!task_of<kBwd>(p, kb, cload.my_row0, t, n, kcol, arow, aoff)) return;
        const int g = group_of(p, n);
        const int64_t nl = n - p.gstart[g];  // the row within linear g
        const uint8_t* src = p.codes[g] + nl * (p.K / 2) + kcol / 2;
        cb0 = ldg_nc_v4(src);
        cb1 = ldg_nc_v4(src + 16);
        const int64_t blk = nl * (p.K / kBK) + kcol / kBK;
        sbyte = __ldg(p.c2_fp8[g] + blk);
        sc1 = __ldg(p.c1[g] + (blk >> 8));
        smu = __ldg(p.mean[g]);
    };

    issue(part);
    for (int local = part; local < n_local; local += kStages) {
        int kb;
        const int seg = seg_for(cconv, local, kb);
        const int s = part;  // == local % kStages
        const uint32_t ph = static_cast<uint32_t>(local / kStages) & 1u;
        const bool weight = kb < p.kb_w;
        uint32_t v[32];
        int64_t n = 0, kcol = 0;
        int arow = 0, aoff = 0;
        if (weight) {
            const bool valid = task_of<kBwd>(p, kb, cconv.my_row0, t, n, kcol, arow, aoff);
            // runs outside W are zero (in the backward they are part of the contraction)
            const float sc = valid ? dq_constant(static_cast<uint8_t>(sbyte), sc1, smu) : 0.0f;
            convert_run(cb0, cb1, sc, p.q, v);
        }
        if (!warp_wait(P.empty(s), ph ^ 1u, lane)) return;
        if (weight) {
            store_swizzled_row(P.sA(s) + static_cast<uint32_t>(aoff), arow, v);
            fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(full_a_leader0 + 8u * s);
        while (next_epi < seg) {  // segments before the current one: never the last
            seg_epilogue<kBwd, false>(P, p, R, next_epi++, part, quarter, lane, ok);
            if (!ok) return;
        }
        // the loads of the next own stage go out after the hand-off, so that
        // nothing above waits for them
        issue(local + kStages);
    }
    while (next_epi < R.nseg) {
        if (next_epi + 1 < R.nseg)
            seg_epilogue<kBwd, false>(P, p, R, next_epi, part, quarter, lane, ok);
        else
            seg_epilogue<kBwd, true>(P, p, R, next_epi, part, quarter, lane, ok);
        ++next_epi;
        if (!ok) return;
    }
}

template <bool kBwd>
__global__ void __launch_bounds__(kThreads, 1)
k_nf4_gemm_pair(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_lact,
                const __grid_constant__ CUtensorMap tm_lw, const __grid_constant__ PairParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base (the swizzle atoms), by pointer arithmetic so
    // every access below stays a 32-bit shared-memory access; the offset is
    // the same in both CTAs of the pair
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 3);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    Pipe P;
    P.smem = smem_u32(smem);
    P.bar0 = smem_u32(bars);
    P.rank = cluster_ctarank();
    P.pair = static_cast<int>(blockIdx.x >> 1);
    P.num_pairs = static_cast<int>(gridDim.x >> 1);
    __shared__ Range s_range;
    if (threadIdx.x == 0) {
        s_range = pair_range(p, P.pair, P.num_pairs);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(P.full_b(s), 1);          // the even CTA's expect_tx arrival (+ both CTAs' bytes)
            mbar_init(P.full_a(s), 2 * 4);      // the part's four warps in each CTA
            mbar_init(P.empty(s), 1);           // the pair MMA's commit
        }
        mbar_init(P.acc_full(), 1);
        mbar_init(P.acc_empty(), 2 * kDqWarps);  // every converter warp of both CTAs
        mbar_init(P.drain(), 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&tm_act);
        tma_prefetch_desc(&tm_lact);
        tma_prefetch_desc(&tm_lw);
    }
    tc_fence_before();
    __syncthreads();
    cluster_arrive();  // both CTAs' barriers are initialised before any remote arrive
    cluster_wait();
    tc_fence_after();
    P.tmem = *tmem_slot;
    const Range& R = s_range;  // read from shared memory where used, not held in registers
    if (warp == 0) {
        if (lane == 0) role_tma<kBwd>(P, p, R, &tm_act, &tm_lact, &tm_lw);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && P.rank == 0) {
            role_mma<kBwd>(P, p, R);
            // every pair MMA issued (also on an early exit) has completed
            // before the tensor memory can be freed
            tc_commit_pair_mc(P.drain(), 1);
            mbar_wait(P.drain(), 0u, &g_pair_error);
        }
        __syncwarp();
    } else {
        role_convert<kBwd>(P, p, R, warp, lane);
    }
    tc_fence_before();
    __syncthreads();
    cluster_arrive();  // neither CTA frees its tensor memory or leaves while the pair may still use it
    cluster_wait();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(P.tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host
// Row-major bf16 matrix (outer x inner), 128-byte swizzled boxes of
// box_inner (<= 64) x box_outer elements, zero fill outside.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                   uint32_t box_outer) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of two kernels that can be resident at once, asked once per
// context.
template <bool kBwd>
int max_pairs() {
    static ContextMemo<int> memo;
    uint64_t ctx = 0;
    if (!current_context_id(&ctx)) return 0;
    int n = 0;
    memo.get(ctx, &n, [](int* v) {
        cudaLaunchConfig_t cfg{};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * static_cast<unsigned>(num_sms()));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemBytes;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int c = 0;
        if (cudaOccupancyMaxActiveClusters(&c, k_nf4_gemm_pair<kBwd>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            c = 0;
        }
        *v = c;
        return true;
    });
    return n;
}

// Workspace of the split tiles for `pairs` pairs: the flags (one int per
// pair), then one partial-sum slot per pair.
size_t flag_bytes(int pairs) { return static_cast<size_t>(round_up(static_cast<int64_t>(pairs) * 4, 256)); }
size_t ws_bytes_for(int pairs) { return flag_bytes(pairs) + static_cast<size_t>(pairs) * kSlotFloats * 4; }

template <bool kBwd>
cudaError_t launch_pair(const CUtensorMap& ma, const CUtensorMap& ml, const CUtensorMap& mw, PairParams p, void* ws,
                        size_t ws_bytes, cudaStream_t st) {
    static ContextMemo<int> attr_memo;
    cudaError_t e = ensure_smem_limit(attr_memo, k_nf4_gemm_pair<kBwd>, kSmemBytes);
    if (e != cudaSuccess) return e;
    int pairs = max_pairs<kBwd>();
    if (pairs <= 0) return cudaErrorNotSupported;
    // no more pairs than the workspace has slots for, and at least a few
    // stages for each
    while (pairs > 1 && (ws == nullptr || ws_bytes < ws_bytes_for(pairs))) --pairs;
    const int64_t by_work = p.iters / kMinStagesPerPair;
    if (by_work < pairs) pairs = static_cast<int>(by_work > 1 ? by_work : 1);
    // Splitting the last round's tiles evens out the pairs' work but costs
    // an accumulator hand-off per extra segment (the epilogue is exposed
    // then): measured, it pays when that round would leave at least half of
    // the pairs idle, not when it is fuller.
    const int rem = p.num_tiles % pairs;
    p.split_tail = (rem != 0 && 2 * rem <= pairs) ? 1 : 0;
    if (pairs > 1) {  // a single pair splits no tile and needs no workspace
        p.flags = reinterpret_cast<int*>(ws);
        p.partial = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + flag_bytes(pairs));
        e = cudaMemsetAsync(p.flags, 0, static_cast<size_t>(pairs) * 4, st);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * static_cast<unsigned>(pairs));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_nf4_gemm_pair<kBwd>, ma, ml, mw, p);
    note_launches(1);
    return e;
}

PairParams base_params(const Nf4Weight& w, int64_t M, int r, uint16_t* out, bool bwd) {
    PairParams p{};
    p.G = 1;
    p.codes[0] = w.codes;
    p.c2_fp8[0] = w.c2_fp8;
    p.c1[0] = w.c1;
    p.mean[0] = w.mean;
    p.gstart[0] = 0;
    p.gstart[1] = static_cast<int>(w.N);
    p.r_lora_off = 0;
    p.out = out;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(w.N);
    p.K = static_cast<int>(w.K);
    p.r = r;
    p.rows = bwd ? p.K : p.N;
    p.ctr = bwd ? p.N : p.K;
    p.kb_w = static_cast<int>(ceil_div(p.ctr, kBK));
    p.kb_total = p.kb_w + static_cast<int>(ceil_div(r, kBK));
    p.num_t = static_cast<int>(ceil_div(M, kTileTok));
    p.num_tiles = p.num_t * static_cast<int>(ceil_div(p.rows, kRowsPair));
    p.iters = static_cast<int64_t>(p.num_tiles) * p.kb_total;
    for (int i = 0; i < 16; ++i) p.q[i] = tables(w.qtype).q[i];
    return p;
}

// The failure-detection self-test: one thread waits, with the given limit,
// for a phase of an mbarrier that nothing ever arrives on.  No copy or MMA
// is in flight, so when the limit passes the wait records QLORA_ERR_TIMEOUT
// in the sticky word and the kernel simply returns.
__global__ void k_wait_selftest(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0u, &g_pair_error, limit_ns);
    __syncthreads();
}

}  // namespace

bool pair_gemm_supported(int64_t M, const Nf4Weight& w, int r, bool bwd) {
    // TMA row strides: X / dY / T / U / A / B rows a multiple of 16 bytes;
    // the stage count of all tiles below 2^31
    const int64_t rows = bwd ? w.K : w.N, ctr = bwd ? w.N : w.K;
    const int64_t iters = ceil_div(M, kTileTok) * ceil_div(rows, kRowsPair) * (ceil_div(ctr, kBK) + ceil_div(r, kBK));
    return iters < (int64_t(1) << 31) && M >= 1 && M < (int64_t(1) << 31) && w.K >= kBK && w.K % kBK == 0 && w.N >= 1 &&
           w.N < (int64_t(1) << 31) && w.K < (int64_t(1) << 31) && r >= 8 && r % 8 == 0 && r <= 256 &&
           (!bwd || w.N % 8 == 0) && tensor_map_encoder() != nullptr;
}

// Enough for one slot per pair of SMs of the current device.
size_t pair_gemm_workspace() {
    const int pairs = num_sms() / 2 > 0 ? num_sms() / 2 : 1;
    return ws_bytes_for(pairs);
}

cudaError_t launch_fwd_gemm_pair(const uint16_t* X, const Nf4Weight& w, const uint16_t* T, const uint16_t* B,
                                 int64_t M, int r, uint16_t* Y, void* ws, size_t ws_bytes, cudaStream_t st) {
    PairParams p = base_params(w, M, r, Y, false);
    CUtensorMap ma, ml, mw;
    if (!make_map_bf16(&ma, X, static_cast<uint64_t>(w.K), static_cast<uint64_t>(M), kBK, kHalfTok) ||
        !make_map_bf16(&ml, T, static_cast<uint64_t>(r), static_cast<uint64_t>(M), kBK, kHalfTok) ||
        !make_map_bf16(&mw, B, static_cast<uint64_t>(r), static_cast<uint64_t>(w.N), kBK, kRowsCta))
        return cudaErrorInvalidValue;
    return launch_pair<false>(ma, ml, mw, p, ws, ws_bytes, st);
}

cudaError_t launch_bwd_dx_gemm_pair(const uint16_t* dY, const Nf4Weight& w, const uint16_t* U, const uint16_t* A,
                                    int64_t M, int r, uint16_t* dX, void* ws, size_t ws_bytes, cudaStream_t st) {
    PairParams p = base_params(w, M, r, dX, true);
    CUtensorMap ma, ml, mw;
    if (!make_map_bf16(&ma, dY, static_cast<uint64_t>(w.N), static_cast<uint64_t>(M), kBK, kHalfTok) ||
        !make_map_bf16(&ml, U, static_cast<uint64_t>(r), static_cast<uint64_t>(M), kBK, kHalfTok) ||
        !make_map_bf16(&mw, A, static_cast<uint64_t>(w.K), static_cast<uint64_t>(r), 64, kBK))
        return cudaErrorInvalidValue;
    return launch_pair<true>(ma, ml, mw, p, ws, ws_bytes, st);
}

bool pair_group_supported(int64_t M, const Nf4Group& g, int r) {
    if (g.G < 1 || g.G > kMaxGroups || r < 8 || r % 8 != 0 || g.G * r > 256) return false;
    int64_t n = 0;
    for (int i = 0; i < g.G; ++i) {
        if (g.w[i].N < 1 || g.w[i].N % kRowsPair != 0 || g.w[i].K != g.w[0].K || g.w[i].qtype != g.w[0].qtype)
            return false;
        n += g.w[i].N;
    }
    Nf4Weight all = g.w[0];
    all.N = n;
    return n < (int64_t(1) << 31) && pair_gemm_supported(M, all, g.G * r, true);
}

// The stacked weight: rows gstart[i] .. of the product are linear i's.
PairParams group_params(const Nf4Group& g, int64_t M, int r_slabs, uint16_t* out, bool bwd) {
    Nf4Weight all = g.w[0];
    int64_t n = 0;
    for (int i = 0; i < g.G; ++i) n += g.w[i].N;
    all.N = n;
    PairParams p = base_params(all, M, r_slabs, out, bwd);
    p.G = g.G;
    int64_t start = 0;
    for (int i = 0; i < g.G; ++i) {
        p.codes[i] = g.w[i].codes;
        p.c2_fp8[i] = g.w[i].c2_fp8;
        p.c1[i] = g.w[i].c1;
        p.mean[i] = g.w[i].mean;
        p.gstart[i] = static_cast<int>(start);
        start += g.w[i].N;
    }
    p.gstart[g.G] = static_cast<int>(start);
    return p;
}

cudaError_t launch_fwd_gemm_pair_group(const uint16_t* X, const Nf4Group& g, const uint16_t* T, const uint16_t* B_cat,
                                       int64_t M, int r, uint16_t* Y, void* ws, size_t ws_bytes, cudaStream_t st) {
    PairParams p = group_params(g, M, r, Y, false);
    p.r_lora_off = r;
    const int64_t K = g.w[0].K;
    CUtensorMap ma, ml, mw;
    if (!make_map_bf16(&ma, X, static_cast<uint64_t>(K), static_cast<uint64_t>(M), kBK, kHalfTok) ||
        !make_map_bf16(&ml, T, static_cast<uint64_t>(g.G) * r, static_cast<uint64_t>(M), kBK, kHalfTok) ||
        !make_map_bf16(&mw, B_cat, static_cast<uint64_t>(r), static_cast<uint64_t>(p.N), kBK, kRowsCta))
        return cudaErrorInvalidValue;
    return launch_pair<false>(ma, ml, mw, p, ws, ws_bytes, st);
}

cudaError_t launch_bwd_dx_gemm_pair_group(const uint16_t* dY, const Nf4Group& g, const uint16_t* U,
                                          const uint16_t* A_cat, int64_t M, int r, uint16_t* dX, void* ws,
                                          size_t ws_bytes, cudaStream_t st) {
    const int rc = g.G * r;  // the LoRA contraction: every linear's rank
    PairParams p = group_params(g, M, rc, dX, true);
    const int64_t K = g.w[0].K;
    CUtensorMap ma, ml, mw;
    if (!make_map_bf16(&ma, dY, static_cast<uint64_t>(p.N), static_cast<uint64_t>(M), kBK, kHalfTok) ||
        !make_map_bf16(&ml, U, static_cast<uint64_t>(rc), static_cast<uint64_t>(M), kBK, kHalfTok) ||
        !make_map_bf16(&mw, A_cat, static_cast<uint64_t>(K), static_cast<uint64_t>(rc), 64, kBK))
        return cudaErrorInvalidValue;
    return launch_pair<true>(ma, ml, mw, p, ws, ws_bytes, st);
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st) {
    k_wait_selftest<<<1, 32, 0, st>>>(limit_ns);
    note_launches(1);
    return cudaGetLastError();
}

int pair_device_error(int reset) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_pair_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    if (reset && v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_pair_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return v;
}

}  // namespace qlora
