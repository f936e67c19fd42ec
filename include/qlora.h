/*
 * qlora.h -- C ABI of the B200 (sm_100a) QLoRA NF4 linear-layer library.
 *
 * The hot path of QLoRA (Dettmers et al., "QLoRA: Efficient Finetuning of
 * Quantized LLMs", arXiv:2305.14314) for one frozen linear layer with a LoRA
 * side path.  Citations name the QLoRA study-notes page (gitcode.csdn.net) by
 * section and equation.
 *
 * Notation (row-major, "out x in" like torch.nn.Linear):
 *   W  N x K   frozen weight, stored as NF4 codes + double-quantized constants
 *   X  M x K   input activations (bf16)
 *   A  r x K   LoRA down projection (the pages' L1 = A^T)
 *   B  N x r   LoRA up projection   (the pages' L2 = B^T)
 *   s          the LoRA scalar of eq. (3) (usually alpha / r)
 *   Y  M x N   output; dY, dX, dA, dB the matching gradients
 *
 * Conventions for every entry point:
 *   - Array pointers are DEVICE pointers owned by the caller, except the one
 *     host array of qlora_nf4_codebook.  The library never allocates or frees
 *     memory; scratch space is passed in as a workspace (ws, ws_bytes).
 *   - Every device pointer must be 16-byte aligned; tensors are contiguous.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously; no call synchronizes the device.
 *   - Every call returns a qlora_status.  Argument errors are detected on
 *     the host before anything is enqueued.  QLORA_ERR_CUDA means a launch
 *     failed (the CUDA error was consumed with cudaGetLastError).
 *   - Calls that share a workspace must be ordered on one stream.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qlora_status {
    QLORA_OK = 0,
    QLORA_ERR_INVALID_ARG = 1, /* null / negative / misaligned / bad dtype          */
    QLORA_ERR_UNSUPPORTED = 2, /* block sizes other than 64/256, K % 64 != 0, r > 256 */
    QLORA_ERR_WORKSPACE = 3,   /* ws NULL or ws_bytes below the documented size       */
    QLORA_ERR_CUDA = 4,        /* a kernel launch or CUDA runtime call failed          */
    QLORA_ERR_NONFINITE = 5,   /* written to the device status word: NaN/Inf in W      */
    QLORA_ERR_TIMEOUT = 6      /* from qlora_device_error: a device-side wait gave up  */
} qlora_status;

/* The 4-bit data types (section 3.2 builds NF4; FP4 and Int4 are the types
 * it is compared with): the codes are indices into a sorted table of 16
 * values in [-1, 1], scaled by the block constant. */
#define QLORA_TYPE_NF4 0   /* NormalFloat: eq. (4), the default everywhere    */
#define QLORA_TYPE_FP4 1   /* OCP E2M1 values / 6: 15 distinct, top repeated   */
#define QLORA_TYPE_INT4 2  /* eq. (1) at 4 bits: k / 7, k = -7..7, top repeated */

#define QLORA_BLOCK 64       /* first-level block: elements per absmax constant  */
#define QLORA_BLOCK2 256     /* second-level block: constants per FP8 scale       */
#define QLORA_MAX_RANK 256   /* largest LoRA rank r                              */

/*
 * qlora_nf4_codebook -- the 16 values of the 4-bit NormalFloat type
 * (section 3.2, eq. 4 and the asymmetric construction that keeps an exact
 * zero): 7 negative quantiles of N(0,1), one 0 and 8 positive quantiles,
 * normalised into [-1, 1].  Each half places its points at evenly spaced
 * probabilities from 1/2 out to delta = ((1 - 1/30) + (1 - 1/32)) / 2.
 * out_host: HOST array of 16 floats, sorted ascending (out[7] == 0,
 * out[0] == -1, out[15] == +1).  Pure host function; never touches the GPU.
 * Returns QLORA_ERR_INVALID_ARG for a NULL pointer.
 */
int qlora_nf4_codebook(float out_host[16]);

/*
 * qlora_codebook -- the 16 values of a 4-bit data type (QLORA_TYPE_*),
 * ascending, into the HOST array out_host.  NF4 as qlora_nf4_codebook.
 * FP4: the OCP E2M1 magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} with both signs,
 * divided by 6 (15 distinct values; its two zeros are one value), the top
 * value repeated at index 15.  Int4: k / 7 for k = -7 .. 7, the top value
 * repeated at index 15.  A repeated value is never chosen by the nearest-
 * value rule (ties go to the lower index).  QLORA_ERR_INVALID_ARG for a NULL
 * pointer or an unknown type.
 */
int qlora_codebook(int qtype, float out_host[16]);

/*
 * Workspace bytes that qlora_quantize_nf4_dq needs for `numel` weights:
 *   2048 (exact-sum bins) + 16 (flags) + round_up_16(4 * ceil(numel / 64)).
 */
size_t qlora_quantize_workspace_size(int64_t numel);

/*
 * qlora_quantize_nf4_dq -- block-wise NF4 quantization of a frozen weight
 * with double quantization of its constants (sections 3.1-3.3, 3.5).
 *
 *   W       in : numel fp32 values (the flattened tensor).
 *   block   in : must be 64 (QLORA_BLOCK); block2 must be 256 (QLORA_BLOCK2).
 *   codes   out: ceil(numel/2) bytes; element 2t in the high nibble, 2t+1 in
 *                the low nibble; an odd tail leaves a zero low nibble.
 *   c2_fp8  out: nb = ceil(numel/64) bytes, the per-block absmax c2 after
 *                double quantization, as OCP E4M3 codes.
 *   c1      out: ceil(nb/256) fp32 second-level scales.
 *   mean    out: 1 fp32, the mean of all c2, subtracted before the FP8 pass.
 *   ws           scratch of qlora_quantize_workspace_size(numel) bytes.
 *   status  out: nullable device int32; receives QLORA_OK, or
 *                QLORA_ERR_NONFINITE if W holds a NaN or Inf (outputs then
 *                unspecified).
 *
 * Definition (all steps IEEE fp32, round to nearest even, unfused):
 *   c2[j]  = max |w| over the 64 consecutive elements of block j
 *   code   = argmin_i |w / c2[j] - q_i| (ties to the lower i); c2 = 0 -> 7
 *   mean   = RN32(RN64(S) / nb), S the exact sum of all c2
 *   c1[g]  = max_{j in g} |c2[j] - mean| / 448
 *   c2_fp8 = E4M3_rne_satfinite((c2[j] - mean) / c1[g]); 0 where c1[g] == 0
 * numel == 0 enqueues nothing.  numel must be below 2^46.
 */
int qlora_quantize_nf4_dq(const float* W, int64_t numel, int block, int block2,
                          uint8_t* codes, uint8_t* c2_fp8, float* c1, float* mean,
                          void* ws, size_t ws_bytes, int32_t* status, void* stream);

/*
 * qlora_quantize_4bit_dq, qlora_dequantize_4bit, qlora_linear_fwd_4bit,
 * qlora_linear_bwd_4bit -- the same calls for any of the 4-bit data types:
 * `qtype` (QLORA_TYPE_*) first, then exactly the arguments of
 * qlora_quantize_nf4_dq, qlora_dequantize, qlora_linear_fwd and
 * qlora_linear_bwd, with the same definitions with q_i the type's table
 * (qlora_codebook).  The NF4 calls are these with QLORA_TYPE_NF4.  An
 * unknown type returns QLORA_ERR_INVALID_ARG.
 */
int qlora_quantize_4bit_dq(int qtype, const float* W, int64_t numel, int block, int block2,
                           uint8_t* codes, uint8_t* c2_fp8, float* c1, float* mean,
                           void* ws, size_t ws_bytes, int32_t* status, void* stream);
int qlora_dequantize_4bit(int qtype, const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                          const float* mean, int64_t numel, int block, int block2,
                          void* out, int out_dtype, void* stream);
int qlora_linear_fwd_4bit(int qtype, const uint16_t* X, int64_t M, int64_t N, int64_t K,
                          const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                          const float* mean, const uint16_t* A, const uint16_t* B, int r,
                          float s, uint16_t* Y, uint16_t* T_save, void* ws, size_t ws_bytes,
                          void* stream);
int qlora_linear_bwd_4bit(int qtype, const uint16_t* dY, const uint16_t* X, int64_t M, int64_t N,
                          int64_t K, const uint8_t* codes, const uint8_t* c2_fp8,
                          const float* c1, const float* mean, const uint16_t* A,
                          const uint16_t* B, int r, float s, const uint16_t* T,
                          uint16_t* dX, uint16_t* dA, uint16_t* dB, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * qlora_quantize_nf4_dq_noalloc -- the same quantization as
 * qlora_quantize_nf4_dq (same arguments minus ws / ws_bytes, same outputs,
 * bit for bit), for callers that cannot give the library a workspace: for
 * example a plugin whose host program owns all device memory and offers no
 * allocator, or a loop that cannot afford cudaMalloc's implicit
 * synchronisation.  The paper has no counterpart; this is a library
 * convenience.
 *
 * Its scratch is one fixed device array inside the library, reserved on
 * every GPU that loads it until the process exits: 2064 bytes plus 4 bytes
 * per 64-block, sized for numel <= QLORA_NOALLOC_MAX_NUMEL (2^28 weights,
 * about 16 MiB).  Larger numel returns QLORA_ERR_WORKSPACE without
 * launching anything.  The call allocates nothing (no cudaMalloc/cudaFree).
 * The first call in each CUDA context (i.e. per device, with that device
 * current) looks up the array's device address (cudaGetSymbolAddress) and
 * remembers it for that context; make that first call before any stream
 * capture.  After a device reset the next call runs in a new context and
 * looks the address up again, so it never uses an address from before the
 * reset (the array's contents do not survive a reset; nothing relies on
 * them between calls).  All calls share the one array: calls
 * whose kernels overlap on the GPU (different streams without ordering,
 * or several host threads) race on it and must be serialised by the
 * caller.  Each call clears the parts that must start at zero.
 */
#define QLORA_NOALLOC_MAX_NUMEL (1LL << 28)
int qlora_quantize_nf4_dq_noalloc(const float* W, int64_t numel, int block, int block2,
                                  uint8_t* codes, uint8_t* c2_fp8, float* c1, float* mean,
                                  int32_t* status, void* stream);

/*
 * qlora_dequantize -- double dequantization (section 3.5, eq. 6):
 *   c2' = RN32(RN32(E4M3(c2_fp8[j]) * c1[j / 256]) + mean)
 *   w   = RN32(q[code] * c2')                 (out_dtype 0: fp32)
 *   w   = bf16_rne(RN32(q[code] * c2'))       (out_dtype 1: bf16 bits)
 * Inputs as written by qlora_quantize_nf4_dq; `mean` is a device pointer.
 * out: numel elements of the chosen dtype.
 */
int qlora_dequantize(const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                     const float* mean, int64_t numel, int block, int block2,
                     void* out, int out_dtype, void* stream);

/*
 * Workspace bytes for qlora_linear_fwd / qlora_linear_bwd.  The forward
 * needs M*r*2 bytes for T (used when T_save is NULL); the backward needs U
 * and T (M*r*2 bytes each, 256-byte aligned).  Both add the GEMM's scratch
 * for output tiles whose contraction is split between SM pairs: one 512 KiB
 * fp32 slot per pair of SMs of the current device plus a few flags (about
 * 37 MiB on a 148-SM part).  A workspace of the larger size serves both.
 */
size_t qlora_linear_fwd_workspace_size(int64_t M, int64_t N, int64_t K, int r);
size_t qlora_linear_bwd_workspace_size(int64_t M, int64_t N, int64_t K, int r);

/*
 * qlora_linear_fwd -- the QLoRA linear (section 3.5 eq. 5 with the LoRA
 * scalar of section 4 eq. 3):
 *   T = bf16(s * X A^T)                       (M x r; saved to T_save if given)
 *   Y = bf16(X W'^T + T B^T)                  fp32 accumulation
 * where W' = bf16 of the double-dequantized weight (eq. 6).  W is given by
 * the four buffers of qlora_quantize_nf4_dq for an N x K row-major weight.
 * Requires K % 64 == 0, 1 <= r <= 256, M >= 0, N >= 1.
 * Small batches (1 <= M <= 16 with N % 16 == 0, 8 <= r <= 64, r % 8 == 0,
 * K <= 21504) take a single weight-streaming kernel that applies each
 * 64-block's constant c2' to the block's partial dot product, i.e. the
 * weight enters as bf16(q[code]) * c2' rather than bf16(q[code] * c2'):
 * the same value up to one bf16 rounding, within the forward's tolerance.
 * That path uses no workspace and computes T itself.
 */
int qlora_linear_fwd(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                     const uint8_t* codes, const uint8_t* c2_fp8, const float* c1,
                     const float* mean, const uint16_t* A, const uint16_t* B, int r,
                     float s, uint16_t* Y, uint16_t* T_save, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * qlora_linear_bwd -- gradients of the QLoRA linear (section 3.5: gradients
 * only for the adapters; the input gradient flows through the dequantized
 * frozen weight in bf16; there is no gradient for W):
 *   U  = bf16(s * dY B)                       (M x r)
 *   dX = bf16(dY W' + U A)                    (nullable: skipped)
 *   dA = bf16(U^T X)                          (r x K)
 *   dB = bf16(dY^T T)                         (N x r), T = bf16(s X A^T)
 * T: the T_save of the forward, or NULL to recompute it.  fp32 accumulation
 * throughout.  Same shape rules as qlora_linear_fwd.
 */
int qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, int64_t N,
                     int64_t K, const uint8_t* codes, const uint8_t* c2_fp8,
                     const float* c1, const float* mean, const uint16_t* A,
                     const uint16_t* B, int r, float s, const uint16_t* T,
                     uint16_t* dX, uint16_t* dA, uint16_t* dB, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * The frozen 4-bit weight of one linear: the four device buffers
 * qlora_quantize_4bit_dq writes for an N x K row-major weight.
 */
typedef struct qlora_weight_4bit {
    const uint8_t* codes;  /* N*K/2 bytes      */
    const uint8_t* c2_fp8; /* N*K/64 bytes     */
    const float* c1;       /* ceil(N*K/16384)  */
    const float* mean;     /* 1 float          */
    int64_t N;             /* output features  */
} qlora_weight_4bit;

/*
 * qlora_linear_group_fwd / qlora_linear_group_bwd -- G QLoRA linears that
 * read the same input (an attention block's q, k and v projections; an MLP's
 * gate and up projections), each with its own frozen weight W_g (N_g x K,
 * all of one 4-bit type) and its own rank-r adapter (A_g, B_g), run as one:
 * the products are exactly those of G qlora_linear_fwd / _bwd calls (same
 * definitions, same rounding points), stacked.  Buffers:
 *   W      in : host array of G descriptors (device buffers inside).
 *   A_cat  in : (G r) x K bf16, A_1 .. A_G stacked by rows.
 *   B_cat  in : (sum N_g) x r bf16, B_1 .. B_G stacked by rows.
 *   Y     out : M x (sum N_g) bf16, Y_g in columns n_g .. n_g + N_g - 1
 *               (n_g = N_1 + .. + N_{g-1}).
 *   T_save / T: M x (G r) bf16, T_g in columns g r .. (nullable as in the
 *               single calls).
 *   dY     in : M x (sum N_g), laid out like Y.
 *   dX    out : M x K = sum_g dY_g W_g' + U_g A_g, one bf16 rounding of the
 *               fp32 sum (nullable: skipped).
 *   dA_cat out: (G r) x K, dA_g stacked like A_cat.
 *   dB_cat out: (sum N_g) x r, dB_g stacked like B_cat.
 * Requires 1 <= G <= 4, every N_g a multiple of 256, K % 64 == 0, r % 8 == 0
 * and G r <= 256 (else QLORA_ERR_UNSUPPORTED; use the single calls), M >= 0.
 * The frozen-weight GEMM of the group is one kernel over the stacked weight,
 * its dX GEMM one kernel whose contraction runs over all G weights and the
 * G r adapter columns.  Workspace: the _workspace_size functions (fwd: T;
 * bwd: U and T, each M x G r bf16; both plus the GEMM scratch).
 */
size_t qlora_linear_group_fwd_workspace_size(int64_t M, int G, int r);
size_t qlora_linear_group_bwd_workspace_size(int64_t M, int G, int r);
int qlora_linear_group_fwd(int qtype, const uint16_t* X, int64_t M, int64_t K,
                           const qlora_weight_4bit* W, int G, const uint16_t* A_cat,
                           const uint16_t* B_cat, int r, float s, uint16_t* Y,
                           uint16_t* T_save, void* ws, size_t ws_bytes, void* stream);
int qlora_linear_group_bwd(int qtype, const uint16_t* dY, const uint16_t* X, int64_t M,
                           int64_t K, const qlora_weight_4bit* W, int G,
                           const uint16_t* A_cat, const uint16_t* B_cat, int r, float s,
                           const uint16_t* T, uint16_t* dX, uint16_t* dA_cat,
                           uint16_t* dB_cat, void* ws, size_t ws_bytes, void* stream);

/*
 * qlora_fp8_e4m3_encode -- the FP8 encoder the double quantization uses
 * (section 3.3 names 8-bit floats; read as OCP E4M3): out[i] =
 * E4M3_rne_satfinite(x[i]), NaN -> 0x7f.  n elements, device pointers.
 */
int qlora_fp8_e4m3_encode(const float* x, uint8_t* out, int64_t n, void* stream);

/*
 * qlora_device_error -- the sticky error word of the tensor-core kernels on
 * the current device: QLORA_OK, or QLORA_ERR_TIMEOUT if a pipeline wait
 * inside a kernel gave up (the kernel then ended early and its outputs are
 * invalid).  Synchronizes with the device to read it; reset != 0 clears it.
 * Returns QLORA_ERR_CUDA if the word cannot be read.
 */
int qlora_device_error(int reset);

/*
 * qlora_debug_fill / qlora_debug_read -- measurement aids, not part of the
 * method: the DRAM write and read ceilings that the HBM-bound kernels
 * (quantize, dequantize, the small-batch forward) are compared with.
 * qlora_debug_fill writes `value` to n_words 32-bit words at dst;
 * qlora_debug_read reads n_words words at src and writes their XOR-fold to
 * *sink only if it equals `never` (so the reads are kept; pass a value the
 * data cannot fold to, and the call writes nothing).  Both use 16-byte
 * accesses in whole 512-byte warp runs.  n_words must be a
 * multiple of 4 and the pointers 16-byte aligned (device memory), else
 * QLORA_ERR_INVALID_ARG; n_words == 0 launches nothing.
 */
int qlora_debug_fill(uint32_t* dst, int64_t n_words, uint32_t value, void* stream);
int qlora_debug_read(const uint32_t* src, int64_t n_words, uint32_t never, uint32_t* sink, void* stream);

/*
 * qlora_int8_quantize -- block-wise Int8 absmax quantization, the 8-bit
 * baseline of section 3.1, eq. (1), applied to consecutive blocks of
 * `block` elements of the flattened tensor (block in {32, 64, 128, 256};
 * the last block may be partial):
 *   c[j]    = RN32(127 / absmax(block j))           (0 for an all-zero block)
 *   code[i] = round_half_away_from_zero(RN32(c[j] * x[i]))   in [-127, 127]
 *   x       in : numel fp32;  codes out: numel int8;  c out: ceil(numel/block) fp32
 *   status  out: nullable device int32, cleared to QLORA_OK then set to
 *                QLORA_ERR_NONFINITE if a block holds a NaN or Inf (or its
 *                constant overflows fp32); the outputs are then unspecified.
 * Pointers 16-byte aligned.  numel == 0 enqueues nothing.
 */
int qlora_int8_quantize(const float* x, int64_t numel, int block, int8_t* codes, float* c,
                        int32_t* status, void* stream);

/*
 * qlora_int8_dequantize -- eq. (2): x'[i] = RN32(code[i] / c[j]), 0 where
 * c[j] == 0.  Same layout as qlora_int8_quantize; out: numel fp32.
 */
int qlora_int8_dequantize(const int8_t* codes, const float* c, int64_t numel, int block, float* out,
                          void* stream);

/*
 * qlora_debug_wait_timeout -- failure-detection self-test (no counterpart
 * in the paper).  Launches one single-thread kernel on `stream` whose
 * bounded wait (the same wait every pipeline stage of the tensor-core
 * kernels uses) is never satisfied: after limit_ns nanoseconds of GPU time
 * it gives up, records QLORA_ERR_TIMEOUT in the sticky word that
 * qlora_device_error reads, and returns.  Nothing else is in flight in that
 * kernel, so the context stays usable and later calls work as usual.
 * 0 < limit_ns <= 1e9, else QLORA_ERR_INVALID_ARG (nothing launched).
 */
int qlora_debug_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * qlora_kernel_launch_count -- number of kernels this library has launched
 * in the calling process since it was loaded (all devices, all streams).
 * A diagnostic for benchmarks that report how many kernels ran.
 */
uint64_t qlora_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
