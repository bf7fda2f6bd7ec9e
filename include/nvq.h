/*
 * nvq.h: C ABI of the group-wise affine quantized products for NVIDIA B200 (sm_100a).
 *
 * The format (nuvec documentation, "Docs / Quantization", section "Affine"):
 * a weight row is divided into runs of group_size consecutive values (32, 64
 * or 128); a run stores one scale and one bias, and every value is stored as a
 * `bits`-wide unsigned integer, several to a uint32 word, with
 *     w ~= scale * code + bias.
 * Code j of a word sits at bits [j*bits, (j+1)*bits). Scales and biases have
 * the weights' dtype (nuvec crate docs, "Structs": Quantized). This library
 * quantizes and dequantizes at bits 1, 2, 4 and 8 (the widths that divide 32)
 * and runs products at bits 2, 4 and 8.
 *
 * Layouts (all dense, row-major, no padding):
 *   weights [rows, cols], grouped along cols:
 *     codes  uint32 [rows, cols * bits / 32]
 *     scales dtype  [rows, cols / group_size]
 *     biases dtype  [rows, cols / group_size]
 *   For products, transpose = 1 means the weights are stored [N, K] (row n holds
 *   output feature n, grouped along K) and y = x . w^T; transpose = 0 means they
 *   are stored [K, N], grouped along N, and y = x . w.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is a DEVICE pointer (unless stated otherwise) owned
 *     by the caller; the library allocates no device memory and never
 *     synchronises the stream (except nv_gather_qmm_flags and
 *     nv_pipeline_error, whose job is to read a word back). The only state kept
 *     between calls is the sticky pipeline error word (nv_pipeline_error) and
 *     the fixed routing array of nv_gather_qmm_noalloc. All work is enqueued
 *     on `stream` (NULL = the legacy default stream), in call order.
 *   - Device pointers must be 16-byte aligned.
 *   - Argument errors are found on the host before anything is launched and
 *     are returned synchronously: NV_ERR_INVALID_ARG (a shape, pointer or
 *     alignment is wrong), NV_ERR_UNSUPPORTED (a valid-looking combination this
 *     library does not implement, e.g. bits = 3), NV_ERR_WORKSPACE (too small).
 *     A failed launch returns NV_ERR_CUDA. Nothing traps on the device: data
 *     errors found while running (an expert id out of range) set flag bits that
 *     nv_gather_qmm_flags reads.
 *   - Results are deterministic: the same call on the same inputs gives the same
 *     bits, run to run (nuvec crate docs, section "Determinism").
 */
#ifndef NVQ_H
#define NVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* The same type as cudaStream_t. */
typedef struct CUstream_st* nv_stream_t;

typedef enum nv_status {
    NV_OK = 0,
    NV_ERR_INVALID_ARG = 1,
    NV_ERR_UNSUPPORTED = 2,
    NV_ERR_WORKSPACE = 3,
    NV_ERR_CUDA = 4
} nv_status;

typedef enum nv_dtype {
    NV_F32 = 0,  /* IEEE binary32 */
    NV_BF16 = 1  /* bfloat16 */
} nv_dtype;

/* Largest row count for which row_exact holds: each row's output is then
 * bitwise equal to a one-row call (nuvec crate docs: constant
 * ROW_INDEPENDENT_ROWS and function with_row_exact; "Docs / Quantization",
 * section "Products on the GPU", which sends at most 8 rows to the
 * matrix-vector kernels). */
#define NV_ROW_INDEPENDENT_ROWS 8

/* Device anomaly flags written by nv_gather_qmm into its workspace. */
#define NV_FLAG_EXPERT_OUT_OF_RANGE 0x1u /* an rhs id >= E: that row's output is zero */
#define NV_FLAG_NOT_SORTED 0x2u          /* sorted = 1 but rhs ids decrease somewhere */
#define NV_FLAG_TOKEN_OUT_OF_RANGE 0x4u  /* an lhs id >= x_rows: that row's output is zero */

/* Readable text for a status code (static storage, never NULL). */
const char* nv_status_string(nv_status s);

/*
 * Affine quantizer ("Docs / Quantization", section "Affine", and its first
 * example: affine mode, group size 64, 4 bits).
 *
 * w       [rows, cols] in `dt` (NV_F32 or NV_BF16), grouped along cols.
 * codes   uint32 [rows, cols * bits / 32] (output).
 * scales, biases  `dt` [rows, cols / group_size] (outputs).
 * Per group, in IEEE fp32 with round-to-nearest-even at every step:
 *   scale = (max - min) / (2^bits - 1), bias = min,
 *   code  = clamp(round_half_even((w - bias) / scale), 0, 2^bits - 1),
 *   a constant group (scale == 0) gets code 0; scale and bias are stored in
 *   `dt` (bf16 by round-to-nearest-even). The minimum of a group holding both
 *   -0 and +0 is -0, the maximum +0. Inputs must be finite.
 * group_size in {32, 64, 128}; bits in {1, 2, 4, 8}; cols % group_size == 0.
 * Bits 3, 5 and 6 return NV_ERR_UNSUPPORTED (no packing of widths that do not
 * divide 32 is specified), any other width NV_ERR_INVALID_ARG.
 */
nv_status nv_quantize_affine(const void* w, nv_dtype dt, int64_t rows, int64_t cols,
                             int group_size, int bits, uint32_t* codes, void* scales,
                             void* biases, nv_stream_t stream);

/*
 * Dequantizer: the weights back from their codes ("Docs / Quantization",
 * section "Affine": w ~= scale * code + bias; the nuvec crate docs list
 * dequantize beside the quantizer).
 *
 * codes   uint32 [rows, cols * bits / 32]; scales, biases `dt` [rows,
 *         cols / group_size] (inputs, the layout nv_quantize_affine writes).
 * w       `dt` [rows, cols] (output): w[r, c] = scale * code + bias, the exact
 *         value rounded once (to nearest, ties to even) to `dt`: one fused
 *         multiply-add in fp32 or in bf16. Deterministic.
 * dt in {NV_F32, NV_BF16}; group_size in {32, 64, 128}; bits in {1, 2, 4, 8};
 * cols % group_size == 0; rows == 0 is a no-op returning NV_OK. Bits 3, 5, 6
 * return NV_ERR_UNSUPPORTED.
 */
nv_status nv_dequantize_affine(const uint32_t* codes, const void* scales, const void* biases,
                               nv_dtype dt, int64_t rows, int64_t cols, int group_size,
                               int bits, void* w, nv_stream_t stream);

/*
 * Floating-point quantization modes ("Docs / Quantization", section
 * "Floating-point formats": every value stored as a small float with one
 * shared scale per group, scales stored as uint8 codes, no biases; the
 * dequantized weights are bfloat16; quantized_matmul(q, true) returns x's
 * dtype). The pages' table of the formats did not survive; the modes are the
 * published definitions of their names:
 *   NV_MXFP4  E2M1 codes (4 bits), one E8M0 scale (2^(s - 127)) per 32 values;
 *   NV_MXFP8  E4M3 codes (8 bits, no infinities), one E8M0 scale per 32;
 *   NV_NVFP4  E2M1 codes, one E4M3 scale per 16 values.
 * Codes pack like the affine codes (code j of a uint32 at bits [j*b, (j+1)*b)).
 * Parity with MLX's own quantizer (which the pages say these equal) is not
 * established: the scale rule used here is written out at nv_quantize_fp.
 */
typedef enum nv_fp_mode {
    NV_MXFP4 = 1,
    NV_MXFP8 = 2,
    NV_NVFP4 = 3
} nv_fp_mode;

/*
 * Quantizer of the floating-point modes.
 * w       [rows, cols] in dt (NV_F32 or NV_BF16), grouped along cols
 *         (input); cols a multiple of 32.
 * codes   uint32 [rows, cols * b / 32] (b = 4, or 8 for NV_MXFP8), output.
 * scales  uint8 [rows, cols / group] (group 32, or 16 for NV_NVFP4), output.
 * Per group: amax = max |w|. MX modes: scale 2^(floor(log2 amax) - emax),
 * emax = 2 (E2M1) or 8 (E4M3), code clamped to 0..254 (0 for an all-zero
 * group); each code is w / scale rounded to the nearest element (ties to the
 * even mantissa, saturated at the largest finite one: 6 or 448). NVFP4: scale
 * = fl32(amax / 6) rounded to E4M3 the same way; codes from fl32(w / scale),
 * all 0 when the scale is 0. Bit-exact with the oracle. Deterministic.
 * Errors: NV_ERR_INVALID_ARG (mode, shape, null or unaligned pointers;
 * 16-byte alignment of w and codes), NV_ERR_UNSUPPORTED (dtype).
 */
nv_status nv_quantize_fp(const void* w, nv_dtype dt, int64_t rows, int64_t cols, nv_fp_mode mode,
                         uint32_t* codes, uint8_t* scales, nv_stream_t stream);

/*
 * Dequantizer of the floating-point modes: out bf16 [rows, cols] (16-byte
 * aligned), element value times scale value, rounded once to bf16 (exact
 * unless the product underflows bf16). Errors as nv_quantize_fp.
 */
nv_status nv_dequantize_fp(const uint32_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                           nv_fp_mode mode, void* out, nv_stream_t stream);

/*
 * Product with floating-point-mode weights stored [N, K] (codes and scales
 * as nv_quantize_fp writes them for rows = N, cols = K): y [M, N] = x [M, K]
 * . w^T, bf16 x and y (dt must be NV_BF16, else NV_ERR_UNSUPPORTED); K a
 * multiple of 32. M <= 8: a matrix-vector kernel (every row computed as in a
 * one-row call: row-exact); M > 8 with K a multiple of 64: the tiled
 * tcgen05 kernel with the weights dequantized exactly into its bf16 tiles.
 * Tolerance as nv_qmm. Errors as nv_quantize_fp; M == 0 or N == 0 is a no-op.
 */
nv_status nv_qmm_fp(const void* x, nv_dtype dt, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
                    const uint8_t* scales, nv_fp_mode mode, void* y, nv_stream_t stream);

/*
 * Quantized product ("Docs / Quantization", sections "Affine" (example
 * x.quantized_matmul(&q, true)) and "Products on the GPU").
 *
 * x      [M, K] in `dt`; y [M, N] in `dt` (the output follows x's dtype).
 * transpose = 1: weights stored [N, K] (codes [N, K*bits/32], scales/biases
 *   [N, K/group_size]), y = x . w^T.  transpose = 0: weights stored [K, N]
 *   (codes [K, N*bits/32], scales/biases [K, N/group_size]), y = x . w.
 * Scales and biases have dtype `dt` too: supported pairs are (F32, F32) and
 * (BF16, BF16). Accumulation is fp32.
 * row_exact = 1 (M <= NV_ROW_INDEPENDENT_ROWS, else NV_ERR_INVALID_ARG): each
 *   row's result equals, bit for bit, the same call with that row alone (M = 1).
 * Routing is a pure function of (M, N, K, dt, group_size, bits, transpose,
 * row_exact): matrix-vector kernels for M <= 8, tensor-core tiles above.
 * bits in {2, 4, 8}; 1-bit codes return NV_ERR_UNSUPPORTED here.
 * M == 0 or N == 0 is a no-op returning NV_OK.
 */
nv_status nv_qmm(const void* x, nv_dtype dt, int64_t M, int64_t K, int64_t N,
                 const uint32_t* codes, const void* scales, const void* biases, int group_size,
                 int bits, int transpose, int row_exact, void* y, nv_stream_t stream);

/*
 * Batched quantized product: B items of L rows each, all with the same
 * weights ("Docs / Quantization", section "Products on the GPU"; nuvec crate
 * docs, section "Determinism": batch items of quantized products give each
 * item the bits of its own call, the split-K partitions being counted per
 * item).
 *
 * x      [B, L, K] in `dt`; y [B, L, N] in `dt`; weights as for nv_qmm.
 * Routing (kernel, tile shape and split-K partition count) is the function of
 * (L, N, K, dt, group_size, bits, transpose) that nv_qmm applies to an L-row
 * call, so that item b of the result is bitwise equal to
 * nv_qmm(x[b], M = L, row_exact = 0). B * L == 0 or N == 0 is a no-op
 * returning NV_OK; B * L above 2^40 returns NV_ERR_INVALID_ARG.
 */
nv_status nv_qmm_batched(const void* x, nv_dtype dt, int64_t B, int64_t L, int64_t K, int64_t N,
                         const uint32_t* codes, const void* scales, const void* biases,
                         int group_size, int bits, int transpose, void* y, nv_stream_t stream);

/*
 * K-partitions (split-K; "Docs / Quantization", section "Products on the
 * GPU": split-K when the output is small but the inner dimension long) that
 * nv_qmm uses for an M-row product: 1 when it does not split. Host only, no
 * launch. Products of more than 8 bf16 rows (either layout) split K over a
 * cluster of up to 8 CTAs when their 128 x BN output tiles would occupy fewer
 * than half of the SMs and K holds at least 8 steps of 64; the partial sums
 * are reduced in a fixed order, so results stay deterministic.
 */
int nv_qmm_splits(int64_t M, int64_t K, int64_t N, int bits, int group_size, int transpose,
                  nv_dtype dt);

/* Bytes of device workspace nv_gather_qmm needs for R pairs and E experts. */
size_t nv_gather_qmm_workspace_size(int64_t R, int64_t E);

/*
 * Mixture-of-experts product ("Docs / Quantization", section "Mixture of
 * experts": every row is multiplied by its own expert's quantized weights,
 * read in place, with no gathered copy of the weights).
 *
 * x        [x_rows, K] in `dt`.
 * lhs_idx  uint32 [R] or NULL: pair r reads row lhs_idx[r] of x (NULL: row r).
 * rhs_idx  uint32 [R]: pair r uses expert rhs_idx[r] in [0, E).
 * codes/scales/biases: E experts back to back, each laid out as for nv_qmm
 *   (transpose = 1: [E, N, K]; transpose = 0: [E, K, N]).
 * y        [R, N] in `dt`: row r is x[lhs[r]] times expert rhs[r], in pair order.
 * sorted   = 1 is the caller's promise that rhs_idx never decreases (the
 *   option sorted_indices); a broken promise is flagged (NV_FLAG_NOT_SORTED)
 *   and the result is still correct.
 * row_exact = 1: each row's output is bitwise equal to nv_qmm(M = 1) of that
 *   row with its expert's weights.
 * workspace: device memory of at least nv_gather_qmm_workspace_size(R, E)
 *   bytes, 16-byte aligned, owned by the caller; its contents on entry do not
 *   matter. Calls that share a workspace must not overlap on the GPU.
 */
nv_status nv_gather_qmm(const void* x, nv_dtype dt, int64_t x_rows, int64_t K,
                        const uint32_t* lhs_idx, const uint32_t* rhs_idx, int64_t R, int64_t E,
                        int64_t N, const uint32_t* codes, const void* scales, const void* biases,
                        int group_size, int bits, int transpose, int sorted, int row_exact,
                        void* workspace, size_t workspace_bytes, void* y, nv_stream_t stream);

/*
 * Mixture-of-experts product with full-precision experts, gather_mm (the
 * unquantized companion of gather_qmm; "Docs / Quantization", section
 * "Mixture of experts", and the nuvec crate docs).
 *
 * x, lhs_idx, rhs_idx, sorted, workspace, y: as for nv_gather_qmm (the same
 *   routing and workspace size; nv_gather_qmm_flags reads its flags).
 * w        bf16 [E, N, K]: expert e's weights, row n = output feature n.
 * y[r, n] = sum_k x[lhs[r], k] * w[rhs[r], n, k], fp32 accumulation, stored
 *   in bf16; pairs with an out-of-range id get zero rows and a flag.
 * dt must be NV_BF16, K a multiple of 64 and x_rows * K below 2^35
 * (NV_ERR_UNSUPPORTED otherwise).
 */
nv_status nv_gather_mm(const void* x, nv_dtype dt, int64_t x_rows, int64_t K,
                       const uint32_t* lhs_idx, const uint32_t* rhs_idx, int64_t R, int64_t E,
                       int64_t N, const void* w, int sorted, void* workspace,
                       size_t workspace_bytes, void* y, nv_stream_t stream);

/* Bytes of device workspace nv_moe_swiglu needs for T tokens with topk
 * experts each, E experts, hidden size I and model size K (0 for invalid
 * sizes). */
size_t nv_moe_swiglu_workspace_size(int64_t T, int64_t topk, int64_t E, int64_t I, int64_t K);

/*
 * The routed SwiGLU mixture-of-experts block over quantized experts
 * ("Docs / Quantization", section "Mixture of experts": gather_qmm multiplies
 * every row by its own expert's quantized weights without gathering them; the
 * block around it is the gate and up products, silu(gate) * up, the down
 * product, and the sum over each token's experts):
 *   y[t] = sum_j rw[t, j] * down_e( silu(gate_e(x[t])) * up_e(x[t]) ),
 *   e = ids[t, j], silu(z) = z / (1 + e^-z),
 * in one routed pass: the pairs (t, j) are sorted by expert once, the gate
 * and up products run on the grouped tensor-core kernel (the up product's
 * epilogue applies silu(gate) * up), the down product runs on the pairs'
 * hidden rows, and the combine sums each token's experts in j order (fp32,
 * rounded once to bf16).
 *
 * x       bf16 [T, K]; ids uint32 [T, topk]; rw fp32 [T, topk] (routing weights).
 * gate_*, up_*: quantized [E, I, K] (codes [E, I, K*bits/32], scales/biases
 *   [E, I, K/group_size], grouped along K); down_*: quantized [E, K, I].
 * y       bf16 [T, K] (output).
 * workspace: >= nv_moe_swiglu_workspace_size(T, topk, E, I, K) bytes, 16-byte
 *   aligned, caller-owned; it holds the routing tables and flags (the flags
 *   first: nv_gather_qmm_flags(workspace, ...) reads them), the hidden rows
 *   and the down products. Calls sharing a workspace must not overlap.
 * An expert id >= E contributes nothing to y and sets NV_FLAG_EXPERT_OUT_OF_RANGE.
 * dt must be NV_BF16, K and I multiples of 128 with (K / group_size) and
 * (I / group_size) multiples of 8, 1 <= topk <= 64, E <= 1023
 * (NV_ERR_UNSUPPORTED otherwise); bits in {2, 4, 8}. T == 0 is a no-op.
 */
nv_status nv_moe_swiglu(const void* x, nv_dtype dt, int64_t T, int64_t K, const uint32_t* ids,
                        const float* rw, int topk, int64_t E, int64_t I,
                        const uint32_t* gate_codes, const void* gate_scales,
                        const void* gate_biases, const uint32_t* up_codes, const void* up_scales,
                        const void* up_biases, const uint32_t* down_codes,
                        const void* down_scales, const void* down_biases, int group_size,
                        int bits, void* workspace, size_t workspace_bytes, void* y,
                        nv_stream_t stream);

/* Copy the anomaly flags of the last nv_gather_qmm (or nv_gather_mm) that used
 * `workspace` into *host_flags (a HOST pointer). Synchronises `stream`. */
nv_status nv_gather_qmm_flags(const void* workspace, uint32_t* host_flags, nv_stream_t stream);

/*
 * Read and clear the sticky error word of the asynchronous (TMA / tensor-core)
 * pipelines into *host_code (a HOST pointer): 0 when every wait inside the
 * kernels completed; otherwise a nonzero code naming the first wait that gave
 * up after its time limit (2 s; the launch that owned it then stopped early,
 * and its outputs are not valid). A wait that gave up affects only its own
 * launch: later launches run normally whether or not the word was read.
 * Synchronises the device. A diagnostic of this library (the pages have no
 * counterpart): nothing on the device traps or spins without a limit.
 */
nv_status nv_pipeline_error(uint32_t* host_code);

/*
 * Self-test of the bounded waits behind nv_pipeline_error (a diagnostic of
 * this library; the pages have no counterpart). Enqueues on `stream` one
 * kernel whose single thread waits, through the pipelines' own bounded wait,
 * on a barrier that nothing completes; after limit_us microseconds the wait
 * gives up, records code 0x5E in the error word and the kernel returns, so
 * that nv_pipeline_error then reports 0x5E. limit_us in [1, 2000000], else
 * NV_ERR_INVALID_ARG. Writes no caller memory.
 */
nv_status nv_pipeline_selftest(uint32_t limit_us, nv_stream_t stream);

/*
 * nv_gather_qmm without a workspace argument, for callers that cannot allocate
 * device memory (a host runtime that owns all memory and forbids allocation
 * on its hot path, a plugin without an allocator, a real-time loop where
 * cudaMalloc may block). The pages have no counterpart: this is an addition of
 * this library. Arguments and results as nv_gather_qmm.
 * The routing tables live in one fixed device array built into the library
 * (about 200 KB, kept on every GPU that loads the library until exit):
 * R <= 32768 pairs and E <= 256 experts, else NV_ERR_WORKSPACE before any
 * launch. The first call on a device looks the array's address up (with that
 * device current) and should come before any stream capture; the address is
 * kept for the life of the process, so a cudaDeviceReset between calls
 * leaves a stale address behind (do not reset a device this entry point has
 * been called on). Every call shares the array: calls that may overlap on
 * the GPU race and must be serialised by the caller (one stream, or events).
 * Nothing in the array needs to start at zero (each call writes every entry
 * it reads). The anomaly flags of nv_gather_qmm are written into the array
 * too and cannot be read back (nv_gather_qmm_flags needs a workspace
 * pointer); a caller that needs them uses nv_gather_qmm. No device memory is
 * allocated or freed.
 */
nv_status nv_gather_qmm_noalloc(const void* x, nv_dtype dt, int64_t x_rows, int64_t K,
                                const uint32_t* lhs_idx, const uint32_t* rhs_idx, int64_t R,
                                int64_t E, int64_t N, const uint32_t* codes, const void* scales,
                                const void* biases, int group_size, int bits, int transpose,
                                int sorted, int row_exact, void* y, nv_stream_t stream);

/* Name of the CUDA error behind the last NV_ERR_CUDA this thread received
 * (static storage; "cudaSuccess" if none). Diagnostics only. */
const char* nv_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* NVQ_H */
