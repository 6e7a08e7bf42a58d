/*
 * qlora.h -- C ABI of libqlora: the QLoRA linear layer on NVIDIA B200 (sm_100a).
 *
 * The layer keeps a frozen weight W0 (d x k) as blockwise 4-bit NormalFloat
 * (NF4) codes, optionally with double quantisation (DQ) of the per-block
 * constants, and trains a rank-r LoRA adapter (A: r x k, B: d x r) beside it:
 *
 *     Y = X * deq(W0)^T + (alpha / r) * (X * A^T) * B^T
 *
 * Sources (page title, section):
 *   "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora): sections
 *     "How does it work?" (h = W0 x + (alpha/r) B (A x), A is r x k, B is d x r),
 *     "First, how does k-bit quantization work?" (Int8 absmax),
 *     "NF4: Choose the codebook to fit the distribution" (the 16-value table),
 *     "Quantizing and dequantizing with the codebook" (blockwise NF4, blocks of 64),
 *     "Double quantization and double dequantization" (8-bit block constants in
 *       groups of 256 with an FP32 second-level scale and a stored mean, Int8 or
 *       the "c2_FP8" E4M3 variant; the QLoRA expression; backpropagation through
 *       the reconstructed base),
 *     "Merging LoRA weights for inference" (qlora_lora_merge).
 *   "LoRA and QLoRA: Efficient Fine-Tuning of Large Language Models"
 *     (fromzero2ai.dev): section "Low-Rank Matrix Factorization".
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers into caller-owned memory.  The
 *     library never allocates device memory; scratch space is passed in as
 *     `workspace`.  Host-side structs (qlora_nf4_t) are read during the call only.
 *   - bf16 tensors are passed as uint16_t bit patterns, row-major, densely
 *     packed, 16-byte aligned.  fp32 outputs are row-major, 16-byte aligned.
 *   - Every compute call is asynchronous: it validates its arguments on the
 *     host, enqueues kernels on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns.  Results are ready when the stream reaches them.
 *   - Return value: QLORA_OK (0) or a negative qlora_status.  Nothing is
 *     enqueued when a call returns an error.  qlora_last_error() gives a
 *     human-readable reason (thread-local, valid until the next call on the
 *     same thread).
 *   - Kernels never trap.  A kernel that detects a failed internal check (a
 *     bounded wait that ran out) records it in a per-device status word that
 *     qlora_device_status() reads and clears.
 *   - No NaN/Inf handling is promised: W0 and the activations must be finite;
 *     non-finite inputs give unspecified (but memory-safe) results.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = -1,  /* null pointer, negative size, mismatched struct  */
  QLORA_ERR_UNSUPPORTED = -2,  /* valid but not implemented (blocksize != 64, ...) */
  QLORA_ERR_ALIGNMENT = -3,    /* a pointer is not 16-byte aligned               */
  QLORA_ERR_WORKSPACE = -4,    /* workspace missing or smaller than required      */
  QLORA_ERR_CUDA = -5,         /* a CUDA runtime/driver call failed               */
  QLORA_ERR_DEVICE = -6        /* a kernel reported a failed check (see status)   */
} qlora_status;

/* A cudaStream_t, passed as an opaque pointer so this header needs no CUDA headers. */
typedef void *qlora_stream_t;

/* Quantized weight.  Element i of W0 (flat row-major index, N = d*k) lies in
 * block j = i / 64 and DQ group g = j / 256.
 *   codes : ceil(N/2) bytes; byte t = code[2t] | code[2t+1] << 4 (low nibble
 *           first); an odd N pads the last high nibble with 0.
 *   absmax: M_b = ceil(N/64) fp32 block scales (the block's max |w|); used and
 *           written only when double_quant == 0 (may be NULL otherwise).
 *   c2    : M_b 8-bit quantized deviations (s_j - mean) * c1[g]; DQ only.
 *           double_quant == 1: int8, round half to even.
 *           double_quant == 2: OCP FP8 E4M3 bytes (the page's "c2_FP8"), round
 *           to nearest even, saturating at 448.
 *   c1    : G = ceil(M_b/256) fp32 second-level scales over the group, 127 /
 *           max|s - mean| (Int8) or 448 / max|s - mean| (E4M3); 1.0 for an
 *           all-zero group; DQ only.
 *   mean  : 1 fp32, the mean of all M_b block scales; DQ only.
 * All pointers are device pointers.  Alignment (checked on the host, else
 * QLORA_ERR_ALIGNMENT): codes 4 bytes for nf4_quantize / nf4_dequantize and
 * 16 bytes for qlora_linear_fwd / qlora_linear_bwd (read by TMA); c2 8 bytes;
 * absmax, c1 and mean 4 bytes. */
typedef struct {
  int64_t d;
  int64_t k;
  int32_t blocksize;     /* weights per NF4 block; only 64 is supported       */
  int32_t double_quant;  /* 0: fp32 absmax per block; 1: int8 c2 + fp32 c1;   *
                          * 2: E4M3 c2 + fp32 c1.  Every entry point accepts   *
                          * all three modes.                                   */
  uint8_t *codes;
  float *absmax;
  int8_t *c2;
  float *c1;
  float *mean;
} qlora_nf4_t;

/* Index of each buffer in qlora_nf4_sizes()'s `sizes` array. */
enum { QLORA_BUF_CODES = 0, QLORA_BUF_ABSMAX = 1, QLORA_BUF_C2 = 2, QLORA_BUF_C1 = 3, QLORA_BUF_MEAN = 4 };

/* Byte sizes of the five quantized-weight buffers for a d x k weight, and the
 * workspace nf4_quantize needs.  Buffers not used by the chosen mode get size
 * 0.  With blocksize 64 and DQ on, sizes[1..4] add up to the page's
 * 8/64 + 32/(256*64) bits per weight ("Double quantization and double
 * dequantization", the 0.373-bit accounting) plus the 4-byte mean.
 * Host-only; touches no GPU. */
int qlora_nf4_sizes(int64_t d, int64_t k, int32_t blocksize, int32_t double_quant,
                    size_t sizes[5], size_t *quant_workspace_bytes);

/* Blockwise NF4 quantisation of W0 ("Quantizing and dequantizing with the
 * codebook") followed, when q->double_quant, by double quantisation of the
 * block scales ("Double quantization and double dequantization").
 *   W0        : d*k bf16 (device, 16-byte aligned).
 *   q         : host struct describing the output buffers (device pointers,
 *               sizes from qlora_nf4_sizes).
 *   workspace : device scratch of at least quant_workspace_bytes (16-byte
 *               aligned); unused and may be NULL when DQ is off.
 * Per block: s = max |w|; code = the index of the nearest NF4 value to
 * RN32(w / s) measured by fp32 distance, the smaller index on ties; an
 * all-zero block gets the exact-zero code 7.  DQ: mean = RN32(RN64(exact sum
 * of s_j) / M_b); per group of 256, c1 = RN32(127 / max|RN32(s_j - mean)|),
 * c2_j = round_half_even(RN32(c1 * RN32(s_j - mean))).  Deterministic and
 * bit-reproducible. */
int nf4_quantize(const uint16_t *W0, const qlora_nf4_t *q, void *workspace, size_t workspace_bytes,
                 qlora_stream_t stream);

/* Largest weight (d * k elements) that nf4_quantize_noalloc accepts. */
#define QLORA_NOALLOC_MAX_WEIGHTS ((int64_t)1 << 28)

/* nf4_quantize for callers that cannot allocate device memory.  The pages have
 * no counterpart to this entry point; it is a convenience of this library.
 * Callers such as a plugin inside an application whose memory manager owns all
 * device memory, or a service that reserves its memory at start-up and must
 * not call cudaMalloc afterwards, have no workspace to pass.  This variant
 * needs none: the scratch that double quantisation uses lives in a fixed
 * array inside the library (about 8 MiB on every GPU that loads the library,
 * kept until the process exits).  Outputs are bit-identical to nf4_quantize.
 *   - d * k above QLORA_NOALLOC_MAX_WEIGHTS returns QLORA_ERR_UNSUPPORTED;
 *     use nf4_quantize with a workspace for larger weights.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, a host-side lookup that allocates nothing; it is
 *     not cached, so a context destroyed and recreated by the caller is
 *     handled).  The first call on a device may load the library's device
 *     code there; make that first call before any stream capture.
 *   - All calls share the one array, and each call clears the part that must
 *     start at zero.  Calls whose kernels may overlap on the GPU (for instance
 *     on two streams without ordering) race on it and give wrong results. */
int nf4_quantize_noalloc(const uint16_t *W0, const qlora_nf4_t *q, qlora_stream_t stream);

/* doubleDequant ("Double quantization and double dequantization"): writes the
 * reconstructed weights W_out[i] = BF16(RN32(C[code_i] * s^_j)) with
 * s^_j = RN32(RN32(c2_j / c1_g) + mean) (DQ on) or s^_j = absmax_j (DQ off).
 *   W_out : d*k bf16 (device, 16-byte aligned). */
int nf4_dequantize(const qlora_nf4_t *q, uint16_t *W_out, qlora_stream_t stream);

/* LoRA merge ("LoRA and QLoRA", "Merging LoRA weights for inference"): folds a
 * trained adapter into the weight so inference needs one path,
 *     W_out[n][c] = BF16(fma(s, acc[n][c], W^[n][c])),
 *     acc[n][c]   = sum_j B[n][j] A[j][c]   (fp32 accumulation, order unspecified),
 * with s = RN32(alpha / r) and W^ the reconstructed weight nf4_dequantize writes
 * (the bf16 weight the forward uses), rounded once to bf16 (nearest even).  So
 * X W_out^T equals the two-path qlora_linear_fwd output up to rounding.
 * Re-quantising the merged weight is nf4_quantize on W_out (the page notes
 * that merging into a quantized model costs precision).
 *   q     : the quantized base, as for qlora_linear_fwd (k % 64 == 0,
 *           d % 8 == 0, d <= 4194240; codes 16-byte aligned).
 *   A     : r x k bf16, row-major;  B : d x r bf16, row-major;  1 <= r <= 256.
 *   W_out : d x k bf16, row-major (device, 16-byte aligned); may not alias the
 *           inputs.
 * Stream-ordered; errors as for the other entry points. */
int qlora_lora_merge(const qlora_nf4_t *q, const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                     uint16_t *W_out, qlora_stream_t stream);

/* Columns of the saved adapter activation T_save (and of the internal U):
 * r rounded up to a multiple of 64. */
int32_t qlora_rank_pad(int32_t r);

/* Workspace bytes needed by qlora_linear_fwd (backward == 0) or
 * qlora_linear_bwd (backward == 1) for M tokens and a d x k weight of rank r.
 * Host-only. */
int qlora_linear_workspace_size(int64_t M, int64_t d, int64_t k, int32_t r, int32_t backward,
                                size_t *bytes);

/* Forward of the QLoRA linear layer (the QLoRA expression in "Double
 * quantization and double dequantization"; scaling alpha/r from "How does
 * alpha/r control adapter strength?"):
 *     Y = X * W^T + s * (X * A^T) * B^T,  s = RN32(alpha / r),
 * where W = doubleDequant(q) in bf16 is formed tile by tile in on-chip memory
 * and never written to device memory.
 *   X      : M x k bf16.        A : r x k bf16.       B : d x r bf16.
 *   Y      : M x d bf16 (written, not accumulated).
 *   T_save : M x qlora_rank_pad(r) bf16, receives BF16(s * X * A^T) with zero
 *            padding columns, for reuse by qlora_linear_bwd; may be NULL.
 *   workspace : qlora_linear_workspace_size(M, d, k, r, 0) bytes, 16-byte
 *            aligned (may be NULL only when that size is 0).
 * Requirements: k % 64 == 0, d % 8 == 0, 1 <= r <= 256, M >= 0 (M == 0 is a
 * no-op).  Accumulation is fp32 on the tensor cores. */
int qlora_linear_fwd(const uint16_t *X, int64_t M, const qlora_nf4_t *q, const uint16_t *A,
                     const uint16_t *B, int32_t r, float alpha, uint16_t *Y, uint16_t *T_save,
                     void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/* Backward of the QLoRA linear layer.  The base weight is frozen ("we
 * backpropagate through the reconstructed base transformations to train those
 * adapters; the stored 4-bit weights are not updated"), so there is no dW0:
 *     U  = s * dY * B                    (M x r)
 *     dX = dY * W + U * A                (M x k, bf16)
 *     dA = U^T * X  = s * (dY B)^T X     (r x k, fp32)
 *     dB = s * dY^T * (X A^T)            (d x r, fp32)
 *   T_save : the buffer filled by qlora_linear_fwd with the same X, A, r,
 *            alpha; NULL recomputes it into the workspace.
 *   dX, dA, dB are written, not accumulated.  dX may be NULL to skip it.
 *   workspace : qlora_linear_workspace_size(M, d, k, r, 1) bytes. */
int qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, int64_t M, const qlora_nf4_t *q,
                     const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                     const uint16_t *T_save, uint16_t *dX, float *dA, float *dB,
                     void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/* Grouped projections ("LoRA and QLoRA: Efficient Fine-Tuning of Large
 * Language Models" (fromzero2ai.dev), "4. Define LoRA Target Modules and
 * Config": q_proj, k_proj, v_proj and o_proj carry adapters; q, k and v read
 * the same input, as gate and up do in the MLP).  Projections that share X
 * run as one layer over their stacked rows, so X is read once per pass
 * instead of once per projection:
 *     Y_i = X W_i^T + s (X A_i^T) B_i^T,   i = 0 .. n-1,
 * each W_i quantised on its own (own blocks, groups and mean; bit for bit what
 * nf4_quantize gives for W_i alone), each with its own adapter of rank r.
 *
 * Layout (all row-major, projections in order i = 0 .. n-1):
 *   w      : the stacked weight, w.d = d[0] + ... + d[n-1]; codes, c2 (or
 *            absmax) and c1 hold the projections' buffers back to back (quantise
 *            W_i with nf4_quantize into its slice: codes + (rows before i) * k / 2,
 *            c2 + (rows before i) * k / 64, c1 + (rows before i) * k / 16384);
 *            w.mean points to n means, one per projection.
 *   A      : (n r) x k, the A_i stacked.        B : w.d x r, the B_i stacked.
 *   Y, dY  : M x w.d, Y_i in columns [rows before i, + d[i]).
 *   T_save : M x qlora_rank_pad(n r), T_i = BF16(s X A_i^T) in columns [i r, (i+1) r).
 *   dA     : (n r) x k (fp32), the dA_i stacked.   dB : w.d x r (fp32), the dB_i stacked.
 *   dX     : M x k, the sum over the projections.
 * Requirements: 1 <= n <= 4; d[i] a multiple of 256 for i < n - 1; n r <= 256;
 * r % 8 == 0 when n > 1; otherwise as for qlora_linear_fwd / _bwd. */
#define QLORA_MAX_GROUP 4
typedef struct {
  int32_t n;                   /* projections sharing the input, 1..4 */
  int64_t d[QLORA_MAX_GROUP];  /* output rows of each                 */
  qlora_nf4_t w;               /* the stacked weight                  */
} qlora_nf4_group_t;

/* Workspace bytes of the grouped forward (backward == 0) or backward. */
int qlora_grouped_workspace_size(int64_t M, const qlora_nf4_group_t *g, int32_t r, int32_t backward,
                                 size_t *bytes);

/* Forward of n projections sharing X (layout above); s = RN32(alpha / r). */
int qlora_linear_fwd_grouped(const uint16_t *X, int64_t M, const qlora_nf4_group_t *g, const uint16_t *A,
                             const uint16_t *B, int32_t r, float alpha, uint16_t *Y, uint16_t *T_save,
                             void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/* Backward of the grouped forward: dX = sum_i (dY_i W_i + s (dY_i B_i) A_i),
 * dA_i = s (dY_i B_i)^T X, dB_i = s dY_i^T (X A_i^T). */
int qlora_linear_bwd_grouped(const uint16_t *dY, const uint16_t *X, int64_t M, const qlora_nf4_group_t *g,
                             const uint16_t *A, const uint16_t *B, int32_t r, float alpha, const uint16_t *T_save,
                             uint16_t *dX, float *dA, float *dB, void *workspace, size_t workspace_bytes,
                             qlora_stream_t stream);

/* Adapter dropout ("LoRA and QLoRA: Efficient Fine-Tuning of Large Language
 * Models" (fromzero2ai.dev), "Python Implementation: Fine-Tuning with PEFT and
 * BitsAndBytes", step 4: lora_dropout = 0.05).  Dropout acts on the adapter's
 * input only; the frozen base path sees X unchanged:
 *     Y = X W^T + s (drop(X) A^T) B^T,   drop(X) = X . keep / (1 - p).
 * The keep decision of element i = m * k + j of X comes from the counter-based
 * generator Philox4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy as
 * 1, 2, 3", SC 2011): output word i % 4 at counter (i / 4 low 32 bits, i / 4
 * high 32 bits, offset low, offset high) under key (seed low, seed high);
 * with u = (word >> 8) * 2^-24 the element is kept when u >= p.  Kept values
 * are scaled by RN32(1 / RN32(1 - p)).  The backward regenerates the same
 * decisions from (seed, offset), so no mask is stored between the calls; use
 * a new offset (or seed) for every training step. */
typedef struct {
  float p;           /* drop probability, 0 <= p < 1 (0: the plain layer, bit for bit) */
  uint64_t seed;     /* generator key                                                  */
  uint64_t offset;   /* generator counter offset                                       */
} qlora_dropout_t;

/* Writes the keep bitmask of an M x k activation: bit b of keep_bits[w] is the
 * decision for flat element 32 w + b (1 = kept); ceil(M * k / 32) words,
 * bits past M * k are 0.  keep_bits: device, 4-byte aligned. */
int qlora_dropout_mask(int64_t M, int64_t k, const qlora_dropout_t *drop, uint32_t *keep_bits,
                       qlora_stream_t stream);

/* Workspace bytes of qlora_linear_fwd_dropout (backward == 0) or
 * qlora_linear_bwd_dropout (backward == 1): the plain layer's workspace plus
 * the keep bitmask of X (M * k / 8 bytes, rounded up to 256).  Host-only. */
int qlora_linear_dropout_workspace_size(int64_t M, int64_t d, int64_t k, int32_t r, int32_t backward,
                                        size_t *bytes);

/* qlora_linear_fwd with adapter dropout `drop` (NULL or p == 0: no dropout).
 * T_save receives BF16(s * drop(X) * A^T).  Other arguments and requirements
 * as for qlora_linear_fwd; workspace from qlora_linear_dropout_workspace_size.
 * A probability outside [0, 1) returns QLORA_ERR_INVALID_ARG. */
int qlora_linear_fwd_dropout(const uint16_t *X, int64_t M, const qlora_nf4_t *q, const uint16_t *A,
                             const uint16_t *B, int32_t r, float alpha, const qlora_dropout_t *drop, uint16_t *Y,
                             uint16_t *T_save, void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/* qlora_linear_bwd for the dropout forward with the same `drop`:
 *     U  = s dY B,   dX = dY W + (U A) . keep / (1 - p),
 *     dA = U^T drop(X),   dB = s dY^T (drop(X) A^T).
 * T_save: the buffer the dropout forward filled (NULL recomputes it with the
 * same mask).  Workspace from qlora_linear_dropout_workspace_size. */
int qlora_linear_bwd_dropout(const uint16_t *dY, const uint16_t *X, int64_t M, const qlora_nf4_t *q,
                             const uint16_t *A, const uint16_t *B, int32_t r, float alpha,
                             const qlora_dropout_t *drop, const uint16_t *T_save, uint16_t *dX, float *dA, float *dB,
                             void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/* The library's NF4 table C[0..15] (fp32, ascending) copied to host memory. */
int qlora_nf4_codebook(float out[16]);

/* Synchronizes `stream`, then reads and clears the current device's status
 * word: *status = 0 when no kernel reported a failed check since the last
 * read, otherwise the code of the first failure.  Returns QLORA_ERR_DEVICE
 * when *status != 0. */
int qlora_device_status(qlora_stream_t stream, int32_t *status);

/* Self-test of the device-side failure path (not a paper operation).  Every
 * wait inside the library's kernels is bounded; when one runs out the kernel
 * records a code in the status word, releases what it holds (TMEM) and
 * returns, so the context stays usable.  This call exercises exactly that path
 * without any fault: one CTA takes 32 TMEM columns and waits on a barrier that
 * nothing arrives at, for limit_us microseconds (1 .. 1000000).  It then
 * records code 7 in the status word, frees the TMEM and writes 2 to *result
 * (device int32, 4-byte aligned).  qlora_device_status afterwards returns
 * QLORA_ERR_DEVICE with status 7 and clears it. */
int qlora_selftest_wait_timeout(uint32_t limit_us, int32_t *result, qlora_stream_t stream);

/* Tracing: every kernel launch of the library belongs to one class. */
enum {
  QLORA_KC_QUANT = 0,      /* blockwise NF4 code search + packing            */
  QLORA_KC_DQ_CONST = 1,   /* exact mean and 8-bit quantisation of the scales */
  QLORA_KC_DEQUANT = 2,    /* standalone doubleDequant                         */
  QLORA_KC_FWD_GEMM = 3,   /* fused dequant + LoRA forward GEMM                */
  QLORA_KC_BWD_GEMM = 4,   /* fused dequant + LoRA backward (dX) GEMM          */
  QLORA_KC_LORA_GEMM = 5,  /* low-rank GEMMs: s X A^T, s dY B, dA, dB          */
  QLORA_KC_AUX = 6,        /* split-K reductions, transposes                   */
  QLORA_KC_COUNT = 7
};

/* Turn per-launch device timing on (1) or off (0).  While on, each launch is
 * bracketed by two CUDA events on the call's stream (pooled; no allocation in
 * steady state).  Launch counting is always on.  Host-only. */
int qlora_profile_enable(int on);

/* Wait for the recorded events, write the summed device milliseconds per
 * kernel class (ms, may be NULL) and the launches per class since the last
 * read (launches, may be NULL), then reset both.  Not a paper operation: a
 * tracing aid for benchmarks. */
int qlora_profile_read(double ms[QLORA_KC_COUNT], int64_t launches[QLORA_KC_COUNT]);

/* Reason for the last error returned on this thread ("" if none). */
const char *qlora_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
