/*
 * qlr.h -- C ABI of the quantised-base + LoRA linear library for NVIDIA B200 (sm_100a).
 *
 * The layer is  Y = X dequant(Wq)^T + s (P(X) A^T) B^T  with a frozen low-bit base
 * weight Wq and a trainable low-rank adapter (A, B); P is the identity (QLoRA, LQ-LoRA)
 * or the group mean over L input channels (QA-LoRA).
 *
 * Conventions shared by every entry point
 *   - Return value: QLR_OK (0) or a negative QLR_ERR_* code.  Arguments are validated on the
 *     host before anything is launched; an invalid call launches nothing and leaves every
 *     buffer untouched.
 *   - Pointers are caller-owned DEVICE memory unless stated otherwise; the library keeps no
 *     allocation of its own.  Scratch space is passed in as `workspace` (device memory of at
 *     least the size the matching *_workspace_bytes query returns, 256-byte aligned).
 *   - bf16 and fp16 buffers are passed as uint16_t bit patterns.  Matrices are row-major and
 *     densely packed (leading dimension = number of columns); every pointer must be 16-byte
 *     aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  All work is
 *     asynchronous on that stream.
 *   - `status` (optional, may be NULL) is a device int32 that kernels set to a negative
 *     QLR_ERR_* code when they detect a fault at run time (non-finite weights in a quantiser,
 *     a pipeline wait that ran past its bound).  The caller zeroes it and reads it after
 *     synchronising the stream.  Kernels never trap.
 *   - Shapes: W is [N, K] (out_features x in_features), X is [M, K], Y is [M, N], A is [r, Ka]
 *     (Ka = K, or K / group for the pooled adapter), B is [N, r].
 */
#ifndef QLR_H
#define QLR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLR_API __attribute__((visibility("default")))
#else
#define QLR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  QLR_OK = 0,
  QLR_ERR_ARG = -1,         /* null pointer, unknown enum value, negative size */
  QLR_ERR_SHAPE = -2,       /* sizes the kernels do not support (see each call) */
  QLR_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned */
  QLR_ERR_UNSUPPORTED = -4, /* a valid combination this build does not implement */
  QLR_ERR_NONFINITE = -5,   /* set in *status by a quantiser that met a NaN or infinity */
  QLR_ERR_TIMEOUT = -6,     /* set in *status by a pipelined kernel whose wait ran out */
  QLR_ERR_CUDA = -7,        /* a CUDA runtime/driver call failed */
  QLR_ERR_WORKSPACE = -8    /* workspace missing or smaller than the query's answer */
};

enum { QLR_FMT_NFK = 1, QLR_FMT_INT4G = 2 };

/* Parts of a quantised weight, for qlr_qweight_part_bytes. */
enum { QLR_PART_CODES = 0, QLR_PART_C1 = 1, QLR_PART_C1_FP8 = 2, QLR_PART_S2 = 3,
       QLR_PART_SCALE = 4, QLR_PART_ZERO = 5 };

/*
 * A quantised base weight.  The struct is plain data owned by the caller; its pointers are
 * caller-allocated device buffers of the sizes qlr_qweight_part_bytes reports.
 *
 * NF-k (fmt = QLR_FMT_NFK; QLoRA explainer, "Innovation 1: 4-bit NormalFloat (NF4)" and
 * "Innovation 2: Double Quantization"; LQ-LoRA abstract for k = 2, 3 and block 64/128):
 *   codes   packed k-bit codes of the row-major flattened W.  k=4: two per byte, element 2j in
 *           the low nibble; k=2: four per byte, element 4j+t at bits 2t..2t+1; k=3: per 32
 *           codes three little-endian uint32 bit planes (word p holds bit p of code t at bit t).
 *   c1      fp32 absmax per block of `block` consecutive weights (only when dq_block == 0).
 *   c1_fp8  E4M3 byte per block: c1 / s2 rounded to nearest even, saturated (dq_block > 0).
 *   s2      fp32 per group of dq_block blocks: max(c1 in group) / 448 (dq_block > 0).
 * INT4 group (fmt = QLR_FMT_INT4G; QA-LoRA abstract, group-wise INT4):
 *   codes   packed like NF-4, row-major [N, K];
 *   scale   fp16 [N, K / group];  zero  fp16 [N, K / group] (integer before a merge).
 */
typedef struct qlr_qweight {
  int32_t fmt;
  int32_t bits;
  int32_t block;
  int32_t dq_block;
  int32_t group;
  int32_t reserved;
  int64_t N;
  int64_t K;
  uint8_t* codes;
  float* c1;
  uint8_t* c1_fp8;
  float* s2;
  uint16_t* scale;
  uint16_t* zero;
} qlr_qweight;

/* Static text for a return code.  Never NULL. */
QLR_API const char* qlr_error_string(int code);

/* Library ABI version (major * 100 + minor). */
QLR_API int qlr_version(void);

/* Number of bytes a part of a quantised weight occupies (0 when the format has no such part,
 * negative QLR_ERR_* for invalid arguments).  Pure host arithmetic. */
QLR_API int64_t qlr_qweight_part_bytes(int fmt, int64_t N, int64_t K, int bits, int block, int dq_block, int group,
                               int part);

/* The fp32 NF-k levels the library uses (2^bits values, ascending), derived on the host from
 * an inverse normal CDF (AS241) by the quantile construction: positive levels at 2^(k-1)
 * evenly spaced probabilities from delta toward 1/2, negative levels at 2^(k-1)-1, an exact
 * zero, divided by the quantile at delta, delta = 1 - (1/(2(2^k-1)) + 1/(2^(k+1)))/2.
 * (QLoRA explainer, "Innovation 1: 4-bit NormalFloat (NF4)": equal share of a normal
 * distribution per bin.)  `out` is HOST memory of 2^bits floats. */
QLR_API int qlr_nf_levels(int bits, float* out);

/* The decision table the NF-k quantiser uses for its nearest-level search (QLoRA explainer,
 * "Background: what is quantization?": each normalised weight u = fp32(w / absmax) in [-1, 1] takes
 * the nearest level; ties go to the lower index).  For fixed levels that choice is a step function of
 * u, so it is fixed by 2^bits - 1 fp32 thresholds.  The table splits [-1, 1] into 33 cells, cell
 * k = round-half-even(16 u) + 16 (computed as the bits of fma(u, 16, 1.5 * 2^23 + 16) minus those of
 * 1.5 * 2^23), each holding at most one threshold:  code(u) = base[k] + (u >= threshold[k]), with
 * threshold[k] = +inf for a cell without one.  `threshold` and `base` are HOST arrays of 33 entries.
 * Returns QLR_ERR_ARG for bits outside 2 .. 4 and QLR_ERR_UNSUPPORTED if a cell would hold two
 * thresholds (it does not for the NF-2/3/4 levels of qlr_nf_levels).  Pure host arithmetic. */
QLR_API int qlr_nf_decision_table(int bits, float* threshold, int32_t* base);

/*
 * Blockwise NF-k quantisation with optional double quantisation of the constants.
 * (QLoRA explainer, "Background: what is quantization?", "Innovation 1", the page's code
 * sketch for absmax / nearest level, "Innovation 2: Double Quantization".)
 *   W         fp32 [N, K] device, read only.
 *   bits      2, 3 or 4;  block  64 or 128;  dq_block  256 or 0.
 *   out       describes the destination buffers (out->fmt/bits/block/dq_block/N/K are checked
 *             against the arguments); codes, and c1 or (c1_fp8, s2), are written.
 * Per element: u = fp32(w / absmax) (IEEE division), code = first index minimising
 * fp32 |u - level|; an all-zero block takes the zero level.  Non-finite W sets
 * *status = QLR_ERR_NONFINITE (outputs are then unspecified).
 * Shapes: N*K a multiple of 128 (so blocks, bit-plane groups and bytes never straddle a unit).
 */
QLR_API int qlr_quantize_nf4(const float* W, int64_t N, int64_t K, int bits, int block, int dq_block,
                     const qlr_qweight* out, int32_t* status, void* stream);

/*
 * Group-wise asymmetric INT4 quantisation (QA-LoRA abstract: group-wise operators, INT4).
 * Per (row o, group g of `group` consecutive inputs): lo = min(0, min w), hi = max(0, max w),
 * scale = fp16(fp32(hi - lo) / 15), z = clamp(rne(-lo / scale), 0, 15),
 * code = clamp(rne(fp32(w / scale) + z), 0, 15); a zero scale gives z = 0 and codes 0.
 *   W fp32 [N, K] device;  group 32, 64 or 128, dividing K.
 *   out->codes [N, K/2] bytes, out->scale and out->zero fp16 [N, K/group].
 */
QLR_API int qlr_quantize_int4_group(const float* W, int64_t N, int64_t K, int group, const qlr_qweight* out,
                            int32_t* status, void* stream);

/*
 * Dequantise a whole weight to bf16 (W_out [N, K] device).  NF-k:
 * bf16(level[code] * (fp32(E4M3(c1_fp8)) * s2)) (or level * c1 without double
 * quantisation); INT4 group: bf16(fp32(code - zero) * scale).  Each product is one fp32
 * multiplication rounded to nearest; the result is the exact value every GEMM of this
 * library multiplies with.  (QLoRA explainer, "The QLoRA recipe", stage 3: dequantised to
 * BFloat16.)
 */
QLR_API int qlr_dequant(const qlr_qweight* w, uint16_t* W_out, int32_t* status, void* stream);

/*
 * LQ-LoRA initialisation (LQ-LoRA abstract: an iterative method splits each pretrained matrix into a
 * low-rank part kept in high precision plus a quantised part that is cheap to store; the quantised
 * part stays frozen and the low-rank part is the adapter).  Read as the alternation
 *   Q_0 = 0;  for t = 1..iters:  L_t = rank-r truncated SVD of (W - dequant(Q_{t-1})),
 *                                Q_t = NF-k quantisation (bits, block, dq_block) of (W - L_t)
 * with, from the last SVD L = U_r S_r V_r^T,  A = bf16(sqrt(S_r) V_r^T)  [r, K]  and
 * B = bf16(U_r sqrt(S_r) / s)  [N, r], so that dequant(Q) + s B A approximates W.  iters = 0 is plain
 * quantisation with A = B = 0.
 *   W       fp32 [N, K] row-major (device, 16-byte aligned), read only.
 *   out     NF-k weight descriptor with buffers sized by qlr_qweight_part_bytes (fmt, bits, block,
 *           dq_block, N, K must match the arguments); codes and constants are written.
 *   r       1 .. 64 and <= min(N, K);  s > 0;  iters 0 .. 64.
 *   workspace  qlr_lqlora_init_workspace_bytes(N, K, r) bytes, 256-byte aligned (residual, Gram
 *           matrix, factors and the eigensolver's work area; about N K + min(N, K)^2 floats).
 * The truncated SVD comes from the r largest eigenpairs of the Gram matrix on the smaller side
 * (R^T R when K <= N, else R R^T) and one projection of R onto them; the Gram matrix and the projection
 * are single-precision cuBLAS products and the eigenpairs cuSOLVER's syevdx (index range), both loaded
 * at run time; without them the call returns QLR_ERR_UNSUPPORTED (iters = 0 needs neither).  This is
 * an offline, once-per-weight call: it synchronises the stream (the eigensolver's status is read back
 * every iteration).  The solver and BLAS handles are created once per device, on the first call made
 * while that device is current (the libraries allocate a little device memory for them then), and
 * kept until the process exits; make that first call outside any stream capture.  Singular vectors are
 * unique up to sign, so A and B may differ in sign from another implementation's; their product does not.
 */
QLR_API size_t qlr_lqlora_init_workspace_bytes(int64_t N, int64_t K, int r);
QLR_API int qlr_lqlora_init(const float* W, int64_t N, int64_t K, int bits, int block, int dq_block, int r, float s,
                            int iters, qlr_qweight* out, uint16_t* A, uint16_t* B, void* workspace,
                            size_t workspace_bytes, int32_t* status, void* stream);

/*
 * Squared reconstruction error of NF-k quantisation, ||W - dequant(Q(W))||_F^2 with the dequantised
 * bf16 weight the layer uses: the per-option input of qlr_lqlora_allocate.
 *   W        fp32 [N, K] (device, 16-byte aligned);  bits 2..4, block 64 or 128, dq_block 0 or 256.
 *   err_out  one double in DEVICE memory (8-byte aligned), written on the stream.
 *   workspace  qlr_nf_quant_error_workspace_bytes(...) bytes, 256-byte aligned (the quantised weight
 *            and the fp64 partial sums).  Deterministic: fixed mapping and reduction order.
 */
QLR_API size_t qlr_nf_quant_error_workspace_bytes(int64_t N, int64_t K, int bits, int block, int dq_block);
QLR_API int qlr_nf_quant_error(const float* W, int64_t N, int64_t K, int bits, int block, int dq_block,
                               double* err_out, void* workspace, size_t workspace_bytes, int32_t* status,
                               void* stream);

/*
 * LQ-LoRA's budgeted allocation (LQ-LoRA abstract: an integer linear programme picks each matrix's
 * bit width and block size so that the whole model meets a memory budget).  Read as a multiple-choice
 * knapsack: matrix i takes one option o out of n_opt with error err[i * n_opt + o] and storage
 * cost_bits[i * n_opt + o]; the summed error is minimised with the summed storage within budget_bits.
 * Exact dynamic programming over the budget in whole units of unit_bits (costs rounded up, so the plan
 * never exceeds the budget); the plan is read back last matrix first, each taking the lowest option
 * index among its minima.  HOST memory, no GPU:
 *   err        double [n_mat * n_opt];  cost_bits  int64 [n_mat * n_opt];  n_opt <= 255.
 *   choice     int [n_mat], the option of each matrix;  total_err (optional) the plan's summed error.
 * QLR_ERR_SHAPE when the budget is below the cheapest plan, or when (budget_bits / unit_bits + 1) *
 * n_mat exceeds 2^30 (use a larger unit).
 */
QLR_API int qlr_lqlora_allocate(const double* err, const int64_t* cost_bits, int n_mat, int n_opt, int64_t budget_bits,
                                int64_t unit_bits, int* choice, double* total_err);

/*
 * QA-LoRA merge (QA-LoRA abstract: once fine-tuned, the adapter folds into the quantised weight
 * and the model loses no accuracy).  With the pooled adapter, s (B A)[o, g] / L is
 * added to every weight of group g of row o, which is a shift of the zero point:
 *   zero'[o, g] = fp16( zero - s * (B A)[o, g] / (group * scale[o, g]) ),  in fp64;
 * groups with scale == 0 keep their zero.  w->zero is rewritten in place.
 *   A bf16 [r, K/group], B bf16 [N, r];  w->fmt must be QLR_FMT_INT4G.
 */
QLR_API int qlr_qalora_merge(const qlr_qweight* w, const uint16_t* A, const uint16_t* B, int r, float s,
                     int32_t* status, void* stream);

/*
 * Forward pass of the layer (QLoRA explainer, "The QLoRA recipe", stage 3 and "The complete
 * QLoRA forward pass"; QA-LoRA pooled adapter when w->fmt == QLR_FMT_INT4G and pooled != 0):
 *   T_save = bf16( s * P(X) A^T )                               [M, r]
 *   Y      = bf16( X dequant(W)^T + T_save B^T )                 [M, N]
 * The dequantised weight never reaches global memory: the fused kernel streams the packed
 * codes into shared memory, dequantises them there and feeds tcgen05 tensor-core tiles;
 * the adapter term is added as r extra reduction columns of the same accumulator.
 * Token counts M <= 16 with 4-bit NF codes, double quantisation over 256 blocks and K a multiple of
 * 256 take a memory-streaming decode kernel instead.
 *   X bf16 [M, K];  A bf16 [r, Ka];  B bf16 [N, r];  Y bf16 [M, N];  T_save bf16 [M, r].
 *   r in {8, 16, 32, 64};  K a multiple of 64 (and of w->block);  N a multiple of 8.
 */
QLR_API size_t qlr_forward_workspace_bytes(const qlr_qweight* w, int64_t M, int r, int pooled);
QLR_API int qlr_forward(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* A, const uint16_t* B, int r,
                float s, int pooled, uint16_t* Y, uint16_t* T_save, void* workspace, size_t workspace_bytes,
                int32_t* status, void* stream);

/* The two stages of qlr_forward, callable separately (same arguments and buffers):
 *   qlr_lora_down     T_save = bf16(s * P(X) A^T)      (split-K tensor-core GEMM + fixed-order sum; for
 *                     1..16 tokens without pooling, and for the pooled adapter, one fixed-order
 *                     reduction kernel straight from X and no workspace; for r in {16, 32, 64} at 1024
 *                     or more tokens without pooling, one launch of 4-CTA clusters that split K and sum
 *                     their partials in shared memory in a fixed order, no workspace)
 *   qlr_forward_base  Y = bf16(X dequant(W)^T + T_save B^T)   (the fused dequant + tcgen05 kernel)
 * qlr_lora_down uses the workspace of qlr_forward_workspace_bytes; qlr_forward_base needs none. */
QLR_API int qlr_lora_down(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* A, int r, float s,
                          int pooled, uint16_t* T_save, void* workspace, size_t workspace_bytes, int32_t* status,
                          void* stream);
QLR_API int qlr_forward_base(const qlr_qweight* w, const uint16_t* X, int64_t M, const uint16_t* B, int r,
                             const uint16_t* T_save, uint16_t* Y, int32_t* status, void* stream);

/*
 * The MLP block's up projection with the SwiGLU gate fused into its epilogue (the LLaMA-7B-shaped MLP:
 * H = silu(G) * U between the gate/up and down projections).  Same arguments as qlr_forward_base for the up
 * projection, plus the gate projection's output G (bf16 [M, N], from qlr_forward_base of the gate weight):
 *   U = bf16( X dequant(W_up)^T + T_up B_up^T )      written to U  [M, N]
 *   H = bf16( silu(G) * U ),  silu(g) = g / (1 + exp(-g)), fp32 arithmetic on the bf16 G and U
 * in one launch, so U is never read back.  The SwiGLU arithmetic is the same as qlr_swiglu_forward's, so the
 * results are bit-identical to qlr_forward_base followed by qlr_swiglu_forward.  Decode-sized calls (the
 * decode kernel's conditions) run the two steps as two launches.  N a multiple of 8.
 */
QLR_API int qlr_forward_swiglu(const qlr_qweight* w_up, const uint16_t* X, int64_t M, const uint16_t* B_up, int r,
                               const uint16_t* T_up, const uint16_t* G, uint16_t* U, uint16_t* H, int32_t* status,
                               void* stream);

/* Number of kernels this library has launched in this process (all devices, all streams). */
QLR_API uint64_t qlr_launch_count(void);

/*
 * Adapter gradients (QLoRA explainer, "Background: how LoRA works" and "The QLoRA recipe":
 * gradients reach only A and B).  With T_save from qlr_forward:
 *   dT = bf16( s * dY B )          [M, r]   (written to dT_out, consumed by qlr_backward_dx)
 *   dB = dY^T T_save               [N, r]   fp32
 *   dA = dT^T P(X)                 [r, Ka]  fp32  (dT taken in bf16)
 * Each fp32 reduction over tokens is split across CTAs and summed in a fixed order, so the
 * results are deterministic.  With the pooled adapter (QA-LoRA), dA is formed from the group means of
 * X: one kernel writes, per slice of 16 tokens, the products of those means with the tokens' dT rows
 * to the workspace, and a second sums the slices in a fixed order.
 */
QLR_API size_t qlr_backward_lora_workspace_bytes(const qlr_qweight* w, int64_t M, int r, int pooled);
QLR_API int qlr_backward_lora(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY, const uint16_t* T_save,
                      const uint16_t* B, int64_t M, int r, float s, int pooled, float* dA, float* dB,
                      uint16_t* dT_out, void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/*
 * The two halves of qlr_backward_lora, for callers that overlap them with the input gradient: dT (which
 * qlr_backward_dx needs) first, then dB and dA (which nothing in the step waits for) on a second stream that
 * waits for dT, beside qlr_backward_dx on the first.  Same arithmetic and results as qlr_backward_lora; each
 * takes the workspace of qlr_backward_lora_workspace_bytes (calls that may run at the same time need
 * separate workspaces).
 *   qlr_backward_lora_dT     dT = bf16( s dY B )                              (no pooled variant is needed)
 *   qlr_backward_lora_dAdB   dB = dY^T T_save,  dA = dT^T P(X)   from the dT of qlr_backward_lora_dT
 */
QLR_API int qlr_backward_lora_dT(const qlr_qweight* w, const uint16_t* dY, int64_t M, const uint16_t* B, int r,
                                 float s, uint16_t* dT_out, void* workspace, size_t workspace_bytes, int32_t* status,
                                 void* stream);
QLR_API int qlr_backward_lora_dAdB(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY, const uint16_t* T_save,
                                   const uint16_t* dT, int64_t M, int r, int pooled, float* dA, float* dB,
                                   void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/* Size in bytes of the scratch array built into the library for qlr_backward_lora_noalloc: one per
 * GPU that loads the library, held until the process exits. */
#define QLR_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * qlr_backward_lora for callers that cannot allocate device memory (the pages have no counterpart:
 * this is a property of the library's interface, not of the method).  Such callers include a
 * framework that owns all device memory through its own pool, a runtime with a fixed memory plan,
 * and latency-critical loops that must not pay cudaMalloc/cudaFree.  Same arguments, results and
 * errors as qlr_backward_lora, without workspace: the split partial sums go to a scratch array of
 * QLR_NOALLOC_SCRATCH_BYTES compiled into the library.  It allocates nothing.
 *   - A problem whose workspace would exceed QLR_NOALLOC_SCRATCH_BYTES is rejected with
 *     QLR_ERR_WORKSPACE before anything is launched.
 *   - The array's device address is looked up once per GPU, on the first call made while that GPU
 *     is current; make that first call outside any stream capture.
 *   - All calls share the array and leave their partial sums in it (nothing needs to start at zero).
 *     Calls that can overlap on the GPU -- different streams, or several host threads -- race on it
 *     and must be serialised by the caller.
 */
QLR_API int qlr_backward_lora_noalloc(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY,
                                      const uint16_t* T_save, const uint16_t* B, int64_t M, int r, float s,
                                      int pooled, float* dA, float* dB, uint16_t* dT_out, int32_t* status,
                                      void* stream);

/*
 * LoQA: gradients of the loss with respect to the quantiser's own parameters (LoQA abstract: the scale and
 * the zero point of a quantised model are fine-tuned, through a form of the quantisation operator that works
 * with LoRA and equals the original).  Read on the group-wise INT4 format: the dequantised weight is
 * W[o, k] = scale[o, g] (code[o, k] - zero[o, g]), g = k / group, with the codes frozen; the bf16 rounding of
 * W is passed straight through.  With G = dY^T X (the gradient with respect to W, never formed in memory):
 *   dscale[o, g] = sum_{k in g} G[o, k] (code[o, k] - zero[o, g])      fp32 [N, K / group]
 *   dzero[o, g]  = -scale[o, g] sum_{k in g} G[o, k]                    fp32 [N, K / group]
 * A tcgen05 GEMM forms 128 x 256 tiles of G in tensor memory (the tokens are the reduction) and its epilogue
 * reduces them group by group with the codes.  Each result is one fixed-order sum (deterministic).
 *   w       QLR_FMT_INT4G, group 32, 64 or 128;  N a multiple of 8;  K a multiple of the group.
 *   X bf16 [M, K], dY bf16 [M, N] (device, row-major, 16-byte aligned);  M = 0 writes zeros.
 */
QLR_API int qlr_loqa_grad(const qlr_qweight* w, const uint16_t* X, const uint16_t* dY, int64_t M, float* dscale,
                          float* dzero, int32_t* status, void* stream);

/*
 * Input gradient through the frozen quantised weight (QLoRA explainer, "The contribution":
 * backpropagate through the frozen 4-bit weights into the adapters):
 *   dX = bf16( dY dequant(W) + P^T(dT A) )  [M, K]
 * With accumulate != 0 the previous contents of dX are added to the fp32 result before its one rounding:
 *   dX = bf16( dY dequant(W) + P^T(dT A) + dX_old )   (how the MLP block's up projection adds onto the gate's)
 * P^T spreads each pooled column over its group with weight 1/group.  Same fused
 * dequant + tcgen05 design as the forward, with the weight tile laid out MN-major.
 */
QLR_API size_t qlr_backward_dx_workspace_bytes(const qlr_qweight* w, int64_t M, int r, int pooled);
QLR_API int qlr_backward_dx(const qlr_qweight* w, const uint16_t* dY, int64_t M, const uint16_t* A, const uint16_t* dT,
                    int r, int pooled, int accumulate, uint16_t* dX, void* workspace, size_t workspace_bytes,
                    int32_t* status, void* stream);

/*
 * The MLP block's down-projection input gradient with the SwiGLU backward fused into its epilogue: with
 * dH = bf16( dY dequant(W_down) + dT A )  [M, K]  (K = the down weight's inputs = the gate/up outputs), which
 * is never stored, writes
 *   dG = bf16( dH U sig(G) (1 + G (1 - sig(G))) ),   dU = bf16( dH silu(G) )     bf16 [M, K]
 * from the forward's G and U.  Same arithmetic as qlr_backward_dx followed by qlr_swiglu_backward, so the
 * results are bit-identical to that pair; dH's write and read are saved.  No pooled adapter; K a multiple of 8.
 */
QLR_API int qlr_backward_dx_swiglu(const qlr_qweight* w_down, const uint16_t* dY, int64_t M, const uint16_t* A,
                                   const uint16_t* dT, int r, const uint16_t* G, const uint16_t* U, uint16_t* dG,
                                   uint16_t* dU, int32_t* status, void* stream);

/*
 * SwiGLU between the gate/up and down projections of an MLP block (the LLaMA-7B-shaped
 * workload): H = silu(G) * U;  backward dG = dH U sig(G) (1 + G (1 - sig(G))), dU = dH silu(G).
 * All bf16 [n] device buffers, fp32 arithmetic, n >= 0.
 */
QLR_API int qlr_swiglu_forward(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n, void* stream);
QLR_API int qlr_swiglu_backward(const uint16_t* dH, const uint16_t* G, const uint16_t* U, uint16_t* dG, uint16_t* dU,
                        int64_t n, void* stream);

/*
 * Bound of the pipeline waits (failure detection; the pages have no counterpart).  Every handshake of the
 * pipelined kernels (fused GEMM, adapter GEMM, decode) waits at most this many SM clock cycles; past it
 * the kernel raises an abort flag, every role leaves its loop, the CTA waits (with a fixed bound) for its
 * own TMA copies and tensor-core work still in flight, releases its tensor memory and sets
 * *status = QLR_ERR_TIMEOUT, so the context stays usable.  The process-wide default is 4e9 cycles (about
 * 2 s at the B200 boost clock); cycles < 0 restores it.  Applies to the launches that follow the call;
 * returns the previous bound.  Meant for tests of the timeout path: a short bound makes a healthy kernel
 * time out too.
 */
QLR_API long long qlr_set_wait_limit(long long cycles);

/*
 * Launches one small kernel that holds tensor memory and waits on a barrier nothing will complete, with
 * the current wait bound: it must set *status = QLR_ERR_TIMEOUT (status: one device int32, required),
 * release the tensor memory and return.  A test of the timeout path that needs no fault.
 */
QLR_API int qlr_wait_selftest(int32_t* status, void* stream);

/* Number of SMs of the current device (used to size persistent grids); <= 0 on error. */
QLR_API int qlr_device_sm_count(void);

#ifdef __cplusplus
}
#endif

#endif /* QLR_H */
