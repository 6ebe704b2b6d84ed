/*
 * gptq.h — C ABI of the B200 (sm_100a) GPTQ layer-quantization library (libgptq_b200.so).
 *
 * The library runs the per-layer hot path of GPTQ on one GPU:
 *   gptq_hessian_accumulate  H = 2 X X^T over calibration activations      (SYRK, tcgen05)
 *   gptq_prepare_hinv        dead columns, damping, act-order, U = upper Cholesky factor of H^-1
 *   gptq_quantize_layer      column sweep with OBS compensation and lazy block updates
 *   gptq_pack                codes -> packed int words, scales/zeros -> fp16
 *   gptq_quantize_pack_layer the sweep writing the packed words and fp16 scales/zeros directly
 *   rtn_quantize             round-to-nearest baseline with the same quantizer
 *   gptq_dequant_gemv        Y = X W_hat^T on the packed layer (batch 1 to 8), the format's consumer
 *   gptq_dequant_gemm        Y = X W_hat^T on the packed 4-bit layer for prefill-sized batches
 *   gptq_gemm_f32            C = alpha op(A) op(B) + beta C at fp32 accuracy: the product kernel
 *                            of prepare and of the lazy block update, exposed on its own
 *   gptq_quantize_layer_noalloc  gptq_quantize_layer on a fixed device scratch array
 *
 * Sources (page title, section):
 *   [INT4-GPTQ] "INT4 and GPTQ Quantization" (beta.fermi.ai wiki)
 *   [Q-INT8]    "Quantization (INT8, INT4, GPTQ)" (brentwoodlivery.com)
 *   [GPTQ-MATH] "GPTQ: Mathematical Foundations, Optimal Brain Surgeon Inversion, and
 *               Second-Order Error Minimization in LLM Quantization" (llms.blog)
 *
 * Conventions shared by every call
 *   - Array arguments are DEVICE pointers owned by the caller; the library allocates no device
 *     memory. Scratch memory comes from the caller as (ws, ws_bytes), sized by
 *     gptq_workspace_size().
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream). The int it returns reports only what is checked on the host before launching:
 *     GPTQ_OK, GPTQ_ERR_INVALID_ARG, GPTQ_ERR_UNSUPPORTED, GPTQ_ERR_WORKSPACE, GPTQ_ERR_CUDA.
 *     Nothing is launched when the return value is not GPTQ_OK.
 *   - Errors found on the device are written to `dev_status` (device int32[2]: code, index),
 *     which the caller zeroes once and reads after synchronising. Kernels of later calls given
 *     the same dev_status do no work while dev_status[0] != 0. dev_status may be NULL (no
 *     device-side reporting, no skipping).
 *   - Matrices are row-major with an explicit leading dimension (elements) where stated.
 *   - Calls never trap, never block the host, and never spin without a time limit: a wait on
 *     the device that exceeds its limit records GPTQ_ERR_TIMEOUT and the kernel returns.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gptq_stream_t; /* cudaStream_t */

/* Status codes. Host-side (returned) and device-side (written to dev_status[0]). */
enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad parameter combination */
  GPTQ_ERR_UNSUPPORTED = 2,  /* dtype or layout the kernels do not handle */
  GPTQ_ERR_WORKSPACE = 3,    /* ws_bytes smaller than gptq_workspace_size() */
  GPTQ_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  GPTQ_ERR_NOT_SPD = 16,     /* device: a Cholesky pivot <= 0 or non-finite; index = column */
  GPTQ_ERR_NONFINITE = 17,   /* device: a non-finite value met in the sweep; index = column */
  GPTQ_ERR_TIMEOUT = 18      /* device: a bounded wait ran out; index = kernel-specific site */
};

/* Element types of X and W. */
enum { GPTQ_BF16 = 0, GPTQ_F32 = 1 };

/* Column orders ([GPTQ-MATH] §1 Arbitrary Order Quantization; §Activation Ordering). */
enum {
  GPTQ_ORDER_NATURAL = 0,  /* columns 0..d_in-1 */
  GPTQ_ORDER_DESC_ACT = 1, /* pi = stable argsort of diag(H), descending (act-order / desc_act) */
  GPTQ_ORDER_GIVEN = 2     /* pi supplied by the caller in `perm` */
};

/* Quantization parameters ([GPTQ-MATH] §GPTQ Algorithm Execution Walkthrough signature:
 * bits, block_size, percdamp, group_size; [RA-GPTQ] hyperparameters: bits, group size,
 * act-order, damping). */
typedef struct {
  int32_t bits;       /* 2, 3, 4 or 8 */
  int32_t group_size; /* -1: one (scale, zero) per output row; otherwise a divisor of
                         block_size that is a multiple of 4 (typically 128) */
  int32_t sym;        /* 0: asymmetric min/max; 1: symmetric max|w| (codes offset by 2^(b-1)) */
  int32_t order;      /* GPTQ_ORDER_* */
  int32_t block_size; /* lazy-update block B; must be 128 */
  float percdamp;     /* relative damping alpha: lambda = alpha * mean(diag H); 0.01 */
  int32_t static_groups; /* 0: a group's (scale, zero) comes from its columns' current values
                            when the sweep reaches it (groups are runs of group_size columns in
                            sweep order). 1: groups are runs of group_size columns in the
                            ORIGINAL order and their (scale, zero) are taken from the original
                            weights (dead columns zero) before the sweep; with act-order each
                            swept column uses its original group's parameters, and g_idx is
                            c / group_size. Needs group_size > 0. Read by gptq_quantize_layer;
                            0 when the caller zero-initialises the struct. */
} gptq_params;

/*
 * gptq_workspace_size — bytes of scratch (ws) that gptq_prepare_hinv and gptq_quantize_layer
 * need for a layer of this shape; one buffer of this size serves both. Returns 0 for invalid
 * arguments.
 */
size_t gptq_workspace_size(int64_t d_out, int64_t d_in, const gptq_params* p);

/*
 * gptq_hessian_accumulate — H_upper (+)= alpha * X^T X.
 *
 * Defines: H = 2 X X^T ([INT4-GPTQ] §The Quantization Error and Layerwise Objective; [Q-INT8]
 * §Where the Hessian comes from; [GPTQ-MATH] §Second-Order Taylor Expansion and the Hessian).
 *
 *   H          fp32 [d_in, ldh] device, row-major. Only the upper triangle (i <= j, i,j < d_in)
 *              is written; the strictly lower triangle is neither read nor changed.
 *   X          device, token-major [n_tokens, ldx] (one row per calibration token; the pages'
 *              X in R^{d_in x N} is its transpose). The first d_in columns are used.
 *              x_dtype GPTQ_BF16: tensor-core bf16 products with fp32 accumulation; base
 *              16-byte aligned, ldx a multiple of 8. GPTQ_F32: fp32 arithmetic (3xTF32 split);
 *              ldx a multiple of 4, base 16-byte aligned.
 *   alpha      2.0 for the pages' H.
 *   accumulate 0: H_upper = alpha X^T X. 1: H_upper += alpha X^T X (chunked calibration sets;
 *              also how a caller resumes accumulation).
 *   Errors: INVALID_ARG for null pointers, d_in < 1, n_tokens < 0, ldx < d_in, ldh < d_in,
 *   misaligned X; the device status reports TIMEOUT only.
 */
int gptq_hessian_accumulate(float* H, int64_t d_in, int64_t ldh, const void* X, int x_dtype,
                            int64_t n_tokens, int64_t ldx, float alpha, int accumulate,
                            int32_t* dev_status, gptq_stream_t stream);

/*
 * gptq_prepare_hinv — from the raw Hessian to U, the upper Cholesky factor of H_damped^-1.
 *
 * Defines ([GPTQ-MATH] §GPTQ Algorithm Execution Walkthrough steps 1-2, §Hessian Damping and
 * Numerical Regularization, §Activation Ordering, §3 Cholesky Decomposition and Pre-computation):
 *   pi    = identity | stable argsort(diag H) descending | caller's perm   (p->order)
 *   H'    = H[pi][:, pi]
 *   dead  = diag(H') == 0;   H'_jj = 1 for dead j
 *   H_d   = H' + lambda I,   lambda = p->percdamp * mean(diag H')
 *   U     upper triangular with positive diagonal and H_d^-1 = U^T U.
 * U is computed as the inverse of the factor V of H_d = V V^T with V upper triangular (a
 * Cholesky factorization from the last column), which equals the pages' three-step route
 * chol -> cholesky_inverse -> chol(upper) in exact arithmetic.
 *
 *   H          fp32 [d_in, d_in] device (ld = d_in): input raw H, upper triangle valid.
 *              Clobbered (used as working storage).
 *   U          fp32 [d_in, d_in] device (ld = d_in), output, row-major; the strictly lower
 *              triangle is written with zeros. Read-only input of gptq_quantize_layer, so one U
 *              serves every layer that shares H (q/k/v, gate/up).
 *   perm       int32 [d_in] device: output pi for NATURAL / DESC_ACT, input for GIVEN
 *              (must be a permutation; not validated on the device).
 *   dead       uint8 [d_in] device, output, in sweep order (dead[k] refers to column pi[k]).
 *   ws         scratch of at least gptq_workspace_size(1, d_in, p) bytes.
 *   Device errors: NOT_SPD (index = sweep position of the failing pivot) when H_d is not
 *   positive definite in fp32 (for example percdamp = 0 on a singular H).
 */
int gptq_prepare_hinv(float* H, int64_t d_in, const gptq_params* p, float* U, int32_t* perm,
                      uint8_t* dead, void* ws, size_t ws_bytes, int32_t* dev_status,
                      gptq_stream_t stream);

/*
 * gptq_quantize_layer — the GPTQ column sweep for one layer.
 *
 * Defines ([GPTQ-MATH] §The GPTQ Algorithmic Innovations 1-3, §Quantization Formats and Group
 * Size, walkthrough step 3; [INT4-GPTQ] §The GPTQ Update Rule, §Group Quantization): columns
 * are visited in the order pi; for each column j of every row
 *   (s, z) of the group starting at j from the current values of its g columns (or of the whole
 *          row at the start of the sweep when group_size = -1),
 *   q_j    = clamp(rne(w_j / s) + z, 0, 2^b - 1),  w_hat_j = s (q_j - z),
 *   err_j  = (w_j - w_hat_j) / U_jj,   w_k -= err_j U_jk for the later columns k,
 * with the updates of later blocks applied lazily as W[:, F] -= Err_B U[B, F].
 *
 *   W          device, [d_out, ldw] row-major, w_dtype GPTQ_BF16 or GPTQ_F32. Not modified.
 *   U, perm, dead  outputs of gptq_prepare_hinv for this layer's H.
 *   codes      uint8 [d_out, d_in] device, output, ORIGINAL column order (codes < 2^bits;
 *              symmetric codes are q + 2^(b-1)).
 *   scales, zeros  fp32 [d_out, n_groups] device, output, in sweep-group order; n_groups =
 *              d_in / group_size, or 1 for group_size = -1. zeros are integers.
 *   g_idx      int32 [d_in] device, output: group of each original column (g_idx[pi[k]] =
 *              k / group_size; 0 for group_size = -1).
 *   ws         scratch of at least gptq_workspace_size(d_out, d_in, p) bytes.
 *   Requirements: d_in a multiple of block_size (128); group_size -1 or a divisor of 128 that
 *   is a multiple of 4.
 */
int gptq_quantize_layer(const void* W, int w_dtype, int64_t ldw, int64_t d_out, int64_t d_in,
                        const float* U, const int32_t* perm, const uint8_t* dead,
                        const gptq_params* p, uint8_t* codes, float* scales, float* zeros,
                        int32_t* g_idx, void* ws, size_t ws_bytes, int32_t* dev_status,
                        gptq_stream_t stream);

/*
 * gptq_pack — storage format of the quantized layer.
 *
 * Defines ([GPTQ-MATH] §Inference Execution and Modern Kernel Architectures: eight 4-bit
 * weights per int32 word; [INT4-GPTQ] §Group Quantization: scale and zero stored in FP16):
 * each row of codes is one LSB-first bit stream along d_in, code k at bits [b*k, b*k+b);
 * qweight word w of a row holds stream bits [32w, 32w+32). For bits = 4 that is code k at bit
 * 4*(k%8) of word k/8; for bits = 3, 32 codes per 3 words. A row's tail word is zero-padded.
 * Scales and zeros are converted fp32 -> fp16 with round-to-nearest-even.
 *
 *   codes      uint8 [d_out, d_in] device (each < 2^bits).
 *   qweight    uint32 [d_out, ceil(d_in*bits/32)] device, output.
 *   scales, zeros   fp32 [d_out, n_groups] device; scales_f16, zeros_f16 uint16 (fp16 bits)
 *              [d_out, n_groups] device, outputs.
 */
int gptq_pack(const uint8_t* codes, int64_t d_out, int64_t d_in, int bits, const float* scales,
              const float* zeros, int64_t n_groups, uint32_t* qweight, uint16_t* scales_f16,
              uint16_t* zeros_f16, gptq_stream_t stream);

/*
 * gptq_quantize_pack_layer — gptq_quantize_layer followed by gptq_pack in one pass: the sweep
 * writes the packed layer directly, with no uint8 codes array and no separate pack step
 * ([GPTQ-MATH] §2 Lazy Batch Updates for the sweep, §Inference Execution and Modern Kernel
 * Architectures for the storage: eight 4-bit weights per int32 word).
 *
 * Same arguments and meaning as gptq_quantize_layer, except the outputs:
 *   qweight      uint32 [d_out, d_in * bits / 32] device, 16-byte aligned: the words gptq_pack
 *                would write from gptq_quantize_layer's codes, bit for bit.
 *   scales_f16, zeros_f16  uint16 (fp16 bits) [d_out, n_groups] device: fp16 of scales/zeros
 *                (round to nearest even), as gptq_pack writes them.
 *   scales, zeros, g_idx   as in gptq_quantize_layer (fp32 parameters, sweep-group order).
 * Natural order: each 32-code chunk of a row is packed in the sweep kernel as the chunk is
 * finished. A permuted order: the sweep writes sweep-order codes into ws (gptq_workspace_size
 * includes them) and one kernel gathers and packs them in the original column order.
 */
int gptq_quantize_pack_layer(const void* W, int w_dtype, int64_t ldw, int64_t d_out,
                             int64_t d_in, const float* U, const int32_t* perm,
                             const uint8_t* dead, const gptq_params* p, uint32_t* qweight,
                             uint16_t* scales_f16, uint16_t* zeros_f16, float* scales,
                             float* zeros, int32_t* g_idx, void* ws, size_t ws_bytes,
                             int32_t* dev_status, gptq_stream_t stream);

/*
 * rtn_quantize — round-to-nearest baseline ([GPTQ-MATH] §Comparison: RTN; [INT4-GPTQ] §Group
 * Quantization): (s, z) from the original W of each group (or row), then every weight
 * quantized independently with the same quantizer as gptq_quantize_layer, in natural column
 * order. fp32 arithmetic with IEEE division and round-half-to-even; bit-exact by design.
 *
 *   W, w_dtype, ldw    as in gptq_quantize_layer.  p->order and p->percdamp are ignored.
 *   codes, scales, zeros   outputs as in gptq_quantize_layer.
 */
int rtn_quantize(const void* W, int w_dtype, int64_t ldw, int64_t d_out, int64_t d_in,
                 const gptq_params* p, uint8_t* codes, float* scales, float* zeros,
                 gptq_stream_t stream);

/*
 * gptq_quantize_layer_noalloc — gptq_quantize_layer for callers that cannot allocate device
 * memory (for example a plugin running inside another runtime that owns all device memory, or a
 * service that must not allocate once it is serving). It takes the same arguments minus
 * (ws, ws_bytes) and produces the same outputs; the scratch comes from one fixed array of
 * GPTQ_NOALLOC_SCRATCH_BYTES compiled into this library. (The source pages have no counterpart:
 * this is an interface variant, not a step of the method.)
 *
 *   Limit: returns GPTQ_ERR_WORKSPACE, launching nothing, when
 *          gptq_workspace_size(d_out, d_in, p) > GPTQ_NOALLOC_SCRATCH_BYTES (32 MiB: for example
 *          4M weights such as 1024 x 4096 in natural order).
 *   Memory: the array occupies GPTQ_NOALLOC_SCRATCH_BYTES of device memory on every GPU that
 *          loads the library, until the process exits. The call itself allocates nothing.
 *   Set-up: the first call on a device looks up the array's device address for that device
 *          (cudaGetSymbolAddress, with the device current) and caches it; make that first call
 *          before any stream capture.
 *   Sharing: every call on a device uses the same array, and the array keeps the last call's
 *          contents (nothing in it needs to start at zero). Calls whose kernels overlap on the GPU
 *          (other streams, other host threads) race on the array: order them on one stream.
 */
#define GPTQ_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int gptq_quantize_layer_noalloc(const void* W, int w_dtype, int64_t ldw, int64_t d_out,
                                int64_t d_in, const float* U, const int32_t* perm,
                                const uint8_t* dead, const gptq_params* p, uint8_t* codes,
                                float* scales, float* zeros, int32_t* g_idx, int32_t* dev_status,
                                gptq_stream_t stream);

/* gptq_status_string — a static, human-readable name for a status code. */
const char* gptq_status_string(int status);

/*
 * gptq_dequant_gemv — Y = X W_hat^T on the packed format: the W4A16 / W3A16 consumer of
 * gptq_pack's output (batch 1 to 8, the low-batch decoding case).
 *   "GPTQ: Mathematical Foundations ...", §Inference Execution and Modern Kernel Architectures:
 *   packed codes are unpacked and dequantized, w_hat = (q - z) * s with the FP16 scale and zero,
 *   and multiplied with FP16 activations, accumulating in higher precision.
 *   Y[b, r] = sum_c (code[r, c] - z[r, G(c)]) * s[r, G(c)] * X[b, c], in fp32, with
 *   G(c) = g_idx[c] or, when g_idx is NULL, c / group_size (0 when group_size == -1).
 *
 *   qweight     uint32 [d_out, d_in * bits / 32], the layout gptq_pack writes; 16-byte aligned
 *   d_in        a multiple of 32; bits 2, 3, 4 or 8
 *   scales_f16, zeros_f16  fp16 bit patterns [d_out, n_groups]; zero points are integers in
 *               [0, 2^bits), as gptq_pack stores them (other values are rounded to an integer)
 *   group_size  with g_idx == NULL: -1 (n_groups == 1) or a divisor of d_in
 *               (n_groups == d_in / group_size); ignored when g_idx is given
 *   g_idx       int32 [d_in] group of every column (values < n_groups), or NULL
 *   X           fp16 bit patterns [batch, ldx], 16-byte aligned, ldx a multiple of 8 and >= d_in
 *   batch       1 .. 8
 *   Y           fp32 [batch, ldy], ldy >= d_out (written, not accumulated into)
 * Returns GPTQ_ERR_INVALID_ARG for any other shape, alignment or parameter combination.
 * With contiguous groups of whole 128-column chunks (or one group per row), d_in a multiple of
 * 128 and no g_idx, the product runs on the tensor cores with every row's work split evenly over
 * the SMs: Y is zeroed on the stream and the partial sums of a row are added into it by atomic
 * adds, so the order of those few additions, and the last bits of Y, can differ between calls.
 * The other cases run one warp per row and are bitwise repeatable.
 */
int gptq_dequant_gemv(const uint32_t* qweight, int64_t d_out, int64_t d_in, int bits,
                      const uint16_t* scales_f16, const uint16_t* zeros_f16, int64_t n_groups,
                      int group_size, const int32_t* g_idx, const uint16_t* X, int64_t batch,
                      int64_t ldx, float* Y, int64_t ldy, gptq_stream_t stream);

/*
 * gptq_dequant_gemm — Y = X W_hat^T on the packed 4-bit format for any number of activation
 * rows (the prefill counterpart of gptq_dequant_gemv), on the tensor cores.
 *   "GPTQ: Mathematical Foundations ...", §Inference Execution and Modern Kernel Architectures:
 *   packed codes are unpacked and dequantized on chip, w_hat = (q - z) * s with the FP16 scale
 *   and zero, and multiplied with FP16 activations, accumulating in higher precision.
 *   Y[i, r] = sum_c (code[r, c] - z[r, G(c)]) * s[r, G(c)] * X[i, c] in fp32, computed as
 *   sum_g s (sum_{c in g} X code - z sum_{c in g} X): the products of activations and codes are
 *   exact, and every 128 columns the fp32 partial sums are scaled and added in registers.
 *
 *   qweight     uint32 [d_out, d_in / 8], the layout gptq_pack writes for 4-bit codes;
 *               16-byte aligned
 *   d_in        a multiple of 128
 *   scales_f16, zeros_f16  fp16 bit patterns [d_out, n_groups]; zero points are integers (other
 *               values are rounded to one)
 *   group_size  -1 (n_groups == 1) or a multiple of 128 dividing d_in (n_groups == d_in /
 *               group_size); act-order g_idx layouts are not taken
 *   X           fp16 bit patterns [m, ldx], 16-byte aligned, ldx a multiple of 8 and >= d_in
 *   m           number of activation rows, >= 1
 *   Y           fp32 [m, ldy], ldy >= d_out (written, not accumulated into)
 *   dev_status  as for the other calls: work is skipped if it already holds an error, and a
 *               wait that runs out records GPTQ_ERR_TIMEOUT (then Y holds no result)
 * Returns GPTQ_ERR_INVALID_ARG for any other shape, alignment or parameter combination.
 * Results are bitwise repeatable.
 */
int gptq_dequant_gemm(const uint32_t* qweight, int64_t d_out, int64_t d_in,
                      const uint16_t* scales_f16, const uint16_t* zeros_f16, int64_t n_groups,
                      int group_size, const uint16_t* X, int64_t m, int64_t ldx, float* Y,
                      int64_t ldy, int32_t* dev_status, gptq_stream_t stream);

/*
 * gptq_gemm_f32 — C = alpha * op(A) * op(B) + beta * C in fp32, the product that
 * gptq_prepare_hinv and gptq_quantize_layer use for their block products: the lazy block
 * update W[:, F] -= Err_B U[B, F] ([GPTQ-MATH] §2 Lazy Batch Updates) and the block steps of
 * the Cholesky factor and its inverse (§3 Cholesky Decomposition and Pre-computation).
 * Exposed so that the kernel can be checked and timed on its own.
 *
 * Large products run on the tcgen05 tensor cores with the three-term TF32 split
 * (x = x_hi + x_lo, a b ~ a_hi b_hi + a_hi b_lo + a_lo b_hi), each accumulator covering a bounded
 * stretch of K and the stretches summed in fp32; products up to 512^3 run on CUDA cores.
 * Either way the result carries fp32-level accuracy (about 2^-21 relative per product).
 *
 *   All matrices row-major fp32, device pointers. op(A) is M x K: A[m*lda + k] when trans_a
 *   is 0, A[k*lda + m] when 1; op(B) is K x N: B[k*ldb + n] when trans_b is 0, B[n*ldb + k]
 *   when 1; C[m*ldc + n]. M, N >= 1, K >= 0 (K = 0 gives C = beta C); leading dimensions at
 *   least the row length they index. beta == 0 means C is not read.
 *   dev_status: as elsewhere (NULL allowed); the kernels do no work while it holds an error.
 * Returns GPTQ_ERR_INVALID_ARG for a null pointer or an impossible shape.
 */
int gptq_gemm_f32(int64_t M, int64_t N, int64_t K, float alpha, const float* A, int64_t lda,
                  int trans_a, const float* B, int64_t ldb, int trans_b, float beta, float* C,
                  int64_t ldc, int32_t* dev_status, gptq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
