// kernels.h — host-side launchers of the library's kernels (internal; not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gptq_host {

// ---- Hessian ----
int syrk_bf16_upper(float* H, int d, long long ldh, const void* X, long long n_tokens,
                    long long ldx, float alpha, int accumulate, int32_t* status,
                    cudaStream_t stream);

// ---- fp32 GEMM: C = alpha * op(A) op(B) + beta * C, row-major; op(A) is M x K, op(B) K x N.
// upper_only: only elements with row <= col of C are written (the rest is left untouched).
// tri: triangular structure of the operands (kTri* flags below); each output tile then runs
// only over the k-range where its terms can be nonzero. Terms outside that range must be
// exact zeros, so skipping them leaves the result unchanged.
enum : int {
  kTriNone = 0,
  kTriAUpper = 1,  // op(A)[m][k] = 0 for k < m
  kTriBUpper = 2,  // op(B)[k][n] = 0 for k > n
  kTriBLower = 4,  // op(B)[k][n] = 0 for k < n
};
// [k_lo, k_hi) of an output tile with rows from m0 and columns [n0, n_end), for inner size K.
__host__ __device__ inline void tri_k_range(int tri, int m0, int n0, int n_end, int K, int& k_lo,
                                            int& k_hi) {
  k_lo = 0;
  k_hi = K;
  if ((tri & kTriAUpper) && m0 > k_lo) k_lo = m0;
  if ((tri & kTriBLower) && n0 > k_lo) k_lo = n0;
  if ((tri & kTriBUpper) && n_end < k_hi) k_hi = n_end;
}

// max_ctas > 0 caps the CTAs of the persistent tensor-core kernel (work that runs beside a
// latency-critical chain on another stream leaves SMs free for it).
// exclusive: products on a latency-critical chain ask for enough shared memory that their CTAs
// have their SMs to themselves (nothing launched beside them on other streams fits next to
// them).
int gemm_f32(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
             const float* B, long long ldb, bool transB, float beta, float* C, long long ldc,
             bool upper_only, const int32_t* status, cudaStream_t stream, int tri = kTriNone,
             int max_ctas = 0, bool exclusive = false);

int gemm_f32_simt(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
                  const float* B, long long ldb, bool transB, float beta, float* C, long long ldc,
                  bool upper_only, const int32_t* status, cudaStream_t stream,
                  int tri = kTriNone);
int gemm_f32_small(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
                   const float* B, long long ldb, bool transB, float beta, float* C,
                   long long ldc, bool upper_only, const int32_t* status, cudaStream_t stream,
                   int tri = kTriNone);
bool gemm_f32_staged_supported(int K, const float* A, long long lda, const float* B,
                               long long ldb);
int gemm_f32_staged(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
                    const float* B, long long ldb, bool transB, float beta, float* C,
                    long long ldc, bool upper_only, const int32_t* status, cudaStream_t stream,
                    int tri = kTriNone, bool exclusive = false);
bool gemm_tf32x3_supported(int M, int N, int K, const float* A, long long lda, const float* B,
                           long long ldb, const float* C, long long ldc);
int gemm_tf32x3(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
                const float* B, long long ldb, bool transB, float beta, float* C, long long ldc,
                bool upper_only, const int32_t* status, cudaStream_t stream,
                int tri = kTriNone, int max_ctas = 0);

// ---- prepare ----
// Every kernel below, like all kernels given a status word, does no work while status[0] != 0.
int prep_permute_sym(const float* H, float* Hp, const int32_t* perm, int d,
                     const int32_t* status, cudaStream_t stream);
int prep_copy_upper(const float* src, float* dst, int d, const int32_t* status,
                    cudaStream_t stream);
int prep_act_order(const float* H, int32_t* perm, int d, const int32_t* status,
                   cudaStream_t stream);
int prep_identity_perm(int32_t* perm, int d, const int32_t* status, cudaStream_t stream);
int prep_dead_damp(float* H, uint8_t* dead, int d, float percdamp, int32_t* status,
                   cudaStream_t stream);
int prep_zero_lower(float* U, int d, const int32_t* status, cudaStream_t stream);
int prep_base_block(float* Hblk, float* Ublk, int n, int ld, int index0, int32_t* status,
                    cudaStream_t stream);
constexpr int kPrepBase = 128;

// ---- sweep ----
// qweight / s16 / z16 (packed output, gptq_quantize_pack_layer) may be null: then the sweep
// writes uint8 codes and the fp32 parameters only.
int sweep_gather_w(const void* W, int w_dtype, long long ldw, int n, int d, const int32_t* perm,
                   const uint8_t* dead, float* Wwork, const int32_t* status, cudaStream_t stream);
int sweep_row_params(const float* Wwork, int n, int d, int bits, int sym, float* scales,
                     float* zeros, uint16_t* s16, uint16_t* z16, const int32_t* status,
                     cudaStream_t stream);
int sweep_block(float* Wwork, const float* U, float* Err, uint8_t* codes, float* scales,
                float* zeros, int n, int d, int col0, int bits, int group_size, int sym,
                const int32_t* perm, int static_groups, uint32_t* qweight, uint16_t* s16,
                uint16_t* z16, int32_t* status, cudaStream_t stream);
// inv = perm^-1.
int sweep_invert_perm(const int32_t* perm, int32_t* inv, int d, const int32_t* status,
                      cudaStream_t stream);
// Static groups: (s, z) [n, d / group_size] of the original-order groups (inv = perm^-1).
int sweep_static_params(const float* Wwork, const int32_t* inv, int n, int d, int group_size,
                        int bits, int sym, float* scales, float* zeros, uint16_t* s16,
                        uint16_t* z16, const int32_t* status, cudaStream_t stream);
int sweep_unpermute_codes(const uint8_t* codes_sweep, const int32_t* perm, uint8_t* codes, int n,
                          int d, const int32_t* status, cudaStream_t stream);
// Sweep-order codes -> packed words in the original column order (inv = perm^-1).
int sweep_unpermute_pack(const uint8_t* codes_sweep, const int32_t* inv, int n, int d, int bits,
                         uint32_t* qweight, const int32_t* status, cudaStream_t stream);
int sweep_g_idx(const int32_t* perm, int32_t* g_idx, int d, int group_size,
                const int32_t* status, cudaStream_t stream);

// ---- dequantizing matrix-vector product on the packed format ----
int dequant_gemv(const uint32_t* qweight, int n, int d, int bits, const uint16_t* scales_f16,
                 const uint16_t* zeros_f16, int n_groups, int group_size, const int32_t* g_idx,
                 const uint16_t* x_f16, int batch, long long ldx, float* y, long long ldy,
                 cudaStream_t stream);
// Y [m, ldy] = X [m, ldx] W_hat^T on the packed 4-bit format, tcgen05 (dequant_gemm.cu).
int dequant_gemm(const uint32_t* qweight, int n, int d, const uint16_t* scales_f16,
                 const uint16_t* zeros_f16, int n_groups, int group_size, const uint16_t* x_f16,
                 int m, long long ldx, float* y, long long ldy, const int32_t* status,
                 cudaStream_t stream);

// ---- RTN and pack ----
int rtn_launch(const void* W, int w_dtype, long long ldw, int n, int d, int bits, int group_size,
               int sym, uint8_t* codes, float* scales, float* zeros, cudaStream_t stream);
int pack_launch(const uint8_t* codes, int n, int d, int bits, const float* scales,
                const float* zeros, long long n_groups, uint32_t* qweight, uint16_t* scales_f16,
                uint16_t* zeros_f16, cudaStream_t stream);

}  // namespace gptq_host
