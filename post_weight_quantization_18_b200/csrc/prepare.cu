// prepare.cu — numerical preparation of the Hessian on the GPU.
//
// "GPTQ: Mathematical Foundations ...":
//   §Activation Ordering (Act-Order / Desc-Act): pi = argsort(diag(H), descending),
//     H <- H[pi][:, pi] (stable order: equal keys keep the lower index first).
//   §GPTQ Algorithm Execution Walkthrough, step 1: dead columns (diag 0) get H_jj = 1; the
//     damping lambda = percdamp * mean(diag H) is added to the diagonal
//     (§Hessian Damping and Numerical Regularization).
//   §3 Cholesky Decomposition and Pre-computation: U upper with H^-1 = U^T U.
//
// U is obtained without forming H^-1: factor H_d = V V^T with V upper triangular (Cholesky
// from the last column), then U = V^-1. (V^-T V^-1 = H_d^-1 and V^-1 is upper with a positive
// diagonal, so it is the unique upper Cholesky factor of H_d^-1.) The host recursion in
// api.cu splits the matrix into halves and uses GEMMs; the base blocks of at most 128 columns
// are factored and inverted here by one CTA in shared memory.
#include "common.cuh"
#include "kernels.h"

namespace {

// Hp[a][b] = H[pi a][pi b] on the upper triangle, reading H's upper triangle symmetrically.
__global__ void permute_sym_kernel(const float* __restrict__ H, float* __restrict__ Hp,
                                   const int32_t* __restrict__ perm, int d) {
  const long long total = (long long)d * d;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(e / d), b = (int)(e % d);
    if (a > b) continue;
    const int i = perm[a], j = perm[b];
    const int lo = i < j ? i : j, hi = i < j ? j : i;
    Hp[(long long)a * d + b] = H[(long long)lo * d + hi];
  }
}

__global__ void copy_upper_kernel(const float* __restrict__ src, float* __restrict__ dst, int d) {
  const long long total = (long long)d * d;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(e / d), b = (int)(e % d);
    if (a <= b) dst[e] = src[e];
  }
}

// Stable descending rank of diag(H): rank_i = #{j : h_j > h_i or (h_j == h_i and j < i)};
// perm[rank_i] = i.
__global__ void act_order_rank_kernel(const float* __restrict__ H, int32_t* __restrict__ perm,
                                      int d) {
  __shared__ float keys[1024];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const float hi = (i < d) ? H[(long long)i * d + i] : 0.f;
  int rank = 0;
  for (int base = 0; base < d; base += 1024) {
    for (int t = threadIdx.x; t < 1024; t += blockDim.x) {
      const int j = base + t;
      keys[t] = (j < d) ? H[(long long)j * d + j] : 0.f;
    }
    __syncthreads();
    const int lim = min(1024, d - base);
    if (i < d) {
      for (int t = 0; t < lim; ++t) {
        const float hj = keys[t];
        const int j = base + t;
        rank += (hj > hi || (hj == hi && j < i)) ? 1 : 0;
      }
    }
    __syncthreads();
  }
  if (i < d) perm[rank] = i;
}

__global__ void identity_perm_kernel(int32_t* perm, int d) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < d; i += gridDim.x * blockDim.x)
    perm[i] = i;
}

// One CTA: dead-column fix, mean of the diagonal (after the fix), damping.
__global__ void dead_damp_kernel(float* __restrict__ H, uint8_t* __restrict__ dead, int d,
                                 float percdamp, int32_t* status) {
  __shared__ double partial[32];
  __shared__ int bad;
  __shared__ float lam_s;
  if (threadIdx.x == 0) bad = gptq::status_bad(status) ? 1 : 0;
  __syncthreads();
  if (bad) return;
  double acc = 0.0;
  int nonfinite = -1;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float h = H[(long long)j * d + j];
    if (!isfinite(h)) nonfinite = j;
    const bool is_dead = (h == 0.0f);
    dead[j] = is_dead ? 1 : 0;
    if (is_dead) {
      h = 1.0f;
      H[(long long)j * d + j] = 1.0f;
    }
    acc += (double)h;
  }
  if (nonfinite >= 0) gptq::set_status(status, GPTQ_ERR_NONFINITE, nonfinite);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) partial[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += partial[w];
    lam_s = (float)((double)percdamp * (s / (double)d));
  }
  __syncthreads();
  const float lam = lam_s;
  for (int j = threadIdx.x; j < d; j += blockDim.x) H[(long long)j * d + j] += lam;
}

__global__ void zero_lower_kernel(float* U, int d) {
  const long long total = (long long)d * d;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(e / d), b = (int)(e % d);
    if (a > b) U[e] = 0.f;
  }
}

// Base block (n <= 128): H_d block (upper triangle, ld) -> U block = V^-1 where H_d = V V^T.
// Phase 1 (Cholesky from the last column), step j: V_jj = sqrt(a_jj), V_ij = a_ij / V_jj, and the
// leading block a_ik -= V_ij V_kj (i <= k < j). Phase 2 (U = V^-1, back substitution on all
// columns at once), step i: row i of U = r_i / V_ii (written straight to global memory, it is
// final) and r_kc -= V_ki U_ic for k < i, c >= i, starting from r = I. Every step reads only a
// column (phase 1) or a row (phase 2) that the step itself does not write, so one barrier per
// step suffices. Thread (ty, tx) of the 16 x 32 layout owns rows ty + 16a and columns = tx mod 32.
constexpr int BASE_THREADS = 512;
constexpr int BASE_LD = gptq_host::kPrepBase + 1;

__global__ void __launch_bounds__(BASE_THREADS)
base_block_kernel(float* __restrict__ Hblk, float* __restrict__ Ublk, int n, int ld, int index0,
                  int32_t* status) {
  extern __shared__ float sm[];
  float* a = sm;                                   // working matrix, then r
  float* v = sm + gptq_host::kPrepBase * BASE_LD;  // V (upper)
  __shared__ int bad;
  const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
  if (tid == 0) bad = gptq::status_bad(status) ? 1 : 0;
  for (int i = ty; i < n; i += 16)
    for (int k = tx; k < n; k += 32) a[i * BASE_LD + k] = (i <= k) ? Hblk[(long long)i * ld + k] : 0.f;
  __syncthreads();
  if (bad) return;
  for (int j = n - 1; j >= 0; --j) {
    const float piv = a[j * BASE_LD + j];
    if (!(piv > 0.f) || !isfinite(piv)) {  // uniform: all threads read the same pivot
      if (tid == 0) gptq::set_status(status, GPTQ_ERR_NOT_SPD, index0 + j);
      return;
    }
    const float vjj = sqrtf(piv);
    const float inv = 1.0f / vjj;
    if (ty == 0) {
      for (int i = tx; i < j; i += 32) v[i * BASE_LD + j] = a[i * BASE_LD + j] * inv;
      if (tx == 0) v[j * BASE_LD + j] = vjj;
    }
    for (int i = ty; i < j; i += 16) {
      const float vij = a[i * BASE_LD + j] * inv;
      for (int k = i + ((tx - i) & 31); k < j; k += 32)
        a[i * BASE_LD + k] = fmaf(-vij, a[k * BASE_LD + j] * inv, a[i * BASE_LD + k]);
    }
    __syncthreads();
  }
  for (int i = ty; i < n; i += 16)
    for (int k = tx; k < n; k += 32) {
      a[i * BASE_LD + k] = (i == k) ? 1.f : 0.f;
      if (k < i) Ublk[(long long)i * ld + k] = 0.f;
    }
  __syncthreads();
  for (int i = n - 1; i >= 0; --i) {
    const float inv = 1.0f / v[i * BASE_LD + i];
    if (ty == 0)
      for (int c = i + tx; c < n; c += 32) Ublk[(long long)i * ld + c] = a[i * BASE_LD + c] * inv;
    for (int k = ty; k < i; k += 16) {
      const float vki = v[k * BASE_LD + i] * inv;
      for (int c = i + ((tx - i) & 31); c < n; c += 32)
        a[k * BASE_LD + c] = fmaf(-vki, a[i * BASE_LD + c], a[k * BASE_LD + c]);
    }
    __syncthreads();
  }
}

inline int grid_for(long long total) {
  long long g = (total + 255) / 256;
  const long long cap = (long long)gptq_host::num_sms() * 8;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

namespace gptq_host {

int prep_permute_sym(const float* H, float* Hp, const int32_t* perm, int d, cudaStream_t stream) {
  permute_sym_kernel<<<grid_for((long long)d * d), 256, 0, stream>>>(H, Hp, perm, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_copy_upper(const float* src, float* dst, int d, cudaStream_t stream) {
  copy_upper_kernel<<<grid_for((long long)d * d), 256, 0, stream>>>(src, dst, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_act_order(const float* H, int32_t* perm, int d, cudaStream_t stream) {
  act_order_rank_kernel<<<(d + 255) / 256, 256, 0, stream>>>(H, perm, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_identity_perm(int32_t* perm, int d, cudaStream_t stream) {
  identity_perm_kernel<<<grid_for(d), 256, 0, stream>>>(perm, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_dead_damp(float* H, uint8_t* dead, int d, float percdamp, int32_t* status,
                   cudaStream_t stream) {
  dead_damp_kernel<<<1, 1024, 0, stream>>>(H, dead, d, percdamp, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_zero_lower(float* U, int d, cudaStream_t stream) {
  zero_lower_kernel<<<grid_for((long long)d * d), 256, 0, stream>>>(U, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_base_block(float* Hblk, float* Ublk, int n, int ld, int index0, int32_t* status,
                    cudaStream_t stream) {
  const size_t smem = 2 * (size_t)kPrepBase * BASE_LD * sizeof(float);
  if (cudaFuncSetAttribute(base_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  base_block_kernel<<<1, BASE_THREADS, smem, stream>>>(Hblk, Ublk, n, ld, index0, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
