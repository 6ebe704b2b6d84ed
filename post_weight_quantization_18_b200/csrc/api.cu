// api.cu — the extern "C" entry points declared in include/gptq.h: argument checks on the host,
// then stream-ordered kernel launches.
//
// Two host-side recursions organise the O(d^3) and O(n d^2) work into large GEMMs:
//
//  * U from H_d (gptq_prepare_hinv). With H = [[A, B], [B^T, C]] split at m:
//        U22 = rec(C);  T = B U22^T;  S = A - T T^T;  U11 = rec(S);  U12 = -U11 (T U22)
//    gives the upper U with H^-1 = U^T U (block form of V^-1 for H = V V^T, V upper; T is V12,
//    S the Schur complement A - B C^-1 B^T). Blocks of <= 128 columns are factored and
//    inverted by one CTA (prepare.cu).
//
//  * The sweep (gptq_quantize_layer). Columns [a, b) split at m: sweep [a, m), then
//        W[:, m:b] -= Err[:, a:m] U[a:m, m:b],
//    then sweep [m, b). Each pair of columns i < j receives its compensation Err_i U_ij exactly
//    once — inside a 128-column leaf eagerly, otherwise at their lowest common split — so this
//    is the lazy batch update of "GPTQ: Mathematical Foundations ...", §2 Lazy Batch Updates,
//    applied at every scale, equal to the column-by-column sweep in exact arithmetic.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool params_ok(const gptq_params* p) {
  if (p == nullptr) return false;
  if (!(p->bits == 2 || p->bits == 3 || p->bits == 4 || p->bits == 8)) return false;
  if (p->block_size != 128) return false;
  if (!(p->group_size == -1 ||
        (p->group_size > 0 && 128 % p->group_size == 0 && p->group_size % 4 == 0)))
    return false;
  if (p->sym != 0 && p->sym != 1) return false;
  if (p->order < GPTQ_ORDER_NATURAL || p->order > GPTQ_ORDER_GIVEN) return false;
  if (!(p->percdamp >= 0.0f) || !isfinite(p->percdamp)) return false;
  return true;
}

struct QuantWs {
  float* Wwork;
  float* Err;
  uint8_t* codes_sweep;
  size_t bytes;
};

QuantWs quant_ws_layout(void* ws, int64_t n, int64_t d, int order) {
  QuantWs w{};
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = 0;
  w.Wwork = reinterpret_cast<float*>(base + off);
  off += align_up((size_t)n * d * sizeof(float));
  w.Err = reinterpret_cast<float*>(base + off);
  off += align_up((size_t)n * d * sizeof(float));
  w.codes_sweep = nullptr;
  if (order != GPTQ_ORDER_NATURAL) {
    w.codes_sweep = base + off;
    off += align_up((size_t)n * d);
  }
  w.bytes = off;
  return w;
}

int split_point(int n) {  // a multiple of 128 near n/2, with 0 < m < n
  int m = ((n / 2) + 127) / 128 * 128;
  if (m >= n) m = n - 128;
  if (m <= 0) m = n / 2;
  return m;
}

// Side streams for work off the recursion's critical path. V = T U22 of a split needs only T,
// so it runs on a side stream while the caller's stream goes on with S and the recursion on S,
// and the caller's stream waits for it before U12 = -U11 V. One stream and one fork/join event
// pair per recursion depth, per device and per host thread, created on first use and kept for
// the thread's lifetime. A thread issues its calls in order, so a pair is never in use by two
// splits at once; event record/wait pairs are captured into CUDA graphs as dependencies.
constexpr int kSideDepth = 24;
constexpr int kSideDevices = 64;

struct SideStreams {
  bool ready = false;
  cudaStream_t stream[kSideDepth] = {};
  cudaEvent_t fork[kSideDepth] = {};
  cudaEvent_t join[kSideDepth] = {};
};

SideStreams* side_streams() {
  thread_local SideStreams per_device[kSideDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSideDevices) return nullptr;
  SideStreams& ss = per_device[dev];
  if (!ss.ready) {
    for (int i = 0; i < kSideDepth; ++i) {
      if (cudaStreamCreateWithFlags(&ss.stream[i], cudaStreamNonBlocking) != cudaSuccess ||
          cudaEventCreateWithFlags(&ss.fork[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&ss.join[i], cudaEventDisableTiming) != cudaSuccess)
        return nullptr;
    }
    ss.ready = true;
  }
  return &ss;
}

// U block [off, off+n) from the damped, permuted Hessian block of the same rows/columns.
// The factors U22 and U11 are upper triangular with exact zeros below the diagonal, so the
// products with them skip the k-ranges where their terms vanish.
int rec_prepare(float* H, float* U, int d, int off, int n, int depth, SideStreams* side,
                int32_t* st, cudaStream_t s) {
  using namespace gptq_host;
  const long long ld = d;
  if (n <= kPrepBase) return prep_base_block(H + off * ld + off, U + off * ld + off, n, d, off, st, s);
  const int m = split_point(n);
  const int n2 = n - m;
  float* Bblk = H + (long long)off * ld + off + m;       // H[off:off+m, off+m:off+n]
  float* Ablk = H + (long long)off * ld + off;          // H[off:off+m, off:off+m]
  float* U11 = U + (long long)off * ld + off;
  float* U12 = U + (long long)off * ld + off + m;
  float* U22 = U + (long long)(off + m) * ld + off + m;
  int rc;
  if ((rc = rec_prepare(H, U, d, off + m, n2, depth + 1, side, st, s))) return rc;
  // T = B U22^T -> U12 slot (U22^T is lower triangular)
  if ((rc = gemm_f32(m, n2, n2, 1.f, Bblk, ld, false, U22, ld, true, 0.f, U12, ld, false, st, s,
                     kTriBLower)))
    return rc;
  // V = T U22 -> B slot (B is no longer needed), on the side stream when there is one
  const bool fork = side != nullptr && depth < kSideDepth;
  cudaStream_t vs = s;
  if (fork) {
    vs = side->stream[depth];
    if (cudaEventRecord(side->fork[depth], s) != cudaSuccess ||
        cudaStreamWaitEvent(vs, side->fork[depth], 0) != cudaSuccess)
      return GPTQ_ERR_CUDA;
  }
  if ((rc = gemm_f32(m, n2, n2, 1.f, U12, ld, false, U22, ld, false, 0.f, Bblk, ld, false, st, vs,
                     kTriBUpper)))
    return rc;
  if (fork && cudaEventRecord(side->join[depth], vs) != cudaSuccess) return GPTQ_ERR_CUDA;
  // S = A - T T^T (upper triangle) in place of A
  if ((rc = gemm_f32(m, m, n2, -1.f, U12, ld, false, U12, ld, true, 1.f, Ablk, ld, true, st, s)))
    return rc;
  if ((rc = rec_prepare(H, U, d, off, m, depth + 1, side, st, s))) return rc;
  if (fork && cudaStreamWaitEvent(s, side->join[depth], 0) != cudaSuccess) return GPTQ_ERR_CUDA;
  // U12 = -U11 V (U11 is upper triangular)
  return gemm_f32(m, n2, m, -1.f, U11, ld, false, Bblk, ld, false, 0.f, U12, ld, false, st, s,
                  kTriAUpper);
}

struct SweepCtx {
  float* Wwork;
  const float* U;
  float* Err;
  uint8_t* codes;
  float* scales;
  float* zeros;
  int n, d, bits, g, sym;
  int32_t* st;
  cudaStream_t s;
};

int rec_sweep(const SweepCtx& c, int a, int b) {
  using namespace gptq_host;
  if (b - a <= 128)
    return sweep_block(c.Wwork, c.U, c.Err, c.codes, c.scales, c.zeros, c.n, c.d, a, c.bits, c.g,
                       c.sym, c.st, c.s);
  const int m = a + split_point(b - a);
  int rc;
  if ((rc = rec_sweep(c, a, m))) return rc;
  // W[:, m:b] -= Err[:, a:m] U[a:m, m:b]
  if ((rc = gemm_f32(c.n, b - m, m - a, -1.f, c.Err + a, c.d, false, c.U + (long long)a * c.d + m,
                     c.d, false, 1.f, c.Wwork + m, c.d, false, c.st, c.s)))
    return rc;
  return rec_sweep(c, m, b);
}

}  // namespace

extern "C" {

const char* gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "GPTQ_OK";
    case GPTQ_ERR_INVALID_ARG: return "GPTQ_ERR_INVALID_ARG";
    case GPTQ_ERR_UNSUPPORTED: return "GPTQ_ERR_UNSUPPORTED";
    case GPTQ_ERR_WORKSPACE: return "GPTQ_ERR_WORKSPACE";
    case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA";
    case GPTQ_ERR_NOT_SPD: return "GPTQ_ERR_NOT_SPD";
    case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE";
    case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT";
    default: return "GPTQ_ERR_UNKNOWN";
  }
}

size_t gptq_workspace_size(int64_t d_out, int64_t d_in, const gptq_params* p) {
  if (!params_ok(p) || d_out < 1 || d_in < 1) return 0;
  return quant_ws_layout(nullptr, d_out, d_in, p->order).bytes;
}

int gptq_hessian_accumulate(float* H, int64_t d_in, int64_t ldh, const void* X, int x_dtype,
                            int64_t n_tokens, int64_t ldx, float alpha, int accumulate,
                            int32_t* dev_status, gptq_stream_t stream) {
  if (H == nullptr || (X == nullptr && n_tokens > 0) || d_in < 1 || d_in > (1 << 30) || n_tokens < 0 ||
      n_tokens > (int64_t(1) << 31) - 1 || ldx < d_in || ldh < d_in)
    return GPTQ_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return GPTQ_ERR_INVALID_ARG;
  if (x_dtype != GPTQ_BF16 && x_dtype != GPTQ_F32) return GPTQ_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (x_dtype == GPTQ_BF16) {
    // TMA: 16-byte aligned bases and row strides.
    if ((n_tokens > 0 && (!aligned(X, 16) || (ldx % 8) != 0)) || !aligned(H, 16) || (ldh % 4) != 0)
      return GPTQ_ERR_INVALID_ARG;
    return gptq_host::syrk_bf16_upper(H, (int)d_in, ldh, X, n_tokens, ldx, alpha, accumulate,
                                      dev_status, s);
  }
  if (!aligned(X, 4)) return GPTQ_ERR_INVALID_ARG;
  if (n_tokens == 0) {
    if (accumulate) return GPTQ_OK;
    // H_upper = 0: alpha * (empty product)
    return gptq_host::gemm_f32((int)d_in, (int)d_in, 0, 0.f, static_cast<const float*>(X), ldx,
                               true, static_cast<const float*>(X), ldx, false, 0.f, H, ldh, true,
                               dev_status, s)
               ? GPTQ_ERR_CUDA
               : GPTQ_OK;
  }
  return gptq_host::gemm_f32((int)d_in, (int)d_in, (int)n_tokens, alpha,
                             static_cast<const float*>(X), ldx, true,
                             static_cast<const float*>(X), ldx, false, accumulate ? 1.f : 0.f, H,
                             ldh, true, dev_status, s)
             ? GPTQ_ERR_CUDA
             : GPTQ_OK;
}

int gptq_prepare_hinv(float* H, int64_t d_in, const gptq_params* p, float* U, int32_t* perm,
                      uint8_t* dead, void* ws, size_t ws_bytes, int32_t* dev_status,
                      gptq_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (!params_ok(p) || H == nullptr || U == nullptr || perm == nullptr || dead == nullptr ||
      d_in < 1 || d_in > (1 << 30) || H == U)
    return GPTQ_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int d = (int)d_in;
  using namespace gptq_host;
  int rc = 0;
  if (p->order == GPTQ_ORDER_NATURAL) {
    rc = prep_identity_perm(perm, d, s);
  } else {
    if (p->order == GPTQ_ORDER_DESC_ACT) rc = prep_act_order(H, perm, d, s);
    if (!rc) rc = prep_permute_sym(H, U, perm, d, s);
    if (!rc) rc = prep_copy_upper(U, H, d, s);
  }
  if (!rc) rc = prep_dead_damp(H, dead, d, p->percdamp, dev_status, s);
  if (!rc) rc = prep_zero_lower(U, d, s);
  if (!rc) rc = rec_prepare(H, U, d, 0, d, 0, side_streams(), dev_status, s);
  return rc ? GPTQ_ERR_CUDA : GPTQ_OK;
}

int gptq_quantize_layer(const void* W, int w_dtype, int64_t ldw, int64_t d_out, int64_t d_in,
                        const float* U, const int32_t* perm, const uint8_t* dead,
                        const gptq_params* p, uint8_t* codes, float* scales, float* zeros,
                        int32_t* g_idx, void* ws, size_t ws_bytes, int32_t* dev_status,
                        gptq_stream_t stream) {
  if (!params_ok(p) || W == nullptr || U == nullptr || perm == nullptr || dead == nullptr ||
      codes == nullptr || scales == nullptr || zeros == nullptr || g_idx == nullptr ||
      ws == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (d_out < 1 || d_in < 128 || d_in % 128 != 0 || ldw < d_in || d_in > (1 << 30) ||
      d_out > (1 << 30))
    return GPTQ_ERR_INVALID_ARG;
  if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_F32) return GPTQ_ERR_UNSUPPORTED;
  if (!aligned(U, 16) || !aligned(codes, 4) || !aligned(ws, 16)) return GPTQ_ERR_INVALID_ARG;
  const QuantWs w = quant_ws_layout(ws, d_out, d_in, p->order);
  if (ws_bytes < w.bytes) return GPTQ_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int n = (int)d_out, d = (int)d_in;
  using namespace gptq_host;
  int rc = sweep_gather_w(W, w_dtype, ldw, n, d, perm, dead, w.Wwork, dev_status, s);
  if (!rc && p->group_size == -1)
    rc = sweep_row_params(w.Wwork, n, d, p->bits, p->sym, scales, zeros, dev_status, s);
  uint8_t* cs = (p->order == GPTQ_ORDER_NATURAL) ? codes : w.codes_sweep;
  SweepCtx c{w.Wwork, U, w.Err, cs, scales, zeros, n, d, p->bits, p->group_size, p->sym,
             dev_status, s};
  if (!rc) rc = rec_sweep(c, 0, d);
  if (!rc && p->order != GPTQ_ORDER_NATURAL)
    rc = sweep_unpermute_codes(cs, perm, codes, n, d, dev_status, s);
  if (!rc) rc = sweep_g_idx(perm, g_idx, d, p->group_size, s);
  return rc ? GPTQ_ERR_CUDA : GPTQ_OK;
}

int gptq_pack(const uint8_t* codes, int64_t d_out, int64_t d_in, int bits, const float* scales,
              const float* zeros, int64_t n_groups, uint32_t* qweight, uint16_t* scales_f16,
              uint16_t* zeros_f16, gptq_stream_t stream) {
  if (codes == nullptr || scales == nullptr || zeros == nullptr || qweight == nullptr ||
      scales_f16 == nullptr || zeros_f16 == nullptr || d_out < 1 || d_in < 1 || n_groups < 1 ||
      d_in > (1 << 30) || d_out > (1 << 30))
    return GPTQ_ERR_INVALID_ARG;
  if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) return GPTQ_ERR_INVALID_ARG;
  return gptq_host::pack_launch(codes, (int)d_out, (int)d_in, bits, scales, zeros, n_groups,
                                qweight, scales_f16, zeros_f16,
                                reinterpret_cast<cudaStream_t>(stream))
             ? GPTQ_ERR_CUDA
             : GPTQ_OK;
}

int rtn_quantize(const void* W, int w_dtype, int64_t ldw, int64_t d_out, int64_t d_in,
                 const gptq_params* p, uint8_t* codes, float* scales, float* zeros,
                 gptq_stream_t stream) {
  if (p == nullptr || W == nullptr || codes == nullptr || scales == nullptr || zeros == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (!(p->bits == 2 || p->bits == 3 || p->bits == 4 || p->bits == 8) ||
      (p->sym != 0 && p->sym != 1))
    return GPTQ_ERR_INVALID_ARG;
  if (d_out < 1 || d_in < 1 || ldw < d_in || d_in > (1 << 30) || d_out > (1 << 30))
    return GPTQ_ERR_INVALID_ARG;
  if (!(p->group_size == -1 || (p->group_size > 0 && d_in % p->group_size == 0)))
    return GPTQ_ERR_INVALID_ARG;
  if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_F32) return GPTQ_ERR_UNSUPPORTED;
  return gptq_host::rtn_launch(W, w_dtype, ldw, (int)d_out, (int)d_in, p->bits, p->group_size,
                               p->sym, codes, scales, zeros,
                               reinterpret_cast<cudaStream_t>(stream))
             ? GPTQ_ERR_CUDA
             : GPTQ_OK;
}

}  // extern "C"
