// api.cu — the extern "C" entry points declared in include/gptq.h: argument checks on the host,
// then stream-ordered kernel launches.
//
// Two host-side recursions organise the O(d^3) and O(n d^2) work into large GEMMs:
//
//  * U from H_d (gptq_prepare_hinv). With H = [[A, B], [B^T, C]] split at m:
//        U22 = rec(C);  T = B U22^T;  S = A - T T^T;  U11 = rec(S);  U12 = -U11 (T U22)
//    gives the upper U with H^-1 = U^T U (block form of V^-1 for H = V V^T, V upper; T is V12,
//    S the Schur complement A - B C^-1 B^T). Up to 32 blocks of 128 columns, the same
//    factorization runs right-looking (one block column at a time, its trailing update beside
//    the critical chain on another stream). Blocks of <= 128 columns are factored and inverted
//    by one CTA (prepare.cu).
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
  if (p->static_groups != 0 && p->static_groups != 1) return false;
  if (p->static_groups && p->group_size == -1) return false;
  if (!(p->percdamp >= 0.0f) || !isfinite(p->percdamp)) return false;
  return true;
}

struct QuantWs {
  float* Wwork;
  float* Err;
  uint8_t* codes_sweep;
  int32_t* inv_perm;  // static groups or a permuted order: the inverse column permutation
  size_t bytes;
};

QuantWs quant_ws_layout(void* ws, int64_t n, int64_t d, int order, int static_groups) {
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
  w.inv_perm = nullptr;
  if (static_groups || order != GPTQ_ORDER_NATURAL) {
    w.inv_perm = reinterpret_cast<int32_t*>(base + off);
    off += align_up((size_t)d * sizeof(int32_t));
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

// Streams and events of the prepare step, per device and host thread, created on first use and
// kept for the thread's lifetime. A thread issues its calls in order, so no stream or event is
// used by two operations at once in a way the code below does not order explicitly; event
// record/wait pairs are captured into CUDA graphs as dependencies.
//  * depth[i], fork[i], join[i]: the halving recursion above the right-looking size runs
//    V = T U22 of a split at depth i on depth[i] while the caller's stream continues.
//  * chain / trail / inv: the three streams of the right-looking part (see rl_prepare); chain and
//    inv have the highest priority, trail the lowest.
constexpr int kSideDepth = 24;
constexpr int kSideDevices = 64;
constexpr int kRLBlocks = 32;  // right-looking nodes hold at most 32 blocks of 128 columns

struct PrepStreams {
  bool ready = false;
  cudaStream_t depth[kSideDepth] = {};
  cudaEvent_t fork[kSideDepth] = {};
  cudaEvent_t join[kSideDepth] = {};
  cudaStream_t chain = nullptr, trail = nullptr, inv = nullptr;
  cudaEvent_t start = nullptr, done_chain = nullptr, done_trail = nullptr, done_inv = nullptr;
  cudaEvent_t ev_base[kRLBlocks] = {}, ev_pd[kRLBlocks] = {}, ev_col[kRLBlocks] = {},
              ev_trail[kRLBlocks] = {};
};

PrepStreams* prep_streams() {
  thread_local PrepStreams per_device[kSideDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSideDevices) return nullptr;
  PrepStreams& ps = per_device[dev];
  if (!ps.ready) {
    auto ev = [](cudaEvent_t* e) {
      return cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    };
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return nullptr;
    for (int i = 0; i < kSideDepth; ++i)
      if (cudaStreamCreateWithFlags(&ps.depth[i], cudaStreamNonBlocking) != cudaSuccess ||
          !ev(&ps.fork[i]) || !ev(&ps.join[i]))
        return nullptr;
    if (cudaStreamCreateWithPriority(&ps.chain, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&ps.inv, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&ps.trail, cudaStreamNonBlocking, least) != cudaSuccess ||
        !ev(&ps.start) || !ev(&ps.done_chain) || !ev(&ps.done_trail) || !ev(&ps.done_inv))
      return nullptr;
    for (int i = 0; i < kRLBlocks; ++i)
      if (!ev(&ps.ev_base[i]) || !ev(&ps.ev_pd[i]) || !ev(&ps.ev_col[i]) || !ev(&ps.ev_trail[i]))
        return nullptr;
    ps.ready = true;
  }
  return &ps;
}

inline int ev_rec(cudaEvent_t e, cudaStream_t s) {
  return cudaEventRecord(e, s) == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}
inline int ev_wait(cudaStream_t s, cudaEvent_t e) {
  return cudaStreamWaitEvent(s, e, 0) == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

struct InvNode {
  int lo, mid, hi;
};
// Ranges are split in halves, except those that start at block 0: their U12 products run after
// the last base block, so they split after at most 4 blocks and leave only products of
// K <= 512 for the end (their large Y = V12 U22 runs while the chain finishes its last blocks).
void inv_tree(int lo, int hi, InvNode* out, int& n) {
  if (hi - lo < 2) return;
  const int half = (hi - lo) / 2;
  const int mid = lo + (lo == 0 && half > 4 ? 4 : half);
  out[n++] = InvNode{lo, mid, hi};
  inv_tree(lo, mid, out, n);
  inv_tree(mid, hi, out, n);
}

// Right-looking form of the same factorization for a node [off, off+n), n <= 32 * 128: block
// columns b = nb-1 .. 0 of 128 (block nb-1 may be shorter), A = the node's part of H.
//   chain (critical path):   base(b): A_bb -> U_bb = V_bb^-1
//                            Pd = A[b-1, b] U_bb^T           (V's block above the diagonal)
//                            A[b-1, b-1] -= Pd Pd^T          (next diagonal block ready)
//   trail (beside it):       P = A[0:b-1, b] U_bb^T          (rest of V's block column b)
//                            A[0:b-1, 0:b] -= P [P; Pd]^T    (upper; next block column and
//                                                             trailing update)
//   inv:                     U = V^-1 over a balanced tree of block ranges [lo, mid, hi):
//                            Y = V12 U22 once the right half is inverted and V's columns
//                            mid.. are final (at level mid), U12 = -U11 Y once the left half is
//                            inverted (at level lo). Only the U12 products of the ranges that
//                            start at block 0 remain after the last base block, and the tree
//                            keeps those small.
// V's off-diagonal blocks are held in U's upper blocks until the inverse overwrites them; Y is
// staged in the same blocks of H, which nothing reads again by then.
// Each wait names the level whose writes the next operation depends on.
int rl_prepare(float* H, float* U, int d, int off, int n, PrepStreams* ps, int32_t* st,
               cudaStream_t s) {
  using namespace gptq_host;
  const long long ld = d;
  const int nb = (n + 127) / 128;
  auto o = [&](int b) { return off + 128 * b; };
  auto sz = [&](int b) { return (n - 128 * b) < 128 ? (n - 128 * b) : 128; };
  auto Hp = [&](int rb, int cb) { return H + (long long)o(rb) * ld + o(cb); };
  auto Up = [&](int rb, int cb) { return U + (long long)o(rb) * ld + o(cb); };
  const bool conc = ps != nullptr;
  cudaStream_t cm = conc ? ps->chain : s, ct = conc ? ps->trail : s, ci = conc ? ps->inv : s;
  // CTA budgets of the persistent GEMMs beside the chain: together they leave 16 SMs for the
  // chain's base block and small products. Over the last few levels the trailing updates are
  // small and the inverse runs uncapped.
  const int sms = num_sms();
  const int cap_inv = sms > 96 ? 24 : 0;
  const int cap_trail = sms > 96 ? sms - 16 - cap_inv : 0;
  // Internal nodes [lo, mid, hi) of the balanced tree over the blocks (nb - 1 of them).
  InvNode nodes[kRLBlocks];
  int n_nodes = 0;
  inv_tree(0, nb, nodes, n_nodes);
  int rc = 0;
  if (conc) {
    if ((rc = ev_rec(ps->start, s)) || (rc = ev_wait(cm, ps->start)) ||
        (rc = ev_wait(ct, ps->start)) || (rc = ev_wait(ci, ps->start)))
      return rc;
  }
  for (int b = nb - 1; b >= 0; --b) {
    // ---- chain ----
    // base(b) needs the trailing updates of levels b+2 and above: the chain waited for them
    // before Pd(b+1), so one cross-stream wait per level (before Pd) covers every dependency.
    if ((rc = prep_base_block(Hp(b, b), Up(b, b), sz(b), d, o(b), st, cm))) return rc;
    if (conc && (rc = ev_rec(ps->ev_base[b], cm))) return rc;
    if (b >= 1) {
      // Pd(b) reads A[b-1, b] and diag(b) writes A[b-1, b-1]; both lie in the region of the
      // trailing update of level b+1.
      if (conc && b + 1 <= nb - 1 && (rc = ev_wait(cm, ps->ev_trail[b + 1]))) return rc;
      if ((rc = gemm_f32(128, sz(b), sz(b), 1.f, Hp(b - 1, b), ld, false, Up(b, b), ld, true, 0.f,
                         Up(b - 1, b), ld, false, st, cm, kTriBLower, 0, true)))
        return rc;
      if (conc && (rc = ev_rec(ps->ev_pd[b], cm))) return rc;
      if ((rc = gemm_f32(128, 128, sz(b), -1.f, Up(b - 1, b), ld, false, Up(b - 1, b), ld, true,
                         1.f, Hp(b - 1, b - 1), ld, true, st, cm, kTriNone, 0, true)))
        return rc;
    }
    // ---- trail ----
    if (b >= 2) {
      const int rows = 128 * (b - 1);
      if (conc && (rc = ev_wait(ct, ps->ev_base[b]))) return rc;
      if ((rc = gemm_f32(rows, sz(b), sz(b), 1.f, Hp(0, b), ld, false, Up(b, b), ld, true, 0.f,
                         Up(0, b), ld, false, st, ct, kTriBLower, cap_trail)))
        return rc;
      if (conc && (rc = ev_wait(ct, ps->ev_pd[b]))) return rc;
      // A[0:b-1, 0:b] -= P [P; Pd]^T (upper): the next block column and the trailing update in
      // one product, [P; Pd] being V's block column b, rows 0 .. b-1 (all of U[0:b, b]).
      if ((rc = gemm_f32(rows, rows + 128, sz(b), -1.f, Up(0, b), ld, false, Up(0, b), ld, true,
                         1.f, Hp(0, 0), ld, true, st, ct, kTriNone, cap_trail)))
        return rc;
      if (conc && ((rc = ev_rec(ps->ev_col[b], ct)) || (rc = ev_rec(ps->ev_trail[b], ct))))
        return rc;
    } else if (conc) {  // nothing to do: record so that later waits find this level's events
      if ((rc = ev_rec(ps->ev_col[b], ct)) || (rc = ev_rec(ps->ev_trail[b], ct))) return rc;
    }
    // ---- inv ----
    if (conc && (rc = ev_wait(ci, ps->ev_base[b]))) return rc;
    // U12 = -U11 Y of the ranges that start at b, smallest first (each one's U11 is the
    // previous one's whole range; the list is in pre-order, parents before their left
    // children, so it is walked backwards); U12 overwrites V12, whose last readers ran at
    // level mid.
    for (int i = n_nodes - 1; i >= 0; --i) {
      const InvNode& t = nodes[i];
      if (t.lo != b) continue;
      const int r1 = 128 * (t.mid - t.lo), r2 = n - 128 * t.mid < 128 * (t.hi - t.mid)
                                                   ? n - 128 * t.mid : 128 * (t.hi - t.mid);
      if (conc && (rc = ev_wait(ci, ps->ev_trail[t.mid]))) return rc;
      if ((rc = gemm_f32(r1, r2, r1, -1.f, Up(t.lo, t.lo), ld, false, Hp(t.lo, t.mid), ld, false,
                         0.f, Up(t.lo, t.mid), ld, false, st, ci, kTriAUpper,
                         b <= 4 ? 0 : cap_inv)))
        return rc;
    }
    // Y = V12 U22 of the ranges split at b: U22 (the range [b, hi)) was completed just above,
    // V's columns b.. are final after this level's panel.
    bool waited = false;
    for (int i = 0; i < n_nodes; ++i) {
      const InvNode& t = nodes[i];
      if (t.mid != b) continue;
      const int r1 = 128 * (t.mid - t.lo), r2 = n - 128 * t.mid < 128 * (t.hi - t.mid)
                                                   ? n - 128 * t.mid : 128 * (t.hi - t.mid);
      if (conc && !waited) {
        if ((rc = ev_wait(ci, ps->ev_pd[b])) || (rc = ev_wait(ci, ps->ev_col[b]))) return rc;
        waited = true;
      }
      if ((rc = gemm_f32(r1, r2, r2, 1.f, Up(t.lo, t.mid), ld, false, Up(t.mid, t.mid), ld, false,
                         0.f, Hp(t.lo, t.mid), ld, false, st, ci, kTriBUpper,
                         b <= 4 ? 0 : cap_inv)))
        return rc;
    }
  }
  if (conc) {
    if ((rc = ev_rec(ps->done_chain, cm)) || (rc = ev_rec(ps->done_trail, ct)) ||
        (rc = ev_rec(ps->done_inv, ci)) || (rc = ev_wait(s, ps->done_chain)) ||
        (rc = ev_wait(s, ps->done_trail)) || (rc = ev_wait(s, ps->done_inv)))
      return rc;
  }
  return 0;
}

// U block [off, off+n) from the damped, permuted Hessian block of the same rows/columns.
// Nodes of at most 32 blocks use the right-looking form; larger ones split in halves:
//   U22 = rec(C); T = B U22^T; S = A - T T^T; U11 = rec(S); U12 = -U11 (T U22).
// The factors U22 and U11 are upper triangular with exact zeros below the diagonal, so the
// products with them skip the k-ranges where their terms vanish.
int rec_prepare(float* H, float* U, int d, int off, int n, int depth, PrepStreams* ps,
                int32_t* st, cudaStream_t s) {
  using namespace gptq_host;
  const long long ld = d;
  if (n <= kRLBlocks * 128) return rl_prepare(H, U, d, off, n, ps, st, s);
  const int m = split_point(n);
  const int n2 = n - m;
  float* Bblk = H + (long long)off * ld + off + m;       // H[off:off+m, off+m:off+n]
  float* Ablk = H + (long long)off * ld + off;          // H[off:off+m, off:off+m]
  float* U11 = U + (long long)off * ld + off;
  float* U12 = U + (long long)off * ld + off + m;
  float* U22 = U + (long long)(off + m) * ld + off + m;
  int rc;
  if ((rc = rec_prepare(H, U, d, off + m, n2, depth + 1, ps, st, s))) return rc;
  // T = B U22^T -> U12 slot (U22^T is lower triangular)
  if ((rc = gemm_f32(m, n2, n2, 1.f, Bblk, ld, false, U22, ld, true, 0.f, U12, ld, false, st, s,
                     kTriBLower)))
    return rc;
  // V = T U22 -> B slot (B is no longer needed), on the depth's stream when there is one
  const bool fork = ps != nullptr && depth < kSideDepth;
  cudaStream_t vs = s;
  if (fork) {
    vs = ps->depth[depth];
    if ((rc = ev_rec(ps->fork[depth], s)) || (rc = ev_wait(vs, ps->fork[depth]))) return rc;
  }
  if ((rc = gemm_f32(m, n2, n2, 1.f, U12, ld, false, U22, ld, false, 0.f, Bblk, ld, false, st, vs,
                     kTriBUpper)))
    return rc;
  if (fork && (rc = ev_rec(ps->join[depth], vs))) return rc;
  // S = A - T T^T (upper triangle) in place of A
  if ((rc = gemm_f32(m, m, n2, -1.f, U12, ld, false, U12, ld, true, 1.f, Ablk, ld, true, st, s)))
    return rc;
  if ((rc = rec_prepare(H, U, d, off, m, depth + 1, ps, st, s))) return rc;
  if (fork && (rc = ev_wait(s, ps->join[depth]))) return rc;
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
  const int32_t* perm;  // static groups: the sweep order, for each column's original group
  int static_groups;
  uint32_t* qweight;    // packed output in natural order (else null: uint8 codes)
  uint16_t* s16;        // fp16 copies of the dynamic group parameters (packed output)
  uint16_t* z16;
  int32_t* st;
  cudaStream_t s;
};

int rec_sweep(const SweepCtx& c, int a, int b) {
  using namespace gptq_host;
  if (b - a <= 128)
    return sweep_block(c.Wwork, c.U, c.Err, c.codes, c.scales, c.zeros, c.n, c.d, a, c.bits, c.g,
                       c.sym, c.perm, c.static_groups, c.qweight, c.s16, c.z16, c.st, c.s);
  const int m = a + split_point(b - a);
  int rc;
  if ((rc = rec_sweep(c, a, m))) return rc;
  // W[:, m:b] -= Err[:, a:m] U[a:m, m:b]
  if ((rc = gemm_f32(c.n, b - m, m - a, -1.f, c.Err + a, c.d, false, c.U + (long long)a * c.d + m,
                     c.d, false, 1.f, c.Wwork + m, c.d, false, c.st, c.s)))
    return rc;
  return rec_sweep(c, m, b);
}

// The rows of the sweep in two panels on two streams. Rows are independent given U
// ([GPTQ-MATH] §The Layer-Wise Reconstruction Problem: the objective is a sum over rows), so
// each panel runs its own block recursion; one panel's latency-bound 128-column sweeps then
// share the SMs with the other panel's tensor-core lazy updates instead of leaving them idle.
struct SweepStreams {
  bool ready = false;
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

SweepStreams* sweep_streams() {
  thread_local SweepStreams per_device[kSideDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSideDevices) return nullptr;
  SweepStreams& ss = per_device[dev];
  if (!ss.ready) {
    if (cudaStreamCreateWithFlags(&ss.side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    ss.ready = true;
  }
  return &ss;
}

constexpr int kPanelMinRows = 8192;  // below this one panel: half the rows make the products too small

int sweep_in_panels(const SweepCtx& c) {
  const int n1 = ((c.n / 2 + 15) / 16) * 16;  // whole 16-row sweep CTAs in the first panel
  if (c.n < kPanelMinRows || n1 >= c.n) return rec_sweep(c, 0, c.d);
  SweepStreams* ss = sweep_streams();
  if (ss == nullptr) return GPTQ_ERR_CUDA;
  const long long G = (c.g > 0) ? c.d / c.g : 1;
  SweepCtx c1 = c, c2 = c;
  c1.n = n1;
  c2.n = c.n - n1;
  c2.Wwork += (long long)n1 * c.d;
  c2.Err += (long long)n1 * c.d;
  c2.codes += (long long)n1 * c.d;
  c2.scales += n1 * G;
  c2.zeros += n1 * G;
  if (c.qweight != nullptr) c2.qweight += (long long)n1 * (c.d / 32) * c.bits;
  if (c.s16 != nullptr) {
    c2.s16 += n1 * G;
    c2.z16 += n1 * G;
  }
  c2.s = ss->side;
  int rc;
  if ((rc = ev_rec(ss->fork, c.s)) || (rc = ev_wait(ss->side, ss->fork))) return rc;
  if ((rc = rec_sweep(c1, 0, c.d)) || (rc = rec_sweep(c2, 0, c.d))) return rc;
  if ((rc = ev_rec(ss->join, ss->side)) || (rc = ev_wait(c.s, ss->join))) return rc;
  return 0;
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
  return quant_ws_layout(nullptr, d_out, d_in, p->order, p->static_groups).bytes;
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
    rc = prep_identity_perm(perm, d, dev_status, s);
  } else {
    if (p->order == GPTQ_ORDER_DESC_ACT) rc = prep_act_order(H, perm, d, dev_status, s);
    if (!rc) rc = prep_permute_sym(H, U, perm, d, dev_status, s);
    if (!rc) rc = prep_copy_upper(U, H, d, dev_status, s);
  }
  if (!rc) rc = prep_dead_damp(H, dead, d, p->percdamp, dev_status, s);
  if (!rc) rc = prep_zero_lower(U, d, dev_status, s);
  if (!rc) rc = rec_prepare(H, U, d, 0, d, 0, prep_streams(), dev_status, s);
  return rc ? GPTQ_ERR_CUDA : GPTQ_OK;
}

// Shared by gptq_quantize_layer (codes != null: uint8 codes) and gptq_quantize_pack_layer
// (qweight != null: packed words and fp16 parameters, no codes array).
static int quantize_impl(const void* W, int w_dtype, int64_t ldw, int64_t d_out, int64_t d_in,
                         const float* U, const int32_t* perm, const uint8_t* dead,
                         const gptq_params* p, uint8_t* codes, uint32_t* qweight,
                         uint16_t* scales_f16, uint16_t* zeros_f16, float* scales, float* zeros,
                         int32_t* g_idx, void* ws, size_t ws_bytes, int32_t* dev_status,
                         gptq_stream_t stream) {
  if (!params_ok(p) || W == nullptr || U == nullptr || perm == nullptr || dead == nullptr ||
      scales == nullptr || zeros == nullptr || g_idx == nullptr || ws == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (d_out < 1 || d_in < 128 || d_in % 128 != 0 || ldw < d_in || d_in > (1 << 30) ||
      d_out > (1 << 30))
    return GPTQ_ERR_INVALID_ARG;
  if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_F32) return GPTQ_ERR_UNSUPPORTED;
  if (!aligned(U, 16) || !aligned(ws, 16)) return GPTQ_ERR_INVALID_ARG;
  if (codes != nullptr && !aligned(codes, 4)) return GPTQ_ERR_INVALID_ARG;
  if (qweight != nullptr && !aligned(qweight, 16)) return GPTQ_ERR_INVALID_ARG;
  const QuantWs w = quant_ws_layout(ws, d_out, d_in, p->order, p->static_groups);
  if (ws_bytes < w.bytes) return GPTQ_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int n = (int)d_out, d = (int)d_in;
  const bool natural = p->order == GPTQ_ORDER_NATURAL;
  using namespace gptq_host;
  int rc = sweep_gather_w(W, w_dtype, ldw, n, d, perm, dead, w.Wwork, dev_status, s);
  if (!rc && w.inv_perm != nullptr) rc = sweep_invert_perm(perm, w.inv_perm, d, dev_status, s);
  if (!rc && p->group_size == -1)
    rc = sweep_row_params(w.Wwork, n, d, p->bits, p->sym, scales, zeros, scales_f16, zeros_f16,
                          dev_status, s);
  if (!rc && p->static_groups)
    rc = sweep_static_params(w.Wwork, w.inv_perm, n, d, p->group_size, p->bits, p->sym, scales,
                             zeros, scales_f16, zeros_f16, dev_status, s);
  // Natural order: the sweep writes the output (codes, or packed words) directly; a permuted
  // order sweeps into sweep-order codes that are then unpermuted (and packed).
  uint8_t* cs = natural ? codes : w.codes_sweep;
  uint32_t* qw_sweep = natural ? qweight : nullptr;
  const bool dyn = p->group_size > 0 && !p->static_groups;  // parameters decided by the sweep
  SweepCtx c{w.Wwork, U, w.Err, cs, scales, zeros, n, d, p->bits, p->group_size, p->sym,
             perm, p->static_groups, qw_sweep, dyn ? scales_f16 : nullptr,
             dyn ? zeros_f16 : nullptr, dev_status, s};
  if (!rc) rc = sweep_in_panels(c);
  if (!rc && !natural) {
    if (qweight != nullptr)
      rc = sweep_unpermute_pack(cs, w.inv_perm, n, d, p->bits, qweight, dev_status, s);
    else
      rc = sweep_unpermute_codes(cs, perm, codes, n, d, dev_status, s);
  }
  if (!rc)
    rc = sweep_g_idx(p->static_groups ? nullptr : perm, g_idx, d, p->group_size, dev_status, s);
  return rc ? GPTQ_ERR_CUDA : GPTQ_OK;
}

int gptq_quantize_layer(const void* W, int w_dtype, int64_t ldw, int64_t d_out, int64_t d_in,
                        const float* U, const int32_t* perm, const uint8_t* dead,
                        const gptq_params* p, uint8_t* codes, float* scales, float* zeros,
                        int32_t* g_idx, void* ws, size_t ws_bytes, int32_t* dev_status,
                        gptq_stream_t stream) {
  if (codes == nullptr) return GPTQ_ERR_INVALID_ARG;
  return quantize_impl(W, w_dtype, ldw, d_out, d_in, U, perm, dead, p, codes, nullptr, nullptr,
                       nullptr, scales, zeros, g_idx, ws, ws_bytes, dev_status, stream);
}

int gptq_quantize_pack_layer(const void* W, int w_dtype, int64_t ldw, int64_t d_out,
                             int64_t d_in, const float* U, const int32_t* perm,
                             const uint8_t* dead, const gptq_params* p, uint32_t* qweight,
                             uint16_t* scales_f16, uint16_t* zeros_f16, float* scales,
                             float* zeros, int32_t* g_idx, void* ws, size_t ws_bytes,
                             int32_t* dev_status, gptq_stream_t stream) {
  if (qweight == nullptr || scales_f16 == nullptr || zeros_f16 == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  return quantize_impl(W, w_dtype, ldw, d_out, d_in, U, perm, dead, p, nullptr, qweight,
                       scales_f16, zeros_f16, scales, zeros, g_idx, ws, ws_bytes, dev_status,
                       stream);
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

int gptq_dequant_gemv(const uint32_t* qweight, int64_t d_out, int64_t d_in, int bits,
                      const uint16_t* scales_f16, const uint16_t* zeros_f16, int64_t n_groups,
                      int group_size, const int32_t* g_idx, const uint16_t* X, int64_t batch,
                      int64_t ldx, float* Y, int64_t ldy, gptq_stream_t stream) {
  if (qweight == nullptr || scales_f16 == nullptr || zeros_f16 == nullptr || X == nullptr ||
      Y == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (d_out < 1 || d_in < 32 || d_in % 32 != 0 || d_in > (1 << 30) || d_out > (1 << 30))
    return GPTQ_ERR_INVALID_ARG;
  if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) return GPTQ_ERR_INVALID_ARG;
  if (batch < 1 || batch > 8 || ldx < d_in || ldx % 8 != 0 || ldy < d_out) return GPTQ_ERR_INVALID_ARG;
  if (!aligned(qweight, 16) || !aligned(X, 16) || !aligned(scales_f16, 2) || !aligned(zeros_f16, 2))
    return GPTQ_ERR_INVALID_ARG;
  if (n_groups < 1 || n_groups > d_in) return GPTQ_ERR_INVALID_ARG;
  if (g_idx == nullptr) {
    if (group_size == -1) {
      if (n_groups != 1) return GPTQ_ERR_INVALID_ARG;
    } else if (group_size < 1 || d_in % group_size != 0 || n_groups != d_in / group_size) {
      return GPTQ_ERR_INVALID_ARG;
    }
  }
  return gptq_host::dequant_gemv(qweight, (int)d_out, (int)d_in, bits, scales_f16, zeros_f16,
                                 (int)n_groups, g_idx ? 0 : group_size, g_idx, X, (int)batch, ldx,
                                 Y, ldy, reinterpret_cast<cudaStream_t>(stream))
             ? GPTQ_ERR_CUDA
             : GPTQ_OK;
}

int gptq_dequant_gemm(const uint32_t* qweight, int64_t d_out, int64_t d_in,
                      const uint16_t* scales_f16, const uint16_t* zeros_f16, int64_t n_groups,
                      int group_size, const uint16_t* X, int64_t m, int64_t ldx, float* Y,
                      int64_t ldy, int32_t* dev_status, gptq_stream_t stream) {
  if (qweight == nullptr || scales_f16 == nullptr || zeros_f16 == nullptr || X == nullptr ||
      Y == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (d_out < 1 || d_in < 128 || d_in % 128 != 0 || d_in > (1 << 30) || d_out > (1 << 30) ||
      m < 1 || m > (1 << 30))
    return GPTQ_ERR_INVALID_ARG;
  if (ldx < d_in || ldx % 8 != 0 || ldy < d_out) return GPTQ_ERR_INVALID_ARG;
  if (!aligned(qweight, 16) || !aligned(X, 16) || !aligned(Y, 4) || !aligned(scales_f16, 2) ||
      !aligned(zeros_f16, 2))
    return GPTQ_ERR_INVALID_ARG;
  if (group_size == -1) {
    if (n_groups != 1) return GPTQ_ERR_INVALID_ARG;
  } else if (group_size < 128 || group_size % 128 != 0 || d_in % group_size != 0 ||
             n_groups != d_in / group_size) {
    return GPTQ_ERR_INVALID_ARG;
  }
  return gptq_host::dequant_gemm(qweight, (int)d_out, (int)d_in, scales_f16, zeros_f16,
                                 (int)n_groups, group_size, X, (int)m, ldx, Y, ldy, dev_status,
                                 reinterpret_cast<cudaStream_t>(stream))
             ? GPTQ_ERR_CUDA
             : GPTQ_OK;
}

int gptq_gemm_f32(int64_t M, int64_t N, int64_t K, float alpha, const float* A, int64_t lda,
                  int trans_a, const float* B, int64_t ldb, int trans_b, float beta, float* C,
                  int64_t ldc, int32_t* dev_status, gptq_stream_t stream) {
  if (C == nullptr || M < 1 || N < 1 || K < 0 || M > (1 << 30) || N > (1 << 30) ||
      K > (1 << 30) || (trans_a != 0 && trans_a != 1) || (trans_b != 0 && trans_b != 1))
    return GPTQ_ERR_INVALID_ARG;
  if (K > 0 && (A == nullptr || B == nullptr)) return GPTQ_ERR_INVALID_ARG;
  const int64_t a_row = trans_a ? M : K, b_row = trans_b ? K : N;
  if (ldc < N || (K > 0 && (lda < a_row || ldb < b_row))) return GPTQ_ERR_INVALID_ARG;
  if (!aligned(C, 4) || (K > 0 && (!aligned(A, 4) || !aligned(B, 4))))
    return GPTQ_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) {  // C = beta C (alpha times an empty product)
    return gptq_host::gemm_f32((int)M, (int)N, 0, 0.f, C, ldc, false, C, ldc, false, beta, C, ldc,
                               false, dev_status, s)
               ? GPTQ_ERR_CUDA
               : GPTQ_OK;
  }
  return gptq_host::gemm_f32((int)M, (int)N, (int)K, alpha, A, lda, trans_a != 0, B, ldb,
                             trans_b != 0, beta, C, ldc, false, dev_status, s)
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
