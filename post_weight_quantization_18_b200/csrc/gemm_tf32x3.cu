// gemm_tf32x3.cu — C = alpha * op(A) op(B) + beta * C in fp32 on tcgen05 tensor cores, with
// fp32-level accuracy from the 3xTF32 split: x = x_hi + x_lo where x_hi is x with the low 13
// mantissa bits cleared (exactly representable in tf32) and x_lo = x - x_hi (exact in fp32);
// a*b ~= a_hi*b_hi + a_hi*b_lo + a_lo*b_hi (the dropped a_lo*b_lo term is ~2^-22 relative).
//
// Serves the lazy block updates of the sweep ("GPTQ: Mathematical Foundations ...", §2 Lazy
// Batch Updates: W[:, F] -= Err_B U[B, F]), the GEMM steps of the U recursion (§3 Cholesky
// Decomposition and Pre-computation) and the Hessian of fp32 calibration inputs.
//
// One CTA per SM (persistent), 128 x 128 output tiles, 32-wide K blocks, 4-stage ring.
//   warp 0      TMA producer: the A tile (for the converters) and the B tile (the MMA operand)
//   warp 1      TMEM owner + MMA issuer: per 8-wide K step three tcgen05.mma kind::tf32 with A
//               read from tensor memory and B from shared memory
//   warps 2-5   converters: each thread splits one row of the A tile into hi and lo and stores
//               both into tensor memory (tcgen05.st); together they write the lo part of the B
//               tile to a second buffer (the landed tile itself is B's hi operand: the tensor core
//               reads an fp32 operand of kind::tf32 as its top 19 bits)
//   warps 6-13  epilogue: two warps per TMEM lane quarter; each thread owns half a row of the
//               tile (64 columns) and adds the accumulator of every K stretch into registers
//               (fp32, round to nearest), then writes C once
// Shared memory is the limiting resource of the three-product scheme: with A in tensor memory the
// MMAs read only B from it, about half of what reading both operands three times would take.
//
// Accuracy: the tensor core adds into its fp32 accumulator with truncation (at most one ulp per
// step, one-sided on sums of like-signed terms), so one accumulator covers at most KCB k-blocks
// (K = 128, 48 accumulate steps) before the epilogue takes it over.
//
// Tile order: bands of GROUP tile rows, column by column inside a band, so that the CTAs running
// together read about GROUP panels of A and GROUP panels of B, which stay in L2.
//
// Every mbarrier wait is bounded (GPTQ_ERR_TIMEOUT on expiry); a CTA that gives up waits
// (bounded) for the loads and MMAs it already issued before it frees TMEM and exits.
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int BM = 128, BN = 128, BK = 32, STAGES = 4;
constexpr int TILE_BYTES = 128 * BK * 4;              // 16 KB: one operand tile (128 x 32 fp32)
constexpr int STAGE_BYTES = 3 * TILE_BYTES;           // A (for the converters), B, B_lo
constexpr int SMEM_DATA = STAGES * STAGE_BYTES;       // 192 KB
constexpr int SMEM_BYTES = SMEM_DATA + 1024 + 256;
constexpr int THREADS = 448;
constexpr int CONV_WARP0 = 2, N_CONV = 4, EPI_WARP0 = 6, N_EPI = 8;
constexpr int EPI_COLS = BN / 2;     // columns of a row per epilogue thread (two warps per quarter)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;      // two 128-column accumulators, at columns 0 and 128
constexpr uint32_t A_COL = 256;      // stage s: A_hi at A_COL + 64 s, A_lo at A_COL + 64 s + 32
static_assert(A_COL + 64 * STAGES <= TMEM_COLS, "A stages and accumulators fit tensor memory");
constexpr int KCB = 4;               // k-blocks per accumulator
constexpr int GROUP = 12;            // tile rows per band of the tile order

struct GemmArgs {
  int M, N, K;
  float alpha, beta;
  float* C;
  long long ldc;
  int a_mn, b_mn;      // 1: operand is MN-major in memory
  int upper_only;
  int tri;             // kTri* flags: triangular operands, per-tile k-ranges
  int tiles_m, tiles_n, n_tiles;
  const int32_t* status;
  int32_t* status_w;
};

// Shared-memory descriptor of the B tile at K offset kk (in units of 8 elements).
// K-major: rows of 128 B (32 fp32 of K), 128-byte swizzle with 16-byte atoms in 8-row groups
// (SBO 1 KB); a K step moves 32 B along the row.
// MN-major: tf32 operands stored MN-major must use the 128-byte swizzle with 32-byte atoms:
// K rows of 128 B (32 fp32 of N) in 4-row groups (SBO 512 B), four 32-element N atoms of BK rows
// each (LBO 4 KB, one TMA box); a K step moves 8 rows = 1 KB.
__device__ __forceinline__ uint64_t b_desc(uint32_t base, int mn_major, int kk) {
  if (mn_major) return gptq::smem_desc(base + kk * 1024, 4096, 512, gptq::kLayoutSW128Atom32B);
  return gptq::smem_desc(base + kk * 32, 16, 1024, gptq::kLayoutSW128);
}

// Tile t -> (tm, tn): bands of GROUP tile rows; inside a band, down each tile column in turn.
__device__ __forceinline__ void tile_of(int t, const GemmArgs& a, int& tm, int& tn) {
  const int band = GROUP * a.tiles_n;
  const int gm = t / band, r = t % band;
  const int h = min(GROUP, a.tiles_m - gm * GROUP);
  tm = gm * GROUP + r % h;
  tn = r / h;
}

__device__ __forceinline__ bool tile_live(int tm, int tn, const GemmArgs& a) {
  return !a.upper_only || (tm * BM <= tn * BN + BN - 1);
}

// K blocks [kb0, kb1) of a tile: the blocks that can hold nonzero terms under the operands'
// triangular structure. Never empty (an extra block only adds exact zeros), so that every tile
// produces at least one accumulator for the epilogue. Every warp role derives the same range.
__device__ __forceinline__ void tile_kb(int tm, int tn, const GemmArgs& a, int nkb, int& kb0,
                                        int& kb1) {
  int k_lo, k_hi;
  gptq_host::tri_k_range(a.tri, tm * BM, tn * BN, tn * BN + BN, a.K, k_lo, k_hi);
  kb0 = k_lo / BK;
  kb1 = (k_hi + BK - 1) / BK;
  if (kb0 > nkb - 1) kb0 = nkb - 1;
  if (kb1 <= kb0) kb1 = kb0 + 1;
}

__device__ __forceinline__ uint32_t hi_bits(float x) { return __float_as_uint(x) & 0xFFFFE000u; }

__global__ void __launch_bounds__(THREADS, 1)
gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   GemmArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_DATA);
  uint64_t* full = bars;                       // TMA landed        [STAGES]
  uint64_t* conv = bars + STAGES;              // split done        [STAGES]
  uint64_t* empty = bars + 2 * STAGES;         // MMA consumed      [STAGES]
  uint64_t* acc_full = bars + 3 * STAGES;      // [2]
  uint64_t* acc_empty = bars + 3 * STAGES + 2; // [2]
  uint64_t* mma_drain = bars + 3 * STAGES + 4; // abort path: the issued MMAs have completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* skip_flag = abort_flag + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *skip_flag = gptq::status_bad(args.status) ? 1 : 0;
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      gptq::mbar_init(&full[s], 1);
      gptq::mbar_init(&conv[s], N_CONV);
      gptq::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      gptq::mbar_init(&acc_full[b], 1);
      gptq::mbar_init(&acc_empty[b], N_EPI);
    }
    gptq::mbar_init(mma_drain, 1);
    gptq::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    gptq::tma_prefetch_desc(&tmA);
    gptq::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    gptq::tmem_alloc(tmem_slot, TMEM_COLS);
    gptq::tmem_relinquish();
  }
  gptq::tc_fence_before();
  __syncthreads();
  gptq::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nkb = (args.K + BK - 1) / BK;

  if (!*skip_flag) {
    if (warp == 0) {
      if (lane == 0) {  // ---------------- TMA producer ----------------
        int stage = 0;
        uint32_t phase = 0;
        uint32_t filled = 0, fill_parity = 0;  // per stage: filled at least once, last parity
        for (int t = blockIdx.x; t < args.n_tiles && !*abort_flag; t += gridDim.x) {
          int tm, tn;
          tile_of(t, args, tm, tn);
          if (!tile_live(tm, tn, args)) continue;
          int kb0, kb1;
          tile_kb(tm, tn, args, nkb, kb0, kb1);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!gptq::mbar_wait_sleep(&empty[stage], phase ^ 1, abort_flag)) break;
            uint8_t* sa = smem + stage * STAGE_BYTES;
            uint8_t* sb = sa + TILE_BYTES;
            gptq::mbar_arrive_expect_tx(&full[stage], 2 * TILE_BYTES);
            const int k0 = kb * BK;
            // A: one box, (m, k) at k*512 + 4m (MN-major, unswizzled) or row m at 128 m with
            // 16-byte chunk c at (c ^ (m & 7)) (K-major, 128-byte swizzle).
            if (args.a_mn) gptq::tma_load_2d(sa, &tmA, &full[stage], tm * BM, k0);
            else gptq::tma_load_2d(sa, &tmA, &full[stage], k0, tm * BM);
            if (args.b_mn) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                gptq::tma_load_2d(sb + q * 4096, &tmB, &full[stage], tn * BN + 32 * q, k0);
            } else {
              gptq::tma_load_2d(sb, &tmB, &full[stage], k0, tn * BN);
            }
            filled |= 1u << stage;
            fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
        if (*abort_flag)  // let the loads already issued land before the CTA exits
          for (int s = 0; s < STAGES; ++s)
            if (filled & (1u << s)) gptq::mbar_drain(&full[s], (fill_parity >> s) & 1u);
      }
    } else if (warp == 1) {
      if (lane == 0) {  // ---------------- MMA issuer ----------------
        const uint32_t idesc = gptq::instr_desc(/*tf32*/ 2, /*A in TMEM*/ 0, args.b_mn, BM, BN);
        int stage = 0;
        uint32_t phase = 0;
        int buf = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < args.n_tiles && !*abort_flag; t += gridDim.x) {
          int tm, tn;
          tile_of(t, args, tm, tn);
          if (!tile_live(tm, tn, args)) continue;
          int kb0, kb1;
          tile_kb(tm, tn, args, nkb, kb0, kb1);
          bool ok = true;
          for (int kc = kb0; kc < kb1 && ok; kc += KCB) {
            const int kc1 = min(kb1, kc + KCB);
            if (!gptq::mbar_wait_sleep(&acc_empty[buf], acc_phase ^ 1, abort_flag)) {
              ok = false;
              break;
            }
            gptq::tc_fence_after();
            const uint32_t d_tmem = tmem_base + ACC_COL + (uint32_t)(buf * BN);
            for (int kb = kc; kb < kc1; ++kb) {
              if (!gptq::mbar_wait_sleep(&conv[stage], phase, abort_flag)) { ok = false; break; }
              gptq::tc_fence_after();
              const uint32_t b_hi = gptq::smem_u32(smem + stage * STAGE_BYTES + TILE_BYTES);
              const uint32_t b_lo = b_hi + TILE_BYTES;
              const uint32_t a_hi = tmem_base + A_COL + 64u * stage;
              const uint32_t a_lo = a_hi + 32u;
#pragma unroll
              for (int kk = 0; kk < BK / 8; ++kk) {
                const uint64_t dbh = b_desc(b_hi, args.b_mn, kk), dbl = b_desc(b_lo, args.b_mn, kk);
                gptq::mma_tf32_tmem_a(d_tmem, a_hi + 8u * kk, dbl, idesc,
                                      (kb > kc || kk > 0) ? 1u : 0u);
                gptq::mma_tf32_tmem_a(d_tmem, a_lo + 8u * kk, dbh, idesc, 1u);
                gptq::mma_tf32_tmem_a(d_tmem, a_hi + 8u * kk, dbh, idesc, 1u);
              }
              gptq::mma_commit(&empty[stage]);
              if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            gptq::mma_commit(&acc_full[buf]);
            if (++buf == 2) { buf = 0; acc_phase ^= 1; }
          }
          if (!ok) break;
        }
        if (*abort_flag) {  // the MMAs already issued finish before TMEM is released
          gptq::mma_commit(mma_drain);
          gptq::mbar_drain(mma_drain, 0);
        }
      }
    } else if (warp < EPI_WARP0) {
      // ------------- converters: A row -> (hi, lo) in TMEM; B -> lo copy -------------
      const int quarter = warp & 3;              // TMEM lanes 32 quarter .. 32 quarter + 31
      const int m = quarter * 32 + lane;         // the A row this thread splits
      const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
      const int ct = threadIdx.x - CONV_WARP0 * 32;  // 0..127
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < args.n_tiles && !*abort_flag; t += gridDim.x) {
        int tm, tn;
        tile_of(t, args, tm, tn);
        if (!tile_live(tm, tn, args)) continue;
        int kb0, kb1;
        tile_kb(tm, tn, args, nkb, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!gptq::mbar_wait_sleep(&full[stage], phase, abort_flag)) break;
          const uint8_t* sa = smem + stage * STAGE_BYTES;
          uint32_t hi[32], lo[32];
          if (args.a_mn) {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const float x = *reinterpret_cast<const float*>(sa + k * 512 + 4 * m);
              hi[k] = hi_bits(x);
              lo[k] = __float_as_uint(x - __uint_as_float(hi[k]));
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 v =
                  *reinterpret_cast<const float4*>(sa + m * 128 + ((c ^ (m & 7)) << 4));
              const float xs[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                hi[4 * c + e] = hi_bits(xs[e]);
                lo[4 * c + e] = __float_as_uint(xs[e] - __uint_as_float(hi[4 * c + e]));
              }
            }
          }
          __syncwarp();  // tcgen05.st is warp-collective
          gptq::tmem_st_32x32b_x32(tmem_base + lane_field + A_COL + 64u * stage, hi);
          gptq::tmem_st_32x32b_x32(tmem_base + lane_field + A_COL + 64u * stage + 32u, lo);
          // B: the landed tile stays in place as the hi operand; its lo part goes to B_lo.
          const float4* bh = reinterpret_cast<const float4*>(sa + TILE_BYTES);
          float4* bl = reinterpret_cast<float4*>(const_cast<uint8_t*>(sa) + 2 * TILE_BYTES);
#pragma unroll 4
          for (int e = ct; e < TILE_BYTES / 16; e += N_CONV * 32) {
            const float4 x = bh[e];
            float4 l;
            l.x = x.x - __uint_as_float(hi_bits(x.x));
            l.y = x.y - __uint_as_float(hi_bits(x.y));
            l.z = x.z - __uint_as_float(hi_bits(x.z));
            l.w = x.w - __uint_as_float(hi_bits(x.w));
            bl[e] = l;
          }
          gptq::tmem_st_wait();
          gptq::fence_proxy_async_smem();
          gptq::tc_fence_before();
          __syncwarp();
          if (lane == 0) gptq::mbar_arrive(&conv[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    } else {
      // ---------------- epilogue: K stretches summed in registers ----------------
      const int quarter = warp & 3;
      const int col_half = (warp - EPI_WARP0) >> 2;  // columns [64 col_half, 64 col_half + 64)
      const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
      int buf = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < args.n_tiles && !*abort_flag; t += gridDim.x) {
        int tm, tn;
        tile_of(t, args, tm, tn);
        if (!tile_live(tm, tn, args)) continue;
        int kb0, kb1;
        tile_kb(tm, tn, args, nkb, kb0, kb1);
        float acc[EPI_COLS];
#pragma unroll
        for (int e = 0; e < EPI_COLS; ++e) acc[e] = 0.f;  // 0 + x is x exactly: no select
        bool ok = true;
        for (int kc = kb0; kc < kb1; kc += KCB) {
          if (!gptq::mbar_wait_sleep(&acc_full[buf], acc_phase, abort_flag)) { ok = false; break; }
          gptq::tc_fence_after();
#pragma unroll
          for (int q = 0; q < EPI_COLS / 32; ++q) {
            uint32_t r[32];
            __syncwarp();  // tcgen05.ld is warp-collective: reconverge before every load
            gptq::tmem_ld_32x32b_x32(tmem_base + lane_field + ACC_COL +
                                         (uint32_t)(buf * BN + EPI_COLS * col_half + 32 * q),
                                     r);
            gptq::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e)
              acc[32 * q + e] += __uint_as_float(r[e]);
          }
          gptq::tc_fence_before();
          __syncwarp();
          if (lane == 0) gptq::mbar_arrive(&acc_empty[buf]);
          if (++buf == 2) { buf = 0; acc_phase ^= 1; }
        }
        if (!ok) break;
        const int row = tm * BM + quarter * 32 + lane;
        if (row < args.M) {
          float* crow = args.C + (long long)row * args.ldc;
          const float alpha = args.alpha, beta = args.beta;
#pragma unroll
          for (int c = 0; c < EPI_COLS / 32; ++c) {
            const int col0 = tn * BN + EPI_COLS * col_half + c * 32;
            if (col0 >= args.N) continue;
            const bool full_vec = (col0 + 32 <= args.N) && (!args.upper_only || row <= col0);
            if (full_vec) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                float4* p = reinterpret_cast<float4*>(crow + col0 + 4 * q);
                float4 o;
                o.x = alpha * acc[32 * c + 4 * q + 0];
                o.y = alpha * acc[32 * c + 4 * q + 1];
                o.z = alpha * acc[32 * c + 4 * q + 2];
                o.w = alpha * acc[32 * c + 4 * q + 3];
                if (beta != 0.f) {
                  const float4 old = *p;
                  o.x = fmaf(beta, old.x, o.x);
                  o.y = fmaf(beta, old.y, o.y);
                  o.z = fmaf(beta, old.z, o.z);
                  o.w = fmaf(beta, old.w, o.w);
                }
                *p = o;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const int col = col0 + e;
                if (col >= args.N || (args.upper_only && row > col)) continue;
                float o = alpha * acc[32 * c + e];
                if (beta != 0.f) o = fmaf(beta, crow[col], o);
                crow[col] = o;
              }
            }
          }
        }
      }
    }
  }

  gptq::tc_fence_before();
  __syncthreads();
  if (warp == 1) gptq::tmem_dealloc(tmem_base, TMEM_COLS);
  if (threadIdx.x == 0 && *abort_flag) gptq::set_status(args.status_w, GPTQ_ERR_TIMEOUT, 2);
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace gptq_host {

bool gemm_tf32x3_supported(int M, int N, int K, const float* A, long long lda, const float* B,
                           long long ldb, const float* C, long long ldc) {
  return M > 0 && N > 0 && K > 0 && al16(A) && al16(B) && al16(C) && (lda % 4) == 0 &&
         (ldb % 4) == 0 && (ldc % 4) == 0;
}

// op(A) is M x K: transA=false -> A[m*lda + k] (K-major); transA=true -> A[k*lda + m] (MN-major).
// op(B) is K x N: transB=false -> B[k*ldb + n] (MN-major); transB=true -> B[n*ldb + k] (K-major).
int gemm_tf32x3(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
                const float* B, long long ldb, bool transB, float beta, float* C, long long ldc,
                bool upper_only, const int32_t* status, cudaStream_t stream, int tri,
                int max_ctas) {
  CUtensorMap ta, tb;
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;               // K-major tiles
  const CUtensorMapSwizzle sw32 = CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;    // MN-major B tiles
  int rc;
  // A feeds the converters only: MN-major as one unswizzled 128 x 32 box (a warp reads one
  // 512-byte K row per load), K-major as one 32 x 128 box with the 128-byte swizzle (a thread
  // reads its own row in 16-byte chunks; the swizzle spreads eight rows over the banks).
  if (transA)  // MN-major: inner = M
    rc = make_tmap_2d(&ta, f32, 4, A, (uint64_t)M, (uint64_t)K, (uint64_t)lda * 4, BM, BK,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  else         // K-major: inner = K
    rc = make_tmap_2d(&ta, f32, 4, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 4, BK, BM, sw);
  if (rc) return GPTQ_ERR_CUDA;
  if (!transB)  // MN-major: inner = N
    rc = make_tmap_2d(&tb, f32, 4, B, (uint64_t)N, (uint64_t)K, (uint64_t)ldb * 4, 32, BK, sw32);
  else          // K-major: inner = K
    rc = make_tmap_2d(&tb, f32, 4, B, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 4, BK, BN, sw);
  if (rc) return GPTQ_ERR_CUDA;
  GemmArgs a;
  a.M = M; a.N = N; a.K = K;
  a.alpha = alpha; a.beta = beta;
  a.C = C; a.ldc = ldc;
  a.a_mn = transA ? 1 : 0;
  a.b_mn = transB ? 0 : 1;
  a.upper_only = upper_only ? 1 : 0;
  a.tri = tri;
  a.tiles_m = (M + BM - 1) / BM;
  a.tiles_n = (N + BN - 1) / BN;
  a.n_tiles = a.tiles_m * a.tiles_n;
  a.status = status;
  a.status_w = const_cast<int32_t*>(status);
  if (ensure_smem_attr(reinterpret_cast<const void*>(gemm_tf32x3_kernel), SMEM_BYTES) != 0)
    return GPTQ_ERR_CUDA;
  int sms = num_sms();
  if (max_ctas > 0 && max_ctas < sms) sms = max_ctas;
  const int grid = a.n_tiles < sms ? a.n_tiles : sms;
  gemm_tf32x3_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(ta, tb, a);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
