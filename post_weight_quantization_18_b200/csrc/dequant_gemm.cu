// dequant_gemm.cu — Y = X W_hat^T on the packed 4-bit format for prefill-sized batches, on the
// tcgen05 tensor cores (the GEMM counterpart of the dequantizing GEMV in gemv.cu).
//
// "GPTQ: Mathematical Foundations ...", §Inference Execution and Modern Kernel Architectures:
// packed codes are streamed from HBM, unpacked with bit shifts and dequantized on chip,
// w_hat = (q - z) * s with the FP16 scale and zero, and multiplied with the FP16 activations,
// accumulating in higher precision.
//
// Exact per-group form. With G(k) the contiguous group of column k,
//   Y[m, n] = sum_g s[n, g] (sum_{k in g} X[m, k] q[n, k]  -  z[n, g] sum_{k in g} X[m, k]),
// so the MMAs multiply the activations by the codes themselves, which are exact in fp16, and
// the scale and zero point enter once per group in fp32. The codes are written to shared memory
// as fp16 subnormals, code * 2^-24 (the bit pattern of the code with a zero exponent field: one
// byte permute and one AND per two codes), so an accumulator holds 2^-24 sum X q. The sums of X
// over a group come from a second MMA of the same A tile with an all-ones B of 16 columns.
//
// One CTA per SM (persistent), 128 x 128 output tiles (m: activation rows, n: weight rows),
// 64-wide K blocks (one 128-byte swizzle atom of fp16), 4-stage ring.
//   warp 0      TMA producer: the X tile (fp16, 128-byte swizzle) and the packed codes of the
//               128 weight rows (32 bytes a row)
//   warp 1      TMEM owner + MMA issuer: per 16-wide K step one kind::f16 MMA into the
//               128-column accumulator and one into the 16-column sum of X
//   warps 2-5   converters: thread n decodes weight row n of the block into the fp16 B tile
//               (128-byte swizzle, K-major) and, at the start of every 128 columns of K, writes
//               the row's s * 2^24 and -s * z for the epilogue
//   warps 6-13  epilogue: two warps per TMEM lane quarter, 64 columns a thread; every 128
//               columns of K (so that the truncating tensor-core accumulation covers at most 8
//               MMAs) it folds the accumulator into fp32 registers with the group's parameters,
//               and writes Y once per tile
// Every mbarrier wait is bounded (GPTQ_ERR_TIMEOUT on expiry); a CTA that gives up waits
// (bounded) for the loads and MMAs it already issued before it frees TMEM and exits.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int BM = 128, BN = 128, BK = 64, STAGES = 4;
constexpr int X_BYTES = BM * BK * 2;                        // 16 KB: X tile, fp16
constexpr int Q_BYTES = BN * BK / 2;                        // 4 KB: 4-bit codes, 32 B a row
constexpr int B_BYTES = BN * BK * 2;                        // 16 KB: decoded codes, fp16
constexpr int STAGE_BYTES = X_BYTES + Q_BYTES + B_BYTES;    // 36 KB
constexpr int ONES_BYTES = 16 * BK * 2;                     // 16 x 64 fp16 ones
constexpr int PAR_FLOATS = 2 * BN;                          // s * 2^24 and -s * z of 128 rows
constexpr int SMEM_DATA = STAGES * STAGE_BYTES + ONES_BYTES + 2 * PAR_FLOATS * 4;
constexpr int SMEM_BYTES = SMEM_DATA + 1024 + 256;
constexpr int THREADS = 448;
constexpr int CONV_WARP0 = 2, N_CONV = 4, EPI_WARP0 = 6, N_EPI = 8;
constexpr int EPI_COLS = BN / 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;    // two 128-column accumulators
constexpr uint32_t XS_COL = 256;   // two 16-column sums of X
constexpr int FOLD_KB = 2;         // k-blocks per accumulator: 128 columns of K
constexpr int GROUP = 8;           // tile rows per band of the tile order
constexpr uint32_t IDESC = gptq::instr_desc(/*f16*/ 0, 0, 0, BM, BN);
constexpr uint32_t IDESC_XS = gptq::instr_desc(/*f16*/ 0, 0, 0, BM, 16);

struct DqArgs {
  int M, N, K;
  const uint16_t* scales;  // fp16 [N, G]
  const uint16_t* zeros;
  int G, group_size;       // group_size -1: one group per row
  float* Y;
  long long ldy;
  int tiles_m, tiles_n, n_tiles;
  const int32_t* status;
  int32_t* status_w;
};

// Tile t -> (tm, tn): bands of GROUP activation-row tiles; inside a band, down each weight-row
// tile column in turn, so that the CTAs running together share a few panels of each operand.
__device__ __forceinline__ void tile_of(int t, const DqArgs& a, int& tm, int& tn) {
  const int band = GROUP * a.tiles_n;
  const int gm = t / band, r = t % band;
  const int h = min(GROUP, a.tiles_m - gm * GROUP);
  tm = gm * GROUP + r % h;
  tn = r / h;
}

__device__ __forceinline__ uint64_t desc_k64(uint32_t base, int kk) {
  // K-major, 128-byte rows (64 fp16 of K), 16-byte chunks swizzled over 8-row groups (SBO 1 KB);
  // a 16-wide K step moves 32 bytes along the row.
  return gptq::smem_desc(base + kk * 32, 16, 1024, gptq::kLayoutSW128);
}

__global__ void __launch_bounds__(THREADS, 1)
dequant_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
                    DqArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ones = smem + STAGES * STAGE_BYTES;
  float* par = reinterpret_cast<float*>(ones + ONES_BYTES);  // [2][2][BN]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_DATA);
  uint64_t* full = bars;                  // TMA landed              [STAGES]
  uint64_t* conv = full + STAGES;         // B tile decoded          [STAGES]
  uint64_t* empty = conv + STAGES;        // MMAs read the stage     [STAGES]
  uint64_t* acc_full = empty + STAGES;    // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]
  uint64_t* par_full = acc_empty + 2;     // [2] parameters of a fold written
  uint64_t* par_empty = par_full + 2;     // [2] parameters of a fold used
  uint64_t* mma_drain = par_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
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
      gptq::mbar_init(&par_full[b], N_CONV);
      gptq::mbar_init(&par_empty[b], N_EPI);
    }
    gptq::mbar_init(mma_drain, 1);
    gptq::fence_barrier_init();
  }
  // The all-ones B operand of the sums of X: every fp16 is 1.0, so the swizzle does not matter.
  for (int i = threadIdx.x; i < ONES_BYTES / 4; i += THREADS)
    reinterpret_cast<uint32_t*>(ones)[i] = 0x3C003C00u;
  gptq::fence_proxy_async_smem();
  if (warp == 0 && lane == 0) {
    gptq::tma_prefetch_desc(&tmX);
    gptq::tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) {
    gptq::tmem_alloc(tmem_slot, TMEM_COLS);
    gptq::tmem_relinquish();
  }
  gptq::tc_fence_before();
  __syncthreads();
  gptq::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nkb = args.K / BK;

  if (!*skip_flag) {
    if (warp == 0) {
      if (lane == 0) {  // ---------------- TMA producer ----------------
        int stage = 0;
        uint32_t phase = 0;
        uint32_t filled = 0, fill_parity = 0;
        for (int t = blockIdx.x; t < args.n_tiles && !*abort_flag; t += gridDim.x) {
          int tm, tn;
          tile_of(t, args, tm, tn);
          for (int kb = 0; kb < nkb; ++kb) {
            if (!gptq::mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
            uint8_t* sx = smem + stage * STAGE_BYTES;
            gptq::mbar_arrive_expect_tx(&full[stage], X_BYTES + Q_BYTES);
            gptq::tma_load_2d(sx, &tmX, &full[stage], kb * BK, tm * BM);
            gptq::tma_load_2d(sx + X_BYTES, &tmQ, &full[stage], kb * (BK / 8), tn * BN);
            filled |= 1u << stage;
            fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
        if (*abort_flag)
          for (int s = 0; s < STAGES; ++s)
            if (filled & (1u << s)) gptq::mbar_drain(&full[s], (fill_parity >> s) & 1u);
      }
    } else if (warp == 1) {
      if (lane == 0) {  // ---------------- MMA issuer ----------------
        const uint32_t ones_base = gptq::smem_u32(ones);
        int stage = 0;
        uint32_t phase = 0;
        int buf = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < args.n_tiles && ok && !*abort_flag; t += gridDim.x) {
          for (int kc = 0; kc < nkb && ok; kc += FOLD_KB) {
            if (!gptq::mbar_wait(&acc_empty[buf], acc_phase ^ 1, abort_flag)) { ok = false; break; }
            gptq::tc_fence_after();
            const uint32_t d_acc = tmem_base + ACC_COL + (uint32_t)(buf * BN);
            const uint32_t d_xs = tmem_base + XS_COL + (uint32_t)(buf * 16);
            for (int kb = kc; kb < kc + FOLD_KB; ++kb) {
              if (!gptq::mbar_wait(&conv[stage], phase, abort_flag)) { ok = false; break; }
              gptq::tc_fence_after();
              const uint32_t sx = gptq::smem_u32(smem + stage * STAGE_BYTES);
              const uint32_t sb = sx + X_BYTES + Q_BYTES;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                const uint32_t accumulate = (kb > kc || kk > 0) ? 1u : 0u;
                const uint64_t da = desc_k64(sx, kk);
                gptq::mma_f16(d_acc, da, desc_k64(sb, kk), IDESC, accumulate);
                gptq::mma_f16(d_xs, da, desc_k64(ones_base, kk), IDESC_XS, accumulate);
              }
              gptq::mma_commit(&empty[stage]);
              if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            gptq::mma_commit(&acc_full[buf]);
            if (++buf == 2) { buf = 0; acc_phase ^= 1; }
          }
        }
        if (*abort_flag) {
          gptq::mma_commit(mma_drain);
          gptq::mbar_drain(mma_drain, 0);
        }
      }
    } else if (warp < EPI_WARP0) {
      // ---------- converters: weight row n of the block -> fp16 codes; fold parameters ----------
      const int n = threadIdx.x - CONV_WARP0 * 32;  // 0..127
      int stage = 0;
      uint32_t phase = 0;
      int pb = 0;
      uint32_t par_phase = 0;
      bool ok = true;
      // The row's fp16 (s, z) of the fold at column k0, read from global memory one fold before
      // they are needed, so that the decoding never waits on them.
      auto fold_params = [&](int row, int k0, uint16_t& sh, uint16_t& zh) {
        sh = 0;
        zh = 0;
        if (row < args.N) {
          const int gi = args.group_size > 0 ? k0 / args.group_size : 0;
          const long long o = (long long)row * args.G + gi;
          sh = __ldg(args.scales + o);
          zh = __ldg(args.zeros + o);
        }
      };
      for (int t = blockIdx.x; t < args.n_tiles && ok && !*abort_flag; t += gridDim.x) {
        int tm, tn;
        tile_of(t, args, tm, tn);
        const int row = tn * BN + n;
        uint16_t nxt_s, nxt_z;
        fold_params(row, 0, nxt_s, nxt_z);
        for (int kb = 0; kb < nkb; ++kb) {
          if (kb % FOLD_KB == 0) {  // this fold's s * 2^24 and -s * z of the row
            const float s = __half2float(__ushort_as_half(nxt_s));
            // zero points are integers; another value is rounded to one
            const float z = rintf(__half2float(__ushort_as_half(nxt_z)));
            if (kb + FOLD_KB < nkb) fold_params(row, (kb + FOLD_KB) * BK, nxt_s, nxt_z);
            if (!gptq::mbar_wait(&par_empty[pb], par_phase ^ 1, abort_flag)) { ok = false; break; }
            par[pb * PAR_FLOATS + n] = s * 16777216.f;  // 0 past the rows: (s, z) = (0, 0)
            par[pb * PAR_FLOATS + BN + n] = -s * z;
            __syncwarp();
            if (lane == 0) gptq::mbar_arrive(&par_full[pb]);
            if (++pb == 2) { pb = 0; par_phase ^= 1; }
          }
          if (!gptq::mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          uint8_t* sq = smem + stage * STAGE_BYTES + X_BYTES;
          uint8_t* sb = sq + Q_BYTES;
          // Row n's 64 codes: 8 words, word i holding codes 8i .. 8i + 7 (nibbles, LSB first).
          // Pair j of word i is (code 8i + 2j, code 8i + 2j + 1): byte j of w and byte j of
          // w >> 4 placed in the two halves, masked to their low nibbles.
          const uint4 q0 = *reinterpret_cast<const uint4*>(sq + n * 32);
          const uint4 q1 = *reinterpret_cast<const uint4*>(sq + n * 32 + 16);
          const uint32_t w8[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t w = w8[i], u = w >> 4;
            uint4 v;
            v.x = __byte_perm(w, u, 0x0400) & 0x000F000Fu;
            v.y = __byte_perm(w, u, 0x0501) & 0x000F000Fu;
            v.z = __byte_perm(w, u, 0x0602) & 0x000F000Fu;
            v.w = __byte_perm(w, u, 0x0703) & 0x000F000Fu;
            // K-major 128-byte swizzle: 16-byte chunk i of row n at chunk i ^ (n & 7).
            *reinterpret_cast<uint4*>(sb + n * 128 + ((i ^ (n & 7)) << 4)) = v;
          }
          gptq::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) gptq::mbar_arrive(&conv[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    } else {
      // ---------------- epilogue ----------------
      const int quarter = warp & 3;
      const int col_half = (warp - EPI_WARP0) >> 2;
      const uint32_t lane_field = (uint32_t)(quarter * 32) << 16;
      int buf = 0;
      uint32_t acc_phase = 0;
      int pb = 0;
      uint32_t par_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.n_tiles && ok && !*abort_flag; t += gridDim.x) {
        int tm, tn;
        tile_of(t, args, tm, tn);
        float y[EPI_COLS];
#pragma unroll
        for (int e = 0; e < EPI_COLS; ++e) y[e] = 0.f;
        for (int kc = 0; kc < nkb; kc += FOLD_KB) {
          if (!gptq::mbar_wait(&acc_full[buf], acc_phase, abort_flag) ||
              !gptq::mbar_wait(&par_full[pb], par_phase, abort_flag)) {
            ok = false;
            break;
          }
          gptq::tc_fence_after();
          uint32_t xs_bits;
          __syncwarp();
          asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];"
                       : "=r"(xs_bits)
                       : "r"(tmem_base + lane_field + XS_COL + (uint32_t)(buf * 16)));
          // the wait names the register, so that no use of it is scheduled before the load lands
          asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(xs_bits)::"memory");
          const float xs = __uint_as_float(xs_bits);
          const float* sp = par + pb * PAR_FLOATS + EPI_COLS * col_half;
          const float* nsz = sp + BN;
#pragma unroll
          for (int q = 0; q < EPI_COLS / 32; ++q) {
            uint32_t r[32];
            __syncwarp();
            gptq::tmem_ld_32x32b_x32(
                tmem_base + lane_field + ACC_COL + (uint32_t)(buf * BN + EPI_COLS * col_half + 32 * q),
                r);
            gptq::tmem_ld_wait();
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 a = *reinterpret_cast<const float4*>(sp + 32 * q + 4 * e4);
              const float4 c = *reinterpret_cast<const float4*>(nsz + 32 * q + 4 * e4);
              const float av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int k = 32 * q + 4 * e4 + e;
                y[k] = fmaf(av[e], __uint_as_float(r[4 * e4 + e]), fmaf(cv[e], xs, y[k]));
              }
            }
          }
          gptq::tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            gptq::mbar_arrive(&acc_empty[buf]);
            gptq::mbar_arrive(&par_empty[pb]);
          }
          if (++buf == 2) { buf = 0; acc_phase ^= 1; }
          if (++pb == 2) { pb = 0; par_phase ^= 1; }
        }
        if (!ok) break;
        const int m = tm * BM + quarter * 32 + lane;
        if (m < args.M) {
          float* yrow = args.Y + (long long)m * args.ldy;
#pragma unroll
          for (int c = 0; c < EPI_COLS / 4; ++c) {
            const int col = tn * BN + EPI_COLS * col_half + 4 * c;
            if (col + 4 <= args.N && (args.ldy & 3) == 0) {
              *reinterpret_cast<float4*>(yrow + col) =
                  make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (col + e < args.N) yrow[col + e] = y[4 * c + e];
            }
          }
        }
      }
    }
  }

  gptq::tc_fence_before();
  __syncthreads();
  if (warp == 1) gptq::tmem_dealloc(tmem_base, TMEM_COLS);
  if (threadIdx.x == 0 && *abort_flag) gptq::set_status(args.status_w, GPTQ_ERR_TIMEOUT, 4);
}

}  // namespace

namespace gptq_host {

int dequant_gemm(const uint32_t* qweight, int n, int d, const uint16_t* scales_f16,
                 const uint16_t* zeros_f16, int n_groups, int group_size, const uint16_t* x_f16,
                 int m, long long ldx, float* y, long long ldy, const int32_t* status,
                 cudaStream_t stream) {
  CUtensorMap tx, tq;
  if (make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x_f16, (uint64_t)d, (uint64_t)m,
                   (uint64_t)ldx * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) != 0)
    return GPTQ_ERR_CUDA;
  // Packed words: row r holds d / 8 words; a box is 8 words (64 codes) of 128 rows.
  if (make_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, qweight, (uint64_t)d / 8, (uint64_t)n,
                   (uint64_t)d / 2, BK / 8, BN, CU_TENSOR_MAP_SWIZZLE_NONE) != 0)
    return GPTQ_ERR_CUDA;
  DqArgs a;
  a.M = m; a.N = n; a.K = d;
  a.scales = scales_f16;
  a.zeros = zeros_f16;
  a.G = n_groups;
  a.group_size = group_size;
  a.Y = y;
  a.ldy = ldy;
  a.tiles_m = (m + BM - 1) / BM;
  a.tiles_n = (n + BN - 1) / BN;
  a.n_tiles = a.tiles_m * a.tiles_n;
  a.status = status;
  a.status_w = const_cast<int32_t*>(status);
  if (ensure_smem_attr(reinterpret_cast<const void*>(dequant_gemm_kernel), SMEM_BYTES) != 0)
    return GPTQ_ERR_CUDA;
  const int sms = num_sms();
  const int grid = a.n_tiles < sms ? a.n_tiles : sms;
  dequant_gemm_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(tx, tq, a);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
