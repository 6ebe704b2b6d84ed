// syrk_bf16.cu — H_upper += alpha * X^T X for token-major bf16 X on tcgen05 tensor cores.
//
// Computes the layer Hessian H = 2 X X^T ("INT4 and GPTQ Quantization", §The Quantization Error
// and Layerwise Objective; "GPTQ: Mathematical Foundations ...", §Second-Order Taylor Expansion
// and the Hessian). X is stored token-major [N, d] (row t = one calibration token), so both
// GEMM operands are X itself read "MN-major": element (t, i) sits at t*ldx + i.
//
// Design (one CTA per SM, persistent):
//   * Work unit = (256 x 256 output tile with i-block <= j-block, token chunk). Only tiles on or
//     above the diagonal are scheduled; the token range is split into chunks of at most 8192
//     tokens (and further only when the tiles alone cannot fill the SMs). Units are ordered by
//     groups of tiles, token range by token range inside a group, so that the CTAs running
//     together share the L2-resident panels of X of one group and one range (syrk_units.cuh).
//   * warp 0: TMA producer — per 64-token k-block, four 64x64 boxes of X for the A tile (rows
//     i0..i0+255) and four for the B tile (j0..j0+255), 128-byte swizzled, 3-stage ring.
//   * warp 1: TMEM owner and MMA issuer — per 16-token step two tcgen05.mma kind::f16 of
//     M=128, N=256, one per half of the A tile, sharing the B operand; both operands MN-major.
//     The 256 x 256 fp32 accumulator fills TMEM (the halves at columns 0 and 256). A 256-row
//     tile needs two thirds of the operand bytes per MMA of a 128-row one, which keeps the
//     L2 -> SM feed and the TMA latency well inside what the ring covers.
//   * warps 2-5: epilogue — tcgen05.ld 32 rows x 32 columns, scale by alpha, zero the strictly
//     lower triangle, stage in 128B-swizzled smem and add into H with a TMA reduce-add
//     (cp.reduce.async.bulk.tensor .add), which also clips the ragged edge of H. The MMA warp
//     starts the next unit once both halves are drained.
//   * Every mbarrier wait is bounded; on timeout the CTA records GPTQ_ERR_TIMEOUT, leaves its
//     loops, waits (bounded) for the loads and MMAs it already issued, frees TMEM and returns.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "syrk_units.cuh"
#include "tri_fill.cuh"

namespace {

constexpr int BM = 256, BN = 256, BK = 64, STAGES = 3;
constexpr int MMA_M = 128;                        // rows per tcgen05.mma (two per k-step)
constexpr int BOX = 64;                           // 64 bf16 = 128 B inner, 64 tokens outer
constexpr int BOX_BYTES = BOX * BOX * 2;          // 8 KB
constexpr int A_BYTES = 4 * BOX_BYTES;            // 32 KB
constexpr int B_BYTES = 4 * BOX_BYTES;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // 64 KB
constexpr int EPI_WARPS = 4;
constexpr int EPI_TILE_BYTES = 32 * 32 * 4;       // 32 rows x 32 fp32 = 4 KB
constexpr int EPI_BUFS = 2;
constexpr int SMEM_DATA = STAGES * STAGE_BYTES + EPI_WARPS * EPI_BUFS * EPI_TILE_BYTES;
constexpr int SMEM_BYTES = SMEM_DATA + 1024 /*align*/ + 256 /*barriers*/;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;               // the two 128 x 256 halves of the tile
constexpr uint32_t IDESC = gptq::instr_desc(/*bf16*/ 1, /*A MN*/ 1, /*B MN*/ 1, MMA_M, BN);

struct SyrkArgs {
  int d, n_tb, n_tiles, n_split, kb_per_split, nkb_total;
  int grp;  // tile rows / columns per group (syrk_units.cuh)
  long long n_units;
  float alpha;
  int32_t* status;
};

__global__ void __launch_bounds__(THREADS, 1)
syrk_bf16_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_x,
                         const __grid_constant__ CUtensorMap tmap_h, SyrkArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SMEM_DATA);
  uint64_t* full = bars;                 // [STAGES]
  uint64_t* empty = bars + STAGES;       // [STAGES]
  uint64_t* acc_full = bars + 2 * STAGES;       // accumulator complete
  uint64_t* acc_empty = bars + 2 * STAGES + 1;  // accumulator drained
  uint64_t* mma_drain = bars + 2 * STAGES + 2;  // abort path: the issued MMAs have completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* skip_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *skip_flag = gptq::status_bad(args.status) ? 1 : 0;
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      gptq::mbar_init(&full[s], 1);
      gptq::mbar_init(&empty[s], 1);
    }
    gptq::mbar_init(acc_full, 1);
    gptq::mbar_init(acc_empty, EPI_WARPS);
    gptq::mbar_init(mma_drain, 1);
    gptq::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    gptq::tma_prefetch_desc(&tmap_x);
    gptq::tma_prefetch_desc(&tmap_h);
  }
  if (warp == 1) {
    gptq::tmem_alloc(tmem_slot, TMEM_COLS);
    gptq::tmem_relinquish();
  }
  gptq::tc_fence_before();
  __syncthreads();
  gptq::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool skip = *skip_flag != 0;

  if (!skip) {
    if (warp == 0) {
      // ------------------------------- TMA producer -------------------------------
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        uint32_t filled = 0, fill_parity = 0;  // per stage: filled at least once, last parity
        for (long long u = blockIdx.x; u < args.n_units && !*abort_flag; u += gridDim.x) {
          int ib, jb, split;
          gptq::syrk_unit_coords(u, args.n_tb, args.grp, args.n_split, ib, jb, split);
          const int kb0 = split * args.kb_per_split;
          const int kb1 = min(args.nkb_total, kb0 + args.kb_per_split);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!gptq::mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
            uint8_t* sa = stage_base + stage * STAGE_BYTES;
            uint8_t* sb = sa + A_BYTES;
            gptq::mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
            const int t = kb * BK;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              gptq::tma_load_2d(sa + q * BOX_BYTES, &tmap_x, &full[stage], ib * BM + q * BOX, t);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              gptq::tma_load_2d(sb + q * BOX_BYTES, &tmap_x, &full[stage], jb * BN + q * BOX, t);
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
      // ------------------------------- MMA issuer ---------------------------------
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        uint32_t acc_phase = 0;
        for (long long u = blockIdx.x; u < args.n_units && !*abort_flag; u += gridDim.x) {
          int ib_, jb_, split;
          gptq::syrk_unit_coords(u, args.n_tb, args.grp, args.n_split, ib_, jb_, split);
          const int kb0 = split * args.kb_per_split;
          const int kb1 = min(args.nkb_total, kb0 + args.kb_per_split);
          if (!gptq::mbar_wait(acc_empty, acc_phase ^ 1, abort_flag)) break;
          gptq::tc_fence_after();
          const uint32_t d_tmem = tmem_base;  // half h at column h * BN
          bool ok = true;
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!gptq::mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
            gptq::tc_fence_after();
            const uint32_t sa = gptq::smem_u32(stage_base + stage * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // MN-major, 128B swizzle: MN atoms (64 elements) every 8 KB (one TMA box),
              // 8-token K groups every 1 KB; K=16 advances 16 rows = 2 KB. The second half of
              // the A tile (rows 128..255) starts two boxes further on.
              const uint64_t bdesc = gptq::smem_desc_sw128(sb + kk * 2048, BOX_BYTES, 1024);
              const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
#pragma unroll
              for (int h = 0; h < BM / MMA_M; ++h) {
                const uint64_t adesc = gptq::smem_desc_sw128(
                    sa + h * 2 * BOX_BYTES + kk * 2048, BOX_BYTES, 1024);
                gptq::mma_f16(d_tmem + (uint32_t)(h * BN), adesc, bdesc, IDESC, acc);
              }
            }
            gptq::mma_commit(&empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
          if (!ok) break;
          gptq::mma_commit(acc_full);
          acc_phase ^= 1;
        }
        if (*abort_flag) {  // the MMAs already issued finish before TMEM is released
          gptq::mma_commit(mma_drain);
          gptq::mbar_drain(mma_drain, 0);
        }
      }
    } else {
      // ------------------------------- epilogue -----------------------------------
      const int quarter = warp & 3;  // TMEM lanes 32*quarter .. 32*quarter+31
      uint8_t* my_bufs = epi_base + (warp - 2) * EPI_BUFS * EPI_TILE_BYTES;
      uint32_t acc_phase = 0;
      uint32_t chunk_counter = 0;
      for (long long u = blockIdx.x; u < args.n_units && !*abort_flag; u += gridDim.x) {
        int ib, jb, split;
        gptq::syrk_unit_coords(u, args.n_tb, args.grp, args.n_split, ib, jb, split);
        if (!gptq::mbar_wait(acc_full, acc_phase, abort_flag)) break;
        gptq::tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < (BM / MMA_M) * (BN / 32); ++cc) {
          const int h = cc / (BN / 32), c = cc % (BN / 32);
          const int row0 = ib * BM + h * MMA_M + quarter * 32;
          const int row = row0 + lane;
          const int col0 = jb * BN + c * 32;
          uint32_t r[32];
          __syncwarp();  // tcgen05.ld is warp-collective: reconverge before every load
          const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                 (uint32_t)(h * BN + c * 32);
          gptq::tmem_ld_32x32b_x32(taddr, r);
          gptq::tmem_ld_wait();
          // Chunk entirely below the diagonal or outside H: nothing to add.
          const bool live = row0 < args.d && col0 < args.d && row0 <= col0 + 31;
          if (!live) continue;
          uint8_t* sbuf = my_bufs + (chunk_counter & 1) * EPI_TILE_BYTES;
          if (chunk_counter >= 2) {
            if (lane == 0) gptq::bulk_wait_read<1>();
            __syncwarp();
          }
          ++chunk_counter;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            float4 v;
            float* vp = reinterpret_cast<float*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int col = col0 + q4 * 4 + e;
              const float x = __uint_as_float(r[q4 * 4 + e]) * args.alpha;
              vp[e] = (row <= col) ? x : 0.0f;
            }
            // 128B swizzle: 16-byte chunk q4 of row `lane` lives at chunk q4 ^ (lane & 7).
            *reinterpret_cast<float4*>(sbuf + lane * 128 + ((q4 ^ (lane & 7)) << 4)) = v;
          }
          gptq::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            gptq::tma_reduce_add_2d(&tmap_h, sbuf, col0, row0);
            gptq::bulk_commit();
          }
        }
        gptq::tc_fence_before();
        __syncwarp();
        if (lane == 0) gptq::mbar_arrive(acc_empty);
        acc_phase ^= 1;
      }
      if (lane == 0) gptq::bulk_wait<0>();
      __syncwarp();
    }
  }

  gptq::tc_fence_before();
  __syncthreads();
  if (warp == 1) gptq::tmem_dealloc(tmem_base, TMEM_COLS);
  if (threadIdx.x == 0 && *abort_flag) gptq::set_status(args.status, GPTQ_ERR_TIMEOUT, 1);
}

// H's upper triangle (with the diagonal) = 0 before a non-accumulating product: rows over the
// blocks, 16-byte stores along each row's span (tri_fill.cuh).
__global__ void zero_upper_kernel(float* H, int d, long long ldh, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  for (long long r = blockIdx.x; r < d; r += gridDim.x) {
    long long lo, hi;
    gptq::tri_row_span(gptq::kUpperWithDiag, r, d, lo, hi);
    gptq::fill_span(H + r * ldh, lo, hi, 0.f, threadIdx.x, blockDim.x);
  }
}

}  // namespace

namespace gptq_host {

int syrk_bf16_upper(float* H, int d, long long ldh, const void* X, long long n_tokens,
                    long long ldx, float alpha, int accumulate, int32_t* status,
                    cudaStream_t stream) {
  if (!accumulate) {
    const int grid = d < num_sms() * 8 ? d : num_sms() * 8;
    zero_upper_kernel<<<grid, 256, 0, stream>>>(H, d, ldh, status);
    if (cudaGetLastError() != cudaSuccess) return GPTQ_ERR_CUDA;
  }
  if (n_tokens == 0) return GPTQ_OK;

  CUtensorMap tx, th;
  if (make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, (uint64_t)d, (uint64_t)n_tokens,
                   (uint64_t)ldx * 2, BOX, BOX, CU_TENSOR_MAP_SWIZZLE_128B) != 0)
    return GPTQ_ERR_CUDA;
  if (make_tmap_2d(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, (uint64_t)d, (uint64_t)d,
                   (uint64_t)ldh * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B) != 0)
    return GPTQ_ERR_CUDA;

  SyrkArgs a;
  a.d = d;
  static_assert(BM == BN, "square tiles: one tile grid for rows and columns");
  a.n_tb = (d + BM - 1) / BM;
  a.n_tiles = a.n_tb * (a.n_tb + 1) / 2;
  a.nkb_total = (int)((n_tokens + BK - 1) / BK);
  // The tensor core rounds toward zero when it adds into its fp32 accumulator (a one-sided
  // error of up to one ulp per step on these like-signed sums), so one accumulator covers at
  // most kMaxKb k-blocks (8192 tokens); the chunks are summed into H by the TMA reduce-add.
  // Beyond that minimum, split the token range only as far as needed to fill the SMs: pick the
  // split count whose last wave is fullest, preferring >= 4 waves.
  constexpr int kMaxKb = 128;
  const int sms = num_sms();
  const int s_min = (a.nkb_total + kMaxKb - 1) / kMaxKb;
  int best_split = s_min;
  double best_score = -1.0;
  for (int s = s_min; s <= s_min + 64 && s <= a.nkb_total; ++s) {
    const int per = (a.nkb_total + s - 1) / s;
    const int s_eff = (a.nkb_total + per - 1) / per;
    if (s_eff != s) continue;
    const double units = (double)a.n_tiles * s;
    const double waves = units / sms;
    const double eff = waves / ceil(waves);
    const double score = eff - (waves < 4.0 ? 0.25 : 0.0) - 0.002 * (s - s_min);
    if (score > best_score) { best_score = score; best_split = s; }
    if ((double)a.n_tiles * s_min >= 8.0 * sms) break;  // plenty of units already
  }
  a.n_split = best_split;
  a.kb_per_split = (a.nkb_total + best_split - 1) / best_split;
  a.n_units = (long long)a.n_tiles * a.n_split;
  a.alpha = alpha;
  a.status = status;
  const int grid = (int)(a.n_units < sms ? a.n_units : sms);
  // Groups: when every 256-channel panel of one token range fits in half of L2, one group (the
  // CTAs share the whole range); otherwise grp x grp tiles with grp^2 about one wave, so the
  // CTAs running together need 2 grp panels.
  const double panel_bytes = (double)BM * a.kb_per_split * BK * 2.0;
  if (a.n_tb * panel_bytes <= 64.0 * 1024 * 1024) {
    a.grp = a.n_tb;
  } else {
    a.grp = (int)floor(sqrt((double)grid));
    if (a.grp < 1) a.grp = 1;
  }

  if (ensure_smem_attr(reinterpret_cast<const void*>(syrk_bf16_tcgen05_kernel), SMEM_BYTES) != 0)
    return GPTQ_ERR_CUDA;
  syrk_bf16_tcgen05_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(tx, th, a);
  return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
