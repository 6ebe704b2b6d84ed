// gemv.cu — dequantizing matrix-vector product on the packed format (the W4A16 / W3A16 consumer
// of gptq_pack's output).
//
// "GPTQ: Mathematical Foundations ...", §Inference Execution and Modern Kernel Architectures:
// packed codes are streamed from HBM, unpacked with bit shifts and dequantized in registers,
// w_hat = (q - z) * s with the FP16 scale and zero, and multiplied with the FP16 activations,
// accumulating in higher precision (fused dequantize-and-GEMV for low-batch decoding).
//
// Y[b, r] = sum_c (code[r, c] - z[r, G(c)]) * s[r, G(c)] * X[b, c], b < batch <= 8, with
// G(c) = g_idx[c], or c / group_size when g_idx is NULL (0 for one group per row).
//
// Warp-per-row path (act-order g_idx, groups shorter than 128 columns, d_in not a multiple of
// 128): one warp per output row. A row of qweight is one LSB-first bit stream along d_in
// (code k at stream bits [b k, b k + b)); lane l takes runs of 32 codes, i.e. exactly BITS words,
// run l, l + 32, ..., so a warp reads 128 * BITS contiguous bytes per step (16-byte loads for
// 4 and 8 bits). The 32 codes of a run come out of the BITS words with compile-time shifts (a
// 3-bit code may straddle two words) and become exact fp32 values code - z by the 2^23
// exponent trick. With contiguous groups of at least 32 columns a run lies in one group:
// Y += s * sum (q - z) x; otherwise the parameters are looked up per column. Activations are
// read 8 halves at a time; all sums are fp32, added across the warp with shuffles.
//
// Tensor-core path (2-, 3-, 4- and 8-bit codes, contiguous groups that are whole multiples of
// 128 columns or one group per row, d_in a multiple of 128): work items are (row tile, 128-column
// chunk); a warp's item is 8 mma.sync m16n8k16 (fp16 in, fp32 accumulate) per 16-row m-tile with
// A = the codes and B = X (16 columns x 8 batch rows, lanes past the batch reading its last row).
// Lane (g, t) holds rows g and g + 8 of each m-tile and the 32 columns [32 t, 32 t + 32) of the
// chunk, exactly `bits` packed words per row. The codes enter A as fp16 subnormals decoded in
// place (gemv_pairs.cuh: one AND per two codes), X takes the same column order with byte
// permutes, and the scale and zero point are applied once per chunk in fp32:
// Y += s 2^(24 - pos) sum_class - s z sum(x), the chunk's sum of x coming from MMAs with an
// all-ones A. The grid is persistent and splits the items evenly over the SMs; partial sums of
// a row tile are added into Y (zeroed first) with atomic adds.
#include <cuda_fp16.h>

#include "common.cuh"
#include "gemv_pairs.cuh"
#include "kernels.h"

namespace {

constexpr int GEMV_THREADS = 256;
constexpr int kMaxBatch = 8;

template <int BITS>
__device__ __forceinline__ void load_run(const uint32_t* __restrict__ src, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 8) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (BITS == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
    w[0] = v.x; w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) w[i] = __ldg(src + i);
  }
}

// Code k (0..31) of a run held in BITS words, as an integer.
template <int BITS, int K>
__device__ __forceinline__ uint32_t code_bits(const uint32_t (&w)[BITS]) {
  constexpr int bit = K * BITS, wi = bit / 32, off = bit % 32;
  constexpr uint32_t mask = (1u << BITS) - 1u;
  uint32_t v = w[wi] >> off;
  if constexpr (off + BITS > 32) v |= w[wi + 1] << (32 - off);
  return v & mask;
}

// code - z, exact in fp32: 2^23 + code is the float with bit pattern 0x4B000000 | code, and
// zoff = 2^23 + z is exact for integer z < 2^23.
template <int BITS, int K>
__device__ __forceinline__ float code_minus_z(const uint32_t (&w)[BITS], float zoff) {
  return __uint_as_float(0x4B000000u | code_bits<BITS, K>(w)) - zoff;
}

template <int BITS, int K = 0>
__device__ __forceinline__ void codes_minus_z(const uint32_t (&w)[BITS], float zoff,
                                              float (&qz)[32]) {
  if constexpr (K < 32) {
    qz[K] = code_minus_z<BITS, K>(w, zoff);
    codes_minus_z<BITS, K + 1>(w, zoff, qz);
  }
}

// dot of 32 fp32 values with 32 fp16 activations at x (16-byte aligned).
__device__ __forceinline__ float dot32(const float (&qz)[32], const __half* __restrict__ x) {
  const uint4* xp = reinterpret_cast<const uint4*>(x);
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = __ldg(xp + i);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[j]));
      dot = fmaf(qz[8 * i + 2 * j], f.x, dot);
      dot = fmaf(qz[8 * i + 2 * j + 1], f.y, dot);
    }
  }
  return dot;
}

// One run of 32 columns starting at c0: acc[b] += sum_k w_hat[k] X[b, c0 + k].
template <int BITS, int MAXB>
__device__ __forceinline__ void run_dot(const uint32_t (&w)[BITS], int c0, bool run_groups,
                                        const __half* __restrict__ srow,
                                        const __half* __restrict__ zrow, int group_size,
                                        const int32_t* __restrict__ g_idx,
                                        const __half* __restrict__ X, long long ldx, int batch,
                                        float (&acc)[MAXB]) {
  float qz[32];
  if (run_groups) {
    const int gi = group_size <= 0 ? 0 : c0 / group_size;
    const float s = __half2float(srow[gi]);
    codes_minus_z<BITS>(w, 8388608.f + __half2float(zrow[gi]), qz);
#pragma unroll
    for (int b = 0; b < MAXB; ++b)
      if (b < batch) acc[b] = fmaf(s, dot32(qz, X + b * ldx + c0), acc[b]);
  } else {
    // Parameters per column: qz holds (code - z) * s.
    codes_minus_z<BITS>(w, 8388608.f, qz);
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int c = c0 + k;
      const int gi = g_idx ? g_idx[c] : (group_size <= 0 ? 0 : c / group_size);
      qz[k] = (qz[k] - __half2float(zrow[gi])) * __half2float(srow[gi]);
    }
#pragma unroll
    for (int b = 0; b < MAXB; ++b)
      if (b < batch) acc[b] += dot32(qz, X + b * ldx + c0);
  }
}

// MAXB: the largest batch this instance handles (1 for decoding one token, kMaxBatch otherwise).
template <int BITS, int MAXB>
__global__ void __launch_bounds__(GEMV_THREADS)
dequant_gemv_kernel(const uint32_t* __restrict__ qweight, int n, int d, long long words_per_row,
                    const __half* __restrict__ scales, const __half* __restrict__ zeros, int G,
                    int group_size, const int32_t* __restrict__ g_idx,
                    const __half* __restrict__ X, long long ldx, int batch, float* __restrict__ Y,
                    long long ldy) {
  const int row = blockIdx.x * (GEMV_THREADS / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n) return;
  const uint32_t* wrow = qweight + (long long)row * words_per_row;
  const __half* srow = scales + (long long)row * G;
  const __half* zrow = zeros + (long long)row * G;
  // Contiguous groups of >= 32 columns (or one group per row): a run lies inside one group.
  const bool run_groups = g_idx == nullptr && (group_size <= 0 || group_size % 32 == 0);
  float acc[MAXB];
#pragma unroll
  for (int b = 0; b < MAXB; ++b) acc[b] = 0.f;
  const int runs = d / 32;
  // Two runs per lane and step, both loads issued before either is used, so that twice the
  // bytes are in flight per warp.
  for (int r = lane; r < runs; r += 64) {
    uint32_t w0[BITS], w1[BITS];
    const bool has1 = r + 32 < runs;
    load_run<BITS>(wrow + (long long)r * BITS, w0);
    if (has1) load_run<BITS>(wrow + (long long)(r + 32) * BITS, w1);
    run_dot<BITS, MAXB>(w0, 32 * r, run_groups, srow, zrow, group_size, g_idx, X, ldx, batch, acc);
    if (has1)
      run_dot<BITS, MAXB>(w1, 32 * (r + 32), run_groups, srow, zrow, group_size, g_idx, X, ldx,
                          batch, acc);
  }
#pragma unroll
  for (int b = 0; b < MAXB; ++b) {
    float v = acc[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && b < batch) Y[b * ldy + row] = v;
  }
}

// ---------------------------------------------------------------------------------------------
// Tensor-core path
// ---------------------------------------------------------------------------------------------
constexpr int kChunk = 128;        // columns of one warp step (8 k-steps of 16)

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Packed words are read once: keep them out of L1, which holds the activations and the group
// parameters that every chunk re-reads.
template <int BITS>
__device__ __forceinline__ void load_stream(const uint32_t* __restrict__ src, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 2) {
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(w[0]), "=r"(w[1]) : "l"(src));
  } else if constexpr (BITS == 3) {  // a lane's run starts on a 12-byte boundary
#pragma unroll
    for (int i = 0; i < 3; ++i)
      asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(w[i]) : "l"(src + i));
  } else {
#pragma unroll
    for (int i = 0; i < BITS; i += 4)
      asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(w[i]), "=r"(w[i + 1]), "=r"(w[i + 2]), "=r"(w[i + 3])
                   : "l"(src + i));
  }
}

// The activations of pair P's two columns as an fp16 pair (xr: the run's 32 halves, two per
// word), in the pairing of gemv_pairs.cuh.
template <int BITS, int P>
__device__ __forceinline__ uint32_t pair_x(const uint32_t (&xr)[16]) {
  constexpr gptq::PairDesc d = gptq::PairSet<BITS>::pair(P);
  if constexpr (d.j2 == d.j1 + 1 && (d.j1 & 1) == 0) {
    return xr[d.j1 >> 1];
  } else {
    constexpr uint32_t lo = (d.j1 & 1) ? 0x32u : 0x10u;
    constexpr uint32_t hi = (d.j2 & 1) ? 0x7600u : 0x5400u;
    return __byte_perm(xr[d.j1 >> 1], xr[d.j2 >> 1], hi | lo);
  }
}

template <int BITS, int Q = 0>
__device__ __forceinline__ void act_pairs(const uint32_t (&xr)[16], uint32_t (&b)[16]) {
  if constexpr (Q < 16) {
    b[Q] = pair_x<BITS, Q>(xr);
    act_pairs<BITS, Q + 1>(xr, b);
  }
}

// The 8 MMAs of one m-tile and chunk: rows g (words wa) and g + 8 (words wb).
template <int BITS, int Q = 0>
__device__ __forceinline__ void tile_mmas(const uint32_t (&wa)[BITS], const uint32_t (&wb)[BITS],
                                          const uint32_t (&b)[16],
                                          float (&dc)[gptq::PairSet<BITS>::NCLS][4]) {
  if constexpr (Q < 8) {
    using gptq::pair_code;
    mma_16816(dc[gptq::PairSet<BITS>::cls(Q)], pair_code<BITS>(wa, 2 * Q),
              pair_code<BITS>(wb, 2 * Q), pair_code<BITS>(wa, 2 * Q + 1),
              pair_code<BITS>(wb, 2 * Q + 1), b[2 * Q], b[2 * Q + 1]);
    tile_mmas<BITS, Q + 1>(wa, wb, b, dc);
  }
}

// Work items are (row tile, chunk) pairs, a row tile being MT m-tiles of 16 rows: the activation
// pairs and the all-ones MMAs of a chunk serve every m-tile. The grid is persistent (every CTA
// resident at once) and the items, in tile-major order, are split evenly over the CTAs and then
// over each CTA's warps, so every SM gets the same work whatever the row count; a warp that
// finishes a row tile (or its range) adds its partial sums into Y, which the launcher zeroes.
// The warps run independently (no barrier), each with a ring of 2 items' packed words per row.
// (Measured on B200 at 8192 x 28672, 4-bit, batch 1: 42.9 us; one producer warp per CTA
// preparing the activation pairs for 4 to 8 lock-stepped consumer warps through shared memory:
// 57 to 67 us.)
constexpr int kTcWarps = 8;

// Row r of this lane in row tile `tile`: m-tile r / 2, half r % 2. Rows past the end read the
// last row (valid memory) and are not written.
template <int MT>
__device__ __forceinline__ int lane_row(int tile, int r, int g, int n) {
  return min(tile * 16 * MT + 16 * (r >> 1) + g + 8 * (r & 1), n - 1);
}

template <int BITS, int MT>
__global__ void __launch_bounds__(kTcWarps * 32)
dequant_gemv_tc_kernel(const uint32_t* __restrict__ qweight, int n, int d, long long wpr,
                       const __half* __restrict__ scales, const __half* __restrict__ zeros, int G,
                       int chunks_per_group, const __half* __restrict__ X, long long ldx,
                       int batch, float* __restrict__ Y, long long ldy) {
  using PS = gptq::PairSet<BITS>;
  constexpr int NR = 2 * MT;                // rows per lane: m-tile m, half h -> 2 m + h
  constexpr int CW = kChunk * BITS / 32;    // words of one row in a chunk
  // sum(code * x) = sum_c 2^(24 - pos_c) d_c; with two classes 2^20 (16 d_0 + d_1).
  constexpr float kScale = PS::NCLS == 2 ? 1048576.f : 16777216.f;
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int chunks = d / kChunk;
  const long long items = (long long)((n + 16 * MT - 1) / (16 * MT)) * chunks;
  const long long c0 = items * blockIdx.x / gridDim.x, c1 = items * (blockIdx.x + 1) / gridDim.x;
  const long long i_begin = c0 + (c1 - c0) * warp / nw;
  const long long i_end = c0 + (c1 - c0) * (warp + 1) / nw;
  if (i_begin >= i_end) return;
  // Batch rows past the batch read the last batch row and land in accumulator columns that are
  // not written.
  const __half* xrow = X + (long long)min(g, batch - 1) * ldx + 32 * t;

  // Position of the current item, and of the item the next prefetch loads (pw: its rows'
  // packed words at chunk 0, this lane's run).
  int tile = (int)(i_begin / chunks), chunk = (int)(i_begin % chunks);
  int p_tile = tile, p_chunk = chunk;
  const uint32_t* pw[NR];
  auto set_prefetch_rows = [&]() {
#pragma unroll
    for (int r = 0; r < NR; ++r)
      pw[r] = qweight + (long long)lane_row<MT>(p_tile, r, g, n) * wpr + t * BITS;
  };
  set_prefetch_rows();
  uint32_t wr[2][NR][BITS];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (i_begin + h < i_end) {
#pragma unroll
      for (int r = 0; r < NR; ++r) load_stream<BITS>(pw[r] + (long long)p_chunk * CW, wr[h][r]);
    }
    if (++p_chunk == chunks) {
      p_chunk = 0;
      ++p_tile;
      set_prefetch_rows();
    }
  }

  // Group bookkeeping without a division per chunk (one per tile change); the next group's
  // parameters are fetched when a group starts.
  int gi = 0, g_next = 0;
  __half nxt_s[NR], nxt_z[NR];
  float sc[NR], nsz[NR];  // s * 2^(24 - pos): the scale of the class sums; -s * z
  long long poff[NR];     // row * G of the current tile's rows
  auto start_tile = [&]() {
    gi = min(chunk / chunks_per_group, G - 1);
    g_next = (gi + 1) * chunks_per_group;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      poff[r] = (long long)lane_row<MT>(tile, r, g, n) * G;
      // zero points are integers; another value is rounded to one, as the other paths do
      const float sv = __half2float(scales[poff[r] + gi]);
      const float zv = rintf(__half2float(zeros[poff[r] + gi]));
      sc[r] = sv * kScale;
      nsz[r] = -sv * zv;
      nxt_s[r] = scales[poff[r] + min(gi + 1, G - 1)];
      nxt_z[r] = zeros[poff[r] + min(gi + 1, G - 1)];
    }
  };
  start_tile();

  float acc[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
  // Accumulator layout: element e is (row g + 8 (e >> 1), batch column 2t + (e & 1)).
  auto flush = [&]() {
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int bcol = 2 * t + (e & 1);
        const int row = tile * 16 * MT + 16 * m + g + 8 * (e >> 1);
        if (bcol < batch && row < n) atomicAdd(Y + (long long)bcol * ldy + row, acc[m][e]);
        acc[m][e] = 0.f;
      }
  };
  const uint32_t ones = 0x3C003C00u;  // fp16 (1, 1)
  for (long long it = i_begin; it < i_end; it += 2) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (it + h < i_end) {
        if (chunk == g_next) {
          ++gi;
          g_next += chunks_per_group;
#pragma unroll
          for (int r = 0; r < NR; ++r) {
            const float sv = __half2float(nxt_s[r]), zv = rintf(__half2float(nxt_z[r]));
            sc[r] = sv * kScale;
            nsz[r] = -sv * zv;
            nxt_s[r] = scales[poff[r] + min(gi + 1, G - 1)];
            nxt_z[r] = zeros[poff[r] + min(gi + 1, G - 1)];
          }
        }
        uint32_t xr[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(xrow + (long long)chunk * kChunk) + i);
          xr[4 * i] = v.x; xr[4 * i + 1] = v.y; xr[4 * i + 2] = v.z; xr[4 * i + 3] = v.w;
        }
        uint32_t b[16];
        act_pairs<BITS>(xr, b);
        float dx[4] = {0.f, 0.f, 0.f, 0.f};  // the chunk's sum of x per batch column
#pragma unroll
        for (int q = 0; q < 8; ++q) mma_16816(dx, ones, ones, ones, ones, b[2 * q], b[2 * q + 1]);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          float dc[PS::NCLS][4];
#pragma unroll
          for (int c = 0; c < PS::NCLS; ++c) dc[c][0] = dc[c][1] = dc[c][2] = dc[c][3] = 0.f;
          tile_mmas<BITS>(wr[h][2 * m], wr[h][2 * m + 1], b, dc);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float cx = PS::NCLS == 2 ? fmaf(16.f, dc[0][e], dc[1][e]) : dc[0][e];
            const int r = 2 * m + (e >> 1);
            acc[m][e] = fmaf(sc[r], cx, acc[m][e]);
            acc[m][e] = fmaf(nsz[r], dx[e], acc[m][e]);
          }
        }
        // Refill this ring slot with the item two ahead.
        if (it + h + 2 < i_end) {
#pragma unroll
          for (int r = 0; r < NR; ++r)
            load_stream<BITS>(pw[r] + (long long)p_chunk * CW, wr[h][r]);
        }
        if (++p_chunk == chunks) {
          p_chunk = 0;
          ++p_tile;
          set_prefetch_rows();
        }
        // Next item.
        if (++chunk == chunks) {
          flush();
          chunk = 0;
          ++tile;
          if (it + h + 1 < i_end) start_tile();
        }
      }
    }
  }
  if (chunk != 0) flush();
}

}  // namespace

namespace gptq_host {

namespace {

// The tensor-core kernel runs persistent: kTcWarps warps per CTA and as many CTAs as are
// resident at once (at most one per 16 work items), each taking an even share of the items. Y is
// zeroed first: the warps add their partial sums into it.
template <class K>
int tc_launch(K kernel, long long items, const uint32_t* qweight, int n, int d, long long wpr,
              const __half* s, const __half* z, int G, int cpg, const __half* x, long long ldx,
              int batch, float* y, long long ldy, cudaStream_t stream) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kTcWarps * 32, 0) !=
      cudaSuccess)
    return GPTQ_ERR_CUDA;
  long long grid = (long long)num_sms() * (per_sm > 0 ? per_sm : 1);
  if (grid > (items + 15) / 16) grid = (items + 15) / 16;
  if (cudaMemset2DAsync(y, (size_t)ldy * 4, 0, (size_t)n * 4, (size_t)batch, stream) !=
      cudaSuccess)
    return GPTQ_ERR_CUDA;
  kernel<<<(int)grid, kTcWarps * 32, 0, stream>>>(qweight, n, d, wpr, s, z, G, cpg, x, ldx, batch,
                                                   y, ldy);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace

int dequant_gemv(const uint32_t* qweight, int n, int d, int bits, const uint16_t* scales_f16,
                 const uint16_t* zeros_f16, int n_groups, int group_size, const int32_t* g_idx,
                 const uint16_t* x_f16, int batch, long long ldx, float* y, long long ldy,
                 cudaStream_t stream) {
  const long long wpr = (long long)d * bits / 32;
  const dim3 grid((n + GEMV_THREADS / 32 - 1) / (GEMV_THREADS / 32));
  const __half* s = reinterpret_cast<const __half*>(scales_f16);
  const __half* z = reinterpret_cast<const __half*>(zeros_f16);
  const __half* x = reinterpret_cast<const __half*>(x_f16);
#define GEMV_LAUNCH(B, M)                                                                      \
  dequant_gemv_kernel<B, M><<<grid, GEMV_THREADS, 0, stream>>>(qweight, n, d, wpr, s, z, n_groups, \
                                                               group_size, g_idx, x, ldx, batch,   \
                                                               y, ldy)
  const bool run_groups = g_idx == nullptr && (n_groups == 1 || group_size % kChunk == 0);
  if (run_groups && d % kChunk == 0 && (bits == 2 || bits == 3 || bits == 4 || bits == 8)) {
    const int cpg = n_groups == 1 ? d / kChunk : group_size / kChunk;
    auto items = [&](int mt) { return (long long)((n + 16 * mt - 1) / (16 * mt)) * (d / kChunk); };
    switch (bits) {
      case 2:
        return tc_launch(dequant_gemv_tc_kernel<2, 2>, items(2), qweight, n, d, wpr, s, z,
                         n_groups, cpg, x, ldx, batch, y, ldy, stream);
      case 3:
        return tc_launch(dequant_gemv_tc_kernel<3, 2>, items(2), qweight, n, d, wpr, s, z,
                         n_groups, cpg, x, ldx, batch, y, ldy, stream);
      case 4:
        return tc_launch(dequant_gemv_tc_kernel<4, 2>, items(2), qweight, n, d, wpr, s, z,
                         n_groups, cpg, x, ldx, batch, y, ldy, stream);
      default:
        return tc_launch(dequant_gemv_tc_kernel<8, 1>, items(1), qweight, n, d, wpr, s, z,
                         n_groups, cpg, x, ldx, batch, y, ldy, stream);
    }
  }
  const bool one = batch == 1;
  switch (bits) {
    case 2: if (one) GEMV_LAUNCH(2, 1); else GEMV_LAUNCH(2, kMaxBatch); break;
    case 3: if (one) GEMV_LAUNCH(3, 1); else GEMV_LAUNCH(3, kMaxBatch); break;
    case 4: if (one) GEMV_LAUNCH(4, 1); else GEMV_LAUNCH(4, kMaxBatch); break;
    case 8: if (one) GEMV_LAUNCH(8, 1); else GEMV_LAUNCH(8, kMaxBatch); break;
    default: return GPTQ_ERR_INVALID_ARG;
  }
#undef GEMV_LAUNCH
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
