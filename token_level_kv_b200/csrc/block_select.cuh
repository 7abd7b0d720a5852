// Block-level selection: the alternative the pages measure token-level
// selection against.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), ablation paragraph -- token-level selection against
// block-level selection with 64-token blocks at the same 1024-token budget;
// 10100.com article, "evolution one" -- block selection keeps whole units of
// 64 or 128 tokens.  Readings (the same as the oracle's): aligned blocks
// c = positions [c*B, (c+1)*B); a block's score is the sum of the selection
// scores sigma of its out-of-window candidates; the k blocks with the largest
// score are taken (ties to the smaller block number; all of them if there
// are at most k); the index row is the forced window, then the candidate
// positions of the chosen blocks ascending, then -1.
//
// One CTA of 256 threads per query row, after the same selection-score pass
// as the token-level path.  The scores of a row are summed per block in a
// fixed order (each of G = min(B, 32) lanes adds B/G scores, then a shuffle
// tree), so a block score carries at most B/G - 1 + log2(G) roundings; the
// block scores (at most 16384 per row; shared memory is sized to the call's
// longest row) stay in shared memory, where an exact
// 4-pass radix select over their fp32 bit patterns (scores are >= 0, so the
// patterns order like the values) finds the k-th largest; two block-wide
// scans then mark the ties taken and place each chosen block's positions.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int BS_THREADS = 256;
constexpr int BS_MAX_BLOCKS = 16384;
// shared memory for rows of at most nb_max blocks: the block scores, then 256 bins
__host__ __device__ constexpr size_t bs_smem(int nb_max) { return ((size_t)nb_max + 256) * 4; }

struct BlockSelParams {
  const float* sigma;    // row r at sigma + r * ld, candidates [0, n_r)
  int64_t ld;
  int64_t p0;            // absolute position of row 0's query
  int64_t pstep;         // 1 for prefill rows, 0 for decode rows
  int window;
  int block;             // B: a power of two in [16, 256]
  int topk_blocks;       // k
  int nb_max;            // the most blocks any row has (sizes shared memory)
  int32_t* idx;          // [rows, window + k * B]
};

// Exclusive prefix sum over the CTA (BS_THREADS threads); `total` gets the sum.
__device__ __forceinline__ uint32_t bs_excl_scan(uint32_t v, uint32_t* scratch, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < BS_THREADS / 32; ++w) {
    const uint32_t s = scratch[w];
    before += w < warp ? s : 0u;
    tot += s;
  }
  total = tot;
  __syncthreads();
  return before + x - v;
}

__global__ void __launch_bounds__(BS_THREADS)
block_select_kernel(BlockSelParams p, DevCtx ctx) {
  extern __shared__ __align__(16) uint8_t smem_bs[];
  uint32_t* bsc = reinterpret_cast<uint32_t*>(smem_bs);               // block scores (fp32 patterns)
  uint32_t* hist = bsc + p.nb_max;                                    // 256 bins
  __shared__ uint32_t scratch[BS_THREADS / 32];
  __shared__ uint32_t pick[2];                                         // chosen bin, count above it

  const int64_t row = blockIdx.x;
  const int64_t pos = p.p0 + row * p.pstep;
  const int W = p.window, B = p.block, k = p.topk_blocks;
  const int width = W + k * B;
  int32_t* out = p.idx + row * (int64_t)width;
  const int64_t n = max((int64_t)0, pos - W + 1);                      // candidates 0 .. pos - W
  const int nb = (int)((n + B - 1) / B);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  for (int w = threadIdx.x; w < W; w += BS_THREADS) {
    const int64_t v = pos - W + 1 + w;
    out[w] = v >= 0 ? (int32_t)v : -1;
  }
  const float* src = p.sigma + row * p.ld;

  // ---- block scores: G lanes per block, B/G scores per lane, then a tree
  const int G = B < 32 ? B : 32;
  const int per_lane = B / G;
  const int bpw = 32 / G;                                              // blocks per warp step
  const int sub = lane / G, gl = lane % G;
  // four block steps of a warp at a time, their loads issued together
  constexpr int U = 4;
  bool bad = false;
  for (int c0 = warp * bpw; c0 < nb; c0 += (BS_THREADS / 32) * bpw * U) {
    float acc[U];
#pragma unroll
    for (int s = 0; s < U; ++s) {
      const int c = c0 + s * (BS_THREADS / 32) * bpw + sub;
      acc[s] = 0.f;
      for (int i = 0; i < per_lane; ++i) {
        const int64_t j = (int64_t)c * B + (int64_t)i * G + gl;
        if (c < nb && j < n) {
          uint32_t u = __float_as_uint(src[j]);
          bad |= u > 0x7f800000u;                                      // NaN or negative: not a probability sum
          acc[s] += __uint_as_float(u > 0x7f800000u ? 0u : u);
        }
      }
    }
#pragma unroll
    for (int s = 0; s < U; ++s) {
      const int c = c0 + s * (BS_THREADS / 32) * bpw + sub;
      float a = acc[s];
      for (int o = G / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (gl == 0 && c < nb) bsc[c] = __float_as_uint(a);
    }
  }
  if (bad) report(ctx, ST_DEVICE_CHECK);
  __syncthreads();

  // ---- the k-th largest pattern T and how many blocks equal to T are taken
  uint32_t T = 0u, need_eq = 0xffffffffu;                              // nb <= k: every block
  if (nb > k) {
    uint32_t prefix = 0u, mask = 0u, krem = (uint32_t)k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      hist[threadIdx.x] = 0u;
      __syncthreads();
      for (int c = threadIdx.x; c < nb; c += BS_THREADS) {
        const uint32_t u = bsc[c];
        if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns bins 8l .. 8l+7; find the bin holding the krem-th largest
        uint32_t h[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h[i] = hist[8 * lane + i];
          tot += h[i];
        }
        uint32_t incl = tot;                                           // sum over lanes >= this one
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += y;
        }
        uint32_t above = incl - tot;                                   // in bins of higher lanes
        if (above < krem && krem <= incl) {
          for (int i = 7; i >= 0; --i) {
            if (krem <= above + h[i]) {
              pick[0] = (uint32_t)(8 * lane + i);
              pick[1] = above;
              break;
            }
            above += h[i];
          }
        }
      }
      __syncthreads();
      prefix |= pick[0] << shift;
      mask |= 255u << shift;
      krem -= pick[1];
      __syncthreads();
    }
    T = prefix;
    need_eq = krem;
  }

  // ---- mark (ties taken in block order) and place: thread t owns blocks
  // [t*per, (t+1)*per), per odd so a warp's 32 lanes hit 32 banks
  const int per = ((nb + BS_THREADS - 1) / BS_THREADS) | 1;
  const int c0 = threadIdx.x * per, c1 = min(nb, c0 + per);
  uint32_t n_eq = 0;
  for (int c = c0; c < c1; ++c) n_eq += bsc[c] == T ? 1u : 0u;
  uint32_t tot;
  uint32_t eq_before = bs_excl_scan(n_eq, scratch, tot);
  // the chosen blocks, in block order, into sel[]: every chosen block but a
  // partial last one holds B positions, and a partial block is the last
  // block of the row, so chosen block r starts at slot r * B
  uint32_t n_take = 0;
  for (int c = c0; c < c1; ++c) {
    const uint32_t u = bsc[c];
    bool take = u > T;
    if (u == T) take = eq_before++ < need_eq;
    n_take += take ? 1u : 0u;
    bsc[c] = take ? 1u : 0u;                                          // own blocks only: no race
  }
  uint32_t n_sel;
  uint32_t rank = bs_excl_scan(n_take, scratch, n_sel);
  uint32_t* sel = hist;                                               // the bins are free again
  for (int c = c0; c < c1; ++c)
    if (bsc[c] && rank < (uint32_t)k) sel[rank++] = (uint32_t)c;
  __syncthreads();
  // one warp per chosen block: its positions, lanes on consecutive slots
  const uint32_t n_blk = min(n_sel, (uint32_t)k);
  for (uint32_t r = warp; r < n_blk; r += BS_THREADS / 32) {
    const int64_t j0 = (int64_t)sel[r] * B;
    const int len = (int)min((int64_t)B, n - j0);
    for (int i = lane; i < B; i += 32) out[W + (int64_t)r * B + i] = i < len ? (int32_t)(j0 + i) : -1;
  }
  for (int i = n_blk * B + threadIdx.x; i < k * B; i += BS_THREADS) out[W + i] = -1;
  if (threadIdx.x == 0 && n_sel > (uint32_t)k) report(ctx, ST_DEVICE_CHECK);
}

}  // namespace hs2
