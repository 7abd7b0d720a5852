// Per-row top-k over the out-of-window candidates and the index-row emit
// (rows a4, a5).
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph -- the 128 most recent tokens are
// forced into the selection and 1024 high-scoring out-of-window tokens added;
// 10100.com article -- *at most* 1024 (fewer candidates: take them all).
//
// One CTA (512 threads) per query row.  Scores are >= 0, so their fp32 bit
// patterns order like the values: a radix select over the bits (13 + 10 + 9)
// finds the k-th largest pattern T and how many keys equal to T are taken
// (ties go to the smaller position).  Keys are then marked in a bitmap over
// positions and written in ascending order by a block-wide popcount scan, so
// no sort is needed.  Rows of up to 32768 candidates are cached in shared
// memory (one read of the row); otherwise the row is read twice from global.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int TK_THREADS = 512;
constexpr int TK_NW = TK_THREADS / 32;
constexpr int TK_BINS1 = 8192;        // digit 1: bits 31..19
constexpr int TK_CAP = 6144;          // collected candidates
constexpr int TK_CACHE = 32768;       // cached row values (u32)
constexpr int TK_BITMAP_WORDS = 32768;// bitmap over up to 2^20 positions
constexpr size_t TK_SMEM = (size_t)TK_BINS1 * 4 + (size_t)TK_CAP * 8 + (size_t)TK_CACHE * 4 + 256;

struct TopkParams {
  const float* sigma;    // row r at sigma + r * ld, candidates [0, n_r)
  int64_t ld;
  int64_t p0;            // absolute position of row 0's query
  int64_t pstep;         // 1 for prefill rows, 0 for decode rows
  int window;
  int topk;
  int32_t* idx;          // [rows, window + topk]
};

// Exclusive prefix sum over the CTA's 512 threads; `total` gets the sum.
__device__ __forceinline__ uint32_t tk_excl_scan(uint32_t v, uint32_t* scratch, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < TK_NW ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < TK_NW) scratch[TK_NW + lane] = w;
  }
  __syncthreads();
  total = scratch[2 * TK_NW - 1];
  const uint32_t r = (warp ? scratch[TK_NW + warp - 1] : 0) + x - v;
  __syncthreads();
  return r;
}

// In a histogram of nbins bins, the bin b holding the k-th largest element:
// above(b) < k <= above(b) + hist[b], above(b) = elements in bins > b.
__device__ __forceinline__ void tk_find_bin(const uint32_t* hist, int nbins, uint32_t k,
                                            uint32_t* scratch, uint32_t* res) {
  const int per = nbins / TK_THREADS;
  const int lo = threadIdx.x * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += hist[lo + i];
  uint32_t total;
  const uint32_t excl = tk_excl_scan(local, scratch, total);
  uint32_t above = total - excl - local;        // elements in bins above this range
  if (local > 0 && above < k && k <= above + local) {
    for (int b = lo + per - 1; b >= lo; --b) {
      if (above + hist[b] >= k) {
        res[0] = (uint32_t)b;
        res[1] = above;
        break;
      }
      above += hist[b];
    }
  }
  __syncthreads();
}

// Ordered positions of set bits: writes out[base + j] for the j-th set bit.
__device__ __forceinline__ uint32_t tk_emit_bitmap(const uint32_t* bm, int64_t n, int32_t* out,
                                                   uint32_t limit, uint32_t* scratch) {
  const int64_t words = (n + 31) >> 5;
  const int64_t wpt = (words + TK_THREADS - 1) / TK_THREADS;
  const int64_t w0 = threadIdx.x * wpt;
  const int64_t w1 = min(words, w0 + wpt);
  uint32_t local = 0;
  for (int64_t w = w0; w < w1; ++w) local += __popc(bm[w]);
  uint32_t total;
  uint32_t pos = tk_excl_scan(local, scratch, total);
  for (int64_t w = w0; w < w1; ++w) {
    uint32_t bits = bm[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < limit) out[pos] = (int32_t)(w * 32 + b);
      ++pos;
    }
  }
  return total;
}

// Position of the r-th (1-based) set bit of the bitmap.
__device__ __forceinline__ int64_t tk_nth_bit(const uint32_t* bm, int64_t n, uint32_t r,
                                              uint32_t* scratch, int64_t* res) {
  const int64_t words = (n + 31) >> 5;
  const int64_t wpt = (words + TK_THREADS - 1) / TK_THREADS;
  const int64_t w0 = threadIdx.x * wpt;
  const int64_t w1 = min(words, w0 + wpt);
  uint32_t local = 0;
  for (int64_t w = w0; w < w1; ++w) local += __popc(bm[w]);
  uint32_t total;
  uint32_t before = tk_excl_scan(local, scratch, total);
  if (local > 0 && before < r && r <= before + local) {
    for (int64_t w = w0; w < w1; ++w) {
      uint32_t bits = bm[w];
      const uint32_t c = __popc(bits);
      if (before + c >= r) {
        for (uint32_t j = before; ; ++j) {
          const int b = __ffs(bits) - 1;
          bits &= bits - 1;
          if (j + 1 == r) { *res = w * 32 + b; break; }
        }
        break;
      }
      before += c;
    }
  }
  __syncthreads();
  return *res;
}

__global__ void __launch_bounds__(TK_THREADS, 1)
topk_select_kernel(TopkParams p, DevCtx ctx) {
  extern __shared__ __align__(16) uint8_t smem_tk[];
  uint8_t* smem = smem_tk;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem);
  uint32_t* cval = hist + TK_BINS1;
  int32_t* cpos = reinterpret_cast<int32_t*>(cval + TK_CAP);
  uint32_t* cache = reinterpret_cast<uint32_t*>(cpos + TK_CAP);
  __shared__ uint32_t scratch[2 * TK_NW];
  __shared__ uint32_t res[2];
  __shared__ uint32_t ncand;
  __shared__ int64_t pstar;

  const int64_t row = blockIdx.x;
  const int64_t pos = p.p0 + row * p.pstep;
  const int W = p.window;
  const uint32_t k = (uint32_t)p.topk;
  int32_t* out = p.idx + row * (int64_t)(W + p.topk);
  const int64_t n = max((int64_t)0, pos - W + 1);

  for (int w = threadIdx.x; w < W; w += TK_THREADS) {
    const int64_t v = pos - W + 1 + w;
    out[w] = v >= 0 ? (int32_t)v : -1;
  }
  if (n <= (int64_t)k) {
    for (int i = threadIdx.x; i < p.topk; i += TK_THREADS) out[W + i] = i < n ? i : -1;
    return;
  }
  const uint32_t* src = reinterpret_cast<const uint32_t*>(p.sigma + row * p.ld);
  const bool cached = n <= TK_CACHE;

  for (int i = threadIdx.x; i < TK_BINS1; i += TK_THREADS) hist[i] = 0;
  __syncthreads();
  for (int64_t i = threadIdx.x; i < n; i += TK_THREADS) {
    uint32_t u = src[i];
    if (u > 0x7f800000u) {                // NaN or negative score: not a probability
      report(ctx, ST_DEVICE_CHECK);
      u = 0;
    }
    if (cached) cache[i] = u;
    atomicAdd(&hist[u >> 19], 1u);
  }
  __syncthreads();
  tk_find_bin(hist, TK_BINS1, k, scratch, res);
  const uint32_t b1 = res[0], above1 = res[1];
  const bool fast = above1 + hist[b1] <= (uint32_t)TK_CAP;
  __syncthreads();
  auto load = [&](int64_t i) -> uint32_t {
    uint32_t u = cached ? cache[i] : src[i];
    return u > 0x7f800000u ? 0u : u;
  };

  uint32_t T, need_eq, eq_count;
  {
    // digit 2: bits 18..9
    uint32_t k2 = k - above1;
    if (fast) {
      if (threadIdx.x == 0) ncand = 0;
      __syncthreads();
      for (int64_t i = threadIdx.x; i < n; i += TK_THREADS) {
        const uint32_t u = load(i);
        if ((u >> 19) >= b1) {
          const uint32_t s = atomicAdd(&ncand, 1u);
          cval[s] = u;
          cpos[s] = (int32_t)i;
        }
      }
    }
    for (int i = threadIdx.x; i < 1024; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
    if (fast) {
      for (uint32_t c = threadIdx.x; c < ncand; c += TK_THREADS)
        if ((cval[c] >> 19) == b1) atomicAdd(&hist[(cval[c] >> 9) & 1023u], 1u);
    } else {
      for (int64_t i = threadIdx.x; i < n; i += TK_THREADS) {
        const uint32_t u = load(i);
        if ((u >> 19) == b1) atomicAdd(&hist[(u >> 9) & 1023u], 1u);
      }
    }
    __syncthreads();
    tk_find_bin(hist, 1024, k2, scratch, res);
    const uint32_t b2 = res[0], above2 = res[1];
    const uint32_t pre2 = (b1 << 10) | b2;
    // digit 3: bits 8..0
    const uint32_t k3 = k2 - above2;
    for (int i = threadIdx.x; i < 1024; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
    if (fast) {
      for (uint32_t c = threadIdx.x; c < ncand; c += TK_THREADS)
        if ((cval[c] >> 9) == pre2) atomicAdd(&hist[cval[c] & 511u], 1u);
    } else {
      for (int64_t i = threadIdx.x; i < n; i += TK_THREADS) {
        const uint32_t u = load(i);
        if ((u >> 9) == pre2) atomicAdd(&hist[u & 511u], 1u);
      }
    }
    __syncthreads();
    // 512 bins: pad the search to 1024 with empty bins
    for (int i = 512 + threadIdx.x; i < 1024; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
    tk_find_bin(hist, 1024, k3, scratch, res);
    const uint32_t b3 = res[0], above3 = res[1];
    T = (pre2 << 9) | b3;
    need_eq = k3 - above3;
    eq_count = hist[b3];
  }

  // bitmap over positions: in the cache area unless the row itself lives there
  uint32_t* bm = (!fast && cached) ? cval : cache;
  const int64_t words = (n + 31) >> 5;
  for (int64_t w = threadIdx.x; w < words; w += TK_THREADS) bm[w] = 0;
  if (threadIdx.x == 0) pstar = INT64_MAX;
  __syncthreads();
  if (need_eq < eq_count) {
    // ties at T: keep the need_eq smallest positions
    if (fast) {
      for (uint32_t c = threadIdx.x; c < ncand; c += TK_THREADS)
        if (cval[c] == T) atomicOr(&bm[cpos[c] >> 5], 1u << (cpos[c] & 31));
    } else {
      for (int64_t i = threadIdx.x; i < n; i += TK_THREADS)
        if (load(i) == T) atomicOr(&bm[i >> 5], 1u << (i & 31));
    }
    __syncthreads();
    tk_nth_bit(bm, n, need_eq, scratch, &pstar);
    for (int64_t w = threadIdx.x; w < words; w += TK_THREADS) bm[w] = 0;
    __syncthreads();
  }
  const int64_t pcut = pstar;
  if (fast) {
    for (uint32_t c = threadIdx.x; c < ncand; c += TK_THREADS) {
      const uint32_t u = cval[c];
      if (u > T || (u == T && cpos[c] <= pcut)) atomicOr(&bm[cpos[c] >> 5], 1u << (cpos[c] & 31));
    }
  } else {
    for (int64_t i = threadIdx.x; i < n; i += TK_THREADS) {
      const uint32_t u = load(i);
      if (u > T || (u == T && i <= pcut)) atomicOr(&bm[i >> 5], 1u << (i & 31));
    }
  }
  __syncthreads();
  const uint32_t got = tk_emit_bitmap(bm, n, out + W, k, scratch);
  if (got != k && threadIdx.x == 0) report(ctx, ST_DEVICE_CHECK);
}

}  // namespace hs2
