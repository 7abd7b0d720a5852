// Per-row top-k over the out-of-window candidates and the index-row emit
// (rows a4, a5).
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph -- the 128 most recent tokens are
// forced into the selection and 1024 high-scoring out-of-window tokens added;
// 10100.com article -- *at most* 1024 (fewer candidates: take them all).
//
// One CTA (512 threads) per query row.  Scores are >= 0, so their fp32 bit
// patterns order like the values.  The k-th largest pattern T is found by a
// range select that adapts to the row: the first pass records min and max,
// then each histogram pass splits the current range [lo, hi] into at most
// 4096 equal bins and keeps the bin that holds the k-th element, so rows whose
// scores are nearly equal (near-uniform attention) still spread over the bins
// and 2-3 passes finish.  Keys are then marked in a bitmap over positions --
// ties at T go to the smaller positions -- and written in ascending order by a
// block-wide popcount scan, so no sort is needed.  Rows of up to 32768
// candidates live in shared memory after one read; longer rows are read again
// for one histogram and then only the candidates of the kept bin are
// collected into shared memory.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int TK_THREADS = 512;
constexpr int TK_NW = TK_THREADS / 32;
constexpr int TK_BINS = 4096;
constexpr int TK_CAP = 8192;          // collected candidates of a long row
constexpr int TK_CACHE = 32768;       // cached row values (u32); also the long-row bitmap (2^20 bits)
constexpr int TK_SMALL_BM = TK_CACHE / 32;
constexpr size_t TK_SMEM = (size_t)TK_BINS * 4 + (size_t)TK_CAP * 8 + (size_t)TK_CACHE * 4 +
                           (size_t)TK_SMALL_BM * 4 + 256;

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

// In a histogram of nbins (<= 4096) bins, the bin b holding the k-th largest
// element: above(b) < k <= above(b) + hist[b]; res = {b, above(b), hist[b]}.
__device__ __forceinline__ void tk_find_bin(const uint32_t* hist, int nbins, uint32_t k,
                                            uint32_t* scratch, uint32_t* res) {
  constexpr int PER = TK_BINS / TK_THREADS;
  const int lo = threadIdx.x * PER;
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) local += (lo + i < nbins) ? hist[lo + i] : 0u;
  uint32_t total;
  const uint32_t excl = tk_excl_scan(local, scratch, total);
  uint32_t above = total - excl - local;        // elements in bins above this range
  if (local > 0 && above < k && k <= above + local) {
    for (int b = lo + PER - 1; b >= lo; --b) {
      const uint32_t h = (b < nbins) ? hist[b] : 0u;
      if (above + h >= k) {
        res[0] = (uint32_t)b;
        res[1] = above;
        res[2] = h;
        break;
      }
      above += h;
    }
  }
  __syncthreads();
}

// Ordered positions of set bits: out[j] = position of the j-th set bit (j < limit).
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

// Position of the r-th (1-based) set bit of the bitmap (INT64_MAX if none).
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
        for (uint32_t j = before;; ++j) {
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

__device__ __forceinline__ uint32_t tk_clean(uint32_t u, const DevCtx& ctx) {
  if (u > 0x7f800000u) {                 // NaN or a negative score: not a probability sum
    report(ctx, ST_DEVICE_CHECK);
    return 0u;
  }
  return u;
}

// f(i, u) for every i < n: 16-byte streaming loads, 4 in flight per thread
// (the rows are read once, so they are marked evict-first).
template <typename F>
__device__ __forceinline__ void tk_stream(const uint32_t* src, int64_t n, F&& f) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  const int64_t n4 = n >> 2;
  for (int64_t j0 = threadIdx.x; j0 < n4; j0 += 4 * TK_THREADS) {
    uint4 v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t j = j0 + (int64_t)r * TK_THREADS;
      if (j < n4) v[r] = __ldcs(s4 + j);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t j = j0 + (int64_t)r * TK_THREADS;
      if (j < n4) {
        f(4 * j, v[r].x);
        f(4 * j + 1, v[r].y);
        f(4 * j + 2, v[r].z);
        f(4 * j + 3, v[r].w);
      }
    }
  }
  for (int64_t i = (n4 << 2) + threadIdx.x; i < n; i += TK_THREADS) f(i, __ldcs(src + i));
}

__global__ void __launch_bounds__(TK_THREADS, 1)
topk_select_kernel(TopkParams p, DevCtx ctx) {
  extern __shared__ __align__(16) uint8_t smem_tk[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_tk);
  uint32_t* cval = hist + TK_BINS;
  int32_t* cpos = reinterpret_cast<int32_t*>(cval + TK_CAP);
  uint32_t* cache = reinterpret_cast<uint32_t*>(cpos + TK_CAP);
  uint32_t* small_bm = cache + TK_CACHE;
  __shared__ uint32_t scratch[2 * TK_NW];
  __shared__ uint32_t res[3];
  __shared__ uint32_t red[2 * TK_NW];
  __shared__ uint32_t ncand;
  __shared__ int64_t pstar;

  const int64_t row = blockIdx.x;
  const int64_t pos = p.p0 + row * p.pstep;
  const int W = p.window;
  const uint32_t k = (uint32_t)p.topk;
  int32_t* out = p.idx + row * (int64_t)(W + p.topk);
  const int64_t n = max((int64_t)0, pos - W + 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

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

  // ---- pass A: min and max (and the row into shared memory if it fits)
  uint32_t lmin = 0xFFFFFFFFu, lmax = 0u;
  tk_stream(src, n, [&](int64_t i, uint32_t raw) {
    const uint32_t u = tk_clean(raw, ctx);
    if (cached) cache[i] = u;
    lmin = min(lmin, u);
    lmax = max(lmax, u);
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lmin = min(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
    lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  }
  if (lane == 0) {
    red[warp] = lmin;
    red[TK_NW + warp] = lmax;
  }
  __syncthreads();
  uint32_t lo = red[0], hi = red[TK_NW];
  for (int w = 1; w < TK_NW; ++w) {
    lo = min(lo, red[w]);
    hi = max(hi, red[TK_NW + w]);
  }

  // ---- range select
  bool listed = false;           // long row whose candidates sit in cval/cpos
  uint32_t krem = k, in_range = (uint32_t)n;
  for (int pass = 0; hi > lo; ++pass) {
    const uint32_t span = hi - lo;
    const int sh = max(0, 32 - __clz((int)span) - 12);   // (span >> sh) < 4096
    const int nb = (int)(span >> sh) + 1;
    for (int b = threadIdx.x; b < nb; b += TK_THREADS) hist[b] = 0;
    __syncthreads();
    if (listed) {
      for (uint32_t c = threadIdx.x; c < ncand; c += TK_THREADS) {
        const uint32_t u = cval[c];
        if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
      }
    } else if (cached) {
      for (int64_t i = threadIdx.x; i < n; i += TK_THREADS) {
        const uint32_t u = cache[i];
        if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
      }
    } else {
      tk_stream(src, n, [&](int64_t, uint32_t raw) {
        const uint32_t u = tk_clean(raw, ctx);
        if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> sh], 1u);
      });
    }
    __syncthreads();
    tk_find_bin(hist, nb, krem, scratch, res);
    const uint32_t b = res[0], above = res[1];
    in_range = res[2];
    const uint32_t nlo = lo + (b << sh);
    const uint32_t nhi = (sh >= 32 || nlo + ((1u << sh) - 1u) > hi || nlo + ((1u << sh) - 1u) < nlo)
                             ? hi : nlo + ((1u << sh) - 1u);
    krem -= above;
    lo = nlo;
    hi = nhi;
    if (!listed && k - krem + in_range <= (uint32_t)TK_CAP) {
      // keep only the elements >= lo (all that can still be chosen): the next
      // passes and the marking then touch about k elements, not the row
      if (threadIdx.x == 0) ncand = 0;
      __syncthreads();
      const uint32_t clo = lo;
      auto take = [&](int64_t i, uint32_t u) {
        if (u >= clo) {               // at most TK_CAP of them (counted above)
          const uint32_t slot = atomicAdd(&ncand, 1u);
          cval[slot] = u;
          cpos[slot] = (int32_t)i;
        }
      };
      if (cached) {
        for (int64_t i = threadIdx.x; i < n; i += TK_THREADS) take(i, cache[i]);
      } else {
        tk_stream(src, n, [&](int64_t i, uint32_t raw) { take(i, tk_clean(raw, ctx)); });
      }
      __syncthreads();
      listed = true;
    }
  }
  const uint32_t T = lo;          // the k-th largest score pattern
  const uint32_t need_eq = krem;  // how many keys equal to T are taken
  const uint32_t eq_count = in_range;

  // ---- mark and emit in position order (a listed row no longer needs the cache)
  uint32_t* bm = (cached && !listed) ? small_bm : cache;
  const int64_t words = (n + 31) >> 5;
  if (threadIdx.x == 0) pstar = INT64_MAX;
  if (listed) {
    for (int64_t w = threadIdx.x; w < words; w += TK_THREADS) bm[w] = 0;
    __syncthreads();
    if (need_eq < eq_count) {
      for (uint32_t c = threadIdx.x; c < ncand; c += TK_THREADS)
        if (cval[c] == T) atomicOr(&bm[cpos[c] >> 5], 1u << (cpos[c] & 31));
      __syncthreads();
      tk_nth_bit(bm, n, need_eq, scratch, &pstar);
      for (int64_t w = threadIdx.x; w < words; w += TK_THREADS) bm[w] = 0;
      __syncthreads();
    }
    const int64_t pcut = pstar;
    for (uint32_t c = threadIdx.x; c < ncand; c += TK_THREADS) {
      const uint32_t u = cval[c];
      if (u > T || (u == T && cpos[c] <= pcut)) atomicOr(&bm[cpos[c] >> 5], 1u << (cpos[c] & 31));
    }
  } else if (!cached) {
    // long row that never fit the candidate list: mark straight from global
    for (int64_t w = threadIdx.x; w < words; w += TK_THREADS) bm[w] = 0;
    __syncthreads();
    if (need_eq < eq_count) {
      tk_stream(src, n, [&](int64_t i, uint32_t raw) {
        if (tk_clean(raw, ctx) == T) atomicOr(&bm[i >> 5], 1u << (i & 31));
      });
      __syncthreads();
      tk_nth_bit(bm, n, need_eq, scratch, &pstar);
      for (int64_t w = threadIdx.x; w < words; w += TK_THREADS) bm[w] = 0;
      __syncthreads();
    }
    const int64_t pcut = pstar;
    tk_stream(src, n, [&](int64_t i, uint32_t raw) {
      const uint32_t u = tk_clean(raw, ctx);
      if (u > T || (u == T && i <= pcut)) atomicOr(&bm[i >> 5], 1u << (i & 31));
    });
  } else {
    // cached row: a warp covers 32 consecutive positions = one bitmap word
    __syncthreads();
    if (need_eq < eq_count) {
      for (int64_t i0 = 0; i0 < n; i0 += TK_THREADS) {
        const int64_t i = i0 + threadIdx.x;
        const unsigned w = __ballot_sync(0xffffffffu, i < n && cache[i] == T);
        if (lane == 0 && i < n) bm[i >> 5] = w;
      }
      __syncthreads();
      tk_nth_bit(bm, n, need_eq, scratch, &pstar);
    }
    const int64_t pcut = pstar;
    for (int64_t i0 = 0; i0 < n; i0 += TK_THREADS) {
      const int64_t i = i0 + threadIdx.x;
      const uint32_t u = i < n ? cache[i] : 0u;
      const unsigned w = __ballot_sync(0xffffffffu, i < n && (u > T || (u == T && i <= pcut)));
      if (lane == 0 && i < n) bm[i >> 5] = w;
    }
  }
  __syncthreads();
  const uint32_t got = tk_emit_bitmap(bm, n, out + W, k, scratch);
  if (got != k && threadIdx.x == 0) report(ctx, ST_DEVICE_CHECK);
}

}  // namespace hs2
