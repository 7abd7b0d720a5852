// Per-row top-k over the out-of-window candidates and the index-row emit
// (rows a4, a5).
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph -- the 128 most recent tokens are
// forced into the selection and 1024 high-scoring out-of-window tokens added;
// 10100.com article -- *at most* 1024 (fewer candidates: take them all).
//
// One CTA of 256 threads per query row, four CTAs per SM, so one row's
// barriers and waits overlap the other rows' streaming.  Scores are >= 0, so
// their fp32 bit patterns order like the values.
//   1. A sample of the row (every sb-th block of 128 candidates, at most 2048)
//      is read into shared memory and its pattern V at rank
//      k*m/n + 4*sqrt(k*m/n) + 8 found: below the row's k-th largest unless the
//      row is extreme.
//   2. One pass over the row lists every candidate >= V (one test per 16-byte
//      group); when that yields between k and 4096 of them, the exact k-th
//      largest pattern T is found on the list, else (the fallback) on the row.
//   3. Range select: each pass splits the current pattern range [lo, hi] into
//      at most 2048 equal bins, histograms the candidates and keeps the bin
//      that holds the k-th element, so rows whose scores are nearly equal still
//      spread over the bins.  Over the row (fallback), the survivors are listed
//      as soon as they fit.
//   4. The selection is every key above T plus the first keys equal to T in
//      position order (ties go to the smaller position), marked in a bitmap
//      over a window of 32768 positions at a time and written in ascending
//      order by a block-wide popcount scan: no sort, and any row length uses
//      the same 4 KB bitmap.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int TK_THREADS = 256;
constexpr int TK_NW = TK_THREADS / 32;
constexpr int TK_BINS = 2048;
constexpr int TK_CAP = 4096;          // listed candidates
constexpr int TK_SAMPLE = 2048;       // sampled candidates
constexpr int TK_WIN = 32768;         // positions per bitmap window
constexpr int TK_BMW = TK_WIN / 32;   // bitmap words
constexpr size_t TK_SMEM = (size_t)TK_BINS * 4 + (size_t)TK_CAP * 8 + (size_t)TK_BMW * 4;

struct TopkParams {
  const float* sigma;    // row r at sigma + r * ld, candidates [0, n_r)
  int64_t ld;
  int64_t p0;            // absolute position of row 0's query
  int64_t pstep;         // 1 for prefill rows, 0 for decode rows
  int window;
  int topk;
  int32_t* idx;          // [rows, window + topk]
};

__device__ __forceinline__ uint32_t tk_clean(uint32_t u, const DevCtx& ctx) {
  if (u > 0x7f800000u) {                 // NaN or a negative score: not a probability sum
    report(ctx, ST_DEVICE_CHECK);
    return 0u;
  }
  return u;
}

// Exclusive prefix sum over the CTA; `total` gets the sum.  Two barriers.
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
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < TK_NW; ++w) {
    const uint32_t s = scratch[w];
    before += w < warp ? s : 0u;
    tot += s;
  }
  total = tot;
  __syncthreads();
  return before + x - v;
}

// In a histogram of nb (<= TK_BINS) bins, the bin b holding the k-th largest
// element: above(b) < k <= above(b) + hist[b]; res = {b, above(b), hist[b]}.
// Warp w owns bins [256w, 256w + 256) as 8 rows of 32, read lane-interleaved;
// the 8 row sums are reduced side by side, so only the row holding the bin is
// scanned.
__device__ __forceinline__ void tk_find_bin(const uint32_t* hist, int nb, uint32_t k, uint32_t* scratch,
                                            uint32_t* res) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int PER = TK_BINS / TK_NW / 32;          // 8 rows of 32 bins per warp
  const int base = warp * (TK_BINS / TK_NW);
  uint32_t v[PER], rs[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int bin = base + 32 * j + lane;
    v[j] = bin < nb ? hist[bin] : 0u;
    rs[j] = v[j];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int j = 0; j < PER; ++j) rs[j] += __shfl_xor_sync(0xffffffffu, rs[j], o);
  uint32_t mine = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) mine += rs[j];
  if (lane == 0) scratch[warp] = mine;
  __syncthreads();
  uint32_t above = 0;
#pragma unroll
  for (int w = 0; w < TK_NW; ++w) above += w > warp ? scratch[w] : 0u;
  if (above < k && k <= above + mine) {
    // the row from the top whose sum reaches k, and its bins
    uint32_t vj = 0;
    int jsel = 0;
    bool found = false;
#pragma unroll
    for (int j = PER - 1; j >= 0; --j) {
      if (!found) {
        if (above + rs[j] >= k) {
          found = true;
          jsel = j;
          vj = v[j];
        } else {
          above += rs[j];
        }
      }
    }
    uint32_t x = vj;                                   // inclusive suffix over lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
      if (lane + o < 32) x += y;
    }
    if (above + x - vj < k && k <= above + x) {
      res[0] = (uint32_t)(base + 32 * jsel + lane);
      res[1] = above + x - vj;
      res[2] = vj;
    }
  }
  __syncthreads();
}

// f(i, u) for every i in [i0, i1) (i0 a multiple of 4): 16-byte loads, 4 in
// flight per thread.
template <typename F>
__device__ __forceinline__ void tk_stream(const uint32_t* src, int64_t i0, int64_t i1, F&& f) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  const int64_t j0 = i0 >> 2, j1 = i1 >> 2;
  for (int64_t jb = j0 + threadIdx.x; jb < j1; jb += 4 * TK_THREADS) {
    uint4 v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t j = jb + (int64_t)r * TK_THREADS;
      if (j < j1) v[r] = s4[j];
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t j = jb + (int64_t)r * TK_THREADS;
      if (j < j1) {
        f(4 * j, v[r].x);
        f(4 * j + 1, v[r].y);
        f(4 * j + 2, v[r].z);
        f(4 * j + 3, v[r].w);
      }
    }
  }
  for (int64_t i = (j1 << 2) + threadIdx.x; i < i1; i += TK_THREADS) f(i, src[i]);
}

// f(i, u, valid) for every i < n with all lanes converged (lanes past the
// end pass valid = false): 16-byte loads, 8 in flight per thread.
template <typename F>
__device__ __forceinline__ void tk_stream_conv(const uint32_t* src, int64_t n, F&& f, const DevCtx& ctx) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  const int64_t n4 = n >> 2;
  constexpr int R = 8;
  for (int64_t jb = 0; jb < n4; jb += R * TK_THREADS) {
    uint4 v[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t j = jb + threadIdx.x + (int64_t)r * TK_THREADS;
      v[r] = j < n4 ? s4[j] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t j = jb + threadIdx.x + (int64_t)r * TK_THREADS;
      const bool ok = j < n4;
      const uint32_t e[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) f(4 * j + q, ok ? tk_clean(e[q], ctx) : 0u, ok);
    }
  }
  for (int64_t i0 = n4 << 2; i0 < n; i0 += TK_THREADS) {
    const int64_t i = i0 + threadIdx.x;
    const bool ok = i < n;
    f(i, ok ? tk_clean(src[i], ctx) : 0u, ok);
  }
}

// Shared-memory histogram add.  With AGG (the first pass of a select, where
// nearly equal scores crowd one bin) a warp whose active lanes all hit one
// bin adds once; later passes spread over the bins and add directly.
template <bool AGG>
__device__ __forceinline__ void tk_hist_add(uint32_t* hist, bool in, uint32_t bin) {
  if (!AGG) {
    if (in) atomicAdd(&hist[bin], 1u);
    return;
  }
  const unsigned act = __ballot_sync(0xffffffffu, in);
  if (act == 0) return;
  const int leader = __ffs(act) - 1;
  const uint32_t b0 = __shfl_sync(0xffffffffu, bin, leader);
  if (__all_sync(0xffffffffu, !in || bin == b0)) {
    if ((threadIdx.x & 31) == leader) atomicAdd(&hist[b0], (uint32_t)__popc(act));
  } else if (in) {
    atomicAdd(&hist[bin], 1u);
  }
}

__global__ void __launch_bounds__(TK_THREADS, 4)
topk_select_kernel(TopkParams p, DevCtx ctx) {
  extern __shared__ __align__(16) uint8_t smem_tk[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_tk);
  uint32_t* cval = hist + TK_BINS;
  int32_t* cpos = reinterpret_cast<int32_t*>(cval + TK_CAP);
  uint32_t* bm = reinterpret_cast<uint32_t*>(cpos + TK_CAP);
  __shared__ uint32_t scratch[TK_NW];
  __shared__ uint32_t res[3];
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

  // every candidate >= v -> the list (stops writing past TK_CAP; ncand
  // still counts them all)
  // (one test per 16-byte group: its largest pattern against v)
  auto collect = [&](uint32_t v) {
    if (threadIdx.x == 0) ncand = 0;
    __syncthreads();
    auto take4 = [&](int64_t i0, uint32_t e0, uint32_t e1, uint32_t e2, uint32_t e3, bool ok) {
      uint32_t mx = max(max(e0, e1), max(e2, e3));
      if (ok && mx > 0x7f800000u) {                  // NaN or negative: cleaned (and reported)
        e0 = tk_clean(e0, ctx); e1 = tk_clean(e1, ctx); e2 = tk_clean(e2, ctx); e3 = tk_clean(e3, ctx);
        mx = max(max(e0, e1), max(e2, e3));
      }
      if (ok && mx >= v) {                           // rare: a group with a candidate
        const uint32_t e[4] = {e0, e1, e2, e3};
        uint32_t c = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) c += e[q] >= v ? 1u : 0u;
        uint32_t slot = atomicAdd(&ncand, c);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (e[q] >= v) {
            if (slot < (uint32_t)TK_CAP) {
              cval[slot] = e[q];
              cpos[slot] = (int32_t)(i0 + q);
            }
            ++slot;
          }
      }
    };
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    const int64_t n4 = n >> 2;
    constexpr int R = 8;
    for (int64_t jb = threadIdx.x; jb < n4; jb += R * TK_THREADS) {
      uint4 w[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t j = jb + (int64_t)r * TK_THREADS;
        w[r] = j < n4 ? s4[j] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t j = jb + (int64_t)r * TK_THREADS;
        take4(4 * j, w[r].x, w[r].y, w[r].z, w[r].w, j < n4);
      }
    }
    for (int64_t i = (n4 << 2) + threadIdx.x; i < n; i += TK_THREADS) {
      const uint32_t u = tk_clean(src[i], ctx);
      if (u >= v) {
        const uint32_t slot = atomicAdd(&ncand, 1u);
        if (slot < (uint32_t)TK_CAP) {
          cval[slot] = u;
          cpos[slot] = (int32_t)i;
        }
      }
    }
    __syncthreads();
  };

  // ---- range select: the pattern of the r-th largest candidate.  On
  // return lo == hi is that pattern, krem how many of the r are equal to it
  // and in_range how many candidates equal it.  Over the list when `listed`,
  // else over the row, which is collected into the list as soon as every
  // element that can still be chosen fits it.
  bool listed = false;                      // candidates >= lo sit in cval/cpos
  uint32_t lo, hi, krem, in_range;
  // With win_hi < 0x7f800000 the first pass bins only [win_lo, win_hi] (every
  // candidate is >= win_lo) plus one overflow bin for the candidates above.
  // With coarse > 0 the select stops as soon as the bin holding the r-th
  // element holds at most `coarse` elements: lo is then a pattern with between
  // r and r + coarse - 1 listed elements at or above it (a bound, not the
  // exact r-th pattern).
  auto range_select = [&](uint32_t r, uint32_t count, uint32_t win_lo, uint32_t win_hi, uint32_t coarse) {
    lo = win_lo;
    hi = win_hi;
    krem = r;
    in_range = count;
    bool over = win_hi < 0x7f800000u;                  // first pass only
    for (int pass = 0; hi > lo || over; ++pass) {
      const uint32_t span = hi - lo;
      int sh = max(0, 32 - __clz((int)span) - 11);     // (span >> sh) < 2048
      if (over && (span >> sh) + 2 > (uint32_t)TK_BINS) ++sh;
      const int nb = (int)(span >> sh) + 1 + (over ? 1 : 0);
      for (int b = threadIdx.x; b < nb; b += TK_THREADS) hist[b] = 0;
      __syncthreads();
      if (listed) {
        const uint32_t m = ncand;
        for (uint32_t c0 = 0; c0 < m; c0 += TK_THREADS) {
          const uint32_t c = c0 + threadIdx.x;
          const uint32_t u = c < m ? cval[c] : 0u;
          const bool in = c < m && u >= lo && (u <= hi || over);
          const uint32_t bin = u > hi ? (uint32_t)(nb - 1) : (u - lo) >> sh;
          if (pass == 0) tk_hist_add<true>(hist, in, bin);
          else tk_hist_add<false>(hist, in, bin);
        }
      } else {
        tk_stream_conv(src, n, [&](int64_t, uint32_t u, bool valid) {
          const bool in = valid && u >= lo && u <= hi;
          tk_hist_add<true>(hist, in, (u - lo) >> sh);
        }, ctx);
      }
      __syncthreads();
      tk_find_bin(hist, nb, krem, scratch, res);
      const uint32_t b = res[0], above = res[1];
      in_range = res[2];
      krem -= above;
      if (over && b == (uint32_t)(nb - 1)) {           // the k-th largest lies above the window
        lo = hi + 1;
        hi = 0x7f800000u;
      } else {
        const uint32_t nlo = lo + (b << sh);
        const uint32_t top = nlo + ((1u << sh) - 1u);
        lo = nlo;
        hi = (top > hi || top < nlo) ? hi : top;
      }
      over = false;
      if (coarse && in_range <= coarse) break;
      if (!listed && r - krem + in_range <= (uint32_t)TK_CAP) {
        collect(lo);                         // exactly r - krem + in_range of them
        listed = true;
      }
    }
  };

  // ---- a bound from a sample: blocks of 128 candidates, every sb-th block,
  // at most TK_SAMPLE of them.  Its pattern V at rank k*m/n + delta (delta a
  // few standard deviations of that rank) lies below the row's k-th largest
  // for any row without extreme structure; one pass then lists every
  // candidate >= V.  Rows where that fails (fewer than k listed, or more
  // than the list holds) fall back to the range select over the row.
  {
    const int64_t nblk = (n + 127) / 128;
    const int64_t sb = (nblk + (TK_SAMPLE / 128) - 1) / (TK_SAMPLE / 128);
    const int64_t nsb = (nblk + sb - 1) / sb;           // sampled blocks
    const uint32_t m = (uint32_t)(nsb * 128 < (int64_t)TK_SAMPLE ? nsb * 128 : (int64_t)TK_SAMPLE);
    {
      constexpr int R = TK_SAMPLE / (4 * TK_THREADS);   // 16-byte loads per thread, all in flight
      uint4 v[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t q = 4 * (threadIdx.x + r * TK_THREADS);
        const int64_t i = (int64_t)(q / 128) * sb * 128 + (q % 128);
        v[r] = make_uint4(0u, 0u, 0u, 0u);               // padding of a short last block ranks last
        if (q < m) {
          if (i + 3 < n) {
            v[r] = reinterpret_cast<const uint4*>(src)[i >> 2];
          } else {
            if (i < n) v[r].x = src[i];
            if (i + 1 < n) v[r].y = src[i + 1];
            if (i + 2 < n) v[r].z = src[i + 2];
          }
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t q = 4 * (threadIdx.x + r * TK_THREADS);
        if (q < m) {
          const int64_t i = (int64_t)(q / 128) * sb * 128 + (q % 128);
          *reinterpret_cast<uint4*>(cval + q) = make_uint4(tk_clean(v[r].x, ctx), tk_clean(v[r].y, ctx),
                                                           tk_clean(v[r].z, ctx), tk_clean(v[r].w, ctx));
          *reinterpret_cast<int4*>(cpos + q) = make_int4((int)i, (int)i + 1, (int)i + 2, (int)i + 3);
        }
      }
    }
    if (threadIdx.x == 0) ncand = sb == 1 ? (uint32_t)n : m;
    __syncthreads();
    listed = true;
    // the selects start from the sample's own pattern range [mn, mx], so
    // near-equal scores spread over the bins from the first pass
    uint32_t mn = 0xffffffffu, mx = 0u;
    {
      const uint32_t cnt = sb == 1 ? (uint32_t)n : m;
      for (uint32_t c = threadIdx.x; c < cnt; c += TK_THREADS) {
        const uint32_t u = cval[c];
        mn = min(mn, u);
        mx = max(mx, u);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      const int warp = threadIdx.x >> 5;
      if ((threadIdx.x & 31) == 0) {
        hist[warp] = mn;                               // the bins are free until the select
        hist[TK_NW + warp] = mx;
      }
      __syncthreads();
#pragma unroll
      for (int w = 0; w < TK_NW; ++w) {
        mn = min(mn, hist[w]);
        mx = max(mx, hist[TK_NW + w]);
      }
      __syncthreads();
    }
    if (sb == 1) {
      range_select(k, (uint32_t)n, mn, mx, 0u);       // the whole row is the sample
    } else {
      const float ks = (float)k * (float)m / (float)n;
      const uint32_t rv = min(m, (uint32_t)(ks + 4.f * sqrtf(ks) + 8.f));
      // the row into L2 while the sample is searched (the next pass reads it all)
      for (int64_t i = (int64_t)threadIdx.x * 32; i < n; i += 32 * TK_THREADS)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(src + i));
      // the bound needs only the bin of the rv-th sample pattern, not the
      // pattern itself: one pass unless that bin is crowded
      range_select(rv, m, mn, mx, 16u);
      const uint32_t V = lo;
      collect(V);
      if (ncand >= k && ncand <= (uint32_t)TK_CAP) {
        // T is within a few sample ranks of V: first look 2^16 patterns above it
        if (V < 0x7f7f0000u) range_select(k, ncand, V, V + 0xffffu, 0u);
        else range_select(k, ncand, 0u, 0x7f800000u, 0u);
      } else {
        listed = false;
        range_select(k, (uint32_t)n, 0u, 0x7f800000u, 0u);
      }
    }
  }
  const uint32_t T = lo;            // the k-th largest score pattern
  const uint32_t need_eq = krem;    // how many keys equal to T are taken
  const uint32_t eq_count = in_range;

  // g(i, u) over the candidates at positions [w0, w1)
  auto each = [&](int64_t w0, int64_t w1, auto&& g) {
    if (listed) {
      const uint32_t m = ncand;
      for (uint32_t c = threadIdx.x; c < m; c += TK_THREADS) {
        const int64_t i = cpos[c];
        if (i >= w0 && i < w1) g(i, cval[c]);
      }
    } else {
      tk_stream(src, w0, w1, [&](int64_t i, uint32_t raw) { g(i, tk_clean(raw, ctx)); });
    }
  };
  auto clear_bm = [&]() {
    for (int w = threadIdx.x; w < TK_BMW; w += TK_THREADS) bm[w] = 0u;
    __syncthreads();
  };

  // ---- the tie cut: position of the need_eq-th key equal to T
  int64_t pcut = INT64_MAX;
  if (need_eq < eq_count) {
    uint32_t seen = 0;
    for (int64_t w0 = 0; w0 < n; w0 += TK_WIN) {
      const int64_t w1 = min(n, w0 + TK_WIN);
      clear_bm();
      each(w0, w1, [&](int64_t i, uint32_t u) {
        if (u == T) atomicOr(&bm[(i - w0) >> 5], 1u << ((i - w0) & 31));
      });
      __syncthreads();
      const uint4 wv = reinterpret_cast<const uint4*>(bm)[threadIdx.x];
      const uint32_t cnt = __popc(wv.x) + __popc(wv.y) + __popc(wv.z) + __popc(wv.w);
      uint32_t tot;
      const uint32_t before = tk_excl_scan(cnt, scratch, tot);
      const uint32_t r = need_eq - seen;     // rank wanted within this window (1-based)
      if (r <= tot) {
        if (before < r && r <= before + cnt) {
          uint32_t left = r - before;
          const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t c = __popc(ws[q]);
            if (left > 0 && left <= c) {
              uint32_t bits = ws[q];
              for (uint32_t j = 1; j < left; ++j) bits &= bits - 1;
              pstar = w0 + (int64_t)(threadIdx.x * 4 + q) * 32 + (__ffs(bits) - 1);
              left = 0;
            } else if (left > 0) {
              left -= c;
            }
          }
        }
        __syncthreads();
        pcut = pstar;
        break;
      }
      seen += tot;
    }
  }

  // ---- mark and emit in position order, one window at a time
  uint32_t written = 0;
  for (int64_t w0 = 0; w0 < n; w0 += TK_WIN) {
    const int64_t w1 = min(n, w0 + TK_WIN);
    clear_bm();
    each(w0, w1, [&](int64_t i, uint32_t u) {
      if (u > T || (u == T && i <= pcut)) atomicOr(&bm[(i - w0) >> 5], 1u << ((i - w0) & 31));
    });
    __syncthreads();
    const uint4 wv = reinterpret_cast<const uint4*>(bm)[threadIdx.x];
    const uint32_t cnt = __popc(wv.x) + __popc(wv.y) + __popc(wv.z) + __popc(wv.w);
    uint32_t tot;
    uint32_t at = written + tk_excl_scan(cnt, scratch, tot);
    const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t bits = ws[q];
      while (bits) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        if (at < k) out[W + at] = (int32_t)(w0 + (int64_t)(threadIdx.x * 4 + q) * 32 + bit);
        ++at;
      }
    }
    written += tot;
  }
  if (written != k && threadIdx.x == 0) report(ctx, ST_DEVICE_CHECK);
}

}  // namespace hs2
