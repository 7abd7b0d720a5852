// Top-k of long decode rows over the whole GPU (rows a4, a5 at decode): a few
// sequences of up to 2^20 candidates would leave a CTA per row (or per slice
// of a row, then a merge of the slices' lists) doing long serial work, so the
// rows are cut into chunks of RX_CHUNK candidates, one CTA each, and the k-th
// largest score is found by a most-significant-digit radix select whose
// histograms every chunk adds to.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph -- the 128 most recent tokens
// are forced into the selection and 1024 high-scoring out-of-window tokens
// added.  Ties go to the smaller position, as in every other top-k here.
//
// Scores are >= 0, so their fp32 bit patterns (31 bits) order like the
// values.  The digits are bits [30:20], [19:9] and [8:0]:
//   radix_hist_kernel<P> (P = 0, 1, 2; grid chunks x rows): each CTA
//     histograms digit P of its chunk's candidates that carry the digits fixed
//     so far, in shared memory, and adds the non-zero bins to the row's global
//     histogram.  The CTA that finishes last (a counter per row and pass; no
//     CTA waits for another) finds the bin holding the k-th largest and
//     stores the digits fixed so far and the rank left within them.
//   radix_count_kernel: with the k-th largest pattern T and the number of
//     candidates equal to it that are taken (need_eq) known, each chunk counts
//     its candidates above T and equal to T; the last CTA turns the counts
//     into each chunk's exclusive prefix.
//   radix_write_kernel: each chunk takes its candidates above T and its ties
//     while the row's tie count stays below need_eq, and writes them in
//     position order after the selected candidates of the chunks before it:
//     an index row (the window, then the selection) or a (score, position)
//     list.
// The histograms, counters and state are zeroed by decode_sigma_kernel,
// which runs first.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int RX_THREADS = 256;
constexpr int RX_CHUNK = 8192;                       // candidates per CTA
constexpr int RX_PER = RX_CHUNK / RX_THREADS;        // 32 consecutive candidates per thread
constexpr int RX_HIST = 2048 + 2048 + 512 + 8;       // per row: the three digits' bins, then RX_ST words
constexpr int RX_ST = 2048 + 2048 + 512;             // [0..3) done counters, [4] prefix, [5] rank left

struct RadixParams {
  const float* sigma;    // row b at sigma + b * ld, candidates [0, n)
  int64_t ld;
  int64_t n;             // candidates per row (> topk)
  int chunks;            // ceil(n / RX_CHUNK)
  int topk;
  int window;
  int64_t pos;           // query position (index rows)
  int64_t pos_offset;    // added to the positions written (a shard's first global position)
  uint32_t* hist;        // [rows, RX_HIST]: histograms, counters, state (zeroed before the first pass)
  uint32_t* cnt;         // [rows, chunks, 2]: candidates above T, equal to T; then their exclusive prefixes
  int32_t* idx;          // index rows [rows, window + topk], or nullptr: lists below
  float* lval;           // lists [rows, topk] (scores), [rows, topk] positions, [rows] lengths
  int32_t* lpos;
  int32_t* lcnt;
};

__device__ __forceinline__ uint32_t rx_clean(uint32_t u, const DevCtx& ctx) {
  if (u > 0x7f800000u) {                 // NaN or a negative score: not a probability sum
    report(ctx, ST_DEVICE_CHECK);
    return 0u;
  }
  return u;
}

// Exclusive prefix sum over the CTA; `total` gets the sum.
__device__ __forceinline__ uint32_t rx_excl_scan(uint32_t v, uint32_t* scratch, uint32_t& total) {
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
  for (int w = 0; w < RX_THREADS / 32; ++w) {
    const uint32_t s = scratch[w];
    before += w < warp ? s : 0u;
    tot += s;
  }
  total = tot;
  __syncthreads();
  return before + x - v;
}

// The bin d of a histogram of nb bins (nb / RX_THREADS consecutive bins per
// thread) holding the r-th largest element: above(d) < r <= above(d) + h[d].
// Returns d and sets r -= above(d).  Every thread gets the same result.
__device__ __forceinline__ uint32_t rx_pick(const uint32_t* h, int nb, uint32_t& r, uint32_t* scratch,
                                            uint32_t* res) {
  const int per = nb / RX_THREADS;
  // thread t owns bins [per * (RX_THREADS-1-t), ...): bins descending with t,
  // so an exclusive scan over t counts the elements in the higher bins
  const int b0 = per * (RX_THREADS - 1 - threadIdx.x);
  uint32_t v[8], sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = i < per ? __ldcg(h + b0 + i) : 0u;
    sum += v[i];
  }
  uint32_t tot;
  uint32_t above = rx_excl_scan(sum, scratch, tot);
  if (above < r && r <= above + sum) {
    for (int i = per - 1; i >= 0; --i) {
      if (r <= above + v[i]) {
        res[0] = (uint32_t)(b0 + i);
        res[1] = above;
        break;
      }
      above += v[i];
    }
  }
  __syncthreads();
  const uint32_t d = res[0];
  r -= res[1];
  __syncthreads();
  return d;
}

// This thread's 32 consecutive candidates of the chunk (16-byte loads; rows
// and chunks start 16-byte aligned), cleaned; past n they read as "absent".
__device__ __forceinline__ int rx_load(const RadixParams& p, int64_t b, int x, uint32_t (&u)[RX_PER],
                                       const DevCtx& ctx) {
  const int64_t j0 = (int64_t)x * RX_CHUNK + threadIdx.x * RX_PER;
  const uint32_t* src = reinterpret_cast<const uint32_t*>(p.sigma + b * p.ld) + j0;
  const int m = (int)max((int64_t)0, min((int64_t)RX_PER, p.n - j0));
  if (m == RX_PER) {
#pragma unroll
    for (int q = 0; q < RX_PER / 4; ++q) {
      const uint4 w = reinterpret_cast<const uint4*>(src)[q];
      u[4 * q] = w.x; u[4 * q + 1] = w.y; u[4 * q + 2] = w.z; u[4 * q + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < RX_PER; ++i) u[i] = i < m ? src[i] : 0u;
  }
  bool bad = false;
#pragma unroll
  for (int i = 0; i < RX_PER; ++i) bad |= i < m && u[i] > 0x7f800000u;
  if (bad) {
#pragma unroll
    for (int i = 0; i < RX_PER; ++i)
      if (i < m) u[i] = rx_clean(u[i], ctx);
  }
  return m;
}

// True in every thread of the CTA that finishes last among the row's chunks
// (each thread's global writes and atomics made visible before the count).
__device__ __forceinline__ bool rx_last(uint32_t* counter, int chunks, uint32_t* flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) flag[0] = atomicAdd(counter, 1u) == (uint32_t)chunks - 1 ? 1u : 0u;
  __syncthreads();
  const bool last = flag[0] != 0u;
  if (last) __threadfence();
  return last;
}

template <int PASS>
__global__ void __launch_bounds__(RX_THREADS)
radix_hist_kernel(RadixParams p, DevCtx ctx) {
  constexpr int NB = PASS == 2 ? 512 : 2048;
  constexpr int SH = PASS == 0 ? 20 : (PASS == 1 ? 9 : 0);
  constexpr int OFF = PASS == 0 ? 0 : (PASS == 1 ? 2048 : 4096);
  __shared__ uint32_t h[NB];
  __shared__ uint32_t scratch[RX_THREADS / 32];
  __shared__ uint32_t res[2];
  const int x = blockIdx.x;
  const int64_t b = blockIdx.y;
  uint32_t* hrow = p.hist + b * RX_HIST;
  uint32_t* st = hrow + RX_ST;
  const uint32_t prefix = PASS == 0 ? 0u : __ldcg(st + 4);
  for (int i = threadIdx.x; i < NB; i += RX_THREADS) h[i] = 0u;
  uint32_t u[RX_PER];
  const int m = rx_load(p, b, x, u, ctx);
  __syncthreads();
  const uint32_t pmask = PASS == 0 ? 0u : (PASS == 1 ? 0x7ff00000u : 0x7ffffe00u);
  // a warp whose lanes all add to one bin adds once (near-equal scores
  // crowd a few bins of the first digits)
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < RX_PER; ++i) {
    const bool in = i < m && (u[i] & pmask) == prefix;
    const uint32_t bin = (u[i] >> SH) & (NB - 1);
    const unsigned act = __ballot_sync(0xffffffffu, in);
    if (act == 0u) continue;
    const int leader = __ffs(act) - 1;
    const uint32_t b0 = __shfl_sync(0xffffffffu, bin, leader);
    if (__all_sync(0xffffffffu, !in || bin == b0)) {
      if (lane == leader) atomicAdd(&h[b0], (uint32_t)__popc(act));
    } else if (in) {
      atomicAdd(&h[bin], 1u);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NB; i += RX_THREADS)
    if (h[i]) atomicAdd(&hrow[OFF + i], h[i]);
  if (!rx_last(&st[PASS], p.chunks, res)) return;
  // the last chunk of the row: fix digit PASS
  uint32_t rank = PASS == 0 ? (uint32_t)p.topk : __ldcg(st + 5);
  const uint32_t d = rx_pick(hrow + OFF, NB, rank, scratch, res);
  if (threadIdx.x == 0) {
    st[4] = prefix | (d << SH);
    st[5] = rank;
  }
}

__global__ void __launch_bounds__(RX_THREADS)
radix_count_kernel(RadixParams p, DevCtx ctx) {
  __shared__ uint32_t scratch[RX_THREADS / 32];
  __shared__ uint32_t flag[1];
  const int x = blockIdx.x;
  const int64_t b = blockIdx.y;
  uint32_t* st = p.hist + b * RX_HIST + RX_ST;
  const uint32_t T = __ldcg(st + 4);
  uint32_t u[RX_PER];
  const int m = rx_load(p, b, x, u, ctx);
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < RX_PER; ++i) {
    gt += (i < m && u[i] > T) ? 1u : 0u;
    eq += (i < m && u[i] == T) ? 1u : 0u;
  }
  uint32_t tg, te;
  rx_excl_scan(gt, scratch, tg);
  rx_excl_scan(eq, scratch, te);
  uint32_t* cr = p.cnt + b * p.chunks * 2;
  if (threadIdx.x == 0) {
    cr[2 * x] = tg;
    cr[2 * x + 1] = te;
  }
  if (!rx_last(&st[3], p.chunks, flag)) return;
  // the last chunk: every chunk's counts -> exclusive prefixes, in place
  // (RX_THREADS consecutive chunks at a time)
  uint32_t run_g = 0, run_e = 0;
  for (int c0 = 0; c0 < p.chunks; c0 += RX_THREADS) {
    const int c = c0 + threadIdx.x;
    const uint32_t a = c < p.chunks ? __ldcg(cr + 2 * c) : 0u;
    const uint32_t e = c < p.chunks ? __ldcg(cr + 2 * c + 1) : 0u;
    uint32_t sa, se;
    const uint32_t pa = rx_excl_scan(a, scratch, sa);
    const uint32_t pe = rx_excl_scan(e, scratch, se);
    if (c < p.chunks) {
      cr[2 * c] = run_g + pa;
      cr[2 * c + 1] = run_e + pe;
    }
    run_g += sa;
    run_e += se;
  }
}

__global__ void __launch_bounds__(RX_THREADS)
radix_write_kernel(RadixParams p, DevCtx ctx) {
  __shared__ uint32_t scratch[RX_THREADS / 32];
  const int x = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int k = p.topk;
  const uint32_t* st = p.hist + b * RX_HIST + RX_ST;
  const uint32_t T = __ldcg(st + 4), need_eq = __ldcg(st + 5);
  // selected candidates and ties of the chunks before this one
  const uint32_t gt_before = __ldcg(p.cnt + (b * p.chunks + x) * 2);
  const uint32_t eq_before = __ldcg(p.cnt + (b * p.chunks + x) * 2 + 1);
  uint32_t u[RX_PER];
  const int m = rx_load(p, b, x, u, ctx);
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < RX_PER; ++i) {
    gt += (i < m && u[i] > T) ? 1u : 0u;
    eq += (i < m && u[i] == T) ? 1u : 0u;
  }
  uint32_t tot;
  const uint32_t eq_rank = eq_before + rx_excl_scan(eq, scratch, tot);   // the row's ties before this thread's
  // this thread's selected count: its candidates above T and its ties still taken
  const uint32_t eq_take = eq_rank >= need_eq ? 0u : min(eq, need_eq - eq_rank);
  uint32_t at = rx_excl_scan(gt + eq_take, scratch, tot) + gt_before + min(eq_before, need_eq);
  const int64_t j0 = (int64_t)x * RX_CHUNK + threadIdx.x * RX_PER;
  uint32_t eq_seen = 0;
  const bool list = p.idx == nullptr;
  int32_t* out = list ? nullptr : p.idx + b * (int64_t)(p.window + k) + p.window;
#pragma unroll
  for (int i = 0; i < RX_PER; ++i) {
    if (i >= m) break;
    bool take = u[i] > T;
    if (u[i] == T) take = eq_seen++ < eq_take;
    if (take) {
      if (at < (uint32_t)k) {
        const int32_t pos = (int32_t)(p.pos_offset + j0 + i);
        if (list) {
          p.lval[b * k + at] = __uint_as_float(u[i]);
          p.lpos[b * k + at] = pos;
        } else {
          out[at] = pos;
        }
      }
      ++at;
    }
  }
  if (x == 0) {
    if (list) {
      if (threadIdx.x == 0) p.lcnt[b] = k;
    } else {
      int32_t* row = p.idx + b * (int64_t)(p.window + k);
      for (int w = threadIdx.x; w < p.window; w += RX_THREADS) {
        const int64_t v = p.pos - p.window + 1 + w;
        row[w] = v >= 0 ? (int32_t)v : -1;
      }
    }
  }
  // the row selects exactly k (n > k): the last thread of the last chunk ends
  // at the row's total, which says otherwise only if the histograms were not
  // zeroed or the scores changed between the passes
  if (x == p.chunks - 1 && threadIdx.x == RX_THREADS - 1 && at != (uint32_t)k) report(ctx, ST_DEVICE_CHECK);
}

}  // namespace hs2
