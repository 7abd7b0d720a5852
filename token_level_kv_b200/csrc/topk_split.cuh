// Top-k lists of slices of a row, and merges of such lists (rows a4, a5 of
// the context-sharded decode): a shard's candidates are cut into S slices
// whose exact top-k lists merge into the shard's list, and the shards' lists
// merge into the index row.  (Long rows of the single-GPU decode take the
// radix select of topk_radix.cuh instead.)
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph -- the 128 most recent tokens
// are forced into the selection and 1024 high-scoring out-of-window tokens
// added; 10100.com article -- *at most* 1024.  Ties go to the smaller
// position, as in the single-CTA top-k.
//
//   topk_slice_kernel (grid S x batch): the exact top-k of one slice, under the
//     order (score descending, position ascending), as (score, position)
//     pairs in position order.  Every key of the row's top-k is in its
//     slice's top-k (the keys that outrank it in its slice outrank it in the
//     row), so the S lists hold the answer.
//   topk_merge_kernel<false> (grid G x batch, when there are many slices):
//     the top-k of each group of `group` consecutive lists, as a list again
//     (the same argument: the top-k of the row lies in its groups' top-k).
//   topk_merge_kernel<true> (grid batch): the top-k of the concatenated lists,
//     which are in ascending position order already, written after the window.
// Both keep their candidates' fp32 patterns in shared memory (scores are
// >= 0, so the patterns order like the values) and find the k-th largest by
// an exact range select over the patterns (256 bins a pass over the range
// still holding it); two block-wide scans then take the keys above it and, in
// position order, the first ties equal to it.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int TS_THREADS = 256;
constexpr int TS_CAP = 45056;                    // candidates a CTA holds (176 KB)
constexpr size_t TS_SMEM = (size_t)TS_CAP * 4 + 256 * 4;
constexpr int64_t TS_SLICE = 32768;              // preferred slice length

struct TopkSplitParams {
  const float* sigma;    // row b at sigma + b * ld, candidates [0, n)
  int64_t ld;
  int64_t n;             // candidates per row
  int64_t slice;         // candidates per slice (the last may be shorter)
  int splits;            // S
  int topk;              // k
  int window;
  int64_t pos;           // query position
  int64_t pos_offset;    // added to the positions stored in the lists (a shard's first global position)
  float* cval;           // [batch, S, k] slice lists (scores)
  int32_t* cpos;         // [batch, S, k] (positions)
  int32_t* ccnt;         // [batch, S] list lengths
  int group;             // lists merged per CTA of the first merge level (0: one level)
  float* gval;           // [batch, G, k] first-level merged lists, G = ceil(S / group)
  int32_t* gpos;
  int32_t* gcnt;         // [batch, G]
  int32_t* idx;          // [batch, window + k]
  // Where the final merge finds list s of row b when they are not the slice
  // lists above (v_list > 0): scores and positions at (b * v_row + s * v_list)
  // and its length at (b * c_row + s * c_list), in elements.
  int64_t v_row, v_list, c_row, c_list;
};

// Exclusive prefix sum over the CTA; `total` gets the sum.
__device__ __forceinline__ uint32_t ts_excl_scan(uint32_t v, uint32_t* scratch, uint32_t& total) {
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
  for (int w = 0; w < TS_THREADS / 32; ++w) {
    const uint32_t s = scratch[w];
    before += w < warp ? s : 0u;
    tot += s;
  }
  total = tot;
  __syncthreads();
  return before + x - v;
}

// The k-th largest of u[0, m) (m > k): *T its pattern, *need_eq how many
// elements equal to it belong to the top k.  Range select: each pass splits
// the pattern range [lo, hi] still holding the k-th element into at most 256
// equal bins (lo, hi start at the extremes of u), so the passes spread the
// elements over the bins whatever the scores' spread, and at most four are
// needed.
__device__ __forceinline__ void ts_radix_select(const uint32_t* u, int m, uint32_t k, uint32_t* hist,
                                                uint32_t* pick, uint32_t* scratch, uint32_t* T,
                                                uint32_t* need_eq) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t mn = 0xffffffffu, mx = 0u;
  for (int c = threadIdx.x; c < m; c += TS_THREADS) {
    mn = min(mn, u[c]);
    mx = max(mx, u[c]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    scratch[warp] = mn;
    hist[warp] = mx;
  }
  __syncthreads();
  uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
  for (int w = 0; w < TS_THREADS / 32; ++w) {
    lo = min(lo, scratch[w]);
    hi = max(hi, hist[w]);
  }
  __syncthreads();
  uint32_t krem = k;                               // rank wanted among the elements in [lo, hi]
  while (hi > lo) {
    const uint32_t span = hi - lo;
    const int sh = max(0, 32 - __clz((int)span) - 8);   // (span >> sh) < 256
    hist[threadIdx.x] = 0u;
    __syncthreads();
    for (int c = threadIdx.x; c < m; c += TS_THREADS) {
      const uint32_t x = u[c];
      if (x >= lo && x <= hi) atomicAdd(&hist[(x - lo) >> sh], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t h[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        h[i] = hist[8 * lane + i];
        tot += h[i];
      }
      uint32_t incl = tot;                         // bins of this lane and the higher lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += y;
      }
      uint32_t above = incl - tot;
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
    const uint32_t nlo = lo + (pick[0] << sh);
    const uint32_t top = nlo + ((1u << sh) - 1u);
    hi = (top > hi || top < nlo) ? hi : top;
    lo = nlo;
    krem -= pick[1];
    __syncthreads();
  }
  *T = lo;
  *need_eq = krem;
}

// Elements per thread of the in-order passes: thread t owns [t*per, (t+1)*per).
// An odd length puts the 32 lanes of a warp on 32 different banks.
__device__ __forceinline__ int ts_per(int m) { return ((m + TS_THREADS - 1) / TS_THREADS) | 1; }

// Marks u[c] = 1 for the top k of u[0, m) (ties in index order), 0 otherwise,
// and returns this thread's exclusive offset among the kept ones (thread t
// owns the elements of ts_per).  With m <= k every element is kept.
__device__ __forceinline__ uint32_t ts_mark(uint32_t* u, int m, uint32_t k, uint32_t* hist, uint32_t* pick,
                                            uint32_t* scratch, uint32_t* total) {
  uint32_t T = 0u, need_eq = 0xffffffffu;
  if (m > (int)k) ts_radix_select(u, m, k, hist, pick, scratch, &T, &need_eq);
  const int per = ts_per(m);
  const int c0 = threadIdx.x * per, c1 = min(m, c0 + per);
  uint32_t n_eq = 0;
  for (int c = c0; c < c1; ++c) n_eq += u[c] == T ? 1u : 0u;
  uint32_t tot;
  uint32_t eq_before = ts_excl_scan(n_eq, scratch, tot);
  uint32_t n_keep = 0;
  for (int c = c0; c < c1; ++c) {
    const uint32_t x = u[c];
    bool keep = x > T;
    if (x == T) keep = eq_before++ < need_eq;
    n_keep += keep ? 1u : 0u;
    u[c] = keep ? 1u : 0u;                       // own elements only
  }
  return ts_excl_scan(n_keep, scratch, *total);
}

__global__ void __launch_bounds__(TS_THREADS)
topk_slice_kernel(TopkSplitParams p, DevCtx ctx) {
  extern __shared__ __align__(16) uint8_t smem_ts[];
  uint32_t* u = reinterpret_cast<uint32_t*>(smem_ts);
  uint32_t* hist = u + TS_CAP;
  __shared__ uint32_t scratch[TS_THREADS / 32];
  __shared__ uint32_t pick[2];
  const int s = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int64_t j0 = (int64_t)s * p.slice;
  const int m = (int)max((int64_t)0, min(p.n, j0 + p.slice) - j0);
  const float* src = p.sigma + b * p.ld + j0;      // 16-byte aligned: ld and slice are multiples of 64
  const int64_t lo = (b * p.splits + s) * (int64_t)p.topk;
  {
    // 16-byte loads, four in flight per thread
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    const int m4 = m >> 2;
    bool bad = false;
    for (int c4 = threadIdx.x; c4 < m4; c4 += 4 * TS_THREADS) {
      uint4 v[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = c4 + r * TS_THREADS;
        v[r] = j < m4 ? s4[j] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = c4 + r * TS_THREADS;
        if (j < m4) {
          uint32_t e[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            bad |= e[q] > 0x7f800000u;           // NaN or negative: not a probability sum
            e[q] = e[q] > 0x7f800000u ? 0u : e[q];
          }
          *reinterpret_cast<uint4*>(u + 4 * j) = make_uint4(e[0], e[1], e[2], e[3]);
        }
      }
    }
    for (int c = (m4 << 2) + threadIdx.x; c < m; c += TS_THREADS) {
      const uint32_t x = __float_as_uint(src[c]);
      bad |= x > 0x7f800000u;
      u[c] = x > 0x7f800000u ? 0u : x;
    }
    if (bad) report(ctx, ST_DEVICE_CHECK);
  }
  __syncthreads();
  const int per = ts_per(m);
  const int c0 = threadIdx.x * per, c1 = min(m, c0 + per);
  uint32_t total;
  // ts_mark turns u into keep flags; the kept scores are read again from the
  // row, which the load above has just brought into L2
  uint32_t at = ts_mark(u, m, (uint32_t)p.topk, hist, pick, scratch, &total);
  for (int c = c0; c < c1; ++c) {
    if (!u[c]) continue;
    uint32_t x = __float_as_uint(src[c]);
    if (x > 0x7f800000u) x = 0u;
    p.cval[lo + at] = __uint_as_float(x);
    p.cpos[lo + at] = (int32_t)(p.pos_offset + j0 + c);
    ++at;
  }
  if (threadIdx.x == 0) p.ccnt[b * p.splits + s] = (int32_t)total;
}

// FINAL: the top-k of all n_in lists of row b (at in_* with n_in lists of k
// slots per row) written as the index row.  Otherwise the top-k of lists
// [g*group, g*group + group) written as list g of the first merge level.
template <bool FINAL>
__global__ void __launch_bounds__(TS_THREADS)
topk_merge_kernel(TopkSplitParams p, DevCtx ctx) {
  extern __shared__ __align__(16) uint8_t smem_ts[];
  uint32_t* u = reinterpret_cast<uint32_t*>(smem_ts);
  uint32_t* hist = u + TS_CAP;
  __shared__ uint32_t scratch[TS_THREADS / 32];
  __shared__ uint32_t pick[2];
  __shared__ int32_t offs[65];
  const int64_t b = FINAL ? blockIdx.x : blockIdx.y;
  const int k = p.topk;
  // the lists this CTA merges: FINAL reads the first-level lists when there
  // is a first level, else the slice lists
  const bool from_groups = FINAL && p.group > 0;
  const int n_lists_row = from_groups ? (p.splits + p.group - 1) / p.group : p.splits;
  const float* in_val = from_groups ? p.gval : p.cval;
  const int32_t* in_pos = from_groups ? p.gpos : p.cpos;
  const int32_t* in_cnt = from_groups ? p.gcnt : p.ccnt;
  const int l0 = FINAL ? 0 : blockIdx.x * p.group;
  const int nl = FINAL ? n_lists_row : min(p.group, p.splits - l0);
  const bool strided = FINAL && !from_groups && p.v_list > 0;
  const int64_t v_row = strided ? p.v_row : (int64_t)n_lists_row * k, v_list = strided ? p.v_list : k;
  const int64_t c_row = strided ? p.c_row : n_lists_row, c_list = strided ? p.c_list : 1;
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int s = 0; s < nl; ++s) {
      offs[s] = acc;
      acc += in_cnt[b * c_row + (l0 + s) * c_list];
    }
    offs[nl] = acc;
  }
  __syncthreads();
  const int M = offs[nl];
  const int64_t lo = b * v_row + l0 * v_list;       // list s of this CTA starts at lo + s * v_list
  // every list slot at once (independent loads); slot i of list s lands at offs[s] + i
  const int n_slot = nl * k;
#pragma unroll 4
  for (int q = threadIdx.x; q < n_slot; q += TS_THREADS) {
    const int s = q / k, i = q - s * k;
    if (i < offs[s + 1] - offs[s]) u[offs[s] + i] = __float_as_uint(in_val[lo + s * v_list + i]);
  }
  __syncthreads();
  const int per = ts_per(M);
  const int c0 = threadIdx.x * per, c1 = min(M, c0 + per);
  uint32_t total;
  uint32_t at = ts_mark(u, M, (uint32_t)k, hist, pick, scratch, &total);
  int s = 0;
  while (s + 1 < nl && offs[s + 1] <= c0) ++s;
  if (FINAL) {
    const int W = p.window;
    int32_t* out = p.idx + b * (int64_t)(W + k);
    for (int w = threadIdx.x; w < W; w += TS_THREADS) {
      const int64_t v = p.pos - W + 1 + w;
      out[w] = v >= 0 ? (int32_t)v : -1;
    }
    for (int c = c0; c < c1; ++c) {
      while (offs[s + 1] <= c) ++s;
      if (!u[c]) continue;
      if (at < (uint32_t)k) out[W + at] = in_pos[lo + s * v_list + (c - offs[s])];
      ++at;
    }
    for (uint32_t i = total + threadIdx.x; i < (uint32_t)k; i += TS_THREADS) out[W + i] = -1;
    if (threadIdx.x == 0 && total != (uint32_t)min((int64_t)k, p.n)) report(ctx, ST_DEVICE_CHECK);
  } else {
    const int n_groups = (p.splits + p.group - 1) / p.group;
    const int64_t olo = (b * n_groups + blockIdx.x) * (int64_t)k;
    for (int c = c0; c < c1; ++c) {
      while (offs[s + 1] <= c) ++s;
      if (!u[c]) continue;
      const int64_t src = lo + s * v_list + (c - offs[s]);
      p.gval[olo + at] = in_val[src];
      p.gpos[olo + at] = in_pos[src];
      ++at;
    }
    if (threadIdx.x == 0) p.gcnt[b * n_groups + blockIdx.x] = (int32_t)total;
  }
}

}  // namespace hs2
