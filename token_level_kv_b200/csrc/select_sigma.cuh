// Selection scores, prefill pass 2 (row a3): for every query t and every
// out-of-window key j <= p - window,
//     sigma[t, j] = sum_h 2^(x_thj - m_th) / l_th,   x = scale*log2(e) * q_th . k_j
// with (m, l) the exact softmax statistics of pass 1 (kept apart, not folded
// into one log-sum-exp, so an fp32 lse of ~10 does not cost 1e-6 of accuracy).
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary): the full-attention layer acts as the oracle selector
// and scores tokens one by one with exact attention scores; the head
// aggregation (sum of the heads' probabilities) is this library's reading.
//
// Design (sm_100a): the product is computed transposed, S^T = K Q^T, with
// M = 128 keys and N = 256 (query, head) columns (16 queries of 16 heads), so a
// TMEM lane is one key and its columns hold every head of every query: the sum
// over heads is thread-local (no shuffles).  K streams through a ring of
// 64-column TMA boxes (16 KB); the 256-row Q block stays resident.  TMEM: two
// S^T buffers of 256 columns.  Sixteen epilogue warps (four per TMEM lane
// quarter, each taking a quarter of the queries) write sigma rows coalesced;
// with fewer the epilogue, not the tensor pipe, set the pace.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int SG_THREADS = 576;     // TMA warp, MMA warp, 16 epilogue warps
constexpr int SG_STAGES = 5;

template <int D>
struct SgLayout {
  static constexpr int Q_BYTES = 256 * D * 2;
  static constexpr int STAGE = 128 * 64 * 2;
  static constexpr int OFF_RING = Q_BYTES;
  static constexpr int OFF_ML = OFF_RING + SG_STAGES * STAGE;
  static constexpr int OFF_BAR = OFF_ML + 256 * 8;
  static constexpr size_t SMEM = OFF_BAR + 256 + 1024;
};

struct SgParams {
  int64_t Tq;
  int64_t q_start;
  int64_t kv_len;
  int H;
  int window;
  float scale_log2;
  const float* ml;        // [Tq*H, 2] from pass 1
  float* sigma;           // [Tq, ld]
  int64_t ld;
  int n_groups;
};

template <int D, int H>
__global__ void __launch_bounds__(SG_THREADS, 1)
select_sigma_kernel(const __grid_constant__ CUtensorMap tmQ256, const __grid_constant__ CUtensorMap tmK,
                    SgParams p, DevCtx ctx) {
  using L = SgLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* ring = smem + L::OFF_RING;
  float* sML = reinterpret_cast<float*>(smem + L::OFF_ML);     // [256] -m, then [256] 1/l
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* full = bars + 1;                    // [SG_STAGES]
  uint64_t* empty = full + SG_STAGES;           // [SG_STAGES]
  uint64_t* s_full = empty + SG_STAGES;         // [2]
  uint64_t* s_free = s_full + 2;                // [2]
  uint64_t* mma_done = s_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = p.n_groups - 1 - blockIdx.x;               // heaviest first
  constexpr int G = 256 / H;                                  // queries per group
  const int64_t g0 = (int64_t)grp * G;
  const int64_t p_last = p.q_start + min(p.Tq, g0 + G) - 1;
  const int64_t max_key = p_last - p.window;                  // last candidate of the group
  const int n_kt = max_key >= 0 ? (int)(max_key / 128) + 1 : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < SG_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], SG_THREADS - 64);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) {
    const int64_t R = g0 * H + i;
    float m = 0.f, inv = 0.f;
    if (R < p.Tq * H) {
      m = p.ml[R * 2];
      const float l = p.ml[R * 2 + 1];
      inv = l > 0.f ? 1.f / l : 0.f;
    }
    sML[i] = -m;
    sML[256 + i] = inv;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (n_kt == 0) {
    // no candidate keys for any query of the group
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
    return;
  }

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ256);
      tma_prefetch_desc(&tmK);
      mbar_expect_tx(q_full, L::Q_BYTES);
      for (int b = 0; b < D / 64; ++b) tma_load_2d(sQ + b * 32768, &tmQ256, q_full, b * 64, grp * 256);
      int stage = 0;
      uint32_t phase = 0;
      int issued[SG_STAGES];
      for (int s = 0; s < SG_STAGES; ++s) issued[s] = -1;
      bool ok = true;
      for (int j = 0; j < n_kt && ok; ++j) {
        for (int b = 0; b < D / 64; ++b) {
          if (!mbar_wait(&empty[stage], phase ^ 1, ctx)) { ok = false; break; }
          mbar_expect_tx(&full[stage], L::STAGE);
          tma_load_2d(ring + stage * L::STAGE, &tmK, &full[stage], b * 64, j * 128);
          issued[stage] = (int)phase;
          if (++stage == SG_STAGES) { stage = 0; phase ^= 1; }
        }
      }
      mbar_drain(q_full, 0);
      for (int s = 0; s < SG_STAGES; ++s)
        if (issued[s] >= 0) mbar_drain(&full[s], (uint32_t)issued[s]);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, 256, false);
      const uint32_t aQ = smem_u32(sQ), aR = smem_u32(ring);
      bool ok = mbar_wait(q_full, 0, ctx), any = false;
      int stage = 0;
      uint32_t phase = 0;
      for (int j = 0; j < n_kt && ok; ++j) {
        const int buf = j & 1;
        if (!mbar_wait(&s_free[buf], ((j >> 1) & 1) ^ 1, ctx)) break;
        tc_fence_after();
        for (int b = 0; b < D / 64; ++b) {
          if (!mbar_wait(&full[stage], phase, ctx)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = umma_desc_sw128(aR + stage * L::STAGE + k * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(aQ + b * 32768 + k * 32, 16, 1024);
            umma_bf16(tmem + buf * 256, ad, bd, idesc, (b | k) != 0 ? 1u : 0u);
          }
          any = true;
          umma_commit(&empty[stage]);
          if (++stage == SG_STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&s_full[buf]);
      }
      if (any) {
        umma_commit(mma_done);
        mbar_drain(mma_done, 0);
      }
    }
  } else {
    const int e = warp - 2;
    const int quarter = warp & 3;                  // TMEM lanes a warp may read: 32 * (warp % 4)
    const int part = e >> 2;                       // columns [64 * part, 64 * part + 64)
    const int kl = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int j = 0; j < n_kt; ++j) {
      const int buf = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (j >> 1) & 1, ctx))) break;
      tc_fence_after();
      const int64_t key = (int64_t)j * 128 + kl;
      // four chunks of 16 columns; chunk c+1's TMEM load is in flight while
      // chunk c is computed (tcgen05.wait::ld waits for all of this thread's
      // loads, so the next one is issued right after the wait)
      const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
      float va[16], vb[16];
      tmem_ld16(lane_base + buf * 256 + part * 64, va);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float* v = (ch & 1) ? vb : va;
        float* nxt = (ch & 1) ? va : vb;
        tmem_wait_ld();
        if (ch < 3) tmem_ld16(lane_base + buf * 256 + part * 64 + (ch + 1) * 16, nxt);
        // column part*64 + 16*ch + i  <->  (query (part*64 + 16*ch + i) / H, head i % H);
        // heads in pairs: one packed FMA for the two exponents' arguments and
        // one for the two terms of the sum (two interleaved partial sums)
#pragma unroll
        for (int qi = 0; qi < 16 / H; ++qi) {
          const int col = part * 64 + ch * 16 + qi * H;
          const int64_t tq = g0 + col / H;
          const int64_t pq = p.q_start + tq;
          uint64_t acc2 = 0ull;
#pragma unroll
          for (int h = 0; h < H; h += 4) {
            const float4 nm = *reinterpret_cast<const float4*>(sML + col + h);        // -m of 4 heads
            const float4 iv = *reinterpret_cast<const float4*>(sML + 256 + col + h);  // 1/l of 4 heads
            const float2 a = f2_unpack(ffma2(f2_pack(v[qi * H + h], v[qi * H + h + 1]), c2, f2_pack(nm.x, nm.y)));
            const float2 b = f2_unpack(ffma2(f2_pack(v[qi * H + h + 2], v[qi * H + h + 3]), c2, f2_pack(nm.z, nm.w)));
            acc2 = ffma2(f2_pack(fast_exp2(a.x), fast_exp2(a.y)), f2_pack(iv.x, iv.y), acc2);
            acc2 = ffma2(f2_pack(fast_exp2(b.x), fast_exp2(b.y)), f2_pack(iv.z, iv.w), acc2);
          }
          const float2 r = f2_unpack(acc2);
          if (tq < p.Tq && key <= pq - p.window) p.sigma[tq * p.ld + key] = r.x + r.y;
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace hs2
