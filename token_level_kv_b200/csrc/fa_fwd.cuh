// Causal MQA full attention, prefill pass 1 (row a2): O and the per-row
// softmax statistics (m, l) the selection pass needs.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary): the full-attention layer is MQA (one KV head) with
// NoPE, causal; it also serves as the oracle selector, so its exact softmax
// normaliser is kept per (query, head).
//
// Design (sm_100a, tcgen05 + TMEM + TMA):
//   * The 128-row MMA tile packs (query, head) pairs: 128/H queries x H heads
//     share each K/V tile (MQA), rows of Q viewed as [Tq*H, D].
//   * Key tiles of 128.  TMEM: two S buffers (2 x 128 columns) + O (D columns).
//   * warp 0: TMA for Q and K; warp 6: TMA for V; warp 1: TMEM owner and the
//     single-thread tcgen05.mma issuer (S_j = Q K_j^T is issued before
//     O += P_{j-1} V_{j-1}, so the tensor pipe works while softmax runs);
//     warps 2..5: one (query, head) row per thread -- tcgen05.ld of S, causal
//     mask, online softmax in base 2, P (bf16) to shared memory in the
//     128-byte-swizzled K-major layout the next MMA reads, and a lazy rescale
//     of O in TMEM only when a row's max grows by more than 2^8.
//   * V is the MN-major B operand (keys x D, D contiguous) read straight from
//     the TMA tiles: leading byte offset = 16 KB between 64-column blocks.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int FA_THREADS = 224;

template <int D>
struct FaLayout {
  static constexpr int Q_BYTES = 128 * D * 2;
  static constexpr int K_BYTES = 128 * D * 2;
  static constexpr int V_BYTES = 128 * D * 2;
  static constexpr int P_BYTES = 128 * 128 * 2;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + K_BYTES;
  static constexpr int OFF_P = OFF_V + V_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr size_t SMEM = OFF_BAR + 256 + 1024;
};

struct FaParams {
  int64_t Tq;
  int64_t q_start;
  int64_t kv_len;
  int H;
  float scale_log2;        // softmax_scale * log2(e)
  __nv_bfloat16* O;        // [Tq*H, D]
  float* ml;               // [Tq*H, 2]: m (log2 units, the reference max used), l; may be null
  int n_qtiles;
  int64_t window;          // 0: every key <= the query; else the keys [p - window + 1, p]
};

template <int D>
__global__ void __launch_bounds__(FA_THREADS, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, FaParams p, DevCtx ctx) {
  using L = FaLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sP = smem + L::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 2;
  uint64_t* v_full = bars + 3;
  uint64_t* v_empty = bars + 4;
  uint64_t* s_full = bars + 5;     // [2]
  uint64_t* s_free = bars + 7;     // [2]
  uint64_t* p_full = bars + 9;
  uint64_t* p_empty = bars + 10;
  uint64_t* o_final = bars + 11;
  uint64_t* mma_done = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.n_qtiles - 1 - blockIdx.x;             // heaviest tiles first
  const int qpt = 128 / p.H;                               // queries per tile
  const int64_t q0 = (int64_t)qt * qpt;
  const int64_t q_last = min(p.Tq, q0 + qpt) - 1;
  const int64_t p_last = p.q_start + q_last;
  // key tiles kt0 .. kt0 + n_kt - 1 (a sliding window starts at the first
  // query's oldest key); loop counters j run from 0 and the tile is kt0 + j
  const int kt0 = p.window > 0 ? (int)(max((int64_t)0, p.q_start + q0 - p.window + 1) / 128) : 0;
  const int n_kt = (int)(p_last / 128) + 1 - kt0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(p_empty, 1);
    mbar_init(o_final, 1);
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ Q, K loads
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_expect_tx(q_full, L::Q_BYTES);
      for (int b = 0; b < D / 64; ++b) tma_load_2d(sQ + b * 16384, &tmQ, q_full, b * 64, qt * 128);
      int last = -1;
      for (int j = 0; j < n_kt; ++j) {
        if (!mbar_wait(k_empty, (j & 1) ^ 1, ctx)) break;
        mbar_expect_tx(k_full, L::K_BYTES);
        for (int b = 0; b < D / 64; ++b) tma_load_2d(sK + b * 16384, &tmK, k_full, b * 64, (kt0 + j) * 128);
        last = j;
      }
      mbar_drain(q_full, 0);
      if (last >= 0) mbar_drain(k_full, last & 1);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ V loads
    if (lane == 0) {
      tma_prefetch_desc(&tmV);
      int last = -1;
      for (int j = 0; j < n_kt; ++j) {
        if (!mbar_wait(v_empty, (j & 1) ^ 1, ctx)) break;
        mbar_expect_tx(v_full, L::V_BYTES);
        for (int b = 0; b < D / 64; ++b) tma_load_2d(sV + b * 16384, &tmV, v_full, b * 64, (kt0 + j) * 128);
        last = j;
      }
      if (last >= 0) mbar_drain(v_full, last & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = umma_idesc_bf16(128, 128, false);
      constexpr uint32_t idO = umma_idesc_bf16(128, D, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, ctx);
      bool any = false;
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(p_full, i & 1, ctx)) return false;
        if (!mbar_wait(v_full, i & 1, ctx)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = umma_desc_sw128(aP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = umma_desc_sw128(aV + kk * 2048, 16384, 1024);
          umma_bf16(tmem + 256, ad, bd, idO, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(v_empty);
        umma_commit(p_empty);
        return true;
      };
      for (int j = 0; j < n_kt && ok; ++j) {
        const int s = j & 1;
        if (!mbar_wait(k_full, j & 1, ctx)) { ok = false; break; }
        if (!mbar_wait(&s_free[s], ((j >> 1) & 1) ^ 1, ctx)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = umma_desc_sw128(aQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = umma_desc_sw128(aK + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          umma_bf16(tmem + s * 128, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        any = true;
        umma_commit(&s_full[s]);
        umma_commit(k_empty);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && issue_pv(n_kt - 1)) umma_commit(o_final);
      if (any) {
        umma_commit(mma_done);
        mbar_drain(mma_done, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax rows
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int64_t R = (int64_t)qt * 128 + r;
    const int64_t ql = R / p.H;
    const bool valid = ql < p.Tq;
    const int64_t pq = p.q_start + ql;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    float x[128];
    for (int j = 0; j < n_kt; ++j) {
      const int s = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[s], (j >> 1) & 1, ctx))) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + s * 128 + c * 32, x + c * 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[s]);

      const int64_t key0 = (int64_t)(kt0 + j) * 128;
      if (key0 + 127 > pq) {                           // the diagonal tile: keys after the query
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (key0 + i > pq) x[i] = -INFINITY;
      }
      if (p.window > 0 && key0 <= pq - p.window) {     // keys older than the sliding window
        const int64_t oldest = pq - p.window + 1;
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (key0 + i < oldest) x[i] = -INFINITY;
      }
      // row max of the raw scores (scale > 0 commutes with max), eight
      // independent chains so the single warp per scheduler is not latency-bound
      float mr[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mr[a] = x[a];
#pragma unroll
      for (int i = 8; i < 128; ++i) mr[i & 7] = fmaxf(mr[i & 7], x[i]);
      const float mt = fmaxf(fmaxf(fmaxf(mr[0], mr[1]), fmaxf(mr[2], mr[3])),
                             fmaxf(fmaxf(mr[4], mr[5]), fmaxf(mr[6], mr[7]))) * p.scale_log2;
      const float m_new = fmaxf(m_ref, mt);
      float alpha = 1.f;
      const bool need = m_new > m_ref + 8.f;
      if (need) {
        alpha = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - m_new);
        m_ref = m_new;
      }
      const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
      // p = 2^(s*c - mu): the argument as one packed FMA per pair, the sums in
      // four packed accumulators
      const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2), nmu2 = f2_pack(-mu, -mu);
      uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int i = 0; i < 128; i += 2) {
        const float2 a = f2_unpack(ffma2(f2_pack(x[i], x[i + 1]), c2, nmu2));
        x[i] = fast_exp2(a.x);
        x[i + 1] = fast_exp2(a.y);
        rs2[(i >> 1) & 3] = fadd2(rs2[(i >> 1) & 3], f2_pack(x[i], x[i + 1]));
      }
      const float2 r01 = f2_unpack(fadd2(rs2[0], rs2[1])), r23 = f2_unpack(fadd2(rs2[2], rs2[3]));
      const float rs = (r01.x + r01.y) + (r23.x + r23.y);
      l = l * alpha + rs;

      if (j >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(p_empty, (j - 1) & 1, ctx))) { ok = false; break; }
        tc_fence_after();
      }
      // P row -> shared memory, K-major 128B swizzle: 2 blocks of 64 keys
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int blk = u >> 3, c = u & 7;
        uint4 w;
        w.x = pack_bf16x2(x[u * 8 + 0], x[u * 8 + 1]);
        w.y = pack_bf16x2(x[u * 8 + 2], x[u * 8 + 3]);
        w.z = pack_bf16x2(x[u * 8 + 4], x[u * 8 + 5]);
        w.w = pack_bf16x2(x[u * 8 + 6], x[u * 8 + 7]);
        *reinterpret_cast<uint4*>(sP + blk * 16384 + r * 128 + ((c ^ (r & 7)) << 4)) = w;
      }
      if (j >= 1 && __any_sync(0xffffffffu, need)) {
        float o[32];
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          tmem_ld32(lane_base + 256 + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(lane_base + 256 + c * 32, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (__all_sync(0xffffffffu, ok && mbar_wait(o_final, 0, ctx))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* out = p.O + R * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(lane_base + 256 + c * 32, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(o[2 * i] * inv, o[2 * i + 1] * inv);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (valid && p.ml) {
        p.ml[R * 2] = m_ref;
        p.ml[R * 2 + 1] = l;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace hs2
