// Sparse prefill layer (row a6) on the tensor cores: for every query row, the
// 16 heads attend over the row's gathered keys idx[t, :] of the shared bf16 KV.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph -- the sparse layers gather only
// the selected tokens (window + top-k) of the full layer's KV; MQA, NoPE.
//
// Design (sm_100a).  One persistent CTA per SM walks the query rows.
//   * Eight producer warps gather the selected K and V rows with cp.async into
//     a ring whose stage is one tile's rows over the whole head dim (128 keys
//     x d dims: 128-dim halves of two 64-dim atom columns in the 128-byte
//     swizzled layout the MMA reads); two lanes per 32-byte sector, so every
//     request is a whole sector of one row.  One commit per stage releases it
//     (every 16 MMAs at d = 256).
//   * One thread issues tcgen05.mma.  Per 128-key tile t it forms
//     S^T_t = K_t Q^T (M = 128 keys, N = 16 heads, K = d) into TMEM columns
//     [16t, 16t+16) of the row's S buffer; after the softmax it adds
//     O^T += V_t^T P_t^T (M = 128 dims per half of d -- V read MN-major
//     straight from the gathered tile --, N = 16 heads, K = 128 keys) into
//     TMEM columns [480, 480 + 16 * d/128).  With N = 16 a row takes 288
//     MMAs, so the issuing thread only adds constants to descriptors built
//     once per stage.
//   * Four softmax warps (one TMEM lane quarter each: a thread is one key of
//     every tile) run an exact two-pass softmax over the whole row: the
//     per-head maximum over all the row's keys, then p = 2^(s*c - m*c) into
//     P^T (bf16, K-major, swizzled) and the per-head sums.  They also write
//     the previous row's output from TMEM (a thread is one dim).
//   * Two rows are in flight: the ring carries K(0), K(1), V(0), K(2), V(1), ...
//     and S^T is double-buffered in TMEM, so row r's softmax overlaps row
//     r+1's gather and Q K^T products.
//   * P^T moves tile by tile through a 2-tile ring: the softmax writes tile t
//     while the tensor cores multiply tile t-1, which leaves shared memory to
//     a 192 KB gather ring (3 stages at d = 256, 6 at d = 128).
// Rows of up to 15 tiles (1920 keys): TMEM 2 x 240 + 32 columns (512 taken),
// shared memory 192 KB ring + 2 x 4 KB P^T + 2 x 8 KB Q.
#pragma once
#include "attn16.cuh"
#include "common.cuh"

namespace hs2 {

template <int D>
struct StcLayout {
  static constexpr int NPROD = 8;                // producer warps (16 key rows of a stage each)
  static constexpr int MMA_WARP = 4 + NPROD;
  static constexpr int NT = (MMA_WARP + 1) * 32; // 4 softmax warps, the producers, 1 MMA warp
  // a stage is one tile's K or V rows over the whole head dim: 128 keys x
  // d/128 halves of 128 dims (two 16 KB atom columns each), so the MMA thread
  // commits once per 16 (d = 256) or 8 (d = 128) MMAs
  static constexpr int HALF = 128 * 256;         // bytes of one 128-dim half of a tile
  static constexpr int STAGE = HALF * (D / 128);
  static constexpr int NSTG = 6 / (D / 128);     // ring stages (192 KB)
  static constexpr int MAXT = 15;                // tiles of 128 keys per row
  static constexpr int SBUF = 16 * MAXT;         // TMEM columns of one S^T buffer
  static constexpr int OCOL = 2 * SBUF;          // O^T: 16 columns per half of d
  static constexpr int HALVES = D / 128;         // 128-dim halves per tile
  static constexpr int P_TILE = 16 * 256;        // P^T of one tile: 16 heads x 128 keys bf16
  static constexpr int NPS = 2;                  // P^T tiles in flight (softmax -> P V products)
  static constexpr int Q_BYTES = 16 * D * 2;     // 16 heads x d, D/64 atom columns of 2 KB
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_P = OFF_RING + NSTG * STAGE;
  static constexpr int OFF_Q = OFF_P + NPS * P_TILE;
  static constexpr int OFF_RED = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_RED + (2 * 4 * 16 + 2 * 16) * 4;
  static constexpr size_t SMEM = OFF_BAR + 256 + 1024;   // + base alignment
};

// Instruction descriptor as umma_idesc_bf16, A MN-major (bit 15).
__host__ __device__ constexpr uint32_t umma_idesc_bf16_amn(int M, int N) {
  return umma_idesc_bf16(M, N, false) | (1u << 15);
}

template <int D>
__global__ void __launch_bounds__(StcLayout<D>::NT, 1)
sparse_tc_kernel(Attn16Params p, DevCtx ctx) {
  using L = StcLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem_stc[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_stc) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem + L::OFF_RING;
  uint8_t* sP = smem + L::OFF_P;
  uint8_t* sQ = smem + L::OFF_Q;
  float* red_m = reinterpret_cast<float*>(smem + L::OFF_RED);        // [4][16]
  float* red_l = red_m + 64;                                          // [4][16]
  float* linv = red_l + 64;                                           // [2][16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* full = bars;                       // [NSTG] producers' cp.async arrivals
  uint64_t* empty = full + L::NSTG;            // [NSTG] MMA commit
  uint64_t* s_full = empty + L::NSTG;          // [2] S^T of a row complete (per S buffer)
  uint64_t* p_full = s_full + 2;               // [NPS] a P^T tile written (the row's S read)
  uint64_t* p_empty = p_full + L::NPS;         // [NPS] its products done
  uint64_t* o_full = p_empty + L::NPS;         // O^T of a row complete
  uint64_t* mma_done = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nT = (p.n_idx + 127) / 128;
  const int64_t n_rows = p.n_rows;
  // rows of this CTA: blockIdx.x + r * gridDim.x, r < R
  const int R = blockIdx.x < n_rows ? (int)((n_rows - 1 - blockIdx.x) / gridDim.x) + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::NSTG; ++s) {
      mbar_init(&full[s], 32 * L::NPROD);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    for (int i = 0; i < L::NPS; ++i) {
      mbar_init(&p_full[i], 128);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == L::MMA_WARP) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 && warp < L::MMA_WARP) {
    // ------------------------------------------------------------ producers
    constexpr int RW = 128 / L::NPROD;            // key rows per producer warp
    const int w = warp - 4;                       // key rows [RW*w, RW*w + RW) of every stage
    const int ur = lane >> 4, uu = lane & 15;     // two rows per copy instruction, 16 units each
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto acquire = [&]() -> uint8_t* {
      // the warp decides together (a lane that timed out stops all of it)
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[slot], phase ^ 1, ctx))) return nullptr;
      return ring + slot * L::STAGE;
    };
    auto release = [&]() {
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[slot])) : "memory");
      if (++slot == L::NSTG) { slot = 0; phase ^= 1; }
    };
    // this lane's copies of a stage: rows RW*w + 2i + ur, 16-byte unit uu
    // (destination offsets in the swizzled stage, fixed for the kernel)
    uint32_t doff[RW / 2];
#pragma unroll
    for (int i = 0; i < RW / 2; ++i) {
      const int kr = RW * w + 2 * i + ur;
      doff[i] = (uint32_t)((uu >> 3) * 16384 + kr * 128 + (((uu & 7) ^ (kr & 7)) << 4));
    }
    // source rows of one tile (lane r holds row r's position)
    const uint8_t* srow[RW / 2];
    uint32_t svalid = 0;
    auto set_rows = [&](const uint8_t* base, int32_t mypos) {
#pragma unroll
      for (int i = 0; i < RW / 2; ++i) {
        const int32_t pr = __shfl_sync(0xffffffffu, mypos, 2 * i + ur);
        srow[i] = base + ((int64_t)(pr < 0 ? 0 : pr) * D + uu * 8) * 2;
        svalid = (svalid & ~(1u << i)) | ((pr >= 0 ? 1u : 0u) << i);
      }
    };
    // one stage: dims [128c, 128c + 128) of the tile's rows
    auto copy_rows = [&](uint8_t* st, int c) {
      const uint32_t sa = smem_u32(st);
#pragma unroll
      for (int i = 0; i < RW / 2; ++i) cp_async16(sa + doff[i], srow[i] + c * 256, (svalid >> i) & 1u);
    };
    // positions of tile t of a row (lane r < RW: row RW*w + r), loaded one
    // tile ahead so their latency hides behind the copies; entries outside
    // [-1, kv_len) are reported (once, in the K pass) and skipped
    auto ldpos = [&](const int32_t* irow, int t) -> int32_t {
      const int sl = t * 128 + RW * w + lane;
      return (t < nT && lane < RW && sl < p.n_idx) ? irow[sl] : -1;
    };
    // step st: the K stages of row st (st < R), then the V stages of row st-1
    for (int st = 0; st <= R && ok; ++st) {
      if (st < R) {
        const int64_t row = blockIdx.x + (int64_t)st * gridDim.x;
        const int32_t* irow = p.idx + row * p.n_idx;
        uint8_t* qb = sQ + (st & 1) * L::Q_BYTES;
        int32_t nextpos = ldpos(irow, 0);
        for (int t = 0; t < nT && ok; ++t) {
          int32_t mypos = nextpos;
          nextpos = ldpos(irow, t + 1);
          if (mypos < -1 || mypos >= p.kv_len) {
            report(ctx, ST_DEVICE_CHECK);
            mypos = -1;
          }
          set_rows(reinterpret_cast<const uint8_t*>(p.K), mypos);
          {
            uint8_t* stg = acquire();
            if (!stg) { ok = false; break; }
            if (t == 0) {
              // the row's Q (16 heads; rows >= H zero) rides with the first stage
              const __nv_bfloat16* q = p.Q + row * p.H * D;
              for (int u = 32 * w + lane; u < 16 * D / 8; u += 32 * L::NPROD) {
                const int h = u / (D / 8), un = u % (D / 8);
                const int ac = un >> 3, u8 = un & 7;
                cp_async16(smem_u32(qb + ac * 2048 + h * 128 + ((u8 ^ (h & 7)) << 4)),
                           q + (h < p.H ? h : 0) * D + un * 8, h < p.H);
              }
            }
            for (int c = 0; c < L::HALVES; ++c) copy_rows(stg + c * L::HALF, c);
            release();
          }
        }
      }
      if (st >= 1) {
        const int32_t* irow = p.idx + (blockIdx.x + (int64_t)(st - 1) * gridDim.x) * p.n_idx;
        int32_t nextpos = ldpos(irow, 0);
        for (int t = 0; t < nT && ok; ++t) {
          int32_t mypos = nextpos;
          nextpos = ldpos(irow, t + 1);
          if (mypos < -1 || mypos >= p.kv_len) mypos = -1;
          set_rows(reinterpret_cast<const uint8_t*>(p.V), mypos);
          uint8_t* stg = acquire();
          if (!stg) { ok = false; break; }
          for (int c = 0; c < L::HALVES; ++c) copy_rows(stg + c * L::HALF, c);
          release();
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == L::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = umma_idesc_bf16(128, 16, false);
      constexpr uint32_t idO = umma_idesc_bf16_amn(128, 16);
      int slot = 0;
      uint32_t phase = 0;
      int pg = 0;                                     // P^T tiles consumed so far
      bool ok = true, any = false;
      // descriptors of stage 0 and P^T slot 0, built once (K: K-major; V: MN-major,
      // 16 KB between 64-dim blocks); the others are a start-address offset away
      const uint64_t dring0 = umma_desc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t dvring0 = umma_desc_sw128(smem_u32(ring), 16384, 1024);
      const uint64_t dpt0 = umma_desc_sw128(smem_u32(sP), 16, 1024);
      for (int st = 0; st <= R && ok; ++st) {
        if (st < R) {
          // S^T_t = K_t Q^T of row st into S buffer st & 1, one stage (128 dims) at a time
          // descriptors advance by adding (byte offset >> 4) to the start-address field
          const uint64_t dQ = umma_desc_sw128(smem_u32(sQ + (st & 1) * L::Q_BYTES), 16, 1024);
          const uint32_t sb = tmem + (st & 1) * L::SBUF;
          for (int t = 0; t < nT && ok; ++t) {
            if (!mbar_wait(&full[slot], phase, ctx)) { ok = false; break; }
            fence_proxy_async_smem();                // cp.async (generic) data -> tensor-core reads
            tc_fence_after();
            const uint64_t dK = dring0 + (uint64_t)(slot * (L::STAGE >> 4));
#pragma unroll
            for (int c = 0; c < L::HALVES; ++c)
#pragma unroll
              for (int k = 0; k < 8; ++k) {           // 8 steps of 16 dims per half
                const uint64_t ad = dK + (uint64_t)((c * L::HALF + (k >> 2) * 16384 + (k & 3) * 32) >> 4);
                const uint64_t bd = dQ + (uint64_t)((c * 4096 + (k >> 2) * 2048 + (k & 3) * 32) >> 4);
                umma_bf16(sb + 16 * t, ad, bd, idS, (c | k) != 0 ? 1u : 0u);
              }
            any = true;
            umma_commit(&empty[slot]);
            if (++slot == L::NSTG) { slot = 0; phase ^= 1; }
          }
          if (!ok) break;
          umma_commit(&s_full[st & 1]);
        }
        if (st >= 1) {
          // O^T[half c] += V_t^T P_t^T of row st-1 over each tile's 128 keys
          for (int t = 0; t < nT && ok; ++t, ++pg) {
            const int ps = pg % L::NPS;
            if (!mbar_wait(&p_full[ps], (uint32_t)((pg / L::NPS) & 1), ctx)) { ok = false; break; }
            tc_fence_after();
            const uint64_t dP = dpt0 + (uint64_t)(ps * (L::P_TILE >> 4));
            if (!mbar_wait(&full[slot], phase, ctx)) { ok = false; break; }
            fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t dV = dvring0 + (uint64_t)(slot * (L::STAGE >> 4));
#pragma unroll
            for (int c = 0; c < L::HALVES; ++c)
#pragma unroll
              for (int k = 0; k < 8; ++k) {           // 8 steps of 16 keys per half
                const uint64_t ad = dV + (uint64_t)((c * L::HALF + k * 2048) >> 4);
                const uint64_t bd = dP + (uint64_t)(((k >> 2) * 2048 + (k & 3) * 32) >> 4);
                umma_bf16(tmem + L::OCOL + 16 * c, ad, bd, idO, (t | k) != 0 ? 1u : 0u);
              }
            umma_commit(&empty[slot]);
            if (++slot == L::NSTG) { slot = 0; phase ^= 1; }
            umma_commit(&p_empty[ps]);
          }
          if (!ok) break;
          umma_commit(o_full);
        }
      }
      if (any) {
        umma_commit(mma_done);
        mbar_drain(mma_done, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp;                              // TMEM lanes 32*q4 .. 32*q4 + 31
    const int kl = 32 * q4 + lane;                    // key of every tile / dim of every half
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    const float c = p.scale_log2;
    bool ok = true;
    int pg = 0;                                        // P^T tiles written so far
    // the output of row r (O^T in TMEM -> bf16 O; a thread is one dim)
    auto epilogue = [&](int r) -> bool {
      if (!bar_and(1, 128, mbar_wait(o_full, r & 1, ctx))) return false;
      tc_fence_after();
      const int64_t row = blockIdx.x + (int64_t)r * gridDim.x;
      const float* li = linv + (r & 1) * 16;
      for (int hv = 0; hv < L::HALVES; ++hv) {
        float o[16];
        tmem_ld16(lane_base + L::OCOL + 16 * hv, o);
        tmem_wait_ld();
        __nv_bfloat16* out = p.O + row * p.H * D + hv * 128 + kl;
#pragma unroll
        for (int h = 0; h < 16; ++h)
          if (h < p.H) out[h * D] = __float2bfloat16_rn(o[h] * li[h]);
      }
      tc_fence_before();
      return true;
    };
    for (int r = 0; r < R && ok; ++r) {
      const int64_t row = blockIdx.x + (int64_t)r * gridDim.x;
      const uint32_t sbuf = lane_base + (r & 1) * L::SBUF;
      // which of this thread's keys (one per tile) are real: bit t
      uint32_t vmask = 0;
      {
        const int32_t* irow = p.idx + row * p.n_idx;
        for (int t = 0; t < nT; ++t) {
          const int sl = t * 128 + kl;
          if (sl < p.n_idx) {
            const int32_t v = irow[sl];
            if (v >= 0 && v < p.kv_len) vmask |= 1u << t;
          }
        }
      }
      if (!bar_and(1, 128, mbar_wait(&s_full[r & 1], (r >> 1) & 1, ctx))) { ok = false; break; }
      tc_fence_after();
      // pass 1: per-head maximum of the raw scores over the row's valid keys
      float m[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) m[h] = -INFINITY;
      for (int t = 0; t < nT; ++t) {
        float v[16];
        tmem_ld16(sbuf + 16 * t, v);
        tmem_wait_ld();
        if ((vmask >> t) & 1u) {
#pragma unroll
          for (int h = 0; h < 16; ++h) m[h] = fmaxf(m[h], v[h]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int h = 0; h < 16; ++h) m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], o));
      if (lane < 16) {
        float mv = m[0];
#pragma unroll
        for (int h = 1; h < 16; ++h) mv = lane == h ? m[h] : mv;
        red_m[q4 * 16 + lane] = mv;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      float mc[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const float mh = fmaxf(fmaxf(red_m[h], red_m[16 + h]), fmaxf(red_m[32 + h], red_m[48 + h]));
        mc[h] = mh == -INFINITY ? 0.f : mh * c;
      }
      // the previous row's O^T must be read before this row's products start
      if (r >= 1 && !epilogue(r - 1)) { ok = false; break; }
      // pass 2: p = 2^(s*c - m*c), the sums, and P^T (K-major, 128-byte
      // swizzle) tile by tile through the P ring
      float l[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) l[h] = 0.f;
      for (int t = 0; t < nT; ++t, ++pg) {
        const int ps = pg % L::NPS;
        if (!bar_and(1, 128, mbar_wait(&p_empty[ps], (uint32_t)(((pg / L::NPS) & 1) ^ 1), ctx))) { ok = false; break; }
        tc_fence_after();
        float v[16];
        tmem_ld16(sbuf + 16 * t, v);
        tmem_wait_ld();
        const bool valid = (vmask >> t) & 1u;
        uint8_t* pt = sP + ps * L::P_TILE + (kl >> 6) * 2048;
        const int u8 = (kl & 63) >> 3, e = kl & 7;
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const float pv = valid ? fast_exp2(fmaf(v[h], c, -mc[h])) : 0.f;
          l[h] += pv;
          *reinterpret_cast<__nv_bfloat16*>(pt + h * 128 + ((u8 ^ (h & 7)) << 4) + e * 2) = __float2bfloat16_rn(pv);
        }
        fence_proxy_async_smem();                      // P^T visible to the tensor cores
        tc_fence_before();
        mbar_arrive(&p_full[ps]);
      }
      if (!ok) break;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int h = 0; h < 16; ++h) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
      if (lane < 16) {
        float lv = l[0];
#pragma unroll
        for (int h = 1; h < 16; ++h) lv = lane == h ? l[h] : lv;
        red_l[q4 * 16 + lane] = lv;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (threadIdx.x < 16) {
        const int h = threadIdx.x;
        const float ls = red_l[h] + red_l[16 + h] + red_l[32 + h] + red_l[48 + h];
        linv[(r & 1) * 16 + h] = ls > 0.f ? 1.f / ls : 0.f;
      }
    }
    if (ok && R > 0) epilogue(R - 1);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == L::MMA_WARP) tmem_dealloc(tmem, 512);
}

}  // namespace hs2
