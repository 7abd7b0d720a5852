// KV Bridging re-projection (row a1): K = H Wk^T and V = H Wv^T for one
// cross-decoder full-attention layer, with an optional FP8 E4M3 epilogue.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Bridging paragraph -- the cross-decoder full
// layer re-projects the self-decoder full layer's hidden state through its own
// K/V projections; results table "KV @1M (FP8)" -- the cache is FP8.
//
// Design (sm_100a): persistent CTAs, one per SM.  A tile is 128 rows x 256
// outputs (all of K or all of V for those rows), so the FP8 row scale
// (amax/448) is a thread-local reduction in the epilogue: TMEM lane = row.
//   warp 0     : TMA producer, 4-stage ring of {A 128x64, B 256x64} bf16
//                (128-byte swizzle, K-major)
//   warp 1     : TMEM allocator + single-thread tcgen05.mma issuer
//                (M=128, N=256, K=16 per instruction), two TMEM accumulators
//                of 256 columns so the epilogue of tile t overlaps tile t+1
//   warps 2..5 : epilogue, one row per thread: tcgen05.ld -> bf16, or
//                amax pass + RNE satfinite E4M3 pass
// Consecutive tiles are (rows m, K) then (rows m, V), so the second read of
// the hidden-state rows hits L2.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int BG_BM = 128;
constexpr int BG_BN = 256;
constexpr int BG_BK = 64;
constexpr int BG_STAGES = 4;
constexpr int BG_A_BYTES = BG_BM * BG_BK * 2;          // 16 KB
constexpr int BG_B_BYTES = BG_BN * BG_BK * 2;          // 32 KB
constexpr int BG_STAGE_BYTES = BG_A_BYTES + BG_B_BYTES;
constexpr int BG_THREADS = 192;
constexpr size_t BG_SMEM = (size_t)BG_STAGES * BG_STAGE_BYTES + 1024 /*align*/ + 256;

struct BridgeParams {
  int64_t rows;
  int kdim;          // hidden size, multiple of 64
  int out_fp8;
  void* K_out;
  void* V_out;
  float* k_scale;
  float* v_scale;
  int num_tiles;     // 2 * ceil(rows / 128)
};

__global__ void __launch_bounds__(BG_THREADS, 1)
bridge_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmWk,
                   const __grid_constant__ CUtensorMap tmWv, BridgeParams p, DevCtx ctx) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BG_STAGES * BG_STAGE_BYTES);
  uint64_t* empty = full + BG_STAGES;
  uint64_t* tfull = empty + BG_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = p.kdim / BG_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < BG_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmWk);
    tma_prefetch_desc(&tmWv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[BG_STAGES];
      for (int s = 0; s < BG_STAGES; ++s) issued[s] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int m = tile >> 1;
        const CUtensorMap* tb = (tile & 1) ? &tmWv : &tmWk;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, ctx)) { ok = false; break; }
          uint8_t* sa = smem + stage * BG_STAGE_BYTES;
          mbar_expect_tx(&full[stage], BG_STAGE_BYTES);
          tma_load_2d(sa, &tmA, &full[stage], kb * BG_BK, m * BG_BM);
          tma_load_2d(sa + BG_A_BYTES, tb, &full[stage], kb * BG_BK, 0);
          issued[stage] = (int)phase;
          if (++stage == BG_STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // every issued copy lands before the CTA may exit
      for (int s = 0; s < BG_STAGES; ++s)
        if (issued[s] >= 0) mbar_drain(&full[s], (uint32_t)issued[s]);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(BG_BM, BG_BN, false);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, any = false;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, ctx)) break;
        tc_fence_after();
        const uint32_t dt = tmem_base + (uint32_t)(acc * BG_BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, ctx)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * BG_STAGE_BYTES);
          const uint32_t sb = sa + BG_A_BYTES;
#pragma unroll
          for (int k = 0; k < BG_BK / 16; ++k) {
            const uint64_t ad = umma_desc_sw128(sa + k * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(sb + k * 32, 16, 1024);
            umma_bf16(dt, ad, bd, idesc, (kb | k) != 0);
          }
          any = true;
          umma_commit(&empty[stage]);
          if (++stage == BG_STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (any) {
        umma_commit(mma_done);
        mbar_drain(mma_done, 0);
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;                 // TMEM lanes 32*quarter ..
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, ctx))) break;
      tc_fence_after();
      const int m = tile >> 1;
      const bool is_v = tile & 1;
      const int64_t r = (int64_t)m * BG_BM + row_in_tile;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BG_BN);
      float v[32];
      if (p.out_fp8) {
        float amax = 0.f;
#pragma unroll 1
        for (int c = 0; c < BG_BN / 32; ++c) {
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
        const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        uint8_t* out = reinterpret_cast<uint8_t*>(is_v ? p.V_out : p.K_out) + r * BG_BN;
#pragma unroll 1
        for (int c = 0; c < BG_BN / 32; ++c) {
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint16_t lo = f32x2_to_e4m3x2(__fdiv_rn(v[4 * i], scale), __fdiv_rn(v[4 * i + 1], scale));
            const uint16_t hi = f32x2_to_e4m3x2(__fdiv_rn(v[4 * i + 2], scale), __fdiv_rn(v[4 * i + 3], scale));
            w[i] = (uint32_t)lo | ((uint32_t)hi << 16);
          }
          if (r < p.rows) {
            uint4* o = reinterpret_cast<uint4*>(out + c * 32);
            o[0] = make_uint4(w[0], w[1], w[2], w[3]);
            o[1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
        if (r < p.rows) (is_v ? p.v_scale : p.k_scale)[r] = scale;
      } else {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(is_v ? p.V_out : p.K_out) + r * BG_BN;
#pragma unroll 1
        for (int c = 0; c < BG_BN / 32; ++c) {
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
          if (r < p.rows) {
            uint4* o = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

}  // namespace hs2
