// Decode-step KV Bridging: the new token of each sequence is re-projected
// into this cross-decoder layer's K/V and appended to its FP8 cache.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Bridging paragraph -- a cross-decoder full
// layer's K/V are its own projections of the self-decoder full layer's hidden
// state; results table "KV @1M (FP8)" -- the cache is FP8.  The arXiv
// abstract: every cross-decoder KV cache is constructed from self-decoder
// hidden states.  Reading: during decode the self-decoder produces one hidden
// row per sequence and step, so each cache grows by one bridged row per
// sequence and step.
//
// Per sequence b and output (K or V):  x = hidden[b] W^T  (fp32), then
// scale = amax(x)/448 (1 for an all-zero row) and code = E4M3_RNE_satfinite(x/scale)
// written at row pos[b] of sequence b.  The same arithmetic as the
// bridging GEMM's FP8 epilogue, at matrix-vector size.
//
// Design: a GEMV is bound by reading W (2 x 256 x hidden_dim bf16 = 2 MB per
// layer at hidden_dim 2048), so every thread streams 16-byte pieces of W rows
// and no tensor cores are involved.  A thread-block cluster of 4 CTAs serves
// one (sequence, K or V): each CTA computes 64 of the 256 outputs (8 per
// warp; the 32 lanes split hidden_dim and meet in a shuffle tree), and the
// row's amax is the max of the 4 CTAs' maxima read through distributed
// shared memory -- one kernel, no scratch.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

namespace hs2 {

constexpr int BA_CLUSTER = 4;                    // CTAs per (sequence, K or V)
constexpr int BA_THREADS = 256;                  // 8 warps
constexpr int BA_OUT = 256 / BA_CLUSTER;         // outputs per CTA (d = 256)
constexpr int BA_PER_WARP = BA_OUT / (BA_THREADS / 32);

struct AppendParams {
  const __nv_bfloat16* hidden;   // [batch, kdim]
  const __nv_bfloat16* Wk;       // [256, kdim]
  const __nv_bfloat16* Wv;
  int kdim;                      // hidden_dim, a multiple of 256
  uint8_t* Kc;                   // [batch, stride, 256] E4M3 codes
  uint8_t* Vc;
  float* ks;                     // [batch, stride]
  float* vs;
  int64_t stride;                // kv_stride_tokens
  const int32_t* pos;            // [batch] row written in each sequence
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// grid (BA_CLUSTER, 2, batch): x = rank in the cluster, y = K (0) or V (1).
__global__ void __cluster_dims__(BA_CLUSTER, 1, 1) __launch_bounds__(BA_THREADS)
bridge_append_kernel(AppendParams p, DevCtx ctx) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int r = (int)cluster.block_rank();
  const int is_v = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16* W = is_v ? p.Wv : p.Wk;
  __shared__ float outv[BA_OUT];
  __shared__ float cmax;                         // this CTA's max |x|, read by the cluster

  // lane l holds hidden elements 256 j + 8 l .. 256 j + 8 l + 7 of piece j
  const int c0 = r * BA_OUT + warp * BA_PER_WARP;
  const uint4* h4 = reinterpret_cast<const uint4*>(p.hidden + b * p.kdim);
  float acc[BA_PER_WARP];
#pragma unroll
  for (int i = 0; i < BA_PER_WARP; ++i) acc[i] = 0.f;
  const int nj = p.kdim / 256;
  for (int j = 0; j < nj; ++j) {
    float hf[8];
    bf16x8_to_f32(h4[j * 32 + lane], hf);
    uint4 wv[BA_PER_WARP];
#pragma unroll
    for (int i = 0; i < BA_PER_WARP; ++i)
      wv[i] = reinterpret_cast<const uint4*>(W + (int64_t)(c0 + i) * p.kdim)[j * 32 + lane];
#pragma unroll
    for (int i = 0; i < BA_PER_WARP; ++i) {
      float wf[8];
      bf16x8_to_f32(wv[i], wf);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[i] = fmaf(hf[e], wf[e], acc[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < BA_PER_WARP; ++i)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < BA_PER_WARP; ++i) outv[warp * BA_PER_WARP + i] = acc[i];
  __syncthreads();
  if (warp == 0) {
    float m = fmaxf(fabsf(outv[lane]), fabsf(outv[lane + 32]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) cmax = m;
  }
  cluster.sync();
  float amax = 0.f;
#pragma unroll
  for (int q = 0; q < BA_CLUSTER; ++q) amax = fmaxf(amax, *cluster.map_shared_rank(&cmax, q));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const int32_t ps = p.pos[b];
  if (ps < 0 || ps >= p.stride) {
    if (threadIdx.x == 0 && r == 0 && is_v == 0) report(ctx, ST_DEVICE_CHECK);
  } else {
    const int64_t row = b * p.stride + ps;
    if (threadIdx.x < BA_OUT / 2) {
      const int c = 2 * threadIdx.x;
      const uint16_t code2 = f32x2_to_e4m3x2(__fdiv_rn(outv[c], scale), __fdiv_rn(outv[c + 1], scale));
      reinterpret_cast<uint16_t*>((is_v ? p.Vc : p.Kc) + row * 256 + r * BA_OUT)[threadIdx.x] = code2;
    }
    if (r == 0 && threadIdx.x == 0) (is_v ? p.vs : p.ks)[row] = scale;
  }
  cluster.sync();                                // peers read cmax until here
}

}  // namespace hs2
