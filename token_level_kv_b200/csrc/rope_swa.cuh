// Partial rotary position embedding for the self-decoder's sliding-window
// attention layers.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary): the self-decoder mixes full attention with sliding
// window attention (each query attends only to the most recent tokens); the
// SWA layers use 64-dim partial RoPE while the full and sparse layers use
// NoPE; MQA (one KV head).  Readings (the pages fix none of them): pairs are
// (i, i + R/2) for i < R/2 on the first R = rope_dims dims (rotate-half); the
// angle of pair i at absolute position p is p * base^(-2i/R); the other dims
// pass through.
//
// rope_table_kernel computes cos/sin of every (position, pair) angle in fp64
// (the angle p * base^(-2i/R) reaches 2.6e5 rad at 262k tokens, far past
// what an fp32 angle holds to 1e-7) and stores them as fp32 pairs;
// rope_rows_kernel rotates bf16 rows in fp32 (one fused multiply-add per
// output) and rounds them to bf16 for the attention kernel, which then runs
// fa_fwd_kernel with its sliding-window key range.
#pragma once
#include "common.cuh"

namespace hs2 {

// cs[pos * half + i] = (cos, sin) of pos * base^(-2i/R), pos < n_pos, i < half.
__global__ void rope_table_kernel(float2* cs, int64_t n_pos, int half, double base) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_pos * half) return;
  const int64_t pos = t / half;
  const int i = (int)(t - pos * half);
  const double inv = pow(base, -2.0 * (double)i / (double)(2 * half));
  double s, c;
  sincos((double)pos * inv, &s, &c);
  cs[t] = make_float2((float)c, (float)s);
}

// out row r = in row r rotated at position pos0 + r / per_pos (Q rows: one
// position per H heads; K rows: per_pos = 1).  One warp per row: lane i < half
// rotates pair i; the dims from R on are copied in 16-byte pieces.
template <int D>
__global__ void __launch_bounds__(256) rope_rows_kernel(const __nv_bfloat16* in, __nv_bfloat16* out, int64_t rows,
                                                        int64_t pos0, int per_pos, const float2* cs, int half) {
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int64_t pos = pos0 + r / per_pos;
  const __nv_bfloat16* src = in + r * D;
  __nv_bfloat16* dst = out + r * D;
  if (lane < half) {
    const float2 t = cs[pos * half + lane];
    const float x1 = __bfloat162float(src[lane]);
    const float x2 = __bfloat162float(src[lane + half]);
    dst[lane] = __float2bfloat16_rn(fmaf(x1, t.x, -x2 * t.y));
    dst[lane + half] = __float2bfloat16_rn(fmaf(x1, t.y, x2 * t.x));
  }
  const int R = 2 * half;
  for (int u = lane; u < (D - R) / 8; u += 32)
    reinterpret_cast<uint4*>(dst + R)[u] = reinterpret_cast<const uint4*>(src + R)[u];
}

}  // namespace hs2
