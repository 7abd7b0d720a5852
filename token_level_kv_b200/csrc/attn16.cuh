// Attention of one token's 16 query heads over a list of keys of the single
// KV head (rows a6, a7, a8): the shape the sparse layers and the decode step
// have.  The 16 heads are the M=16 rows of mma.sync m16n8k16 (bf16 in, fp32
// accumulate); keys stream through a per-warp cp.async ring.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph -- the sparse layers gather only
// the selected tokens (window + top-k) of the full layer's KV; MQA, NoPE.
// Results table "KV @1M (FP8)" -- decode reads an FP8 cache.
//
// Modes (template flags):
//   RANGE=false : keys are idx[item, slot] (gather; -1 = empty slot)
//   RANGE=true  : keys are a contiguous range (decode full attention; also
//                 writes every scaled logit for the selection pass)
//   FP8=true    : K/V are E4M3 codes with per-token fp32 scales; each chunk is
//                 widened to bf16 in shared memory (exact), the key scale is
//                 applied to the logit and the value scale folded into P.
// A CTA (4 warps) owns one item (a query row or a sequence) and one split of
// its keys; warps take 16-key chunks round-robin and are merged through shared
// memory.  With several splits the (m, l, O) partials go to the workspace and
// attn16_combine_kernel merges them.
#pragma once
#include "common.cuh"

namespace hs2 {

constexpr int A16_WARPS = 4;
constexpr int A16_CH = 16;

struct Attn16Params {
  const __nv_bfloat16* Q;   // [items, H, D]
  const void* K;            // bf16 [kv rows, D] or uint8 [B, kv_stride, D]
  const void* V;
  const float* ks;          // [B, kv_stride] (FP8)
  const float* vs;
  const int32_t* idx;       // [items, n_idx] (gather)
  int n_idx;
  int64_t kv_len;           // valid keys per sequence
  int64_t kv_stride;        // tokens between sequences (0: one shared KV)
  int H;
  float scale_log2;         // softmax_scale * log2(e)
  int splits;               // CTAs per item
  int slots_per_split;      // key slots (gather) or keys (range) per CTA
  int final_out;            // 1: normalised O; 0: (m, l, O) partials
  __nv_bfloat16* O;         // [items, H, D]   (final_out)
  float* part;              // [items, splits, 32 + 16*D]   (partials)
  float* logits;            // [items, H, logit_ld] (RANGE)
  int64_t logit_ld;
};

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
               ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;"
               ::"r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// bf16 row of D elements, 16-byte unit u stored at unit u ^ (row & 7).
template <int D>
__device__ __forceinline__ uint32_t swz_off(int row, int unit) {
  return (uint32_t)(row * D * 2 + ((unit ^ (row & 7)) << 4));
}

template <int D, bool FP8>
struct A16Layout {
  static constexpr int NST = FP8 ? 4 : 2;                 // ring stages per warp
  static constexpr int RAW_ROW = FP8 ? D : 2 * D;         // bytes per key row as stored
  static constexpr int RAW_KV = A16_CH * RAW_ROW;         // K (or V) bytes per chunk
  static constexpr int STAGE = 2 * RAW_KV + 2 * A16_CH * 4 /*scales*/ + A16_CH * 4 /*pos*/;
  static constexpr int CONV = FP8 ? 2 * A16_CH * 2 * D : 0;
  static constexpr int WARP = ((NST * STAGE + CONV) + 127) & ~127;
  static constexpr int Q_BYTES = 16 * D * 2;
  static constexpr int COMBINE = A16_WARPS * (16 * D + 32) * 4;
  static constexpr int MAIN = Q_BYTES + A16_WARPS * WARP;
  static constexpr int SMEM = (MAIN > Q_BYTES + COMBINE ? MAIN : Q_BYTES + COMBINE) + 128;
};

template <int D, bool FP8, bool RANGE>
__global__ void __launch_bounds__(128)
attn16_kernel(Attn16Params p, DevCtx ctx) {
  using L = A16Layout<D, FP8>;
  extern __shared__ __align__(128) uint8_t smem_a16[];
  uint8_t* smem = smem_a16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int item = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;

  // ---- Q (16 rows, rows >= H are zero), swizzled bf16
  uint8_t* sQ = smem;
  {
    const __nv_bfloat16* q = p.Q + (int64_t)item * p.H * D;
    for (int u = threadIdx.x; u < 16 * D / 8; u += blockDim.x) {
      const int row = u / (D / 8), un = u % (D / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < p.H) v = *reinterpret_cast<const uint4*>(q + row * D + un * 8);
      *reinterpret_cast<uint4*>(sQ + swz_off<D>(row, un)) = v;
    }
  }

  int64_t slot_begin = (int64_t)split * p.slots_per_split;
  int64_t slot_end = slot_begin + p.slots_per_split;
  const int64_t total = RANGE ? p.kv_len : (int64_t)p.n_idx;
  if (slot_end > total) slot_end = total;
  const int n_chunks = slot_end > slot_begin ? (int)((slot_end - slot_begin + A16_CH - 1) / A16_CH) : 0;
  const int my_n = warp < n_chunks ? (n_chunks - warp + A16_WARPS - 1) / A16_WARPS : 0;

  const int64_t seq_off = (int64_t)item * p.kv_stride;   // 0 for the shared prefill KV
  const uint8_t* Kb = reinterpret_cast<const uint8_t*>(p.K);
  const uint8_t* Vb = reinterpret_cast<const uint8_t*>(p.V);
  uint8_t* wbase = smem + L::Q_BYTES + warp * L::WARP;

  auto stage_ptr = [&](int s) { return wbase + s * L::STAGE; };

  auto issue = [&](int s, int chunk) {
    uint8_t* st = stage_ptr(s);
    int32_t* spos = reinterpret_cast<int32_t*>(st + 2 * L::RAW_KV + 2 * A16_CH * 4);
    const int64_t sl = slot_begin + (int64_t)chunk * A16_CH + lane;
    int32_t pos = -1;
    if (lane < A16_CH && sl < slot_end) {
      if (RANGE) {
        pos = (int32_t)sl;
      } else {
        pos = p.idx[(int64_t)item * p.n_idx + sl];
        if (pos < -1 || pos >= p.kv_len) {
          report(ctx, ST_DEVICE_CHECK);
          pos = -1;
        }
      }
    }
    if (lane < A16_CH) spos[lane] = pos;
    constexpr int UPR = L::RAW_ROW / 16;                   // 16-byte units per row
#pragma unroll 4
    for (int seg = lane; seg < A16_CH * UPR; seg += 32) {
      const int i = seg / UPR, u = seg % UPR;
      const int32_t pi = __shfl_sync(0xffffffffu, pos, i);
      const int64_t row = seq_off + (pi < 0 ? 0 : pi);
      const uint32_t doff = FP8 ? (uint32_t)(i * L::RAW_ROW + u * 16) : swz_off<D>(i, u);
      cp_async16(smem_u32(st + doff), Kb + row * L::RAW_ROW + u * 16, pi >= 0);
      cp_async16(smem_u32(st + L::RAW_KV + doff), Vb + row * L::RAW_ROW + u * 16, pi >= 0);
    }
    if (FP8 && lane < A16_CH) {
      float* sks = reinterpret_cast<float*>(st + 2 * L::RAW_KV);
      const int64_t row = seq_off + (pos < 0 ? 0 : pos);
      cp_async4(smem_u32(sks + lane), p.ks + row, pos >= 0);
      cp_async4(smem_u32(sks + A16_CH + lane), p.vs + row, pos >= 0);
    }
  };

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  __syncthreads();   // sQ ready

#pragma unroll
  for (int s = 0; s < L::NST - 1; ++s) {
    if (s < my_n) issue(s, warp + A16_WARPS * s);
    cp_async_commit();
  }

  for (int it = 0; it < my_n; ++it) {
    {
      const int nxt = it + L::NST - 1;
      if (nxt < my_n) issue(nxt % L::NST, warp + A16_WARPS * nxt);
      cp_async_commit();
    }
    cp_async_wait<L::NST - 1>();
    __syncwarp();
    uint8_t* st = stage_ptr(it % L::NST);
    const int32_t* spos = reinterpret_cast<const int32_t*>(st + 2 * L::RAW_KV + 2 * A16_CH * 4);
    const float* sks = reinterpret_cast<const float*>(st + 2 * L::RAW_KV);
    uint8_t* kst = st;
    uint8_t* vst = st + L::RAW_KV;
    if (FP8) {
      // widen the chunk to bf16 (exact), swizzled like the bf16 path
      uint8_t* conv = wbase + L::NST * L::STAGE;
      constexpr int UPR8 = D / 8;                          // 8-byte fp8 groups per row
      for (int e = lane; e < 2 * A16_CH * UPR8; e += 32) {
        const int which = e / (A16_CH * UPR8);
        const int r = (e / UPR8) % A16_CH, u = e % UPR8;
        const uint2 raw = *reinterpret_cast<const uint2*>(st + which * L::RAW_KV + r * D + u * 8);
        uint4 w;
        w.x = e4m3x2_to_bf16x2((uint16_t)(raw.x & 0xffff));
        w.y = e4m3x2_to_bf16x2((uint16_t)(raw.x >> 16));
        w.z = e4m3x2_to_bf16x2((uint16_t)(raw.y & 0xffff));
        w.w = e4m3x2_to_bf16x2((uint16_t)(raw.y >> 16));
        *reinterpret_cast<uint4*>(conv + which * (A16_CH * 2 * D) + swz_off<D>(r, u)) = w;
      }
      __syncwarp();
      kst = conv;
      vst = conv + A16_CH * 2 * D;
    }

    // ---- S = Q K^T  (16 heads x 16 keys)
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const uint32_t qa = smem_u32(sQ), ka = smem_u32(kst), va = smem_u32(vst);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4], b[4];
      {
        const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int unit = kk * 2 + (lane >> 4);
        ldsm_x4(a, qa + swz_off<D>(row, unit));
      }
      {
        const int key = (lane & 7) + (lane >> 4) * 8;
        const int unit = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(b, ka + swz_off<D>(key, unit));
      }
      mma_bf16_16816(s[0], a, b[0], b[1]);
      mma_bf16_16816(s[1], a, b[2], b[3]);
    }

    // ---- scale, mask, logits, online softmax
    float x[2][4];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = nt * 8 + 2 * t + (e & 1);
        const int32_t pos = spos[key];
        float f = p.scale_log2;
        if (FP8) f *= sks[key];
        float v = s[nt][e] * f;
        if (pos < 0) v = -INFINITY;
        x[nt][e] = v;
        if (e < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
      }
    }
    if (RANGE) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int key = nt * 8 + 2 * t;
        const int32_t pos = spos[key];
        if (pos >= 0) {   // pairs of keys are both valid or the second is past kv_len
          const bool two = spos[key + 1] >= 0;
          float* r0 = p.logits + ((int64_t)item * p.H + g) * p.logit_ld + pos;
          if (g < p.H) {
            if (two) *reinterpret_cast<float2*>(r0) = make_float2(x[nt][0], x[nt][1]);
            else r0[0] = x[nt][0];
          }
          if (g + 8 < p.H) {
            float* r1 = r0 + 8 * p.logit_ld;
            if (two) *reinterpret_cast<float2*>(r1) = make_float2(x[nt][2], x[nt][3]);
            else r1[0] = x[nt][2];
          }
        }
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - mn0);
    const float al1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
    const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
    float pr[2][4];
    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pe = fast_exp2(x[nt][e] - (e < 2 ? mu0 : mu1));
        if (e < 2) ls0 += pe; else ls1 += pe;
        float pv = pe;
        if (FP8) pv *= sks[A16_CH + nt * 8 + 2 * t + (e & 1)];
        pr[nt][e] = pv;
      }
    }
    l0 = l0 * al0 + ls0;
    l1 = l1 * al1 + ls1;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o[i][0] *= al0; o[i][1] *= al0;
      o[i][2] *= al1; o[i][3] *= al1;
    }
    uint32_t ap[4];
    ap[0] = pack_bf16x2(pr[0][0], pr[0][1]);
    ap[1] = pack_bf16x2(pr[0][2], pr[0][3]);
    ap[2] = pack_bf16x2(pr[1][0], pr[1][1]);
    ap[3] = pack_bf16x2(pr[1][2], pr[1][3]);

    // ---- O += P V
#pragma unroll
    for (int nd = 0; nd < D / 16; ++nd) {
      uint32_t b[4];
      const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int unit = nd * 2 + (lane >> 4);
      ldsm_x4_t(b, va + swz_off<D>(key, unit));
      mma_bf16_16816(o[2 * nd], ap, b[0], b[1]);
      mma_bf16_16816(o[2 * nd + 1], ap, b[2], b[3]);
    }
    __syncwarp();
  }
  cp_async_wait<0>();

  // ---- merge the 4 warps
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();
  float* cmb = reinterpret_cast<float*>(smem + L::Q_BYTES);
  float* cm = cmb;                              // [4][16]
  float* cl = cmb + A16_WARPS * 16;             // [4][16]
  float* cO = cmb + A16_WARPS * 32;             // [4][16][D]
  if (t == 0) {
    cm[warp * 16 + g] = m0;
    cm[warp * 16 + g + 8] = m1;
    cl[warp * 16 + g] = l0;
    cl[warp * 16 + g + 8] = l1;
  }
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int col = i * 8 + 2 * t;
    *reinterpret_cast<float2*>(cO + (warp * 16 + g) * D + col) = make_float2(o[i][0], o[i][1]);
    *reinterpret_cast<float2*>(cO + (warp * 16 + g + 8) * D + col) = make_float2(o[i][2], o[i][3]);
  }
  __syncthreads();
  float* part = p.part + ((int64_t)item * p.splits + split) * (32 + 16 * D);
  for (int e = threadIdx.x; e < 16 * D; e += blockDim.x) {
    const int h = e / D, c = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < A16_WARPS; ++w) M = fmaxf(M, cm[w * 16 + h]);
    float Lsum = 0.f, Ov = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < A16_WARPS; ++w) {
        const float f = (cm[w * 16 + h] == -INFINITY) ? 0.f : fast_exp2(cm[w * 16 + h] - M);
        Lsum += cl[w * 16 + h] * f;
        Ov += cO[(w * 16 + h) * D + c] * f;
      }
    }
    if (p.final_out) {
      if (h < p.H) {
        const float r = Lsum > 0.f ? Ov / Lsum : 0.f;
        p.O[((int64_t)item * p.H + h) * D + c] = __float2bfloat16_rn(r);
      }
    } else {
      part[32 + h * D + c] = Ov;
      if (c == 0) {
        part[h] = M;
        part[16 + h] = Lsum;
      }
    }
  }
}

// Merge split partials: m = max m_s, l = sum l_s 2^(m_s-m), O = sum O_s 2^(m_s-m) / l.
// Also stores (m, l) per head (log2 units) for the selection pass.
template <int D>
__global__ void __launch_bounds__(256)
attn16_combine_kernel(const float* part, int splits, int H, __nv_bfloat16* O, float* ml) {
  const int item = blockIdx.x;
  const float* base = part + (int64_t)item * splits * (32 + 16 * D);
  __shared__ float sM[16], sL[16];
  if (threadIdx.x < 16) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, base[s * (32 + 16 * D) + h]);
    float Lsum = 0.f;
    if (M != -INFINITY)
      for (int s = 0; s < splits; ++s) {
        const float ms = base[s * (32 + 16 * D) + h];
        if (ms != -INFINITY) Lsum += base[s * (32 + 16 * D) + 16 + h] * fast_exp2(ms - M);
      }
    sM[h] = M;
    sL[h] = Lsum;
    if (ml != nullptr && h < H) {
      ml[((int64_t)item * H + h) * 2] = M;
      ml[((int64_t)item * H + h) * 2 + 1] = Lsum;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < H * D; e += blockDim.x) {
    const int h = e / D, c = e % D;
    const float M = sM[h];
    float acc = 0.f;
    if (M != -INFINITY)
      for (int s = 0; s < splits; ++s) {
        const float ms = base[s * (32 + 16 * D) + h];
        if (ms != -INFINITY) acc += base[s * (32 + 16 * D) + 32 + h * D + c] * fast_exp2(ms - M);
      }
    O[((int64_t)item * H + h) * D + c] = __float2bfloat16_rn(sL[h] > 0.f ? acc / sL[h] : 0.f);
  }
}

// Decode selection score: sigma[b, j] = sum_h 2^(x_hj - m_h) / l_h for the
// candidates j < n_cand (x: scaled logits in log2 units).
__global__ void __launch_bounds__(256)
decode_sigma_kernel(const float* logits, int64_t logit_ld, const float* ml, int H,
                    int64_t n_cand, float* sigma, int64_t sigma_ld) {
  const int b = blockIdx.y;
  __shared__ float sM[16], sI[16];
  if (threadIdx.x < H) {
    sM[threadIdx.x] = ml[((int64_t)b * H + threadIdx.x) * 2];
    const float l = ml[((int64_t)b * H + threadIdx.x) * 2 + 1];
    sI[threadIdx.x] = 1.f / l;
  }
  __syncthreads();
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n_cand) return;
  float acc = 0.f;
  for (int h = 0; h < H; ++h)
    acc += fast_exp2(logits[((int64_t)b * H + h) * logit_ld + j] - sM[h]) * sI[h];
  sigma[(int64_t)b * sigma_ld + j] = acc;
}

}  // namespace hs2
