// Decode attention over the FP8 E4M3 cache (rows a7, a8): one new query of
// 16 (or 8) heads per sequence against a range of cached keys (the full
// layer, a7) or against the selected keys idx[b, :] (a sparse layer, a8).
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph (the sparse layers gather the
// selected tokens of the full layer's KV) and results table "KV @1M (FP8)".
// Key j of sequence b is E4M3(K[b,j,:]) * k_scale[b,j], likewise V.
//
// Design (sm_100a), HBM-bound: everything serves bytes in flight.
//   * 4 warps per CTA; each warp streams 16-key chunks through its own
//     4-stage cp.async ring (3 chunks in flight), raw FP8 rows at a padded
//     stride so the fragment loads below are bank-conflict free.
//   * The products run on mma.sync m16n8k16 in f16 with fp32 accumulation
//     (the heads are M): every E4M3 code is an f16, so one cvt.rn.f16x2.e4m3x2
//     widens two codes exactly.  Q enters in f16 after an exact power-of-two
//     prescale that puts its largest element in [2^14, 2^15) (f16 then holds
//     every bf16 element exactly except ones below 2^-28 of that maximum);
//     the prescale, the key scale and softmax_scale multiply the fp32 logit.
//     P holds p * v_scale in f16 (p <= 2^8), so dequantised values must stay
//     below the f16 maximum (|v| <= 65504), which real caches do.
//   * S = Q K^T traverses the head dimension in a fixed permutation shared by
//     Q and K (within each block of 16: thread t's k pairs {2t,2t+1} and
//     {2t+8,2t+9} are the dims 4t..4t+3), so a thread's K fragment is ONE
//     4-byte shared load of 4 consecutive codes; the dot products are
//     unchanged by the permutation.
//   * The CTA's index slice is read into shared memory once; each lane copies
//     half of one key row per chunk.
//   * O += P V reads its B fragments straight from the raw FP8 V rows:
//     ldmatrix.x4.trans on the codes viewed as 16-bit pairs hands thread
//     (g, t) the codes V[2t..2t+1][2g..2g+1]; two byte permutes regroup them
//     into key pairs of one dimension, and one cvt per pair widens them.  The
//     O columns of a fragment are thus dims c0 + 2n + parity, a fixed
//     permutation of d undone when the partial is written.
//   * 6 warps per CTA, each with a 3-stage ring.
//   * Online softmax in base 2 with a lazy rescale: the reference max moves
//     only when a row's max grows by more than 2^8.
//   * a7 (RANGE): the CTA owns one split of a sequence's keys, writes every
//     scaled logit (the selection pass needs them) and its (m, l, O) partial;
//     attn16_combine_kernel merges the splits.
//   * a8 (gather), batch large enough to fill the GPU: a thread-block cluster
//     of C <= 8 CTAs per sequence; the partials are merged through distributed
//     shared memory -- one kernel, no scratch.  Smaller batches use more
//     splits than a cluster holds and write partials (PARTIALS) for
//     attn16_combine_kernel.
#pragma once
#include <cooperative_groups.h>

#include "attn16.cuh"
#include "common.cuh"

namespace hs2 {

namespace cg = cooperative_groups;

template <int D>
struct DecLayout {
  static constexpr int NW = 6;                      // warps per CTA
  static constexpr int CH = 16;
  static constexpr int NST = 3;
  static constexpr int KROW = D + 16;               // padded raw K row
  static constexpr int VROW = D + 16;               // padded raw V row (conflict-free ldmatrix)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + CH * KROW;
  static constexpr int OFF_KS = OFF_V + CH * VROW;
  static constexpr int OFF_VS = OFF_KS + CH * 4;
  static constexpr int OFF_POS = OFF_VS + CH * 4;
  static constexpr int STAGE = OFF_POS + CH * 4;
  static constexpr int WARP = NST * STAGE;
  static constexpr int QROW = 2 * D + 16;           // padded bf16 Q row
  static constexpr int Q_BYTES = 16 * QROW;
  static constexpr int PART = (32 + 16 * D) * 4;    // one (m, l, O) partial
  static constexpr int IDX = 2048 * 4;             // the CTA's index slice
  static constexpr int OFF_IDX = Q_BYTES + NW * WARP;
  static constexpr int MAIN = OFF_IDX + IDX;
  static constexpr int MERGE = Q_BYTES + NW * PART + PART;
  static constexpr size_t SMEM = (MAIN > MERGE ? MAIN : MERGE) + 128;
};

struct DecParams {
  const __nv_bfloat16* Q;   // [B, H, D]
  const uint8_t* K;         // [B, kv_stride, D] E4M3 codes
  const uint8_t* V;
  const float* ks;          // [B, kv_stride]
  const float* vs;
  const int32_t* idx;       // [B, n_idx] (gather)
  int n_idx;
  int64_t kv_len;
  int64_t kv_stride;
  int H;
  float scale_log2;
  int splits;               // CTAs per sequence
  int per_split;            // keys (range) or idx slots (gather) per CTA
  __nv_bfloat16* O;         // [B, H, D] (gather)
  float* part;              // [B, splits, 32 + 16*D] (range)
  float* logits;            // [B, H, logit_ld] (range)
  int64_t logit_ld;
};

template <int D, bool RANGE, bool PARTIALS>
__global__ void __launch_bounds__(DecLayout<D>::NW * 32, 1)
decode_attn_kernel(DecParams p, DevCtx ctx) {
  using L = DecLayout<D>;
  extern __shared__ __align__(128) uint8_t smem_dec[];
  uint8_t* smem = smem_dec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int b = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;

  // ---- Q rows (zero beyond H) -> f16 with an exact power-of-two prescale
  uint8_t* sQ = smem;
  __shared__ float red_max[L::NW];
  float qscale_inv;
  {
    const __nv_bfloat16* q = p.Q + (int64_t)b * p.H * D;
    float mx = 0.f;
    for (int e = threadIdx.x; e < p.H * D; e += blockDim.x) mx = fmaxf(mx, fabsf(__bfloat162float(q[e])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red_max[warp] = mx;
    __syncthreads();
    for (int w = 0; w < L::NW; ++w) mx = fmaxf(mx, red_max[w]);
    const int ex = mx > 0.f ? 14 - ilogbf(mx) : 0;        // mx * 2^ex in [2^14, 2^15)
    const float qs = ldexpf(1.f, ex);
    qscale_inv = ldexpf(1.f, -ex);
    for (int u = threadIdx.x; u < 16 * D / 8; u += blockDim.x) {
      const int r = u / (D / 8), un = u % (D / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < p.H) {
        const uint4 raw = *reinterpret_cast<const uint4*>(q + r * D + un * 8);
        const uint32_t* rw = reinterpret_cast<const uint32_t*>(&raw);
        uint32_t* ow = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw[i]));
          __half2 h = __floats2half2_rn(f.x * qs, f.y * qs);
          ow[i] = *reinterpret_cast<uint32_t*>(&h);
        }
      }
      *reinterpret_cast<uint4*>(sQ + r * L::QROW + un * 16) = v;
    }
  }

  const int64_t s_begin = (int64_t)split * p.per_split;
  const int64_t total = RANGE ? p.kv_len : (int64_t)p.n_idx;
  const int64_t s_end = min(total, s_begin + p.per_split);
  const int n_chunks = s_end > s_begin ? (int)((s_end - s_begin + L::CH - 1) / L::CH) : 0;
  const int my_n = warp < n_chunks ? (n_chunks - warp + L::NW - 1) / L::NW : 0;
  const int64_t seq = (int64_t)b * p.kv_stride;
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + L::OFF_IDX);
  if (!RANGE) {
    for (int64_t i = threadIdx.x; i < s_end - s_begin; i += blockDim.x) {
      int32_t v = p.idx[(int64_t)b * p.n_idx + s_begin + i];
      if (v < -1 || v >= p.kv_len) {
        report(ctx, ST_DEVICE_CHECK);
        v = -1;
      }
      sidx[i] = v;
    }
  }
  uint8_t* wb = smem + L::Q_BYTES + warp * L::WARP;

  auto issue = [&](int s, int chunk) {
    uint8_t* st = wb + s * L::STAGE;
    const int64_t sl = s_begin + (int64_t)chunk * L::CH + lane;
    int32_t pos = -1;
    if (lane < L::CH && sl < s_end) {
      pos = RANGE ? (int32_t)sl : sidx[sl - s_begin];
    }
    if (lane < L::CH) reinterpret_cast<int32_t*>(st + L::OFF_POS)[lane] = pos;
    {
      // lane -> key lane/2, half lane%2 of its row: UPR/2 16-byte copies each for K and V
      constexpr int UPR = D / 16;
      const int key = lane >> 1, u0 = (lane & 1) * (UPR / 2);
      const int32_t pk = __shfl_sync(0xffffffffu, pos, key);
      const int64_t row = seq + (pk < 0 ? 0 : pk);
      const uint8_t* ksrc = p.K + row * D + u0 * 16;
      const uint8_t* vsrc = p.V + row * D + u0 * 16;
      const uint32_t kdst = smem_u32(st + L::OFF_K + key * L::KROW + u0 * 16);
      const uint32_t vdst = smem_u32(st + L::OFF_V + key * L::VROW + u0 * 16);
#pragma unroll
      for (int u = 0; u < UPR / 2; ++u) {
        cp_async16(kdst + u * 16, ksrc + u * 16, pk >= 0);
        cp_async16(vdst + u * 16, vsrc + u * 16, pk >= 0);
      }
    }
    if (lane < L::CH) {
      const int64_t row = seq + (pos < 0 ? 0 : pos);
      cp_async4(smem_u32(st + L::OFF_KS + lane * 4), p.ks + row, pos >= 0);
      cp_async4(smem_u32(st + L::OFF_VS + lane * 4), p.vs + row, pos >= 0);
    }
  };

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  __syncthreads();                       // Q and the index slice are in shared memory

#pragma unroll
  for (int s = 0; s < L::NST - 1; ++s) {
    if (s < my_n) issue(s, warp + L::NW * s);
    cp_async_commit();
  }
  const uint32_t qa = smem_u32(sQ);
  for (int it = 0; it < my_n; ++it) {
    {
      const int nxt = it + L::NST - 1;
      if (nxt < my_n) issue(nxt % L::NST, warp + L::NW * nxt);
      cp_async_commit();
    }
    cp_async_wait<L::NST - 1>();
    __syncwarp();
    const uint8_t* st = wb + (it % L::NST) * L::STAGE;
    const int32_t* spos = reinterpret_cast<const int32_t*>(st + L::OFF_POS);
    const float* sks = reinterpret_cast<const float*>(st + L::OFF_KS);
    const float* svs = reinterpret_cast<const float*>(st + L::OFF_VS);

    // S = Q K^T with the shared head-dim permutation (see the header);
    // four independent accumulation chains
    float s4[4][4] = {};
    const uint8_t* kraw = st + L::OFF_K;
#pragma unroll 4
    for (int kk = 0; kk < D / 16; ++kk) {
      const int d0 = kk * 16 + 4 * t;
      uint32_t a[4];
      {
        const uint2 q0 = *reinterpret_cast<const uint2*>(sQ + g * L::QROW + d0 * 2);
        const uint2 q1 = *reinterpret_cast<const uint2*>(sQ + (g + 8) * L::QROW + d0 * 2);
        a[0] = q0.x; a[2] = q0.y; a[1] = q1.x; a[3] = q1.y;
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const uint32_t kw = *reinterpret_cast<const uint32_t*>(kraw + (nt * 8 + g) * L::KROW + d0);
        mma_f16_16816(s4[(kk & 1) * 2 + nt], a, e4m3x2_to_f16x2((uint16_t)(kw & 0xffffu)),
                      e4m3x2_to_f16x2((uint16_t)(kw >> 16)));
      }
    }
    float s[2][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s[0][e] = s4[0][e] + s4[2][e];
      s[1][e] = s4[1][e] + s4[3][e];
    }
    (void)qa;
    float x[2][4];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = nt * 8 + 2 * t + (e & 1);
        float v = s[nt][e] * (p.scale_log2 * qscale_inv * sks[key]);
        if (spos[key] < 0) v = -INFINITY;
        x[nt][e] = v;
        if (e < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
      }
    if (RANGE) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int key = nt * 8 + 2 * t;
        const int32_t pos = spos[key];
        if (pos >= 0) {
          const bool two = spos[key + 1] >= 0;
          float* r0 = p.logits + ((int64_t)b * p.H + g) * p.logit_ld + pos;
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
    // lazy rescale: move the reference max only when it grows by > 2^8
    float al0 = 1.f, al1 = 1.f;
    if (mx0 > m0 + 8.f) {
      al0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - mx0);
      m0 = mx0;
    }
    if (mx1 > m1 + 8.f) {
      al1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - mx1);
      m1 = mx1;
    }
    const float mu0 = (m0 == -INFINITY) ? 0.f : m0;
    const float mu1 = (m1 == -INFINITY) ? 0.f : m1;
    float pr[2][4];
    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pe = fast_exp2(x[nt][e] - (e < 2 ? mu0 : mu1));
        if (e < 2) ls0 += pe; else ls1 += pe;
        pr[nt][e] = pe * svs[nt * 8 + 2 * t + (e & 1)];
      }
    l0 = l0 * al0 + ls0;
    l1 = l1 * al1 + ls1;
    if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[i][0] *= al0; o[i][1] *= al0;
        o[i][2] *= al1; o[i][3] *= al1;
      }
    }
    uint32_t ap[4];
    ap[0] = pack_f16x2(pr[0][0], pr[0][1]);
    ap[1] = pack_f16x2(pr[0][2], pr[0][3]);
    ap[2] = pack_f16x2(pr[1][0], pr[1][1]);
    ap[3] = pack_f16x2(pr[1][2], pr[1][3]);
    // O += P V, B fragments from the raw codes (see the header): per 32 bytes
    // of d, 4 n-tiles j = 4*blk + 2*half + parity covering dims c0 + 2n + parity
    {
      const uint32_t va = smem_u32(st + L::OFF_V);
      const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int blk = 0; blk < D / 32; ++blk) {
        uint32_t r[4];
        ldsm_x4_t(r, va + key * L::VROW + blk * 32 + (lane >> 4) * 16);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t px = __byte_perm(r[2 * half], r[2 * half + 1], 0x6420);
          const uint32_t py = __byte_perm(r[2 * half], r[2 * half + 1], 0x7531);
          mma_f16_16816(o[4 * blk + 2 * half], ap, e4m3x2_to_f16x2((uint16_t)(px & 0xffffu)),
                        e4m3x2_to_f16x2((uint16_t)(px >> 16)));
          mma_f16_16816(o[4 * blk + 2 * half + 1], ap, e4m3x2_to_f16x2((uint16_t)(py & 0xffffu)),
                        e4m3x2_to_f16x2((uint16_t)(py >> 16)));
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();

  // ---- merge the warps into this CTA's partial (m, l, O) in shared memory
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();
  float* cmb = reinterpret_cast<float*>(smem + L::Q_BYTES);    // [NW warps] partials
  float* mine = cmb + L::NW * (L::PART / 4);                    // merged partial of the CTA
  {
    float* wpart = cmb + warp * (L::PART / 4);
    if (t == 0) {
      wpart[g] = m0;
      wpart[g + 8] = m1;
      wpart[16 + g] = l0;
      wpart[16 + g + 8] = l1;
    }
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      // n-tile j: c0 = 16*(j/2), parity j&1; element e at n = 2t + (e&1)
      const int dcol = 16 * (j >> 1) + 4 * t + (j & 1);
      wpart[32 + g * D + dcol] = o[j][0];
      wpart[32 + g * D + dcol + 2] = o[j][1];
      wpart[32 + (g + 8) * D + dcol] = o[j][2];
      wpart[32 + (g + 8) * D + dcol + 2] = o[j][3];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 16 * D; e += blockDim.x) {
    const int h = e / D, c = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < L::NW; ++w) M = fmaxf(M, cmb[w * (L::PART / 4) + h]);
    float Ls = 0.f, Ov = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < L::NW; ++w) {
        const float mw = cmb[w * (L::PART / 4) + h];
        const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
        Ls += cmb[w * (L::PART / 4) + 16 + h] * f;
        Ov += cmb[w * (L::PART / 4) + 32 + h * D + c] * f;
      }
    }
    if (PARTIALS) {
      float* part = p.part + ((int64_t)b * p.splits + split) * (32 + 16 * D);
      part[32 + h * D + c] = Ov;
      if (c == 0) {
        part[h] = M;
        part[16 + h] = Ls;
      }
    } else {
      mine[32 + h * D + c] = Ov;
      if (c == 0) {
        mine[h] = M;
        mine[16 + h] = Ls;
      }
    }
  }
  if (!PARTIALS) {
    // ---- merge the cluster's partials through distributed shared memory
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    cluster.sync();
    const int hp = (16 + C - 1) / C;                 // heads merged by this CTA
    const int h0 = r * hp, h1 = min(16, h0 + hp);
    for (int e = threadIdx.x; e < (h1 - h0) * D; e += blockDim.x) {
      const int h = h0 + e / D, c = e % D;
      if (h >= p.H) continue;
      float M = -INFINITY;
      for (int q = 0; q < C; ++q) M = fmaxf(M, cluster.map_shared_rank(mine, q)[h]);
      float Ls = 0.f, Ov = 0.f;
      if (M != -INFINITY) {
        for (int q = 0; q < C; ++q) {
          const float* pq = cluster.map_shared_rank(mine, q);
          const float mq = pq[h];
          const float f = (mq == -INFINITY) ? 0.f : fast_exp2(mq - M);
          Ls += pq[16 + h] * f;
          Ov += pq[32 + h * D + c] * f;
        }
      }
      p.O[((int64_t)b * p.H + h) * D + c] = __float2bfloat16_rn(Ls > 0.f ? Ov / Ls : 0.f);
    }
    cluster.sync();                                    // peers read our partial until here
  }
}

}  // namespace hs2
