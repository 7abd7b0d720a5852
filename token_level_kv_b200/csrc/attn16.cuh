// Attention of one token's 16 query heads over a list of keys of the single
// KV head: the shape of the sparse layers (row a6, here) and of the decode
// step (rows a7, a8: decode_attn.cuh).  The 16 heads are the M = 16 rows of
// mma.sync m16n8k16 (bf16 in, fp32 accumulate).  Also the split merge and the
// decode selection-score kernels.
//
// Method: "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (agihunt.info summary), KV Reuse paragraph -- the sparse layers gather only
// the selected tokens (window + top-k) of the full layer's KV; MQA, NoPE.
#pragma once
#include "common.cuh"

namespace hs2 {

struct Attn16Params {
  const __nv_bfloat16* Q;   // [n_rows, H, D]
  const void* K;            // bf16 [kv_len, D]
  const void* V;
  const int32_t* idx;       // [n_rows, n_idx]
  int n_idx;
  int64_t kv_len;
  int H;
  float scale_log2;         // softmax_scale * log2(e)
  __nv_bfloat16* O;         // [n_rows, H, D]
  int64_t n_rows;
};

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
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

// Sparse prefill layer (row a6) over the shared bf16 KV.  A PAIR of warps
// owns one query row; warp half h holds dims [h*D/2, (h+1)*D/2) of Q, of the
// gathered K and V rows and of O (16 heads = the M of mma.sync).  Per 16-key
// chunk each warp forms the partial S over its half of d; the two partials
// meet in shared memory (double-buffered, one pair barrier per chunk) and both
// warps add them in the same order, so both hold the same S and run the same
// online softmax, and each adds P V for its half of d.  Halving O (64 fp32
// registers a thread) puts 8 warps on an SM where one warp per row fitted 4.
// Q stays in registers as mma A fragments, so shared memory holds only the
// gather: K and V half rows of a chunk travel as separate stages of a
// per-warp 6-stage cp.async ring (K_c, V_c, K_c+1, ...), up to 5 stages in
// flight (the bytes in flight per SM set the gather rate); rows are stored at a
// D + 16 byte stride, which keeps the ldmatrix loads of 8 rows on 8 different
// bank groups.  The reference max of the online softmax moves only when a
// row's max grows by more than 2^8 (lazy rescale of O).
template <int D>
struct SpfLayout {
  static constexpr int CH = 16;
  static constexpr int HD = D / 2;                 // dims per warp
  static constexpr int NST = 6;                    // stages per warp (K or V half rows of one chunk)
  static constexpr int NPAIR = 4;                  // query rows in flight per CTA
  static constexpr int NT = NPAIR * 64;
  static constexpr int ROW = 2 * HD + 16;          // half row + pad
  static constexpr int STAGE = CH * ROW + CH * 4;  // rows + positions
  static constexpr int WARP = NST * STAGE;
  static constexpr int XCH = 2 * 2 * 32 * 8 * 4;   // per pair: [chunk parity][half][8 floats x 32 lanes]
  static constexpr size_t SMEM = 2 * NPAIR * (size_t)WARP + NPAIR * (size_t)XCH;
};

template <int D>
__global__ void __launch_bounds__(SpfLayout<D>::NT, 1)
sparse_prefill_kernel(Attn16Params p, DevCtx ctx) {
  using L = SpfLayout<D>;
  constexpr int HD = L::HD;
  extern __shared__ __align__(128) uint8_t smem_spf[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = warp >> 1, h = warp & 1;
  const int g = lane >> 2, t = lane & 3;
  uint8_t* wb = smem_spf + warp * L::WARP;
  float4* xch = reinterpret_cast<float4*>(smem_spf + 2 * L::NPAIR * L::WARP + pair * L::XCH);
  const int cpi = (p.n_idx + L::CH - 1) / L::CH;
  const int64_t n_rows = p.n_rows;
  const int dcol0 = h * HD;                          // this warp's first dim
  auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(1 + pair) : "memory"); };
  int xc = 0;                                        // chunks so far (exchange buffer parity)

  for (int64_t row = (int64_t)blockIdx.x * L::NPAIR + pair; row < n_rows; row += (int64_t)gridDim.x * L::NPAIR) {
    const int32_t* irow = p.idx + row * p.n_idx;
    // positions of a chunk (lanes 0-15, lanes 16-31 mirror them), loaded two
    // chunks before their stages are issued so the load latency is hidden
    auto ldpos = [&](int c) -> int32_t {
      const int sl = c * L::CH + (lane & 15);
      return (c < cpi && sl < p.n_idx) ? irow[sl] : -1;
    };
    // stage sequence: 2c = K half rows of chunk c, 2c + 1 = V half rows
    auto issue = [&](int sidx, int32_t pos) {
      const bool is_v = sidx & 1;
      uint8_t* st = wb + (sidx % L::NST) * L::STAGE;
      if (pos < -1 || pos >= p.kv_len) {
        if (!is_v && h == 0 && lane < 16) report(ctx, ST_DEVICE_CHECK);
        pos = -1;
      }
      if (lane < 16) reinterpret_cast<int32_t*>(st + L::CH * L::ROW)[lane] = pos;
      const uint8_t* base = reinterpret_cast<const uint8_t*>(is_v ? p.V : p.K) + dcol0 * 2;
      constexpr int UPR = 2 * HD / 16;
#pragma unroll
      for (int seg = lane; seg < L::CH * UPR; seg += 32) {
        const int i = seg / UPR, u = seg % UPR;
        const int32_t pi = __shfl_sync(0xffffffffu, pos, i);
        cp_async16(smem_u32(st + i * L::ROW + u * 16), base + (int64_t)(pi < 0 ? 0 : pi) * (2 * D) + u * 16,
                   pi >= 0);
      }
    };
    const int nstages = 2 * cpi;
    {
      const int32_t p0 = ldpos(0), p1 = ldpos(1);
      const int32_t p2 = ldpos(2);
      issue(0, p0);
      cp_async_commit();
      issue(1, p0);
      cp_async_commit();
      if (nstages > 2) issue(2, p1);
      cp_async_commit();
      if (nstages > 3) issue(3, p1);
      cp_async_commit();
      if (nstages > 4) issue(4, p2);
      cp_async_commit();
    }
    // positions of chunks c + 2 and c + 3 (their stages are issued in chunk c)
    int32_t q1 = ldpos(2), q2 = ldpos(3);
    // this warp's half of Q as mma A fragments (rows >= H are zero): per
    // 16-dim step kk, {Q[g][2t,2t+1], Q[g+8][2t,2t+1], Q[g][2t+8,2t+9], Q[g+8][2t+8,2t+9]}
    uint32_t qf[HD / 16][4];
    {
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(p.Q + (row * p.H + g) * D + dcol0) + t;
      const uint32_t* q1 = q0 + 8 * (D / 2);
      const bool h0 = g < p.H, h1 = g + 8 < p.H;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        qf[kk][0] = h0 ? q0[kk * 8] : 0u;
        qf[kk][1] = h1 ? q1[kk * 8] : 0u;
        qf[kk][2] = h0 ? q0[kk * 8 + 4] : 0u;
        qf[kk][3] = h1 ? q1[kk * 8 + 4] : 0u;
      }
    }
    float o[HD / 8][4];
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int c = 0; c < cpi; ++c, ++xc) {
      // K stage of chunk c: 2c; keep NST-1 = 5 stages issued ahead
      static_assert(L::NST == 6, "stage schedule below assumes a 6-stage ring");
      {
        const int nxt = 2 * c + L::NST - 1;           // V stage of chunk c + 2
        if (nxt < nstages) issue(nxt, q1);
        cp_async_commit();
      }
      cp_async_wait<L::NST - 1>();
      __syncwarp();
      const uint8_t* ks = wb + ((2 * c) % L::NST) * L::STAGE;
      const int32_t* spos = reinterpret_cast<const int32_t*>(ks + L::CH * L::ROW);
      const uint32_t ka = smem_u32(ks);
      // partial S over this warp's half of d: four independent chains
      float s4[4][4] = {};
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        uint32_t b[4];
        {
          const int key = (lane & 7) + (lane >> 4) * 8;
          ldsm_x4(b, ka + key * L::ROW + (kk * 2 + ((lane >> 3) & 1)) * 16);
        }
        mma_bf16_16816(s4[(kk & 1) * 2 + 0], qf[kk], b[0], b[1]);
        mma_bf16_16816(s4[(kk & 1) * 2 + 1], qf[kk], b[2], b[3]);
      }
      // exchange the partials; S = S_half0 + S_half1 in both warps
      float s[2][4];
      {
        float4* mine = xch + ((xc & 1) * 2 + h) * 64;
        const float4* other = xch + ((xc & 1) * 2 + (h ^ 1)) * 64;
        const float4 w0 = make_float4(s4[0][0] + s4[2][0], s4[0][1] + s4[2][1], s4[0][2] + s4[2][2], s4[0][3] + s4[2][3]);
        const float4 w1 = make_float4(s4[1][0] + s4[3][0], s4[1][1] + s4[3][1], s4[1][2] + s4[3][2], s4[1][3] + s4[3][3]);
        mine[lane] = w0;
        mine[32 + lane] = w1;
        pair_sync();
        const float4 v0 = other[lane], v1 = other[32 + lane];
        if (h == 0) {
          s[0][0] = w0.x + v0.x; s[0][1] = w0.y + v0.y; s[0][2] = w0.z + v0.z; s[0][3] = w0.w + v0.w;
          s[1][0] = w1.x + v1.x; s[1][1] = w1.y + v1.y; s[1][2] = w1.z + v1.z; s[1][3] = w1.w + v1.w;
        } else {
          s[0][0] = v0.x + w0.x; s[0][1] = v0.y + w0.y; s[0][2] = v0.z + w0.z; s[0][3] = v0.w + w0.w;
          s[1][0] = v1.x + w1.x; s[1][1] = v1.y + w1.y; s[1][2] = v1.z + w1.z; s[1][3] = v1.w + w1.w;
        }
      }
      float x[2][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = nt * 8 + 2 * t + (e & 1);
          float v = s[nt][e] * p.scale_log2;
          if (spos[key] < 0) v = -INFINITY;
          x[nt][e] = v;
          if (e < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
        }
      __syncwarp();            // K stage fully read: it is reissued below
      {
        const int nxt = 2 * c + L::NST;               // K stage of chunk c + 3
        if (nxt < nstages) issue(nxt, q2);
        cp_async_commit();
      }
      q1 = q2;
      q2 = ldpos(c + 4);
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
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
          pr[nt][e] = pe;
        }
      l0 = l0 * al0 + ls0;
      l1 = l1 * al1 + ls1;
      if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
        for (int i = 0; i < HD / 8; ++i) {
          o[i][0] *= al0; o[i][1] *= al0;
          o[i][2] *= al1; o[i][3] *= al1;
        }
      }
      uint32_t ap[4];
      ap[0] = pack_bf16x2(pr[0][0], pr[0][1]);
      ap[1] = pack_bf16x2(pr[0][2], pr[0][3]);
      ap[2] = pack_bf16x2(pr[1][0], pr[1][1]);
      ap[3] = pack_bf16x2(pr[1][2], pr[1][3]);
      // V stage of chunk c: 2c + 1
      cp_async_wait<L::NST - 1>();
      __syncwarp();
      const uint32_t va = smem_u32(wb + ((2 * c + 1) % L::NST) * L::STAGE);
#pragma unroll
      for (int nd = 0; nd < HD / 16; ++nd) {
        uint32_t b[4];
        const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
        ldsm_x4_t(b, va + key * L::ROW + (nd * 2 + (lane >> 4)) * 16);
        mma_bf16_16816(o[2 * nd], ap, b[0], b[1]);
        mma_bf16_16816(o[2 * nd + 1], ap, b[2], b[3]);
      }
      __syncwarp();            // V stage fully read before it is reissued
    }
    cp_async_wait<0>();
    __syncwarp();
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    __nv_bfloat16* out = p.O + row * p.H * D + dcol0;
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      const int col = i * 8 + 2 * t;
      if (g < p.H) *reinterpret_cast<uint32_t*>(out + g * D + col) = pack_bf16x2(o[i][0] * i0, o[i][1] * i0);
      if (g + 8 < p.H)
        *reinterpret_cast<uint32_t*>(out + (g + 8) * D + col) = pack_bf16x2(o[i][2] * i1, o[i][3] * i1);
    }
  }
}

// Merge split partials of one (item, head) per CTA: m = max m_s,
// l = sum l_s 2^(m_s-m), O = sum O_s 2^(m_s-m) / l.  Also stores (m, l) per
// head (log2 units) for the selection pass.  The split factors are computed
// once, cooperatively, into shared memory; then G groups of D threads (one
// output dim per thread) each sum every G-th split, so a sequence with
// hundreds of splits has G times the loads in flight, and group 0 adds the
// groups' sums in a fixed order.  G = 4 for many splits, 1 for few (where
// the extra threads only add start-up).
constexpr int kCombineMaxSplits = 1024;
constexpr int kCombineManySplits = 64;
// With O32 set, the merged O is written unnormalised (fp32, relative to m) for
// a later merge across shards of the context, and O is not written.
template <int D, int G>
__global__ void __launch_bounds__(D * G)
attn16_combine_kernel(const float* part, int splits, int H, __nv_bfloat16* O, float* ml, float* O32) {
  constexpr int NT = D * G;
  const int item = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int c = tid % D, grp = tid / D;
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int PS = 32 + 16 * D;                   // floats per partial
  __shared__ float fac[kCombineMaxSplits];
  __shared__ float red[NT / 32];
  __shared__ float osum[G > 1 ? G - 1 : 1][D];
  const float* base = part + (int64_t)item * splits * PS;
  float M = -INFINITY;
  for (int s = tid; s < splits; s += NT) M = fmaxf(M, base[(int64_t)s * PS + h]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  float ls = 0.f;
  for (int s = tid; s < splits; s += NT) {
    const float ms = base[(int64_t)s * PS + h];
    const float f = (M == -INFINITY || ms == -INFINITY) ? 0.f : fast_exp2(ms - M);
    fac[s] = f;
    ls += base[(int64_t)s * PS + 16 + h] * f;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  if (lane == 0) red[warp] = ls;
  __syncthreads();
  float Ls = 0.f;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) Ls += red[w];
  const float* col = base + 32 + h * D + c;
  float acc0 = 0.f, acc1 = 0.f;
  int s = grp;
#pragma unroll 4
  for (; s + G < splits; s += 2 * G) {
    acc0 += col[(int64_t)s * PS] * fac[s];
    acc1 += col[(int64_t)(s + G) * PS] * fac[s + G];
  }
  if (s < splits) acc0 += col[(int64_t)s * PS] * fac[s];
  float acc = acc0 + acc1;
  if (grp > 0) osum[grp - 1][c] = acc;
  __syncthreads();
  if (grp != 0) return;
#pragma unroll
  for (int q = 0; q < G - 1; ++q) acc += osum[q][c];
  if (c == 0 && ml != nullptr) {
    const int64_t r = (int64_t)item * H + h;
    if (O32 != nullptr) {                           // a shard's partial: m, then l, each [items, H]
      ml[r] = M;
      ml[(int64_t)gridDim.x * H + r] = Ls;
    } else {
      ml[r * 2] = M;
      ml[r * 2 + 1] = Ls;
    }
  }
  if (O32 != nullptr) O32[((int64_t)item * H + h) * D + c] = acc;
  else O[((int64_t)item * H + h) * D + c] = __float2bfloat16_rn(Ls > 0.f ? acc / Ls : 0.f);
}

// Merge of partials across the R shards of a context.  ml_all holds every
// shard's (m, l) as [R][2][items * H] (m in log2 units; an all-gather of
// each shard's planar (m, l) gives it); for each (item, head) the kernel takes
// M = max_q m_q and L = sum_q l_q 2^(m_q - M), rescales this shard's
// unnormalised O by 2^(m_shard - M) (0 for a shard that saw no key), so that
// the shards' O then add up, and writes (M, L) interleaved to ml_out.  Every
// shard computes the same M and L in the same order.
template <int D>
__global__ void __launch_bounds__(D)
partial_merge_kernel(const float* ml_all, int R, int shard, float* O32, float* ml_out, int H) {
  const int item = blockIdx.x, h = blockIdx.y, c = threadIdx.x;
  const int64_t n = (int64_t)gridDim.x * H;
  const int64_t r = (int64_t)item * H + h;
  float M = -INFINITY;
  for (int q = 0; q < R; ++q) M = fmaxf(M, ml_all[q * 2 * n + r]);
  float L = 0.f;
  for (int q = 0; q < R; ++q) {
    const float m = ml_all[q * 2 * n + r];
    L += (m == -INFINITY) ? 0.f : ml_all[q * 2 * n + n + r] * fast_exp2(m - M);
  }
  const float m = ml_all[shard * 2 * n + r];
  const float f = m == -INFINITY ? 0.f : fast_exp2(m - M);
  O32[r * D + c] *= f;
  if (c == 0) {
    ml_out[r * 2] = M;
    ml_out[r * 2 + 1] = L;
  }
}

// The merged output: O = (sum of the shards' rescaled O) / (sum of their l).
template <int D>
__global__ void __launch_bounds__(D)
partial_finalize_kernel(const float* ml, const float* O32, __nv_bfloat16* O, int H) {
  const int item = blockIdx.x, h = blockIdx.y, c = threadIdx.x;
  const int64_t r = (int64_t)item * H + h;
  const float l = ml[r * 2 + 1];
  O[r * D + c] = __float2bfloat16_rn(l > 0.f ? O32[r * D + c] / l : 0.f);
}

// Decode selection score: sigma[b, j] = sum_h 2^(x_hj - m_h) / l_h for the
// candidates j < n_cand (x: scaled logits in log2 units).  A thread takes four
// consecutive candidates with 16-byte loads (rows start 16-byte aligned: the
// leading dimensions are multiples of 64), the heads added in order.  With
// `zero` set, n_zero words per row from zero + b * n_zero are cleared.
__global__ void __launch_bounds__(256)
decode_sigma_kernel(const float* logits, int64_t logit_ld, const float* ml, int H,
                    int64_t n_cand, float* sigma, int64_t sigma_ld, uint32_t* zero, int n_zero) {
  const int b = blockIdx.y;
  __shared__ float sM[16], sI[16];
  if (zero != nullptr && blockIdx.x == 0)           // the row's top-k histograms, for the passes after this one
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[(int64_t)b * n_zero + i] = 0u;
  if (threadIdx.x < H) {
    sM[threadIdx.x] = ml[((int64_t)b * H + threadIdx.x) * 2];
    const float l = ml[((int64_t)b * H + threadIdx.x) * 2 + 1];
    sI[threadIdx.x] = 1.f / l;
  }
  __syncthreads();
  const int64_t j = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (j >= n_cand) return;
  const float* row = logits + (int64_t)b * H * logit_ld + j;
  float* out = sigma + (int64_t)b * sigma_ld + j;
  if (j + 4 <= n_cand) {
    float4 x[16];
#pragma unroll
    for (int h = 0; h < 16; ++h)
      if (h < H) x[h] = *reinterpret_cast<const float4*>(row + h * logit_ld);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int h = 0; h < 16; ++h)
      if (h < H) {
        acc.x += fast_exp2(x[h].x - sM[h]) * sI[h];
        acc.y += fast_exp2(x[h].y - sM[h]) * sI[h];
        acc.z += fast_exp2(x[h].z - sM[h]) * sI[h];
        acc.w += fast_exp2(x[h].w - sM[h]) * sI[h];
      }
    *reinterpret_cast<float4*>(out) = acc;
    return;
  }
  for (int e = 0; e < 4 && j + e < n_cand; ++e) {
    float acc = 0.f;
    for (int h = 0; h < H; ++h) acc += fast_exp2(row[h * logit_ld + e] - sM[h]) * sI[h];
    out[e] = acc;
  }
}

}  // namespace hs2
