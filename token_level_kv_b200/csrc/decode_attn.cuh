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
//   * Producer warps stream 32-key chunks into a shared ring of NS stages,
//     so almost the whole ring is in flight whatever the consumers are doing
//     (one warp for a range, three for a gather, which needs a copy
//     instruction per two rows); the consumer warp pairs take chunk i from
//     stage i % NS (pair i % NP) and hand the stage back through its empty
//     barrier.  A range (a7) is
//     contiguous in the cache: one elected lane moves each chunk's K and V
//     with 3-D TMA tiles (box 128 bytes x 16 keys, 128-byte swizzle; keys past
//     kv_len arrive as zeros), which keeps the whole copy off the load/store
//     pipe.  A gather (a8) copies one row per lane pair with cp.async into
//     rows padded to D + 16 bytes.  Both layouts make the fragment loads below
//     bank-conflict free; the per-key scales always come by cp.async, and
//     completion is tracked on the stage's mbarrier (transaction bytes plus
//     cp.async.mbarrier.arrive).
//   * The products run on mma.sync m16n8k16 in f16 with fp32 accumulation
//     (the heads are M): every E4M3 code is an f16, so one cvt.rn.f16x2.e4m3x2
//     widens two codes exactly.  Q enters in f16 after an exact power-of-two
//     prescale that puts its largest element in [2^14, 2^15) (f16 then holds
//     every bf16 element exactly except ones below 2^-28 of that maximum);
//     the prescale, the key scale and softmax_scale multiply the fp32 logit.
//     P holds p * v_scale * 2^-e in f16, e the exponent of the largest V scale
//     a pair has seen (raised with an exact power-of-two rescale of O when a
//     chunk brings a larger one, and undone when the pairs merge), so P stays
//     below 2^9 (p <= 2^8) and neither overflows nor underflows whatever the
//     magnitude of the scales: the result scales exactly with them.
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
//   * The index slice is copied to shared memory alongside the Q loads, so the
//     first K/V requests leave after one round trip; Q is converted while
//     they are in flight.
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

template <int D, bool RANGE>
struct DecLayout {
  // A range moves each stage with one TMA instruction per box, so one
  // producer warp keeps the ring full; a gather issues a copy instruction per
  // two rows, and one warp could not issue them fast enough (measured: 1.6x
  // slower than the random-row gather rate of the memory), so three warps
  // share it.
  static constexpr int NP = RANGE ? 5 : 4;          // consumer warp pairs
  static constexpr int NC = 2 * NP;                 // consumer warps
  static constexpr int NPROD = RANGE ? 1 : 3;       // producer warps
  static constexpr int HD = D / 2;                  // dims per consumer warp
  static constexpr int NT = (NC + NPROD) * 32;      // 11 warps: <= 168 registers
  static constexpr int NS = 10;                     // ring stages (32 keys each)
  static constexpr int CH = 32;
  // gather stage: K rows, V rows at a padded stride, then the two scale rows
  static constexpr int KROW = RANGE ? 128 : D + 16;
  static constexpr int VROW = D + 16;
  static constexpr int BOX = CH * 128;              // range stage: one TMA box, 128 bytes x 32 keys
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = RANGE ? CH * D : CH * KROW;
  static constexpr int STAGE = RANGE ? 2 * CH * D : 2 * CH * (D + 16) + 2 * CH * 4;
  static constexpr int QROW = 2 * D + 32;           // padded f16 Q row (8-byte fragment loads conflict free)
  static constexpr int Q_BYTES = 16 * QROW;
  static constexpr int PART = (32 + 16 * D) * 4;    // one (m, l, O) partial
  static constexpr int PROW = D + 16;               // padded O row of a pair's partial (conflict-free float4 stores)
  static constexpr int PPART = (32 + 16 * PROW) * 4;
  static constexpr int OFF_RING = (Q_BYTES + 1023) / 1024 * 1024;   // swizzled TMA boxes want 1 KB
  static constexpr int OFF_SC = OFF_RING + NS * STAGE;              // range: scales [NS][2][CH]
  static constexpr int IDX = 2048 * 4;              // the CTA's index slice
  static constexpr int OFF_IDX = OFF_SC + (RANGE ? NS * 2 * CH * 4 : 0);
  static constexpr int XCH = 2 * 2 * 32 * 8 * 4 + 16;   // per pair: [chunk parity][half][8 floats x 32 lanes] + flags
  static constexpr int OFF_XCH = OFF_IDX + (RANGE ? 0 : IDX);
  static constexpr int OFF_BAR = OFF_XCH + NP * XCH;
  static constexpr int MAIN = OFF_BAR + 2 * NS * 8;
  static constexpr int MERGE = Q_BYTES + NP * PPART + PART;
  static constexpr size_t SMEM = (MAIN > MERGE ? MAIN : MERGE) + 1024;   // + base alignment
  // scale rows of stage s
  __device__ static float* kscale(uint8_t* smem, int s) {
    return RANGE ? reinterpret_cast<float*>(smem + OFF_SC) + s * 2 * CH
                 : reinterpret_cast<float*>(smem + OFF_RING + s * STAGE + 2 * CH * (D + 16));
  }
};

constexpr int kNoVexp = -1000;   // no V scale seen yet

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
  int64_t idx_offset;       // gather over one shard of the context: idx entries are global positions and
                            // only [idx_offset, idx_offset + kv_len) are this shard's (rebased); -1: no shard
  float* part;              // [B, splits, 32 + 16*D] (range)
  float* logits;            // [B, H, logit_ld] (range)
  int64_t logit_ld;
};

// tmK / tmV: 3-D maps {D, kv_len, batch} over the codes (range only; a gather
// passes unused maps).
template <int D, bool RANGE, bool PARTIALS>
__global__ void __launch_bounds__(DecLayout<D, RANGE>::NT, 1)
decode_attn_kernel(DecParams p, DevCtx ctx, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV) {
  using L = DecLayout<D, RANGE>;
  extern __shared__ __align__(128) uint8_t smem_dec[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dec) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int b = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;
  uint8_t* ring = smem + L::OFF_RING;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + L::NS;

  const int64_t s_begin = (int64_t)split * p.per_split;
  const int64_t total = RANGE ? p.kv_len : (int64_t)p.n_idx;
  const int64_t s_end = min(total, s_begin + p.per_split);
  const int n_chunks = s_end > s_begin ? (int)((s_end - s_begin + L::CH - 1) / L::CH) : 0;
  const int64_t seq = (int64_t)b * p.kv_stride;
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + L::OFF_IDX);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::NS; ++s) {
      mbar_init(&full[s], RANGE ? 33 : 32);  // the producer lanes' cp.async arrivals (+ the TMA lane)
      mbar_init(&empty[s], 2);             // the consuming warp pair
    }
    fence_barrier_init();
  }
  // ---- start-up: the index slice -> shared memory (cp.async, then each
  // thread checks the entries it copied) while Q comes into registers
  if (!RANGE) {
    for (int64_t i = threadIdx.x; i < s_end - s_begin; i += blockDim.x)
      cp_async4(smem_u32(sidx + i), p.idx + (int64_t)b * p.n_idx + s_begin + i, true);
  }
  cp_async_commit();
  constexpr int QV = 16 * D / 8;                     // uint4 groups of the 16 Q rows
  constexpr int QPT = (QV + L::NT - 1) / L::NT;
  uint4 qraw[QPT];
  float mx = 0.f;
  {
    const __nv_bfloat16* q = p.Q + (int64_t)b * p.H * D;
#pragma unroll
    for (int k = 0; k < QPT; ++k) {
      const int u = threadIdx.x + k * L::NT;
      const int r = u / (D / 8), un = u % (D / 8);
      qraw[k] = make_uint4(0, 0, 0, 0);
      if (u < QV && r < p.H) qraw[k] = *reinterpret_cast<const uint4*>(q + r * D + un * 8);
      const uint32_t* rw = reinterpret_cast<const uint32_t*>(&qraw[k]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw[i]));
        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  __shared__ float red_max[L::NC + L::NPROD];
  if (lane == 0) red_max[warp] = mx;
  cp_async_wait<0>();
  if (!RANGE) {
    for (int64_t i = threadIdx.x; i < s_end - s_begin; i += blockDim.x) {
      const int32_t v = sidx[i];
      if (p.idx_offset >= 0) {                       // a shard: other shards' keys are not errors
        sidx[i] = (v >= p.idx_offset && v < p.idx_offset + p.kv_len) ? (int32_t)(v - p.idx_offset) : -1;
        if (v < -1) report(ctx, ST_DEVICE_CHECK);
      } else if (v < -1 || v >= p.kv_len) {
        report(ctx, ST_DEVICE_CHECK);
        sidx[i] = -1;
      }
    }
  }
  __syncthreads();                                   // barriers, index slice, maxima

  uint8_t* sQ = smem;
  // ------------------------------------------------------------ producer
  // chunk i -> stage i % NS; the first ring round needs no empty wait, so it
  // is issued before the block-wide barrier below (nothing can block there)
  constexpr int UPR = D / 16;                        // 16-byte units per FP8 row
  constexpr int RPI = 32 / UPR;                      // rows per copy instruction (gather)
  auto produce = [&](int i) -> bool {
    const int s = i % L::NS;
    // the warp decides together (a lane that timed out stops all of it)
    if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], (uint32_t)(((i / L::NS) & 1) ^ 1), ctx))) return false;
    uint8_t* st = ring + s * L::STAGE;
    if (RANGE) {
      const int64_t pos0 = s_begin + (int64_t)i * L::CH;
      if (lane == 0) {
        mbar_expect_tx(&full[s], 2 * L::CH * D);
#pragma unroll
        for (int bx = 0; bx < D / 128; ++bx) {
          tma_load_3d(st + L::OFF_K + bx * L::BOX, &tmK, &full[s], bx * 128, (int)pos0, b);
          tma_load_3d(st + L::OFF_V + bx * L::BOX, &tmV, &full[s], bx * 128, (int)pos0, b);
        }
      }
      float* sc = L::kscale(smem, s);
      if (lane < L::CH) {
        const bool ok = pos0 + lane < s_end;
        const int64_t row = seq + (ok ? pos0 + lane : 0);
        cp_async4(smem_u32(sc + lane), p.ks + row, ok);
        cp_async4(smem_u32(sc + L::CH + lane), p.vs + row, ok);
      }
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[s])) : "memory");
      return true;
    }
    // lane j holds the position of stage row j; each copy instruction moves
    // RPI whole rows (consecutive lanes, consecutive 16-byte units)
    const int64_t sl = s_begin + (int64_t)i * L::CH + lane;
    const int32_t pk = sl < s_end ? sidx[sl - s_begin] : -1;
    {
      const int64_t row = seq + (pk < 0 ? 0 : pk);
      float* sc = L::kscale(smem, s);
      cp_async4(smem_u32(sc + lane), p.ks + row, pk >= 0);
      cp_async4(smem_u32(sc + L::CH + lane), p.vs + row, pk >= 0);
    }
    const int ur = lane / UPR, uu = lane % UPR;
#pragma unroll 4
    for (int j = 0; j < L::CH / RPI; ++j) {
      const int r = j * RPI + ur;
      const int32_t pr_ = __shfl_sync(0xffffffffu, pk, r);
      const int64_t row = seq + (pr_ < 0 ? 0 : pr_);
      cp_async16(smem_u32(st + L::OFF_K + r * L::KROW + uu * 16), p.K + row * D + uu * 16, pr_ >= 0);
      cp_async16(smem_u32(st + L::OFF_V + r * L::VROW + uu * 16), p.V + row * D + uu * 16, pr_ >= 0);
    }
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[s])) : "memory");
    return true;
  };
  // producer warp pw issues chunks pw, pw + NPROD, ... in increasing order;
  // a chunk's slot waits only for the chunk NS before it, which some producer
  // issues first, so the producers never wait on each other in a cycle
  const int first_round = min(n_chunks, L::NS);
  const int pw = warp - L::NC;
  bool prod_ok = true;
  int issued = pw;                                   // next chunk of this producer
  if (warp >= L::NC) {
    if (RANGE && lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    while (issued < first_round && prod_ok)
      if ((prod_ok = produce(issued))) issued += L::NPROD;
  }

  float o[L::HD / 8][4];
#pragma unroll
  for (int i = 0; i < L::HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float qscale_inv = 1.f;
  float vinv = 1.f;
  // ---- Q -> f16 with an exact power-of-two prescale (largest element in
  // [2^14, 2^15)), written while the first chunks are in flight
  {
    float m = 0.f;
    for (int w = 0; w < L::NC + L::NPROD; ++w) m = fmaxf(m, red_max[w]);
    const int ex = m > 0.f ? 14 - ilogbf(m) : 0;
    const float qs = ldexpf(1.f, ex);
    qscale_inv = ldexpf(1.f, -ex);
#pragma unroll
    for (int k = 0; k < QPT; ++k) {
      const int u = threadIdx.x + k * L::NT;
      if (u < QV) {
        const int r = u / (D / 8), un = u % (D / 8);
        const uint32_t* rw = reinterpret_cast<const uint32_t*>(&qraw[k]);
        uint4 v;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw[i]));
          __half2 h = __floats2half2_rn(f.x * qs, f.y * qs);
          ow[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(sQ + r * L::QROW + un * 16) = v;
      }
    }
  }
  __syncthreads();                                   // Q in shared memory

  int vexp = kNoVexp;                                // power-of-two reference of the V scales (consumers)
  if (warp >= L::NC) {
    while (issued < n_chunks && prod_ok)
      if ((prod_ok = produce(issued))) issued += L::NPROD;
    asm volatile("cp.async.wait_all;" ::: "memory");  // every issued copy lands before the merge reuses the ring
    static_assert(!RANGE || L::NPROD == 1, "the TMA drain below walks one producer's chunks");
    if (RANGE && lane == 0)                           // and every TMA tile (already done unless a wait gave up)
      for (int i = max(0, issued - L::NS); i < issued; ++i) mbar_drain(&full[i % L::NS], (uint32_t)((i / L::NS) & 1));
  } else {
    // ------------------------------------------------------------ consumers
    // pair `pr` takes steps i = pr, pr + NP, ... of 32 keys.  Warp half `hf`
    // forms S over the whole head dim for keys [16*hf, 16*hf + 16) of the
    // stage; the two halves of S meet in shared memory, both warps run the
    // same online softmax over the 32 keys and each adds P V for dims
    // [hf*HD, (hf+1)*HD) of O.
    const int pr = warp >> 1, hf = warp & 1;
    float4* xch = reinterpret_cast<float4*>(smem + L::OFF_XCH + pr * L::XCH);
    volatile int* xok = reinterpret_cast<volatile int*>(xch + 4 * 64);   // [step parity][half]
    int xc = 0;
    for (int i = pr; i < n_chunks; i += L::NP, ++xc) {
      const int slot = i % L::NS;
      bool both_ok;
      // both warps of the pair reach the pair barrier below on every step and
      // leave the loop together: a timed-out wait still takes part in the
      // exchange (its S is junk) and both warps then see the failure
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[slot], (uint32_t)((i / L::NS) & 1), ctx));
      const uint8_t* st = ring + slot * L::STAGE;
      const float* sks = L::kscale(smem, slot);
      const float* svs = sks + L::CH;
      const int64_t sl0 = s_begin + (int64_t)i * L::CH;
      // S = Q K^T for this warp's 16 keys with the shared head-dim permutation
      // (see the header); four independent accumulation chains
      float s4[4][4] = {};
      const uint8_t* kraw = st + L::OFF_K;
#pragma unroll
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
          // range: row r of box kk/8, 16-byte unit (kk%8) ^ (r%8) (128-byte swizzle)
          const int r = 16 * hf + nt * 8 + g;
          const int koff = RANGE ? (kk >> 3) * L::BOX + r * 128 + (((kk & 7) ^ g) << 4) + 4 * t
                                 : r * L::KROW + d0;
          const uint32_t kw = *reinterpret_cast<const uint32_t*>(kraw + koff);
          mma_f16_16816(s4[(kk & 1) * 2 + nt], a, e4m3x2_to_f16x2((uint16_t)(kw & 0xffffu)),
                        e4m3x2_to_f16x2((uint16_t)(kw >> 16)));
        }
      }
      // n-tiles 0, 1: keys 0-15 (warp 0's); 2, 3: keys 16-31 (warp 1's)
      float s[4][4];
      {
        float4* mine = xch + ((xc & 1) * 2 + hf) * 64;
        const float4* other = xch + ((xc & 1) * 2 + (hf ^ 1)) * 64;
        const float4 w0 = make_float4(s4[0][0] + s4[2][0], s4[0][1] + s4[2][1], s4[0][2] + s4[2][2], s4[0][3] + s4[2][3]);
        const float4 w1 = make_float4(s4[1][0] + s4[3][0], s4[1][1] + s4[3][1], s4[1][2] + s4[3][2], s4[1][3] + s4[3][3]);
        mine[lane] = w0;
        mine[32 + lane] = w1;
        if (lane == 0) xok[(xc & 1) * 2 + hf] = ok ? 1 : 0;
        asm volatile("bar.sync %0, 64;" ::"r"(1 + pr) : "memory");
        const float4 v0 = other[lane], v1 = other[32 + lane];
        both_ok = ok && xok[(xc & 1) * 2 + (hf ^ 1)] != 0;
        const float4 t0 = hf ? v0 : w0, t1 = hf ? v1 : w1, t2 = hf ? w0 : v0, t3 = hf ? w1 : v1;
        s[0][0] = t0.x; s[0][1] = t0.y; s[0][2] = t0.z; s[0][3] = t0.w;
        s[1][0] = t1.x; s[1][1] = t1.y; s[1][2] = t1.z; s[1][3] = t1.w;
        s[2][0] = t2.x; s[2][1] = t2.y; s[2][2] = t2.z; s[2][3] = t2.w;
        s[3][0] = t3.x; s[3][1] = t3.y; s[3][2] = t3.z; s[3][3] = t3.w;
      }
      if (!both_ok) break;
      // positions of this thread's keys 8*nt + 2t + e (-1: empty slot)
      int32_t kpos[4][2];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int64_t sl = sl0 + nt * 8 + 2 * t + e;
          kpos[nt][e] = sl < s_end ? (RANGE ? (int32_t)sl : sidx[sl - s_begin]) : -1;
        }
      float x[4][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = nt * 8 + 2 * t + (e & 1);
          float v = s[nt][e] * (p.scale_log2 * qscale_inv * sks[key]);
          if (kpos[nt][e & 1] < 0) v = -INFINITY;
          x[nt][e] = v;
          if (e < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
        }
      if (RANGE) {                                   // each warp writes the logits of its own keys
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const int32_t pos = kpos[nt][0];
          if ((nt >> 1) == hf && pos >= 0) {
            const bool two = kpos[nt][1] >= 0;
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
      // P enters the f16 product as p * v_scale * 2^-vexp, vexp the exponent
      // of the largest V scale seen so far (raised, with an exact rescale of
      // O, when a stage brings a larger one): p <= 2^8 keeps it below 2^9,
      // and it no longer underflows when the scales themselves are small
      float vmx = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) vmx = fmaxf(vmx, svs[(j >> 1) * 8 + 2 * t + (j & 1)]);
      vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, 1));
      vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, 2));
      if (vmx > 0.f) {
        const int ev = (int)((__float_as_uint(vmx) >> 23) & 0xffu) - 127;   // floor(log2) of a normal scale
        if (ev > vexp) {
          if (vexp != kNoVexp) {
            const float r = ldexpf(1.f, vexp - ev);
#pragma unroll
            for (int j = 0; j < L::HD / 8; ++j) {
              o[j][0] *= r; o[j][1] *= r; o[j][2] *= r; o[j][3] *= r;
            }
          }
          vexp = ev;
          vinv = ldexpf(1.f, -ev);
        }
      }
      float pv[4][4];
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pe = fast_exp2(x[nt][e] - (e < 2 ? mu0 : mu1));
          if (e < 2) ls0 += pe; else ls1 += pe;
          pv[nt][e] = pe * (svs[nt * 8 + 2 * t + (e & 1)] * vinv);
        }
      l0 = l0 * al0 + ls0;
      l1 = l1 * al1 + ls1;
      if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
        for (int j = 0; j < L::HD / 8; ++j) {
          o[j][0] *= al0; o[j][1] *= al0;
          o[j][2] *= al1; o[j][3] *= al1;
        }
      }
      // O += P V over this warp's half of d, in two k-steps of 16 keys; B
      // fragments from the raw codes (see the header): per 32 bytes of d, 4
      // n-tiles j = 4*blk + 2*half + parity covering dims c0 + 2n + parity
      const uint32_t va = smem_u32(st + L::OFF_V);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        uint32_t ap[4];
        ap[0] = pack_f16x2(pv[2 * ks][0], pv[2 * ks][1]);
        ap[1] = pack_f16x2(pv[2 * ks][2], pv[2 * ks][3]);
        ap[2] = pack_f16x2(pv[2 * ks + 1][0], pv[2 * ks + 1][1]);
        ap[3] = pack_f16x2(pv[2 * ks + 1][2], pv[2 * ks + 1][3]);
        const int key = 16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int b2 = 0; b2 < L::HD / 32; ++b2) {
          const int blk = hf * (L::HD / 32) + b2;
          uint32_t r[4];
          const int vu = (blk & 3) * 2 + (lane >> 4);  // range: 16-byte unit within box blk/4
          ldsm_x4_t(r, RANGE ? va + (blk >> 2) * L::BOX + key * 128 + ((vu ^ (lane & 7)) << 4)
                             : va + key * L::VROW + blk * 32 + (lane >> 4) * 16);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t px = __byte_perm(r[2 * half], r[2 * half + 1], 0x6420);
            const uint32_t py = __byte_perm(r[2 * half], r[2 * half + 1], 0x7531);
            mma_f16_16816(o[4 * b2 + 2 * half], ap, e4m3x2_to_f16x2((uint16_t)(px & 0xffffu)),
                          e4m3x2_to_f16x2((uint16_t)(px >> 16)));
            mma_f16_16816(o[4 * b2 + 2 * half + 1], ap, e4m3x2_to_f16x2((uint16_t)(py & 0xffffu)),
                          e4m3x2_to_f16x2((uint16_t)(py >> 16)));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
  }

  // ---- merge the pairs into this CTA's partial (m, l, O) in shared memory
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();
  __shared__ int pexp[L::NP];
  float* cmb = reinterpret_cast<float*>(smem + L::Q_BYTES);    // [NP pairs] partials, O rows padded
  float* mine = cmb + L::NP * (L::PPART / 4);                   // merged partial of the CTA
  if (warp < L::NC) {
    const int pr = warp >> 1, hf = warp & 1;
    float* wpart = cmb + pr * (L::PPART / 4);
    if (t == 0 && hf == 0) {
      wpart[g] = m0;
      wpart[g + 8] = m1;
      wpart[16 + g] = l0;
      wpart[16 + g + 8] = l1;
      if (g == 0) pexp[pr] = vexp == kNoVexp ? 0 : vexp;
    }
    // n-tiles 2q and 2q+1 (q = 2*b2 + half) hold, for rows g and g+8, the four
    // consecutive dims c0 + 4t .. c0 + 4t + 3 (c0 = hf*HD + 16q): one float4 each
#pragma unroll
    for (int q = 0; q < L::HD / 16; ++q) {
      const int dcol = hf * L::HD + 16 * q + 4 * t;
      *reinterpret_cast<float4*>(wpart + 32 + g * L::PROW + dcol) =
          make_float4(o[2 * q][0], o[2 * q + 1][0], o[2 * q][1], o[2 * q + 1][1]);
      *reinterpret_cast<float4*>(wpart + 32 + (g + 8) * L::PROW + dcol) =
          make_float4(o[2 * q][2], o[2 * q + 1][2], o[2 * q][3], o[2 * q + 1][3]);
    }
  }
  // per-head merge factors of the pairs, once: fac[w][h] = 2^(m_w - M_h) for
  // l, times 2^vexp_w for O (undoing the pair's V-scale reference)
  __shared__ float fac[L::NP][16];
  __shared__ float cfac[8][16];
  __shared__ float cinv[16];
  __syncthreads();
  if (threadIdx.x < 16) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int w = 0; w < L::NP; ++w) M = fmaxf(M, cmb[w * (L::PPART / 4) + h]);
    float Ls = 0.f;
    for (int w = 0; w < L::NP; ++w) {
      const float mw = cmb[w * (L::PPART / 4) + h];
      const float f = (M == -INFINITY || mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
      fac[w][h] = f * ldexpf(1.f, pexp[w]);
      Ls += cmb[w * (L::PPART / 4) + 16 + h] * f;
    }
    float* dst = PARTIALS ? p.part + ((int64_t)b * p.splits + split) * (32 + 16 * D) : mine;
    dst[h] = M;
    dst[16 + h] = Ls;
  }
  __syncthreads();
  {
    float* dst = PARTIALS ? p.part + ((int64_t)b * p.splits + split) * (32 + 16 * D) : mine;
    for (int e4 = threadIdx.x; e4 < 16 * D / 4; e4 += blockDim.x) {
      const int h = (e4 * 4) / D;
      const int src = h * L::PROW + (e4 * 4) % D;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < L::NP; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(cmb + w * (L::PPART / 4) + 32 + src);
        const float f = fac[w][h];
        acc.x += v.x * f; acc.y += v.y * f; acc.z += v.z * f; acc.w += v.w * f;
      }
      reinterpret_cast<float4*>(dst + 32)[e4] = acc;
    }
  }
  if (!PARTIALS) {
    // ---- merge the cluster's partials through distributed shared memory
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int r = (int)cluster.block_rank();
    cluster.sync();
    if (threadIdx.x < 16) {
      const int h = threadIdx.x;
      float M = -INFINITY;
      for (int q = 0; q < C; ++q) M = fmaxf(M, cluster.map_shared_rank(mine, q)[h]);
      float Ls = 0.f;
      for (int q = 0; q < C; ++q) {
        const float* pq = cluster.map_shared_rank(mine, q);
        const float f = (M == -INFINITY || pq[h] == -INFINITY) ? 0.f : fast_exp2(pq[h] - M);
        cfac[q][h] = f;
        Ls += pq[16 + h] * f;
      }
      cinv[h] = Ls > 0.f ? 1.f / Ls : 0.f;
    }
    __syncthreads();
    const int hp = (16 + C - 1) / C;                 // heads merged by this CTA
    const int h0 = r * hp, h1 = min(min(16, h0 + hp), p.H);
    const int n4 = h1 > h0 ? (h1 - h0) * D / 4 : 0;
    for (int e4 = threadIdx.x; e4 < n4; e4 += blockDim.x) {
      const int h = h0 + (e4 * 4) / D;
      const int off4 = (h0 * D) / 4 + e4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < C; ++q) {
        const float4 v = reinterpret_cast<const float4*>(cluster.map_shared_rank(mine, q) + 32)[off4];
        const float f = cfac[q][h];
        acc.x += v.x * f; acc.y += v.y * f; acc.z += v.z * f; acc.w += v.w * f;
      }
      const float inv = cinv[h];
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(p.O + ((int64_t)b * p.H) * D + (int64_t)off4 * 4) = pk;
    }
    cluster.sync();                                    // peers read our partial until here
  }
}

}  // namespace hs2
