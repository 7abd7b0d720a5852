// libhs2.so: the C ABI declared in include/hs2.h.  Argument checks, workspace
// sizing, TMA tensor maps and kernel launches; all compute is in the kernels
// included below (one translation unit).
#include "hs2.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "attn16.cuh"
#include "bridge_append.cuh"
#include "block_select.cuh"
#include "bridge_gemm.cuh"
#include "common.cuh"
#include "decode_attn.cuh"
#include "fa_fwd.cuh"
#include "rope_swa.cuh"
#include "select_sigma.cuh"
#include "topk.cuh"
#include "topk_radix.cuh"
#include "topk_split.cuh"
#include "sparse_tc.cuh"

namespace hs2 {

__device__ unsigned g_status_word;

namespace {

constexpr int kMaxDevices = 64;
constexpr long long kDefaultSpin = 1ll << 40;   // the 4 s time cap bounds it
thread_local char g_err[512] = "";
long long g_spin[kMaxDevices];
unsigned* g_status_ptr[kMaxDevices];
int g_num_sms[kMaxDevices];
std::mutex g_mu;

hs2_status fail(hs2_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

#define HS2_CHECK(cond, status, ...)        \
  do {                                      \
    if (!(cond)) return fail(status, __VA_ARGS__); \
  } while (0)

hs2_status cuda_fail(cudaError_t e, const char* what) {
  return fail(HS2_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Per-device state: status-word address, SM count, spin limit.
hs2_status device_ctx(DevCtx* ctx, int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(HS2_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_status_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) return fail(HS2_ERR_UNSUPPORTED, "libhs2 is built for sm_100a (compute capability 10.x), device has %d.x", major);
    g_status_ptr[dev] = static_cast<unsigned*>(p);
    g_num_sms[dev] = sms;
  }
  ctx->status = g_status_ptr[dev];
  ctx->spin_limit = g_spin[dev] > 0 ? g_spin[dev] : kDefaultSpin;
  if (num_sms) *num_sms = g_num_sms[dev];
  return HS2_OK;
}

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [outer, inner] (row stride in elements), 128-byte swizzle.
hs2_status make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t stride_elems,
                         uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {stride_elems * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return HS2_OK;
}

// 3-D u8 tensor {inner, mid, outer} with byte strides (mid_stride, outer_stride),
// 128-byte swizzle; out-of-range boxes read as zeros.
hs2_status make_map_u8_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                          uint64_t mid_stride, uint64_t outer_stride, uint32_t box_inner, uint32_t box_mid) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {mid_stride, outer_stride};
  cuuint32_t box[3] = {box_inner, box_mid, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HS2_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return HS2_OK;
}

// ------------------------------------------------------------------ profiling
constexpr int kMaxProf = 4096;
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
thread_local bool g_prof_on = false;
thread_local int g_prof_n = 0;
thread_local ProfRec g_prof[kMaxProf];
thread_local int g_prof_events = 0;      // event pairs created so far (reused)

// Records the "before" event of the next launch on stream st.
void prof_begin(cudaStream_t st) {
  if (!g_prof_on || g_prof_n >= kMaxProf) return;
  ProfRec& r = g_prof[g_prof_n];
  if (g_prof_n >= g_prof_events) {
    cudaEventCreate(&r.a);
    cudaEventCreate(&r.b);
    ++g_prof_events;
  }
  cudaEventRecord(r.a, st);
}

hs2_status after_launch(const char* what, cudaStream_t st) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  if (g_prof_on) {
    if (g_prof_n < kMaxProf) {
      g_prof[g_prof_n].name = what;
      cudaEventRecord(g_prof[g_prof_n].b, st);
    }
    ++g_prof_n;
  }
  return HS2_OK;
}

// Raises a kernel's dynamic shared memory limit on the current device, once
// per (kernel, device, size): the attribute call costs microseconds of host
// time, which small decode launches would otherwise pay every call.
struct SmemSet {
  const void* kernel;
  int dev;
  size_t bytes;
};
constexpr int kMaxSmemSet = 256;
SmemSet g_smem_set[kMaxSmemSet];
int g_n_smem_set = 0;

template <typename K>
hs2_status set_smem(K kernel, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const void* kp = reinterpret_cast<const void*>(kernel);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_n_smem_set; ++i)
      if (g_smem_set[i].kernel == kp && g_smem_set[i].dev == dev && g_smem_set[i].bytes >= bytes) return HS2_OK;
  }
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_n_smem_set; ++i)
    if (g_smem_set[i].kernel == kp && g_smem_set[i].dev == dev) {
      if (bytes > g_smem_set[i].bytes) g_smem_set[i].bytes = bytes;
      return HS2_OK;
    }
  if (g_n_smem_set < kMaxSmemSet) g_smem_set[g_n_smem_set++] = {kp, dev, bytes};
  return HS2_OK;
}

bool shape_ok(int Hq, int d) { return (Hq == 8 || Hq == 16) && (d == 128 || d == 256); }

// ------------------------------------------------------------------ workspace
struct PrefillWs {
  size_t ml, sigma, total;
  int64_t ld;
};
PrefillWs prefill_ws(int64_t Tq, int64_t kv_len, int Hq) {
  PrefillWs w;
  w.ld = round_up(kv_len, 64);
  w.ml = up256((size_t)Tq * Hq * 2 * sizeof(float));
  w.sigma = up256((size_t)Tq * (size_t)w.ld * sizeof(float));
  w.total = w.ml + w.sigma;
  return w;
}

constexpr int kDecodeKeysPerSplit = 2048;   // the smallest split; workspaces are sized for it

// Keys per CTA of the decode full-attention pass.  One CTA runs per SM, and a
// CTA's start-up and partial merge cost about as much as streaming ~300 more
// keys, so the split is the one of 2048, 4096 or 8192 keys that minimises
// waves x (keys + 300); ties keep the smaller split.  (Measured: 64 sequences
// of 131072 keys run 6% faster with 8192 than with 2048, 4 sequences of 2^20
// 9% faster with 4096, 4 context shards of 2^18 fastest with 8192.)
int decode_split_keys(int batch, int64_t kv_len, int sms) {
  int best = kDecodeKeysPerSplit;
  double best_t = 1e300;
  for (int per = kDecodeKeysPerSplit; per <= 4 * kDecodeKeysPerSplit; per *= 2) {
    const int64_t ctas = (int64_t)batch * ((kv_len + per - 1) / per);
    const double t = (double)((ctas + sms - 1) / sms) * (double)(per + 300);
    if (t < best_t) {
      best_t = t;
      best = per;
    }
  }
  return best;
}


// Decode rows of more than this many candidates take the grid-wide radix
// select (topk_radix.cuh): a few long rows otherwise leave most SMs idle.
constexpr int64_t kRadixMinCand = 4 * TS_SLICE;
int radix_chunks(int64_t n, int k) {
  return (n > kRadixMinCand && n > k) ? (int)((n + RX_CHUNK - 1) / RX_CHUNK) : 0;
}
size_t radix_bytes(int batch, int chunks) {
  return chunks ? up256((size_t)batch * RX_HIST * 4) + up256((size_t)batch * chunks * 8) : 0;
}

// The five radix-select launches over rp.chunks x batch CTAs (the histograms
// were zeroed by decode_sigma_kernel).
hs2_status launch_radix(const RadixParams& rp, int batch, cudaStream_t st, const DevCtx& ctx) {
  const dim3 g((unsigned)rp.chunks, (unsigned)batch);
  hs2_status s;
  prof_begin(st);
  radix_hist_kernel<0><<<g, RX_THREADS, 0, st>>>(rp, ctx);
  if ((s = after_launch("radix_hist_kernel", st)) != HS2_OK) return s;
  prof_begin(st);
  radix_hist_kernel<1><<<g, RX_THREADS, 0, st>>>(rp, ctx);
  if ((s = after_launch("radix_hist_kernel", st)) != HS2_OK) return s;
  prof_begin(st);
  radix_hist_kernel<2><<<g, RX_THREADS, 0, st>>>(rp, ctx);
  if ((s = after_launch("radix_hist_kernel", st)) != HS2_OK) return s;
  prof_begin(st);
  radix_count_kernel<<<g, RX_THREADS, 0, st>>>(rp, ctx);
  if ((s = after_launch("radix_count_kernel", st)) != HS2_OK) return s;
  prof_begin(st);
  radix_write_kernel<<<g, RX_THREADS, 0, st>>>(rp, ctx);
  return after_launch("radix_write_kernel", st);
}

struct DecodeWs {
  size_t logits, part, ml, sigma, radix, total;
  int64_t ld;
  int splits;        // key splits of the full-attention pass (at the smallest split)
  int rx_chunks;     // chunks of the radix select (0: one CTA per row)
};
DecodeWs decode_ws(int batch, int64_t kv_len, int Hq, int d, int window, int topk) {
  DecodeWs w;
  w.ld = round_up(kv_len, 64);
  w.splits = (int)((kv_len + kDecodeKeysPerSplit - 1) / kDecodeKeysPerSplit);
  w.rx_chunks = radix_chunks(std::max<int64_t>(0, kv_len - window), topk);
  w.radix = radix_bytes(batch, w.rx_chunks);
  w.logits = up256((size_t)batch * Hq * (size_t)w.ld * sizeof(float));
  w.part = up256((size_t)batch * w.splits * (32 + 16 * (size_t)d) * sizeof(float));
  w.ml = up256((size_t)batch * Hq * 2 * sizeof(float));
  w.sigma = up256((size_t)batch * (size_t)w.ld * sizeof(float));
  w.total = w.logits + w.part + w.ml + w.sigma + w.radix;
  return w;
}

// CTAs per sequence of the sparse decode.  Up to 8 they form one thread-block
// cluster and merge in distributed shared memory (no workspace); a batch too
// small to fill the GPU that way uses more splits and a workspace.
constexpr int kMaxCluster = 8;
int sparse_decode_splits(int batch, int n_idx, int num_sms) {
  const int max_s = std::max(1, (n_idx + 63) / 64);
  int s = num_sms / batch;
  if (s <= kMaxCluster) return std::max(1, std::min(s, std::min(max_s, kMaxCluster)));
  return std::min((num_sms + batch - 1) / batch, max_s);
}

// ------------------------------------------------------------------ launches
template <int D>
hs2_status launch_combine(const float* part, int splits, int H, __nv_bfloat16* O, float* ml, int items,
                          cudaStream_t st, float* O32 = nullptr) {
  if (splits > kCombineMaxSplits) return fail(HS2_ERR_UNSUPPORTED, "%d split partials (at most %d)", splits, kCombineMaxSplits);
  prof_begin(st);
  if (splits >= kCombineManySplits)
    attn16_combine_kernel<D, 4><<<dim3(items, H), D * 4, 0, st>>>(part, splits, H, O, ml, O32);
  else
    attn16_combine_kernel<D, 1><<<dim3(items, H), D, 0, st>>>(part, splits, H, O, ml, O32);
  return after_launch("attn16_combine_kernel", st);
}

// Rows of up to 1920 keys run on the tensor cores (sparse_tc_kernel, one CTA
// per SM); longer ones on the warp-pair kernel (4 rows per SM).
template <int D>
hs2_status launch_sparse_prefill(const Attn16Params& p, int sms, cudaStream_t st, const DevCtx& ctx) {
  hs2_status s;
  if ((p.n_idx + 127) / 128 <= StcLayout<D>::MAXT) {
    if ((s = set_smem(sparse_tc_kernel<D>, StcLayout<D>::SMEM)) != HS2_OK) return s;
    const int grid = (int)std::min<int64_t>(p.n_rows, sms);
    prof_begin(st);
    sparse_tc_kernel<D><<<grid, StcLayout<D>::NT, StcLayout<D>::SMEM, st>>>(p, ctx);
    return after_launch("sparse_tc_kernel", st);
  }
  if ((s = set_smem(sparse_prefill_kernel<D>, SpfLayout<D>::SMEM)) != HS2_OK) return s;
  const int grid = (int)std::min<int64_t>((p.n_rows + SpfLayout<D>::NPAIR - 1) / SpfLayout<D>::NPAIR, sms);
  prof_begin(st);
  sparse_prefill_kernel<D><<<grid, SpfLayout<D>::NT, SpfLayout<D>::SMEM, st>>>(p, ctx);
  return after_launch("sparse_prefill_kernel", st);
}

template <int D>
hs2_status launch_decode_parts(const DecParams& p, int batch, cudaStream_t st, const DevCtx& ctx) {
  using L = DecLayout<D, false>;
  auto k = decode_attn_kernel<D, false, true>;
  hs2_status s = set_smem(k, L::SMEM);
  if (s != HS2_OK) return s;
  const CUtensorMap unused{};
  prof_begin(st);
  k<<<batch * p.splits, L::NT, L::SMEM, st>>>(p, ctx, unused, unused);
  return after_launch("decode_attn_kernel", st);
}

// One thread-block cluster of p.splits CTAs per sequence.
template <int D>
hs2_status launch_decode_cluster(const DecParams& p, int batch, cudaStream_t st, const DevCtx& ctx) {
  using L = DecLayout<D, false>;
  auto k = decode_attn_kernel<D, false, false>;
  hs2_status s = set_smem(k, L::SMEM);
  if (s != HS2_OK) return s;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(batch * p.splits));
  cfg.blockDim = dim3(L::NT);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_begin(st);
  const CUtensorMap unused{};
  cudaError_t e = cudaLaunchKernelEx(&cfg, k, p, ctx, unused, unused);
  if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx(decode_attn_kernel)");
  return after_launch("decode_attn_kernel", st);
}

// The last stage of a full layer: top-k tokens (block == 0) or top-k blocks
// of `block` tokens per row, from the selection scores in the workspace.
hs2_status launch_select(const float* sigma, int64_t ld, int64_t p0, int64_t pstep, int window, int topk, int block,
                         int32_t* idx, int64_t rows, cudaStream_t st, const DevCtx& ctx) {
  hs2_status s;
  if (block == 0) {
    TopkParams tp;
    tp.sigma = sigma;
    tp.ld = ld;
    tp.p0 = p0;
    tp.pstep = pstep;
    tp.window = window;
    tp.topk = topk;
    tp.idx = idx;
    if ((s = set_smem(topk_select_kernel, TK_SMEM)) != HS2_OK) return s;
    prof_begin(st);
    topk_select_kernel<<<(unsigned)rows, TK_THREADS, TK_SMEM, st>>>(tp, ctx);
    return after_launch("topk_select_kernel", st);
  }
  BlockSelParams bp;
  bp.sigma = sigma;
  bp.ld = ld;
  bp.p0 = p0;
  bp.pstep = pstep;
  bp.window = window;
  bp.block = block;
  bp.topk_blocks = topk;
  // the last row has the most candidates (prefill: the largest position; decode: all rows alike)
  bp.nb_max = (int)((std::max<int64_t>(0, p0 + (rows - 1) * pstep - window + 1) + block - 1) / block);
  bp.idx = idx;
  const size_t smem = bs_smem(bp.nb_max);
  if ((s = set_smem(block_select_kernel, smem)) != HS2_OK) return s;
  prof_begin(st);
  block_select_kernel<<<(unsigned)rows, BS_THREADS, smem, st>>>(bp, ctx);
  return after_launch("block_select_kernel", st);
}

template <int D>
hs2_status prefill_select(const void* Q, const void* K, const void* V, int64_t q_start, int64_t Tq, int64_t kv_len,
                          int Hq, int window, int topk, int block, float scale, void* O, int32_t* idx, void* ws,
                          cudaStream_t st, const DevCtx& ctx) {
  const PrefillWs w = prefill_ws(Tq, kv_len, Hq);
  float* ml = reinterpret_cast<float*>(ws);
  float* sigma = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.ml);
  const float sl2 = scale * 1.4426950408889634f;
  CUtensorMap mQ, mQ256, mK, mV;
  hs2_status s;
  if ((s = make_map_bf16(&mQ, Q, D, (uint64_t)Tq * Hq, D, 64, 128)) != HS2_OK) return s;
  if ((s = make_map_bf16(&mQ256, Q, D, (uint64_t)Tq * Hq, D, 64, 256)) != HS2_OK) return s;
  if ((s = make_map_bf16(&mK, K, D, (uint64_t)kv_len, D, 64, 128)) != HS2_OK) return s;
  if ((s = make_map_bf16(&mV, V, D, (uint64_t)kv_len, D, 64, 128)) != HS2_OK) return s;

  FaParams fp;
  fp.Tq = Tq;
  fp.q_start = q_start;
  fp.kv_len = kv_len;
  fp.H = Hq;
  fp.scale_log2 = sl2;
  fp.O = static_cast<__nv_bfloat16*>(O);
  fp.ml = ml;
  fp.n_qtiles = (int)((Tq * Hq + 127) / 128);
  fp.window = 0;
  if ((s = set_smem(fa_fwd_kernel<D>, FaLayout<D>::SMEM)) != HS2_OK) return s;
  prof_begin(st);
  fa_fwd_kernel<D><<<fp.n_qtiles, FA_THREADS, FaLayout<D>::SMEM, st>>>(mQ, mK, mV, fp, ctx);
  if ((s = after_launch("fa_fwd_kernel", st)) != HS2_OK) return s;

  SgParams sp;
  sp.Tq = Tq;
  sp.q_start = q_start;
  sp.kv_len = kv_len;
  sp.H = Hq;
  sp.window = window;
  sp.scale_log2 = sl2;
  sp.ml = ml;
  sp.sigma = sigma;
  sp.ld = w.ld;
  sp.n_groups = (int)((Tq * Hq + 255) / 256);
  if (Hq == 16) {
    if ((s = set_smem(select_sigma_kernel<D, 16>, SgLayout<D>::SMEM)) != HS2_OK) return s;
    prof_begin(st);
    select_sigma_kernel<D, 16><<<sp.n_groups, SG_THREADS, SgLayout<D>::SMEM, st>>>(mQ256, mK, sp, ctx);
  } else {
    if ((s = set_smem(select_sigma_kernel<D, 8>, SgLayout<D>::SMEM)) != HS2_OK) return s;
    prof_begin(st);
    select_sigma_kernel<D, 8><<<sp.n_groups, SG_THREADS, SgLayout<D>::SMEM, st>>>(mQ256, mK, sp, ctx);
  }
  if ((s = after_launch("select_sigma_kernel", st)) != HS2_OK) return s;
  return launch_select(sigma, w.ld, q_start, 1, window, topk, block, idx, Tq, st, ctx);
}

template <int D>
hs2_status decode_select(const void* Q, const void* K, const void* V, const float* ks, const float* vs, int batch,
                         int64_t kv_len, int64_t kv_stride, int Hq, int window, int topk, int block, float scale,
                         void* O, int32_t* idx, void* ws, int sms, cudaStream_t st, const DevCtx& ctx) {
  const DecodeWs w = decode_ws(batch, kv_len, Hq, D, window, topk);
  const int per = decode_split_keys(batch, kv_len, sms);
  const int splits = (int)((kv_len + per - 1) / per);
  uint8_t* b = static_cast<uint8_t*>(ws);
  float* logits = reinterpret_cast<float*>(b);
  float* part = reinterpret_cast<float*>(b + w.logits);
  float* ml = reinterpret_cast<float*>(b + w.logits + w.part);
  float* sigma = reinterpret_cast<float*>(b + w.logits + w.part + w.ml);
  DecParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const uint8_t*>(K);
  p.V = static_cast<const uint8_t*>(V);
  p.ks = ks;
  p.vs = vs;
  p.kv_len = kv_len;
  p.kv_stride = kv_stride;
  p.H = Hq;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.splits = splits;
  p.per_split = per;
  p.part = part;
  p.logits = logits;
  p.logit_ld = w.ld;
  p.idx_offset = -1;
  using L = DecLayout<D, true>;
  auto k = decode_attn_kernel<D, true, true>;
  hs2_status s = set_smem(k, L::SMEM);
  if (s != HS2_OK) return s;
  CUtensorMap mK, mV;   // {D, kv_len, batch} codes; keys past kv_len read as zeros
  if ((s = make_map_u8_3d(&mK, K, D, (uint64_t)kv_len, (uint64_t)batch, D, (uint64_t)kv_stride * D, 128,
                          L::CH)) != HS2_OK)
    return s;
  if ((s = make_map_u8_3d(&mV, V, D, (uint64_t)kv_len, (uint64_t)batch, D, (uint64_t)kv_stride * D, 128,
                          L::CH)) != HS2_OK)
    return s;
  prof_begin(st);
  k<<<batch * splits, L::NT, L::SMEM, st>>>(p, ctx, mK, mV);
  if ((s = after_launch("decode_attn_kernel", st)) != HS2_OK) return s;
  if ((s = launch_combine<D>(part, splits, Hq, static_cast<__nv_bfloat16*>(O), ml, batch, st)) != HS2_OK) return s;
  const int64_t n_cand = std::max<int64_t>(0, kv_len - window);
  const bool radix = block == 0 && w.rx_chunks > 0;
  uint32_t* rx_hist = reinterpret_cast<uint32_t*>(b + w.logits + w.part + w.ml + w.sigma);
  if (n_cand > 0) {
    dim3 g((unsigned)((n_cand + 1023) / 1024), (unsigned)batch);
    prof_begin(st);
    decode_sigma_kernel<<<g, 256, 0, st>>>(logits, w.ld, ml, Hq, n_cand, sigma, w.ld, radix ? rx_hist : nullptr,
                                           RX_HIST);
    if ((s = after_launch("decode_sigma_kernel", st)) != HS2_OK) return s;
  }
  if (radix) {
    // few rows of many candidates: the radix select over the whole GPU
    RadixParams rp{};
    rp.sigma = sigma;
    rp.ld = w.ld;
    rp.n = n_cand;
    rp.chunks = w.rx_chunks;
    rp.topk = topk;
    rp.window = window;
    rp.pos = kv_len - 1;
    rp.pos_offset = 0;
    rp.hist = rx_hist;
    rp.cnt = rx_hist + up256((size_t)batch * RX_HIST * 4) / 4;
    rp.idx = idx;
    return launch_radix(rp, batch, st, ctx);
  }
  return launch_select(sigma, w.ld, kv_len - 1, 0, window, topk, block, idx, batch, st, ctx);
}

struct SwaWs {
  size_t q, k, table, total;
};
SwaWs swa_ws(int64_t Tq, int64_t kv_len, int Hq, int d, int rope_dims) {
  SwaWs w;
  w.q = up256((size_t)Tq * Hq * d * 2);
  w.k = up256((size_t)kv_len * d * 2);
  w.table = up256((size_t)kv_len * (rope_dims / 2) * sizeof(float2));
  w.total = w.q + w.k + w.table;
  return w;
}

// Sliding-window attention of the self-decoder: RoPE on Q and K into the
// workspace, then the full-attention kernel over each query's window.
template <int D>
hs2_status swa_attn(const void* Q, const void* K, const void* V, int64_t q_start, int64_t Tq, int64_t kv_len, int Hq,
                    int window, int rope_dims, float rope_base, float scale, void* O, void* ws, cudaStream_t st,
                    const DevCtx& ctx) {
  const SwaWs w = swa_ws(Tq, kv_len, Hq, D, rope_dims);
  uint8_t* b = static_cast<uint8_t*>(ws);
  __nv_bfloat16* Qr = reinterpret_cast<__nv_bfloat16*>(b);
  __nv_bfloat16* Kr = reinterpret_cast<__nv_bfloat16*>(b + w.q);
  float2* cs = reinterpret_cast<float2*>(b + w.q + w.k);
  const int half = rope_dims / 2;
  hs2_status s;
  prof_begin(st);
  rope_table_kernel<<<(unsigned)((kv_len * half + 255) / 256), 256, 0, st>>>(cs, kv_len, half, (double)rope_base);
  if ((s = after_launch("rope_table_kernel", st)) != HS2_OK) return s;
  prof_begin(st);
  rope_rows_kernel<D><<<(unsigned)((Tq * Hq + 7) / 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(Q), Qr,
                                                                      Tq * Hq, q_start, Hq, cs, half);
  if ((s = after_launch("rope_rows_kernel", st)) != HS2_OK) return s;
  prof_begin(st);
  rope_rows_kernel<D><<<(unsigned)((kv_len + 7) / 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(K), Kr, kv_len,
                                                                     0, 1, cs, half);
  if ((s = after_launch("rope_rows_kernel", st)) != HS2_OK) return s;
  CUtensorMap mQ, mK, mV;
  if ((s = make_map_bf16(&mQ, Qr, D, (uint64_t)Tq * Hq, D, 64, 128)) != HS2_OK) return s;
  if ((s = make_map_bf16(&mK, Kr, D, (uint64_t)kv_len, D, 64, 128)) != HS2_OK) return s;
  if ((s = make_map_bf16(&mV, V, D, (uint64_t)kv_len, D, 64, 128)) != HS2_OK) return s;
  FaParams fp;
  fp.Tq = Tq;
  fp.q_start = q_start;
  fp.kv_len = kv_len;
  fp.H = Hq;
  fp.scale_log2 = scale * 1.4426950408889634f;
  fp.O = static_cast<__nv_bfloat16*>(O);
  fp.ml = nullptr;
  fp.n_qtiles = (int)((Tq * Hq + 127) / 128);
  fp.window = window;
  if ((s = set_smem(fa_fwd_kernel<D>, FaLayout<D>::SMEM)) != HS2_OK) return s;
  prof_begin(st);
  fa_fwd_kernel<D><<<fp.n_qtiles, FA_THREADS, FaLayout<D>::SMEM, st>>>(mQ, mK, mV, fp, ctx);
  return after_launch("fa_fwd_kernel", st);
}

// ---- context-sharded decode: one shard of every sequence's cache per GPU
struct ShardWs {
  size_t logits, part, sigma, lists, radix, total;
  int64_t ld;
  int splits;      // key splits of the shard's full-attention pass
  int tk_splits;   // slices of the shard's candidates
  int rx_chunks;   // chunks of the radix select over them (0: the slices)
};
// Slices of a shard's candidates: the slices' lists must merge in one CTA.
int shard_slices(int64_t n, int k) {
  int64_t S = std::max<int64_t>(1, (n + TS_SLICE - 1) / TS_SLICE);
  if (S > 1 && S * k > TS_CAP) S = std::max<int64_t>(1, TS_CAP / k);
  return (int)S;
}
ShardWs shard_ws(int batch, int64_t shard_len, int Hq, int d, int topk) {
  ShardWs w;
  w.ld = round_up(shard_len, 64);
  w.splits = (int)((shard_len + kDecodeKeysPerSplit - 1) / kDecodeKeysPerSplit);
  w.tk_splits = shard_slices(shard_len, topk);
  w.logits = up256((size_t)batch * Hq * (size_t)w.ld * sizeof(float));
  w.part = up256((size_t)batch * w.splits * (32 + 16 * (size_t)d) * sizeof(float));
  w.sigma = up256((size_t)batch * (size_t)w.ld * sizeof(float));
  w.lists = up256((size_t)batch * w.tk_splits * ((size_t)topk * 8 + 4));
  w.rx_chunks = radix_chunks(shard_len, topk);
  w.radix = radix_bytes(batch, w.rx_chunks);
  w.total = w.logits + w.part + w.sigma + w.lists + w.radix;
  return w;
}

template <int D>
hs2_status shard_attn(const void* Q, const void* K, const void* V, const float* ks, const float* vs, int batch,
                      int64_t shard_len, int64_t kv_stride, int Hq, float scale, float* ml_out, float* O_out,
                      void* ws, int topk, int sms, cudaStream_t st, const DevCtx& ctx) {
  const ShardWs w = shard_ws(batch, shard_len, Hq, D, topk);
  const int per = decode_split_keys(batch, shard_len, sms);
  const int splits = (int)((shard_len + per - 1) / per);
  uint8_t* b = static_cast<uint8_t*>(ws);
  DecParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const uint8_t*>(K);
  p.V = static_cast<const uint8_t*>(V);
  p.ks = ks;
  p.vs = vs;
  p.kv_len = shard_len;
  p.kv_stride = kv_stride;
  p.H = Hq;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.splits = splits;
  p.per_split = per;
  p.part = reinterpret_cast<float*>(b + w.logits);
  p.logits = reinterpret_cast<float*>(b);
  p.logit_ld = w.ld;
  p.idx_offset = -1;
  using L = DecLayout<D, true>;
  auto k = decode_attn_kernel<D, true, true>;
  hs2_status s = set_smem(k, L::SMEM);
  if (s != HS2_OK) return s;
  CUtensorMap mK, mV;
  if ((s = make_map_u8_3d(&mK, K, D, (uint64_t)shard_len, (uint64_t)batch, D, (uint64_t)kv_stride * D, 128,
                          L::CH)) != HS2_OK)
    return s;
  if ((s = make_map_u8_3d(&mV, V, D, (uint64_t)shard_len, (uint64_t)batch, D, (uint64_t)kv_stride * D, 128,
                          L::CH)) != HS2_OK)
    return s;
  prof_begin(st);
  k<<<batch * splits, L::NT, L::SMEM, st>>>(p, ctx, mK, mV);
  if ((s = after_launch("decode_attn_kernel", st)) != HS2_OK) return s;
  return launch_combine<D>(p.part, splits, Hq, nullptr, ml_out, batch, st, O_out);
}

template <int D>
hs2_status shard_sparse(const DecParams& p0, int batch, int n_idx, int sms, float* ml_out, float* O_out, void* ws,
                        cudaStream_t st, const DevCtx& ctx) {
  DecParams p = p0;
  int splits = sparse_decode_splits(batch, n_idx, sms);
  p.splits = splits;
  p.per_split = (n_idx + splits - 1) / splits;
  p.part = static_cast<float*>(ws);
  hs2_status s = launch_decode_parts<D>(p, batch, st, ctx);
  if (s != HS2_OK) return s;
  return launch_combine<D>(p.part, splits, p.H, nullptr, ml_out, batch, st, O_out);
}

template <int D>
hs2_status launch_partial(bool finalize, const float* ml, int R, int shard, float* O32, float* ml_out,
                          __nv_bfloat16* O, int batch, int H, cudaStream_t st) {
  prof_begin(st);
  if (finalize) {
    partial_finalize_kernel<D><<<dim3(batch, H), D, 0, st>>>(ml, O32, O, H);
    return after_launch("partial_finalize_kernel", st);
  }
  partial_merge_kernel<D><<<dim3(batch, H), D, 0, st>>>(ml, R, shard, O32, ml_out, H);
  return after_launch("partial_merge_kernel", st);
}

}  // namespace
}  // namespace hs2

using namespace hs2;

extern "C" {

const char* hs2_status_string(hs2_status s) {
  switch (s) {
    case HS2_OK: return "HS2_OK";
    case HS2_ERR_INVALID_ARG: return "HS2_ERR_INVALID_ARG";
    case HS2_ERR_UNSUPPORTED: return "HS2_ERR_UNSUPPORTED";
    case HS2_ERR_WORKSPACE: return "HS2_ERR_WORKSPACE";
    case HS2_ERR_CUDA: return "HS2_ERR_CUDA";
    case HS2_ERR_TIMEOUT: return "HS2_ERR_TIMEOUT";
    case HS2_ERR_DEVICE_CHECK: return "HS2_ERR_DEVICE_CHECK";
  }
  return "unknown hs2_status";
}

const char* hs2_last_error(void) { return g_err; }

const char* hs2_version(void) { return "hs2 0.1 sm_100a"; }

hs2_status hs2_bridge_kv(const void* hidden, int64_t rows, int hidden_dim, const void* Wk, const void* Wv, int d,
                         hs2_kv_dtype out_dtype, void* K_out, void* V_out, float* k_scale, float* v_scale,
                         void* stream) {
  g_err[0] = 0;
  HS2_CHECK(hidden && Wk && Wv && K_out && V_out, HS2_ERR_INVALID_ARG, "null tensor pointer");
  HS2_CHECK(aligned16(hidden) && aligned16(Wk) && aligned16(Wv) && aligned16(K_out) && aligned16(V_out),
            HS2_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  HS2_CHECK(rows >= 1 && rows < (1ll << 31), HS2_ERR_INVALID_ARG, "rows = %lld out of range", (long long)rows);
  HS2_CHECK(hidden_dim > 0 && hidden_dim % 64 == 0, HS2_ERR_INVALID_ARG, "hidden_dim must be a positive multiple of 64");
  HS2_CHECK(out_dtype == HS2_KV_BF16 || out_dtype == HS2_KV_FP8_E4M3, HS2_ERR_INVALID_ARG, "bad out_dtype");
  HS2_CHECK(d == 256, HS2_ERR_UNSUPPORTED, "bridging supports d == 256 (got %d)", d);
  if (out_dtype == HS2_KV_FP8_E4M3) {
    HS2_CHECK(k_scale && v_scale && aligned4(k_scale) && aligned4(v_scale), HS2_ERR_INVALID_ARG,
              "FP8 output needs 4-byte aligned k_scale and v_scale");
  } else {
    HS2_CHECK(!k_scale && !v_scale, HS2_ERR_INVALID_ARG, "bf16 output takes no scales");
  }
  DevCtx ctx;
  int sms = 0;
  hs2_status s = device_ctx(&ctx, &sms);
  if (s != HS2_OK) return s;
  CUtensorMap mA, mWk, mWv;
  if ((s = make_map_bf16(&mA, hidden, hidden_dim, rows, hidden_dim, 64, 128)) != HS2_OK) return s;
  if ((s = make_map_bf16(&mWk, Wk, hidden_dim, 256, hidden_dim, 64, 256)) != HS2_OK) return s;
  if ((s = make_map_bf16(&mWv, Wv, hidden_dim, 256, hidden_dim, 64, 256)) != HS2_OK) return s;
  BridgeParams p;
  p.rows = rows;
  p.kdim = hidden_dim;
  p.out_fp8 = out_dtype == HS2_KV_FP8_E4M3;
  p.K_out = K_out;
  p.V_out = V_out;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.num_tiles = (int)(2 * ((rows + BG_BM - 1) / BG_BM));
  if ((s = set_smem(bridge_gemm_kernel, BG_SMEM)) != HS2_OK) return s;
  const int grid = std::min(p.num_tiles, sms);
  prof_begin(static_cast<cudaStream_t>(stream));
  bridge_gemm_kernel<<<grid, BG_THREADS, BG_SMEM, static_cast<cudaStream_t>(stream)>>>(mA, mWk, mWv, p, ctx);
  return after_launch("bridge_gemm_kernel", static_cast<cudaStream_t>(stream));
}

hs2_status hs2_bridge_append(const void* hidden, int batch, int hidden_dim, const void* Wk, const void* Wv, int d,
                             void* Kc, void* Vc, float* k_scale, float* v_scale, int64_t kv_stride_tokens,
                             const int32_t* pos, void* stream) {
  g_err[0] = 0;
  HS2_CHECK(hidden && Wk && Wv && Kc && Vc && k_scale && v_scale && pos, HS2_ERR_INVALID_ARG, "null pointer");
  HS2_CHECK(aligned16(hidden) && aligned16(Wk) && aligned16(Wv) && aligned16(Kc) && aligned16(Vc) &&
                aligned4(k_scale) && aligned4(v_scale) && aligned4(pos),
            HS2_ERR_INVALID_ARG, "misaligned pointer");
  HS2_CHECK(batch >= 1 && batch <= 65535, HS2_ERR_INVALID_ARG, "batch = %d out of range", batch);
  HS2_CHECK(hidden_dim > 0 && hidden_dim % 256 == 0, HS2_ERR_INVALID_ARG, "hidden_dim must be a positive multiple of 256");
  HS2_CHECK(d == 256, HS2_ERR_UNSUPPORTED, "bridging supports d == 256 (got %d)", d);
  HS2_CHECK(kv_stride_tokens >= 1, HS2_ERR_INVALID_ARG, "kv_stride_tokens must be >= 1");
  DevCtx ctx;
  hs2_status s = device_ctx(&ctx, nullptr);
  if (s != HS2_OK) return s;
  AppendParams p;
  p.hidden = static_cast<const __nv_bfloat16*>(hidden);
  p.Wk = static_cast<const __nv_bfloat16*>(Wk);
  p.Wv = static_cast<const __nv_bfloat16*>(Wv);
  p.kdim = hidden_dim;
  p.Kc = static_cast<uint8_t*>(Kc);
  p.Vc = static_cast<uint8_t*>(Vc);
  p.ks = k_scale;
  p.vs = v_scale;
  p.stride = kv_stride_tokens;
  p.pos = pos;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  prof_begin(st);
  bridge_append_kernel<<<dim3(BA_CLUSTER, 2, (unsigned)batch), BA_THREADS, 0, st>>>(p, ctx);
  return after_launch("bridge_append_kernel", st);
}

hs2_status hs2_full_attn_select_workspace(hs2_kv_dtype kv_dtype, int batch, int64_t Tq, int64_t kv_len, int Hq,
                                          int d, int window, int topk, size_t* bytes) {
  g_err[0] = 0;
  HS2_CHECK(bytes, HS2_ERR_INVALID_ARG, "bytes is null");
  HS2_CHECK(batch >= 1 && Tq >= 1 && kv_len >= 1 && window >= 1 && topk >= 1, HS2_ERR_INVALID_ARG, "bad sizes");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  if (kv_dtype == HS2_KV_BF16) {
    *bytes = prefill_ws(Tq, kv_len, Hq).total;
  } else if (kv_dtype == HS2_KV_FP8_E4M3) {
    *bytes = decode_ws(batch, kv_len, Hq, d, window, topk).total;
  } else {
    return fail(HS2_ERR_INVALID_ARG, "bad kv_dtype");
  }
  return HS2_OK;
}

}  // extern "C"

namespace hs2 {
namespace {
// hs2_full_attn_select (block == 0: topk tokens) and
// hs2_full_attn_select_blocks (topk blocks of `block` tokens).
hs2_status full_attn_select_impl(const void* Q, const void* K, const void* V, const float* k_scale,
                                 const float* v_scale, hs2_kv_dtype kv_dtype, int batch, int64_t q_start, int64_t Tq,
                                 int64_t kv_len, int64_t kv_stride_tokens, int Hq, int d, int window, int topk,
                                 int block, float softmax_scale, void* O, int32_t* idx, void* workspace,
                                 size_t ws_bytes, void* stream) {
  HS2_CHECK(Q && K && V && O && idx, HS2_ERR_INVALID_ARG, "null tensor pointer");
  HS2_CHECK(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O) && aligned16(idx), HS2_ERR_INVALID_ARG,
            "tensor pointers must be 16-byte aligned");
  HS2_CHECK(batch >= 1 && Tq >= 1 && kv_len >= 1 && q_start >= 0, HS2_ERR_INVALID_ARG, "bad sizes");
  HS2_CHECK(window >= 1 && topk >= 1, HS2_ERR_INVALID_ARG, "window and topk must be >= 1");
  const int64_t sel_width = (int64_t)topk * (block ? block : 1);
  HS2_CHECK(window + sel_width <= 2048, HS2_ERR_UNSUPPORTED, "the index row (window + selection) must be <= 2048");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256 (got %d, %d)", Hq, d);
  if (block) {
    HS2_CHECK(block >= 16 && block <= 256 && (block & (block - 1)) == 0, HS2_ERR_UNSUPPORTED,
              "block must be a power of two in [16, 256] (got %d)", block);
    HS2_CHECK((kv_len - window + block - 1) / block <= BS_MAX_BLOCKS, HS2_ERR_UNSUPPORTED,
              "at most %d candidate blocks per query", BS_MAX_BLOCKS);
  }
  HS2_CHECK(std::isfinite(softmax_scale) && softmax_scale > 0.f, HS2_ERR_INVALID_ARG, "softmax_scale must be > 0");
  HS2_CHECK(kv_len - window <= (1ll << 20), HS2_ERR_UNSUPPORTED, "at most 2^20 candidate keys per query");
  HS2_CHECK(workspace && ((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0), HS2_ERR_WORKSPACE,
            "workspace must be non-null and 256-byte aligned");
  size_t need = 0;
  hs2_status s = hs2_full_attn_select_workspace(kv_dtype, batch, Tq, kv_len, Hq, d, window, topk, &need);
  if (s != HS2_OK) return s;
  HS2_CHECK(ws_bytes >= need, HS2_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  DevCtx ctx;
  int sms = 0;
  if ((s = device_ctx(&ctx, &sms)) != HS2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kv_dtype == HS2_KV_BF16) {
    HS2_CHECK(batch == 1, HS2_ERR_UNSUPPORTED, "bf16 prefill takes batch == 1");
    HS2_CHECK(!k_scale && !v_scale, HS2_ERR_INVALID_ARG, "bf16 KV takes no scales");
    HS2_CHECK(q_start + Tq <= kv_len, HS2_ERR_INVALID_ARG, "q_start + Tq must be <= kv_len");
    HS2_CHECK(Tq * Hq < (1ll << 31) && kv_len < (1ll << 31), HS2_ERR_UNSUPPORTED, "sizes beyond int32 tiles");
    return d == 256 ? prefill_select<256>(Q, K, V, q_start, Tq, kv_len, Hq, window, topk, block, softmax_scale, O,
                                          idx, workspace, st, ctx)
                    : prefill_select<128>(Q, K, V, q_start, Tq, kv_len, Hq, window, topk, block, softmax_scale, O,
                                          idx, workspace, st, ctx);
  }
  HS2_CHECK(kv_dtype == HS2_KV_FP8_E4M3, HS2_ERR_INVALID_ARG, "bad kv_dtype");
  HS2_CHECK(batch <= 65535, HS2_ERR_UNSUPPORTED, "at most 65535 sequences per call");
  HS2_CHECK(Tq == 1 && q_start == kv_len - 1, HS2_ERR_UNSUPPORTED,
            "FP8 decode takes Tq == 1 with q_start == kv_len - 1");
  HS2_CHECK(k_scale && v_scale && aligned4(k_scale) && aligned4(v_scale), HS2_ERR_INVALID_ARG,
            "FP8 KV needs 4-byte aligned k_scale and v_scale");
  HS2_CHECK(kv_stride_tokens >= kv_len, HS2_ERR_INVALID_ARG, "kv_stride_tokens must be >= kv_len");
  HS2_CHECK(((kv_stride_tokens * d) & 15) == 0, HS2_ERR_INVALID_ARG, "sequence stride must keep 16-byte alignment");
  return d == 256 ? decode_select<256>(Q, K, V, k_scale, v_scale, batch, kv_len, kv_stride_tokens, Hq, window, topk,
                                       block, softmax_scale, O, idx, workspace, sms, st, ctx)
                  : decode_select<128>(Q, K, V, k_scale, v_scale, batch, kv_len, kv_stride_tokens, Hq, window, topk,
                                       block, softmax_scale, O, idx, workspace, sms, st, ctx);
}
}  // namespace
}  // namespace hs2

extern "C" {

hs2_status hs2_full_attn_select(const void* Q, const void* K, const void* V, const float* k_scale,
                                const float* v_scale, hs2_kv_dtype kv_dtype, int batch, int64_t q_start, int64_t Tq,
                                int64_t kv_len, int64_t kv_stride_tokens, int Hq, int d, int window, int topk,
                                float softmax_scale, void* O, int32_t* idx, void* workspace, size_t ws_bytes,
                                void* stream) {
  g_err[0] = 0;
  return full_attn_select_impl(Q, K, V, k_scale, v_scale, kv_dtype, batch, q_start, Tq, kv_len, kv_stride_tokens, Hq,
                               d, window, topk, 0, softmax_scale, O, idx, workspace, ws_bytes, stream);
}

hs2_status hs2_full_attn_select_blocks(const void* Q, const void* K, const void* V, const float* k_scale,
                                       const float* v_scale, hs2_kv_dtype kv_dtype, int batch, int64_t q_start,
                                       int64_t Tq, int64_t kv_len, int64_t kv_stride_tokens, int Hq, int d, int window,
                                       int block, int topk_blocks, float softmax_scale, void* O, int32_t* idx,
                                       void* workspace, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  HS2_CHECK(block >= 1, HS2_ERR_INVALID_ARG, "block must be >= 1");
  return full_attn_select_impl(Q, K, V, k_scale, v_scale, kv_dtype, batch, q_start, Tq, kv_len, kv_stride_tokens, Hq,
                               d, window, topk_blocks, block, softmax_scale, O, idx, workspace, ws_bytes, stream);
}

hs2_status hs2_sparse_attn_prefill(const void* Q, const void* K, const void* V, const int32_t* idx, int64_t Tq,
                                   int64_t kv_len, int n_idx, int Hq, int d, float softmax_scale, void* O,
                                   void* stream) {
  g_err[0] = 0;
  HS2_CHECK(Q && K && V && idx && O, HS2_ERR_INVALID_ARG, "null tensor pointer");
  HS2_CHECK(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O) && aligned4(idx), HS2_ERR_INVALID_ARG,
            "Q, K, V, O must be 16-byte aligned and idx 4-byte aligned");
  HS2_CHECK(Tq >= 1 && Tq < (1ll << 31) && kv_len >= 1 && n_idx >= 1, HS2_ERR_INVALID_ARG, "bad sizes");
  HS2_CHECK(n_idx <= 2048, HS2_ERR_UNSUPPORTED, "n_idx must be <= 2048");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  HS2_CHECK(std::isfinite(softmax_scale) && softmax_scale > 0.f, HS2_ERR_INVALID_ARG, "softmax_scale must be > 0");
  DevCtx ctx;
  hs2_status s;
  Attn16Params p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = K;
  p.V = V;
  p.idx = idx;
  p.n_idx = n_idx;
  p.kv_len = kv_len;
  p.H = Hq;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.n_rows = Tq;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int sms = 0;
  if ((s = device_ctx(&ctx, &sms)) != HS2_OK) return s;
  return d == 256 ? launch_sparse_prefill<256>(p, sms, st, ctx) : launch_sparse_prefill<128>(p, sms, st, ctx);
}

hs2_status hs2_sparse_attn_decode_workspace(int batch, int n_idx, int Hq, int d, size_t* bytes) {
  g_err[0] = 0;
  HS2_CHECK(bytes, HS2_ERR_INVALID_ARG, "bytes is null");
  HS2_CHECK(batch >= 1 && n_idx >= 1, HS2_ERR_INVALID_ARG, "bad sizes");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  DevCtx ctx;
  int sms = 0;
  hs2_status s = device_ctx(&ctx, &sms);
  if (s != HS2_OK) return s;
  const int splits = sparse_decode_splits(batch, n_idx, sms);
  *bytes = splits > kMaxCluster ? up256((size_t)batch * splits * (32 + 16 * (size_t)d) * sizeof(float)) : 0;
  return HS2_OK;
}

}  // extern "C"

namespace hs2 {
namespace {
// Argument checks of the sparse decode (with or without a caller workspace).
hs2_status sparse_decode_args(const void* Q, const void* Kc, const void* Vc, const float* k_scale,
                              const float* v_scale, hs2_kv_dtype kv_dtype, int batch, int64_t kv_len,
                              int64_t kv_stride_tokens, const int32_t* idx, int n_idx, int Hq, int d,
                              float softmax_scale, const void* O) {
  HS2_CHECK(Q && Kc && Vc && k_scale && v_scale && idx && O, HS2_ERR_INVALID_ARG, "null tensor pointer");
  HS2_CHECK(aligned16(Q) && aligned16(Kc) && aligned16(Vc) && aligned16(O) && aligned4(idx) && aligned4(k_scale) &&
                aligned4(v_scale),
            HS2_ERR_INVALID_ARG, "misaligned pointer");
  HS2_CHECK(kv_dtype == HS2_KV_FP8_E4M3, HS2_ERR_UNSUPPORTED, "sparse decode reads an FP8 E4M3 cache");
  HS2_CHECK(batch >= 1 && kv_len >= 1 && n_idx >= 1 && kv_stride_tokens >= kv_len, HS2_ERR_INVALID_ARG, "bad sizes");
  HS2_CHECK(n_idx <= 2048, HS2_ERR_UNSUPPORTED, "n_idx must be <= 2048");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  HS2_CHECK(((kv_stride_tokens * d) & 15) == 0, HS2_ERR_INVALID_ARG, "sequence stride must keep 16-byte alignment");
  HS2_CHECK(std::isfinite(softmax_scale) && softmax_scale > 0.f, HS2_ERR_INVALID_ARG, "softmax_scale must be > 0");
  return HS2_OK;
}
}  // namespace
}  // namespace hs2

extern "C" {

hs2_status hs2_sparse_attn_decode(const void* Q, const void* Kc, const void* Vc, const float* k_scale,
                                  const float* v_scale, hs2_kv_dtype kv_dtype, int batch, int64_t kv_len,
                                  int64_t kv_stride_tokens, const int32_t* idx, int n_idx, int Hq, int d,
                                  float softmax_scale, void* O, void* workspace, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  hs2_status s = sparse_decode_args(Q, Kc, Vc, k_scale, v_scale, kv_dtype, batch, kv_len, kv_stride_tokens, idx,
                                    n_idx, Hq, d, softmax_scale, O);
  if (s != HS2_OK) return s;
  size_t need = 0;
  s = hs2_sparse_attn_decode_workspace(batch, n_idx, Hq, d, &need);
  if (s != HS2_OK) return s;
  HS2_CHECK(ws_bytes >= need && (need == 0 || (workspace && ((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0))),
            HS2_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed (256-byte aligned)", ws_bytes, need);
  DevCtx ctx;
  int sms = 0;
  if ((s = device_ctx(&ctx, &sms)) != HS2_OK) return s;
  const int splits = sparse_decode_splits(batch, n_idx, sms);
  DecParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const uint8_t*>(Kc);
  p.V = static_cast<const uint8_t*>(Vc);
  p.ks = k_scale;
  p.vs = v_scale;
  p.idx = idx;
  p.n_idx = n_idx;
  p.kv_len = kv_len;
  p.kv_stride = kv_stride_tokens;
  p.H = Hq;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.splits = splits;
  p.per_split = (n_idx + splits - 1) / splits;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.idx_offset = -1;
  p.part = static_cast<float*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (splits > kMaxCluster) {
    s = d == 256 ? launch_decode_parts<256>(p, batch, st, ctx) : launch_decode_parts<128>(p, batch, st, ctx);
    if (s != HS2_OK) return s;
    return d == 256 ? launch_combine<256>(p.part, splits, Hq, p.O, nullptr, batch, st)
                    : launch_combine<128>(p.part, splits, Hq, p.O, nullptr, batch, st);
  }
  return d == 256 ? launch_decode_cluster<256>(p, batch, st, ctx) : launch_decode_cluster<128>(p, batch, st, ctx);
}

}  // extern "C"

// Scratch of hs2_sparse_attn_decode_static: the split partials of the sparse
// decode live here instead of in a caller workspace.  Module scope, so every
// device that loads the library holds these 8 MiB until the process exits.
static __device__ __align__(256) float g_static_scratch[HS2_STATIC_SCRATCH_BYTES / sizeof(float)];

namespace {
float* g_static_scratch_ptr[hs2::kMaxDevices];

// Device address of g_static_scratch on the current device, looked up once
// per device (the host-side symbol is only a stand-in, never a device pointer).
hs2_status static_scratch_ptr(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hs2::cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= hs2::kMaxDevices) return hs2::fail(HS2_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lock(hs2::g_mu);
  if (g_static_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return hs2::cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_static_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_static_scratch_ptr[dev];
  return HS2_OK;
}
}  // namespace

extern "C" {

hs2_status hs2_sparse_attn_decode_static(const void* Q, const void* Kc, const void* Vc, const float* k_scale,
                                         const float* v_scale, hs2_kv_dtype kv_dtype, int batch, int64_t kv_len,
                                         int64_t kv_stride_tokens, const int32_t* idx, int n_idx, int Hq, int d,
                                         float softmax_scale, void* O, void* stream) {
  g_err[0] = 0;
  hs2_status s = sparse_decode_args(Q, Kc, Vc, k_scale, v_scale, kv_dtype, batch, kv_len, kv_stride_tokens, idx,
                                    n_idx, Hq, d, softmax_scale, O);
  if (s != HS2_OK) return s;
  size_t need = 0;
  if ((s = hs2_sparse_attn_decode_workspace(batch, n_idx, Hq, d, &need)) != HS2_OK) return s;
  HS2_CHECK(need <= HS2_STATIC_SCRATCH_BYTES, HS2_ERR_UNSUPPORTED,
            "this batch needs %zu bytes of split scratch; the static array holds %u "
            "(use hs2_sparse_attn_decode with a workspace)", need, (unsigned)HS2_STATIC_SCRATCH_BYTES);
  float* scratch = nullptr;
  if ((s = static_scratch_ptr(&scratch)) != HS2_OK) return s;
  return hs2_sparse_attn_decode(Q, Kc, Vc, k_scale, v_scale, kv_dtype, batch, kv_len, kv_stride_tokens, idx,
                                n_idx, Hq, d, softmax_scale, O, scratch, HS2_STATIC_SCRATCH_BYTES, stream);
}

hs2_status hs2_swa_attn_prefill_workspace(int64_t Tq, int64_t kv_len, int Hq, int d, int rope_dims, size_t* bytes) {
  g_err[0] = 0;
  HS2_CHECK(bytes, HS2_ERR_INVALID_ARG, "bytes is null");
  HS2_CHECK(Tq >= 1 && kv_len >= 1, HS2_ERR_INVALID_ARG, "bad sizes");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  HS2_CHECK(rope_dims == 16 || rope_dims == 32 || rope_dims == 64, HS2_ERR_UNSUPPORTED,
            "rope_dims must be 16, 32 or 64 (got %d)", rope_dims);
  *bytes = swa_ws(Tq, kv_len, Hq, d, rope_dims).total;
  return HS2_OK;
}

hs2_status hs2_swa_attn_prefill(const void* Q, const void* K, const void* V, int64_t q_start, int64_t Tq,
                                int64_t kv_len, int Hq, int d, int window, int rope_dims, float rope_base,
                                float softmax_scale, void* O, void* workspace, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  HS2_CHECK(Q && K && V && O, HS2_ERR_INVALID_ARG, "null tensor pointer");
  HS2_CHECK(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O), HS2_ERR_INVALID_ARG,
            "tensor pointers must be 16-byte aligned");
  HS2_CHECK(Tq >= 1 && kv_len >= 1 && q_start >= 0 && q_start + Tq <= kv_len, HS2_ERR_INVALID_ARG,
            "bad sizes (need q_start + Tq <= kv_len)");
  HS2_CHECK(Tq * Hq < (1ll << 31) && kv_len < (1ll << 31), HS2_ERR_UNSUPPORTED, "sizes beyond int32 tiles");
  HS2_CHECK(window >= 1, HS2_ERR_INVALID_ARG, "window must be >= 1");
  HS2_CHECK(std::isfinite(rope_base) && rope_base > 1.f, HS2_ERR_INVALID_ARG, "rope_base must be > 1");
  HS2_CHECK(std::isfinite(softmax_scale) && softmax_scale > 0.f, HS2_ERR_INVALID_ARG, "softmax_scale must be > 0");
  size_t need = 0;
  hs2_status s = hs2_swa_attn_prefill_workspace(Tq, kv_len, Hq, d, rope_dims, &need);
  if (s != HS2_OK) return s;
  HS2_CHECK(workspace && ((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0) && ws_bytes >= need,
            HS2_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed (256-byte aligned)", ws_bytes, need);
  DevCtx ctx;
  if ((s = device_ctx(&ctx, nullptr)) != HS2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 256 ? swa_attn<256>(Q, K, V, q_start, Tq, kv_len, Hq, window, rope_dims, rope_base, softmax_scale, O,
                                  workspace, st, ctx)
                  : swa_attn<128>(Q, K, V, q_start, Tq, kv_len, Hq, window, rope_dims, rope_base, softmax_scale, O,
                                  workspace, st, ctx);
}

hs2_status hs2_decode_shard_workspace(int batch, int64_t shard_len, int n_idx, int Hq, int d, int topk,
                                      size_t* bytes) {
  g_err[0] = 0;
  HS2_CHECK(bytes, HS2_ERR_INVALID_ARG, "bytes is null");
  HS2_CHECK(batch >= 1 && shard_len >= 1 && n_idx >= 1 && topk >= 1, HS2_ERR_INVALID_ARG, "bad sizes");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  DevCtx ctx;
  int sms = 0;
  hs2_status s = device_ctx(&ctx, &sms);
  if (s != HS2_OK) return s;
  const size_t full = shard_ws(batch, shard_len, Hq, d, topk).total;
  const int splits = sparse_decode_splits(batch, n_idx, sms);
  const size_t sparse = up256((size_t)batch * splits * (32 + 16 * (size_t)d) * sizeof(float));
  *bytes = std::max(full, sparse);
  return HS2_OK;
}

hs2_status hs2_decode_shard_attn(const void* Q, const void* Kc, const void* Vc, const float* k_scale,
                                 const float* v_scale, int batch, int64_t shard_len, int64_t kv_stride_tokens,
                                 int Hq, int d, int topk, float softmax_scale, float* ml_out, float* O_out,
                                 void* workspace, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  HS2_CHECK(Q && Kc && Vc && k_scale && v_scale && ml_out && O_out, HS2_ERR_INVALID_ARG, "null pointer");
  HS2_CHECK(aligned16(Q) && aligned16(Kc) && aligned16(Vc) && aligned4(k_scale) && aligned4(v_scale) &&
                aligned4(ml_out) && aligned16(O_out),
            HS2_ERR_INVALID_ARG, "misaligned pointer");
  HS2_CHECK(batch >= 1 && shard_len >= 1 && kv_stride_tokens >= shard_len && topk >= 1, HS2_ERR_INVALID_ARG,
            "bad sizes");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  HS2_CHECK(((kv_stride_tokens * d) & 15) == 0, HS2_ERR_INVALID_ARG, "sequence stride must keep 16-byte alignment");
  HS2_CHECK(std::isfinite(softmax_scale) && softmax_scale > 0.f, HS2_ERR_INVALID_ARG, "softmax_scale must be > 0");
  HS2_CHECK((shard_len + kDecodeKeysPerSplit - 1) / kDecodeKeysPerSplit <= kCombineMaxSplits, HS2_ERR_UNSUPPORTED,
            "shard too long");
  const size_t need = shard_ws(batch, shard_len, Hq, d, topk).total;
  HS2_CHECK(workspace && ((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0) && ws_bytes >= need,
            HS2_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed (256-byte aligned)", ws_bytes, need);
  DevCtx ctx;
  int sms = 0;
  hs2_status s = device_ctx(&ctx, &sms);
  if (s != HS2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 256 ? shard_attn<256>(Q, Kc, Vc, k_scale, v_scale, batch, shard_len, kv_stride_tokens, Hq,
                                    softmax_scale, ml_out, O_out, workspace, topk, sms, st, ctx)
                  : shard_attn<128>(Q, Kc, Vc, k_scale, v_scale, batch, shard_len, kv_stride_tokens, Hq,
                                    softmax_scale, ml_out, O_out, workspace, topk, sms, st, ctx);
}

hs2_status hs2_decode_shard_candidates(void* workspace, size_t ws_bytes, int batch, int64_t shard_len,
                                       int64_t shard_offset, int64_t kv_len, int Hq, int d, int window, int topk,
                                       const float* ml_global, void* cand, void* stream) {
  g_err[0] = 0;
  HS2_CHECK(workspace && ml_global && cand, HS2_ERR_INVALID_ARG, "null pointer");
  HS2_CHECK(aligned4(ml_global) && aligned4(cand), HS2_ERR_INVALID_ARG, "misaligned pointer");
  const size_t n_cand = (size_t)batch * topk;
  float* cand_val = static_cast<float*>(cand);
  int32_t* cand_pos = static_cast<int32_t*>(cand) + n_cand;
  int32_t* cand_cnt = static_cast<int32_t*>(cand) + 2 * n_cand;
  HS2_CHECK(batch >= 1 && batch <= 65535 && shard_len >= 1 && shard_offset >= 0 && shard_offset + shard_len <= kv_len &&
                window >= 1 && topk >= 1,
            HS2_ERR_INVALID_ARG, "bad sizes");
  HS2_CHECK(window + topk <= 2048 && kv_len - window <= (1ll << 30), HS2_ERR_UNSUPPORTED, "index row too wide");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  const ShardWs w = shard_ws(batch, shard_len, Hq, d, topk);
  HS2_CHECK(ws_bytes >= w.total && ((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0), HS2_ERR_WORKSPACE,
            "the workspace of hs2_decode_shard_attn (%zu bytes) is needed", w.total);
  DevCtx ctx;
  hs2_status s = device_ctx(&ctx, nullptr);
  if (s != HS2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* b = static_cast<uint8_t*>(workspace);
  const float* logits = reinterpret_cast<const float*>(b);
  float* sigma = reinterpret_cast<float*>(b + w.logits + w.part);
  // this shard's candidates: global positions offset .. kv_len - 1 - window
  const int64_t n = std::max<int64_t>(0, std::min<int64_t>(shard_len, kv_len - window - shard_offset));
  const int chunks = radix_chunks(n, topk);           // <= w.rx_chunks: n <= shard_len
  uint32_t* rx_hist = reinterpret_cast<uint32_t*>(b + w.logits + w.part + w.sigma + w.lists);
  if (n > 0) {
    dim3 g((unsigned)((n + 1023) / 1024), (unsigned)batch);
    prof_begin(st);
    decode_sigma_kernel<<<g, 256, 0, st>>>(logits, w.ld, ml_global, Hq, n, sigma, w.ld,
                                           chunks ? rx_hist : nullptr, RX_HIST);
    if ((s = after_launch("decode_sigma_kernel", st)) != HS2_OK) return s;
  }
  if (chunks) {
    // a long shard: the radix select over the whole GPU, written as the shard's list
    RadixParams rp{};
    rp.sigma = sigma;
    rp.ld = w.ld;
    rp.n = n;
    rp.chunks = chunks;
    rp.topk = topk;
    rp.window = window;
    rp.pos = kv_len - 1;
    rp.pos_offset = shard_offset;
    rp.hist = rx_hist;
    rp.cnt = rx_hist + up256((size_t)batch * RX_HIST * 4) / 4;
    rp.idx = nullptr;
    rp.lval = cand_val;
    rp.lpos = cand_pos;
    rp.lcnt = cand_cnt;
    return launch_radix(rp, batch, st, ctx);
  }
  const int S = shard_slices(n, topk);
  uint8_t* lists = b + w.logits + w.part + w.sigma;
  const size_t n_list = (size_t)batch * S * topk;
  TopkSplitParams tp{};
  tp.sigma = sigma;
  tp.ld = w.ld;
  tp.n = n;
  tp.splits = S;
  tp.slice = round_up((n + S - 1) / S, 64);
  tp.topk = topk;
  tp.window = window;
  tp.pos = kv_len - 1;
  tp.pos_offset = shard_offset;
  tp.idx = nullptr;
  // one slice: its list is the shard's list; more: a merge of all of them into one
  tp.cval = S == 1 ? cand_val : reinterpret_cast<float*>(lists);
  tp.cpos = S == 1 ? cand_pos : reinterpret_cast<int32_t*>(lists + n_list * 4);
  tp.ccnt = S == 1 ? cand_cnt : reinterpret_cast<int32_t*>(lists + n_list * 8);
  tp.group = S;
  tp.gval = cand_val;
  tp.gpos = cand_pos;
  tp.gcnt = cand_cnt;
  HS2_CHECK(tp.slice <= TS_CAP && (int64_t)S * topk <= TS_CAP, HS2_ERR_UNSUPPORTED, "shard too long for its top-k");
  if ((s = set_smem(topk_slice_kernel, TS_SMEM)) != HS2_OK) return s;
  prof_begin(st);
  topk_slice_kernel<<<dim3((unsigned)S, (unsigned)batch), TS_THREADS, TS_SMEM, st>>>(tp, ctx);
  if ((s = after_launch("topk_slice_kernel", st)) != HS2_OK) return s;
  if (S > 1) {
    if ((s = set_smem(topk_merge_kernel<false>, TS_SMEM)) != HS2_OK) return s;
    prof_begin(st);
    topk_merge_kernel<false><<<dim3(1u, (unsigned)batch), TS_THREADS, TS_SMEM, st>>>(tp, ctx);
    if ((s = after_launch("topk_merge_kernel", st)) != HS2_OK) return s;
  }
  return HS2_OK;
}

hs2_status hs2_decode_merge_candidates(const void* cand_all, int n_shards, int batch, int64_t kv_len, int window,
                                       int topk, int32_t* idx, void* stream) {
  g_err[0] = 0;
  HS2_CHECK(cand_all && idx, HS2_ERR_INVALID_ARG, "null pointer");
  HS2_CHECK(aligned4(cand_all) && aligned4(idx), HS2_ERR_INVALID_ARG, "misaligned pointer");
  HS2_CHECK(batch >= 1 && n_shards >= 1 && kv_len >= 1 && window >= 1 && topk >= 1, HS2_ERR_INVALID_ARG,
            "bad sizes");
  HS2_CHECK(n_shards <= 64 && (int64_t)n_shards * topk <= TS_CAP && window + topk <= 2048, HS2_ERR_UNSUPPORTED,
            "at most 64 shards and %d candidates per row", TS_CAP);
  DevCtx ctx;
  hs2_status s = device_ctx(&ctx, nullptr);
  if (s != HS2_OK) return s;
  // shard q's block: scores [batch, k], positions [batch, k], lengths [batch]
  const int64_t n_cand = (int64_t)batch * topk, P = 2 * n_cand + batch;
  TopkSplitParams tp{};
  tp.n = std::max<int64_t>(0, kv_len - window);
  tp.splits = n_shards;
  tp.topk = topk;
  tp.window = window;
  tp.pos = kv_len - 1;
  tp.cval = const_cast<float*>(static_cast<const float*>(cand_all));
  tp.cpos = const_cast<int32_t*>(static_cast<const int32_t*>(cand_all)) + n_cand;
  tp.ccnt = const_cast<int32_t*>(static_cast<const int32_t*>(cand_all)) + 2 * n_cand;
  tp.group = 0;
  tp.idx = idx;
  tp.v_row = topk;
  tp.v_list = P;
  tp.c_row = 1;
  tp.c_list = P;
  if ((s = set_smem(topk_merge_kernel<true>, TS_SMEM)) != HS2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  prof_begin(st);
  topk_merge_kernel<true><<<(unsigned)batch, TS_THREADS, TS_SMEM, st>>>(tp, ctx);
  return after_launch("topk_merge_kernel", st);
}

hs2_status hs2_sparse_decode_shard(const void* Q, const void* Kc, const void* Vc, const float* k_scale,
                                   const float* v_scale, int batch, int64_t shard_len, int64_t kv_stride_tokens,
                                   int64_t shard_offset, const int32_t* idx, int n_idx, int Hq, int d,
                                   float softmax_scale, float* ml_out, float* O_out, void* workspace,
                                   size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  hs2_status s = sparse_decode_args(Q, Kc, Vc, k_scale, v_scale, HS2_KV_FP8_E4M3, batch, shard_len, kv_stride_tokens,
                                    idx, n_idx, Hq, d, softmax_scale, Q);
  if (s != HS2_OK) return s;
  HS2_CHECK(ml_out && O_out && aligned4(ml_out) && aligned16(O_out), HS2_ERR_INVALID_ARG, "ml_out / O_out");
  HS2_CHECK(shard_offset >= 0, HS2_ERR_INVALID_ARG, "shard_offset must be >= 0");
  DevCtx ctx;
  int sms = 0;
  if ((s = device_ctx(&ctx, &sms)) != HS2_OK) return s;
  const int splits = sparse_decode_splits(batch, n_idx, sms);
  const size_t need = up256((size_t)batch * splits * (32 + 16 * (size_t)d) * sizeof(float));
  HS2_CHECK(workspace && ((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0) && ws_bytes >= need,
            HS2_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed (256-byte aligned)", ws_bytes, need);
  DecParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const uint8_t*>(Kc);
  p.V = static_cast<const uint8_t*>(Vc);
  p.ks = k_scale;
  p.vs = v_scale;
  p.idx = idx;
  p.n_idx = n_idx;
  p.kv_len = shard_len;
  p.kv_stride = kv_stride_tokens;
  p.H = Hq;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.idx_offset = shard_offset;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 256 ? shard_sparse<256>(p, batch, n_idx, sms, ml_out, O_out, workspace, st, ctx)
                  : shard_sparse<128>(p, batch, n_idx, sms, ml_out, O_out, workspace, st, ctx);
}

hs2_status hs2_partial_merge(const float* ml_all, int n_shards, int shard, float* O32, float* ml_out, int batch,
                             int Hq, int d, void* stream) {
  g_err[0] = 0;
  HS2_CHECK(ml_all && O32 && ml_out && aligned4(ml_all) && aligned4(O32) && aligned4(ml_out), HS2_ERR_INVALID_ARG,
            "null or misaligned pointer");
  HS2_CHECK(batch >= 1 && batch <= 65535 && n_shards >= 1 && shard >= 0 && shard < n_shards, HS2_ERR_INVALID_ARG,
            "bad sizes");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 256 ? launch_partial<256>(false, ml_all, n_shards, shard, O32, ml_out, nullptr, batch, Hq, st)
                  : launch_partial<128>(false, ml_all, n_shards, shard, O32, ml_out, nullptr, batch, Hq, st);
}

hs2_status hs2_partial_finalize(const float* ml, const float* O32, void* O, int batch, int Hq, int d, void* stream) {
  g_err[0] = 0;
  HS2_CHECK(ml && O32 && O && aligned4(ml) && aligned4(O32) && aligned16(O), HS2_ERR_INVALID_ARG,
            "null or misaligned pointer");
  HS2_CHECK(batch >= 1 && batch <= 65535, HS2_ERR_INVALID_ARG, "bad batch");
  HS2_CHECK(shape_ok(Hq, d), HS2_ERR_UNSUPPORTED, "Hq must be 8 or 16 and d 128 or 256");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 256 ? launch_partial<256>(true, ml, 1, 0, const_cast<float*>(O32), nullptr,
                                        static_cast<__nv_bfloat16*>(O), batch, Hq, st)
                  : launch_partial<128>(true, ml, 1, 0, const_cast<float*>(O32), nullptr,
                                        static_cast<__nv_bfloat16*>(O), batch, Hq, st);
}

hs2_status hs2_device_status(void* stream) {
  g_err[0] = 0;
  DevCtx ctx;
  hs2_status s = device_ctx(&ctx, nullptr);
  if (s != HS2_OK) return s;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned w = 0;
  e = cudaMemcpyFromSymbol(&w, g_status_word, sizeof(w));
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear status word");
  if (w & ST_TIMEOUT) return fail(HS2_ERR_TIMEOUT, "a device-side wait gave up");
  if (w & ST_DEVICE_CHECK) return fail(HS2_ERR_DEVICE_CHECK, "a device-side input check failed");
  return HS2_OK;
}

hs2_status hs2_profile_enable(int on) {
  g_err[0] = 0;
  g_prof_on = on != 0;
  if (g_prof_on) g_prof_n = 0;
  return HS2_OK;
}

hs2_status hs2_profile_collect(const char** names, float* ms, int max_n, int* n) {
  g_err[0] = 0;
  HS2_CHECK(n && (max_n <= 0 || (names && ms)), HS2_ERR_INVALID_ARG, "null output");
  const int kept = std::min(g_prof_n, kMaxProf);
  for (int i = 0; i < kept && i < max_n; ++i) {
    cudaError_t e = cudaEventSynchronize(g_prof[i].b);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float t = 0.f;
    e = cudaEventElapsedTime(&t, g_prof[i].a, g_prof[i].b);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    names[i] = g_prof[i].name;
    ms[i] = t;
  }
  *n = g_prof_n;
  g_prof_n = 0;
  return HS2_OK;
}

hs2_status hs2_set_spin_limit(int64_t iterations) {
  g_err[0] = 0;
  HS2_CHECK(iterations >= 0, HS2_ERR_INVALID_ARG, "iterations must be >= 0");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(HS2_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  g_spin[dev] = iterations;
  return HS2_OK;
}

}  // extern "C"
