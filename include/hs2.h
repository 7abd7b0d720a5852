/*
 * hs2.h -- C ABI of libhs2.so, the B200 (sm_100a) hot path of HySparse2's
 * token-level KV Reuse attention.
 *
 * Method (cited by page and passage; the pages give no code and no interface):
 *   "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing", agihunt.info
 *   summary, inner-level KV Reuse paragraph -- a causal full-attention layer
 *   scores every past token; per query position the 128 most recent tokens are
 *   forced into the selection and 1024 high-scoring out-of-window tokens are
 *   added; the following sparse layers gather only those tokens from the same
 *   full-attention KV.  Next paragraph: MQA (one KV head), NoPE, the full layer
 *   acts as an oracle selector with exact attention scores.  Outer-level KV
 *   Bridging paragraph: a cross-decoder full layer's K/V are its own linear
 *   projections of a self-decoder full layer's hidden state.  Results table
 *   "KV @1M (FP8)": the cache is stored in FP8.  10100.com article, "evolution
 *   two": *at most* 1024 selected tokens.
 *
 * Readings fixed here where the pages are silent:
 *   - selection score of key j for query i: sigma_ij = sum over the query heads
 *     h of softmax_j(s_hij), s_hij = scale * q_ih . k_j (scale normally 1/sqrt(d));
 *   - forced window of query position p = positions [p-window+1, p];
 *     candidates = [0, p-window]; up to topk of them with the largest sigma;
 *   - FP8 = OCP E4M3FN, round to nearest even, saturating; one fp32 scale per
 *     token row, value = E4M3(code) * scale.
 *
 * Conventions common to every call
 *   - Every tensor pointer is a DEVICE pointer owned by the caller, 16-byte
 *     aligned, dense row-major with the stated shape.  The library allocates
 *     nothing; scratch comes from a caller workspace whose size the matching
 *     *_workspace query returns.
 *   - bf16 = IEEE bfloat16 (uint16 storage); fp8 = E4M3FN (uint8 storage).
 *   - idx rows are int32 absolute key positions; -1 marks an empty slot.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Argument errors are reported synchronously, before any launch,
 *     and nothing is written.  A failed launch returns HS2_ERR_CUDA.  Checks
 *     made on the device (an idx entry out of range) and bounded waits that ran
 *     out set a per-device status word read by hs2_device_status().
 *   - No exception or abort crosses the ABI.  Calls on distinct workspaces may
 *     run concurrently from several host threads.
 *   - Supported in this version: one KV head, Hq in {8, 16}, d in {128, 256},
 *     index rows (window + selection) of at most 2048 entries, window >= 1.
 */
#ifndef HS2_H_
#define HS2_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HS2_API __attribute__((visibility("default")))
#else
#define HS2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HS2_OK = 0,
  HS2_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or shape      */
  HS2_ERR_UNSUPPORTED = 2,   /* valid request outside this version's shapes    */
  HS2_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small     */
  HS2_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed     */
  HS2_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up              */
  HS2_ERR_DEVICE_CHECK = 6   /* a device-side input check failed (bad idx)      */
} hs2_status;

typedef enum { HS2_KV_BF16 = 0, HS2_KV_FP8_E4M3 = 1 } hs2_kv_dtype;

/* Static text for a status code. */
HS2_API const char* hs2_status_string(hs2_status s);

/* Detail of the last error on the calling host thread ("" if none). */
HS2_API const char* hs2_last_error(void);

/* Library version, e.g. "hs2 0.1 sm_100a". */
HS2_API const char* hs2_version(void);

/*
 * KV Bridging re-projection (outer-level KV sharing; agihunt.info summary,
 * KV Bridging paragraph).  For r < rows and c < d:
 *     K[r,c] = sum_e hidden[r,e] * Wk[c,e],   V[r,c] = sum_e hidden[r,e] * Wv[c,e]
 * accumulated in fp32 on the tensor cores.
 *   hidden : bf16 [rows, hidden_dim]    (the self-decoder hidden states)
 *   Wk, Wv : bf16 [d, hidden_dim]       (this layer's own projections, [out, in])
 *   out_dtype HS2_KV_BF16     : K_out, V_out bf16 [rows, d], rounded to nearest even;
 *                               k_scale, v_scale must be NULL.
 *   out_dtype HS2_KV_FP8_E4M3 : K_out, V_out uint8 E4M3 codes [rows, d] and
 *                               k_scale, v_scale fp32 [rows] with
 *                               scale = amax(row)/448 (1 for an all-zero row),
 *                               code = E4M3_RNE_satfinite(x / scale).
 * Requires rows >= 1, hidden_dim a positive multiple of 64, d == 256.
 */
HS2_API hs2_status hs2_bridge_kv(const void* hidden, int64_t rows, int hidden_dim,
                         const void* Wk, const void* Wv, int d, hs2_kv_dtype out_dtype,
                         void* K_out, void* V_out, float* k_scale, float* v_scale,
                         void* stream);

/*
 * Decode-step KV Bridging: append each sequence's new token to this layer's
 * FP8 cache (agihunt.info summary, KV Bridging paragraph; arXiv abstract --
 * every cross-decoder KV cache is built from self-decoder hidden states, so
 * each decode step bridges the new token's hidden row).  For b < batch:
 *     k = hidden[b,:] Wk^T,  v = hidden[b,:] Wv^T      (fp32 accumulation)
 *     k_scale[b,pos[b]] = amax(k)/448 (1 if k is all zero)
 *     Kc[b,pos[b],:]    = E4M3_RNE_satfinite(k / k_scale[b,pos[b]])   (V likewise)
 * the same arithmetic as hs2_bridge_kv's FP8 output, one row per sequence.
 *   hidden : bf16 [batch, hidden_dim] (the new tokens' self-decoder hidden states)
 *   Wk, Wv : bf16 [d, hidden_dim]
 *   Kc, Vc : uint8 [batch, kv_stride_tokens, d]; k_scale, v_scale fp32 [batch, kv_stride_tokens]
 *   pos    : int32 [batch] on the device, the row written in each sequence.
 * Only row pos[b] of each sequence is written.  An entry pos[b] outside
 * [0, kv_stride_tokens) is skipped and raises HS2_ERR_DEVICE_CHECK in
 * hs2_device_status().  Requires 1 <= batch <= 65535, hidden_dim a positive
 * multiple of 256, d == 256.
 */
HS2_API hs2_status hs2_bridge_append(const void* hidden, int batch, int hidden_dim, const void* Wk,
                                     const void* Wv, int d, void* Kc, void* Vc, float* k_scale,
                                     float* v_scale, int64_t kv_stride_tokens, const int32_t* pos,
                                     void* stream);

/*
 * Full-attention layer as the oracle selector (agihunt.info summary, KV Reuse
 * and MQA/NoPE paragraphs).  Query t of sequence b sits at absolute position
 * p = q_start + t and attends causally to keys 0..p of its sequence:
 *     O[b,t,h,:] = sum_j softmax_j(scale * q . k_j) v_j
 *     idx[b,t,0:window]            = p-window+1 .. p (-1 where negative)
 *     idx[b,t,window:window+n]     = the n = min(topk, p-window+1) candidates
 *                                    j <= p-window with the largest sigma_j,
 *                                    ascending; the rest of the row is -1.
 * Two forms are supported:
 *   prefill: kv_dtype HS2_KV_BF16, batch == 1, Tq >= 1, q_start + Tq <= kv_len.
 *            Q bf16 [Tq, Hq, d]; K, V bf16 [kv_len, d]; k_scale/v_scale NULL.
 *            A long prefill may be issued in query chunks (q_start > 0) over
 *            the causal prefix (kv_len = q_start + Tq).
 *   decode : kv_dtype HS2_KV_FP8_E4M3, 1 <= batch <= 65535, Tq == 1,
 *            q_start == kv_len - 1 (the cache already holds the new token).
 *            Q bf16 [batch, Hq, d]; K, V uint8 [batch, kv_stride_tokens, d];
 *            k_scale, v_scale fp32 [batch, kv_stride_tokens]; key j of
 *            sequence b is E4M3(K[b,j,:]) * k_scale[b,j] (V likewise).
 * kv_stride_tokens >= kv_len (prefill: ignored, rows are contiguous).
 * Outputs: O bf16 [batch, Tq, Hq, d]; idx int32 [batch, Tq, window+topk].
 * workspace: device memory of at least hs2_full_attn_select_workspace() bytes,
 * 256-byte aligned; its contents on entry do not matter.
 */
HS2_API hs2_status hs2_full_attn_select(const void* Q, const void* K, const void* V,
                                const float* k_scale, const float* v_scale,
                                hs2_kv_dtype kv_dtype, int batch, int64_t q_start,
                                int64_t Tq, int64_t kv_len, int64_t kv_stride_tokens,
                                int Hq, int d, int window, int topk, float softmax_scale,
                                void* O, int32_t* idx, void* workspace, size_t ws_bytes,
                                void* stream);

/*
 * The same full-attention layer with BLOCK-level selection, the alternative
 * the pages measure token-level selection against (agihunt.info summary,
 * ablation paragraph: 64-token blocks at the same 1024-token budget; 10100.com
 * article, "evolution one").  Blocks are aligned: block c holds positions
 * [c*block, (c+1)*block).  Block c's score is the sum of sigma_j over its
 * candidates j <= p-window (the boundary block counts only those):
 *     idx[b,t,0:window]  = p-window+1 .. p (-1 where negative)
 *     idx[b,t,window:]   = every candidate position of the topk_blocks blocks
 *                          with the largest score (ties to the smaller block;
 *                          all blocks if there are at most topk_blocks),
 *                          ascending, then -1 up to window + topk_blocks*block.
 * Arguments, outputs, workspace (the same query, with topk = topk_blocks) and
 * errors as hs2_full_attn_select; O is the same full-attention output.
 * Requires block a power of two in [16, 256], window + topk_blocks*block <=
 * 2048 and at most 16384 candidate blocks per query.
 */
HS2_API hs2_status hs2_full_attn_select_blocks(const void* Q, const void* K, const void* V,
                                       const float* k_scale, const float* v_scale,
                                       hs2_kv_dtype kv_dtype, int batch, int64_t q_start,
                                       int64_t Tq, int64_t kv_len, int64_t kv_stride_tokens, int Hq,
                                       int d, int window, int block, int topk_blocks,
                                       float softmax_scale, void* O, int32_t* idx, void* workspace,
                                       size_t ws_bytes, void* stream);

/* Workspace bytes hs2_full_attn_select needs for these shape arguments. */
HS2_API hs2_status hs2_full_attn_select_workspace(hs2_kv_dtype kv_dtype, int batch, int64_t Tq,
                                          int64_t kv_len, int Hq, int d, int window,
                                          int topk, size_t* bytes);

/*
 * Sparse layer, prefill (agihunt.info summary, KV Reuse paragraph: the sparse
 * layers reuse the selected tokens of the full layer's KV).  For each query t:
 *     O[t,h,:] = sum_{j in S_t} softmax_{S_t}(scale * q_th . k_j) v_j,
 *     S_t = { idx[t,s] : idx[t,s] >= 0 }.
 *   Q bf16 [Tq, Hq, d] (this sparse layer's own queries); K, V bf16 [kv_len, d]
 *   (the full layer's KV); idx int32 [Tq, n_idx]; O bf16 [Tq, Hq, d].
 * An entry idx >= kv_len (or < -1) is skipped and raises HS2_ERR_DEVICE_CHECK
 * in hs2_device_status(); a row with no valid entry yields O = 0.
 */
HS2_API hs2_status hs2_sparse_attn_prefill(const void* Q, const void* K, const void* V,
                                   const int32_t* idx, int64_t Tq, int64_t kv_len, int n_idx,
                                   int Hq, int d, float softmax_scale, void* O, void* stream);

/*
 * Sparse layer, decode over the FP8 cache: as hs2_sparse_attn_prefill with one
 * query per sequence, keys dequantised as E4M3(code) * scale.
 *   Q bf16 [batch, Hq, d]; Kc, Vc uint8 [batch, kv_stride_tokens, d];
 *   k_scale, v_scale fp32 [batch, kv_stride_tokens]; idx int32 [batch, n_idx]
 *   with entries < kv_len; O bf16 [batch, Hq, d].
 * kv_dtype must be HS2_KV_FP8_E4M3.  workspace may be NULL when
 * hs2_sparse_attn_decode_workspace() returns 0.
 */
HS2_API hs2_status hs2_sparse_attn_decode(const void* Q, const void* Kc, const void* Vc,
                                  const float* k_scale, const float* v_scale,
                                  hs2_kv_dtype kv_dtype, int batch, int64_t kv_len,
                                  int64_t kv_stride_tokens, const int32_t* idx, int n_idx,
                                  int Hq, int d, float softmax_scale, void* O,
                                  void* workspace, size_t ws_bytes, void* stream);

HS2_API hs2_status hs2_sparse_attn_decode_workspace(int batch, int n_idx, int Hq, int d,
                                            size_t* bytes);

/*
 * hs2_sparse_attn_decode without a workspace argument.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory themselves -- e.g. a serving process whose device memory is
 * all reserved up front by its own pool and handed to plugins as fixed
 * buffers, or a decode loop that must not pay for cudaMalloc's implicit
 * synchronisation.  Same arguments, results and errors as
 * hs2_sparse_attn_decode, which it calls with its scratch instead of a
 * caller's workspace.
 *   - Scratch: one file-scope device array of HS2_STATIC_SCRATCH_BYTES
 *     (8 MiB) that every GPU loading the library holds until the process
 *     exits.  A call whose split partials need more than that (see
 *     hs2_sparse_attn_decode_workspace) fails with HS2_ERR_UNSUPPORTED and
 *     launches nothing.  Nothing is allocated, by this call or the library.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - Every call on a device shares the one array.  Its contents need no
 *     clearing (each call writes every partial it reads), but calls whose
 *     executions overlap on the GPU -- on different streams, or from
 *     different host threads -- race on it and give wrong results.
 */
#define HS2_STATIC_SCRATCH_BYTES (8u << 20)
HS2_API hs2_status hs2_sparse_attn_decode_static(const void* Q, const void* Kc, const void* Vc,
                                         const float* k_scale, const float* v_scale,
                                         hs2_kv_dtype kv_dtype, int batch, int64_t kv_len,
                                         int64_t kv_stride_tokens, const int32_t* idx, int n_idx,
                                         int Hq, int d, float softmax_scale, void* O,
                                         void* stream);

/*
 * Sliding-window attention of a self-decoder SWA layer, with partial RoPE
 * (agihunt.info summary: the self-decoder mixes full and sliding-window
 * attention, each SWA query attending only to the most recent tokens; SWA
 * layers use 64-dim partial RoPE, the full and sparse layers NoPE; MQA).
 * These layers produce the hidden states the KV Bridging consumes.  Query t
 * sits at absolute position p = q_start + t and attends to keys
 * [max(0, p - window + 1), p]:
 *     O[t,h,:] = sum_j softmax_j(scale * rope(q_th, p) . rope(k_j, j)) v_j
 * rope(x, p) rotates the pairs (x_i, x_{i+R/2}), i < R/2 = rope_dims/2, by the
 * angle p * rope_base^(-2i/R) and leaves the dims from R on unchanged.  The
 * rotated q and k are rounded to bf16 before the products (fp32 accumulation).
 *   Q bf16 [Tq, Hq, d]; K, V bf16 [kv_len, d] (one KV head); O bf16 [Tq, Hq, d].
 *   workspace: at least hs2_swa_attn_prefill_workspace() bytes, 256-byte
 *   aligned (the rotated Q and K and a cos/sin table); contents on entry do
 *   not matter.
 * Requires q_start + Tq <= kv_len, window >= 1, rope_dims in {16, 32, 64},
 * rope_base > 1 (10000 is the usual value), and the shapes of
 * hs2_full_attn_select's prefill.
 */
HS2_API hs2_status hs2_swa_attn_prefill(const void* Q, const void* K, const void* V, int64_t q_start,
                                        int64_t Tq, int64_t kv_len, int Hq, int d, int window,
                                        int rope_dims, float rope_base, float softmax_scale, void* O,
                                        void* workspace, size_t ws_bytes, void* stream);

HS2_API hs2_status hs2_swa_attn_prefill_workspace(int64_t Tq, int64_t kv_len, int Hq, int d,
                                                  int rope_dims, size_t* bytes);

/*
 * Decode with each sequence's context split over R shards (one per GPU), for
 * the 1M-token regime with few sequences (agihunt.info summary, KV cache
 * table at 1M tokens; the selection and reuse are those of
 * hs2_full_attn_select and hs2_sparse_attn_decode).  Shard q holds the
 * positions [offset_q, offset_q + shard_len_q) of every sequence, offsets
 * ascending with q and the shards tiling [0, kv_len).  One decode step of a
 * full-attention layer and its sparse layers, on every shard:
 *   1. hs2_decode_shard_attn: full attention over the shard -> (m, l) and an
 *      unnormalised O; the shard's logits stay in the workspace.
 *   2. exchange: all-gather the R (m, l) blocks -> ml_all [R][2][batch, Hq].
 *   3. hs2_partial_merge: global (M, L) per head -> ml_global [batch, Hq, 2],
 *      this shard's O rescaled to M.
 *   4. exchange: sum-all-reduce O32 over the shards.
 *   5. hs2_partial_finalize: O = O32 / L (bf16), the full-attention output.
 *   6. hs2_decode_shard_candidates: selection scores of the shard's
 *      candidates under the global (M, L), the shard's top-k as a list.
 *   7. exchange: all-gather the lists -> cand_all [R][...].
 *   8. hs2_decode_merge_candidates: the index row [batch, window + topk],
 *      identical to hs2_full_attn_select's on the whole cache.
 *   9. per sparse layer: hs2_sparse_decode_shard (the index entries that fall
 *      in the shard), then steps 2-5 again for that layer's output.
 * The exchanges are the caller's (e.g. NCCL through torch.distributed).
 * Results equal the single-GPU calls' up to the order of fp32 additions.
 *
 * hs2_decode_shard_attn:
 *   Q bf16 [batch, Hq, d]; Kc, Vc uint8 [batch, kv_stride_tokens, d] and
 *   k_scale, v_scale fp32 [batch, kv_stride_tokens]: the shard's part of the
 *   FP8 cache, local position i = global position offset + i, i < shard_len.
 *   ml_out fp32 [2][batch, Hq]: m (the max of the scaled logits, log2 units)
 *   then l (the sum of 2^(logit - m)); -inf and 0 for no key.
 *   O_out fp32 [batch, Hq, d]: sum_j 2^(logit_j - m) v_j, not normalised.
 *   workspace: hs2_decode_shard_workspace() bytes, 256-byte aligned; it must
 *   be kept, unchanged, for hs2_decode_shard_candidates of the same step.
 *   topk only sizes the workspace; pass the step's topk.
 */
HS2_API hs2_status hs2_decode_shard_workspace(int batch, int64_t shard_len, int n_idx, int Hq, int d,
                                              int topk, size_t* bytes);

HS2_API hs2_status hs2_decode_shard_attn(const void* Q, const void* Kc, const void* Vc,
                                         const float* k_scale, const float* v_scale, int batch,
                                         int64_t shard_len, int64_t kv_stride_tokens, int Hq, int d,
                                         int topk, float softmax_scale, float* ml_out, float* O_out,
                                         void* workspace, size_t ws_bytes, void* stream);

/*
 * ml_all fp32 [n_shards][2][batch, Hq] (every shard's ml_out, shard order);
 * O32 fp32 [batch, Hq, d]: shard `shard`'s O, rescaled in place by
 * 2^(m_shard - M); ml_out fp32 [batch, Hq, 2]: (M, L) with M = max m and
 * L = sum_q l_q 2^(m_q - M), the same on every shard.
 */
HS2_API hs2_status hs2_partial_merge(const float* ml_all, int n_shards, int shard, float* O32,
                                     float* ml_out, int batch, int Hq, int d, void* stream);

/* O bf16 [batch, Hq, d] = O32 / L, with ml = (M, L) [batch, Hq, 2]; 0 where L = 0. */
HS2_API hs2_status hs2_partial_finalize(const float* ml, const float* O32, void* O, int batch, int Hq,
                                        int d, void* stream);

/*
 * The shard's candidates are the global positions offset .. kv_len-1-window
 * that it holds; their selection scores sigma_j = sum_h 2^(logit_hj - M_h)/L_h
 * use the logits hs2_decode_shard_attn left in `workspace` and
 * ml_global = (M, L) from hs2_partial_merge.  cand (4-byte elements):
 * scores fp32 [batch, topk], then global positions int32 [batch, topk], then
 * list lengths int32 [batch]; a row's list is its top min(topk, n) candidates
 * in ascending position (the order of hs2_full_attn_select: score
 * descending, ties to the smaller position).  1 <= batch <= 65535.
 */
HS2_API hs2_status hs2_decode_shard_candidates(void* workspace, size_t ws_bytes, int batch,
                                               int64_t shard_len, int64_t shard_offset, int64_t kv_len,
                                               int Hq, int d, int window, int topk,
                                               const float* ml_global, void* cand, void* stream);

/*
 * cand_all: n_shards (<= 64) blocks of hs2_decode_shard_candidates' cand,
 * shard order.  idx int32 [batch, window + topk]: the window positions
 * kv_len-window .. kv_len-1 (-1 below 0), then the top-k of all lists in
 * ascending position, -1 padded.
 */
HS2_API hs2_status hs2_decode_merge_candidates(const void* cand_all, int n_shards, int batch,
                                               int64_t kv_len, int window, int topk, int32_t* idx,
                                               void* stream);

/*
 * A sparse layer's decode over one shard: hs2_sparse_attn_decode restricted
 * to the entries of idx (global positions) in [shard_offset,
 * shard_offset + shard_len), with the partial outputs of
 * hs2_decode_shard_attn (ml_out [2][batch, Hq], O_out fp32 [batch, Hq, d]).
 * The cache arguments are the shard's, as in hs2_decode_shard_attn.
 * workspace: hs2_decode_shard_workspace() bytes with this n_idx.
 */
HS2_API hs2_status hs2_sparse_decode_shard(const void* Q, const void* Kc, const void* Vc,
                                           const float* k_scale, const float* v_scale, int batch,
                                           int64_t shard_len, int64_t kv_stride_tokens,
                                           int64_t shard_offset, const int32_t* idx, int n_idx, int Hq,
                                           int d, float softmax_scale, float* ml_out, float* O_out,
                                           void* workspace, size_t ws_bytes, void* stream);

/*
 * Synchronises `stream`, then reads and clears the status word of the current
 * device: HS2_OK, HS2_ERR_DEVICE_CHECK or HS2_ERR_TIMEOUT (or HS2_ERR_CUDA if
 * the synchronisation itself failed).
 */
HS2_API hs2_status hs2_device_status(void* stream);

/*
 * Test hook for the bounded device waits: sets the iteration limit of every
 * inter-CTA spin-wait the library launches afterwards on the current device
 * (0 restores the default).  A limit of 1 makes a wait that is not already
 * satisfied give up at once and report HS2_ERR_TIMEOUT.
 */
HS2_API hs2_status hs2_set_spin_limit(int64_t iterations);

/*
 * Kernel timing (instrumentation; no counterpart in the method).  While
 * enabled on the calling host thread, every kernel the library launches is
 * bracketed by CUDA events recorded on its launch stream.
 *   hs2_profile_enable(1) starts a fresh record, hs2_profile_enable(0) stops.
 *   hs2_profile_collect() synchronises on the recorded events and returns, in
 *   launch order, up to max_n entries: names[i] (static strings owned by the
 *   library) and ms[i] (device time of launch i).  *n gets the number recorded
 *   (which may exceed max_n; at most 4096 are kept).  The record is cleared.
 */
HS2_API hs2_status hs2_profile_enable(int on);
HS2_API hs2_status hs2_profile_collect(const char** names, float* ms, int max_n, int* n);

#ifdef __cplusplus
}
#endif
#endif /* HS2_H_ */
