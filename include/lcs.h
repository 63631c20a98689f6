/*
 * lcs.h -- C ABI of liblcs, the B200 (sm_100a) compressed-attention hot path.
 *
 * The method is DeepSeek-V4's hybrid compressed attention as described in
 * "DeepSeek V4 深度解析" (section 2, compressed attention; section 4, FP4 and
 * KV-cache infrastructure) and in the "V3 vs V4" page (inline headings
 * "V4 改进一CSA 与 HCA" and "FP4 为什么能无损"):
 *   CSA  -- every m=4 adjacent tokens' KV pooled into one entry by
 *           position-biased softmax weights with overlapping blocks, a
 *           lightning indexer scoring every entry per query, top-k selection,
 *           and shared-KV MQA over the selection plus the last 128 raw tokens;
 *   HCA  -- the same pooling with m'=128 and dense MQA over all entries plus
 *           the window.
 *
 * Conventions (every function):
 *   - Return LCS_OK (0) or a negative LCS_ERR_* code.  A host-detectable error
 *     (null pointer, bad shape, unsupported dtype combination, short
 *     workspace) returns before anything is enqueued.
 *   - Tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     row-major in the shapes given.  The library allocates no device memory.
 *   - Work is enqueued on `stream` and is asynchronous.  Device-side errors (a
 *     bounded wait that ran out, an index out of range) are written to the
 *     status word at the start of the workspace; lcs_status() reads it.
 *   - Calls that need scratch take (ws, ws_bytes); lcs_workspace_size() gives
 *     the size.  Concurrent calls must not share a workspace.
 *   - No CPU fallback: with no usable sm_100 device every call returns
 *     LCS_ERR_CUDA.
 */
#ifndef LCS_H
#define LCS_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define LCS_API __attribute__((visibility("default")))
#else
#define LCS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define LCS_OK               0
#define LCS_ERR_INVALID     -1   /* null pointer, bad shape or parameter */
#define LCS_ERR_UNSUPPORTED -2   /* dtype / shape combination not implemented */
#define LCS_ERR_CUDA        -3   /* no sm_100 device, or a launch failed */
#define LCS_ERR_TIMEOUT     -4   /* a device-side bounded wait ran out */
#define LCS_ERR_DEVICE      -5   /* device-side check failed (index out of range) */
#define LCS_ERR_WORKSPACE   -6   /* workspace missing or too small */
#define LCS_ERR_TOO_LARGE   -7   /* needs more scratch than csa_attend_noalloc holds */

/* ---- storage types ---- */
#define LCS_F32   0   /* float32 */
#define LCS_BF16  1   /* bfloat16 */
#define LCS_KV_FP8 2  /* mixed-precision KV row ("DeepSeek V4 深度解析" §2, last paragraph:
                         RoPE dims BF16, the rest FP8): for D = 576 (512 content + 64 RoPE)
                         one row is 656 bytes = 512 E4M3 codes | 64 bf16 | 4 fp32 scales,
                         scale b applying to content dims [128b, 128b+128). */
#define LCS_FP4   3   /* FP4 E2M1 with one E4M3 scale per 32 elements ("DeepSeek V4 深度解析"
                         §4: the indexer's QK path is FP4).  A tensor of n vectors of length d
                         is two planes: n*d/2 packed bytes (element 2j in the low nibble of
                         byte j), then n*d/32 scale bytes. */

/* ---- attention modes ---- */
#define LCS_MODE_CSA 0
#define LCS_MODE_HCA 1

/* ---- workspace ops ---- */
#define LCS_OP_INDEX_TOPK 1
#define LCS_OP_ATTEND     2
#define LCS_OP_DECODE     3
#define LCS_OP_TOPK       4
#define LCS_OP_CP_SELECT  5

/*
 * Token compressor, CSA ("DeepSeek V4 深度解析" §2, CSA step 1; "V3 vs V4" page,
 * "V4 改进一": each m adjacent tokens' KV pooled into one entry by softmax
 * weights with a position bias; neighbouring blocks overlap a little).
 *
 * Entry j of request b pools tokens t = m*j - overlap + i, i = 0..m+overlap-1:
 *   p_i = softmax_i(z[b,t] + bias[i]),   e_j = sum_i p_i * x[b,t,:]
 * then rotates its last d_rope dims (rotate-half RoPE, frequency
 * rope_theta^(-2i/d_rope)) at absolute position pos0 + m*j + m - 1.
 * Tokens before the chunk (t < 0) come from x_tail/z_tail (the last `overlap`
 * tokens of the previous chunk); with x_tail == NULL they are left out and the
 * softmax is taken over the remaining positions.
 *
 *   x      [B, T, d]        LCS_F32 or LCS_BF16 (x_dtype)
 *   x_tail [B, overlap, d]  same dtype, or NULL
 *   z_tail [B, overlap]     fp32, non-NULL iff x_tail is
 *   z      [B, T]           fp32 pooling logits
 *   bias   [m + overlap]    fp32 position bias
 *   out    [B, T/m, d]      out_dtype (LCS_F32 or LCS_BF16), rounded to nearest even
 * T must be a multiple of m; 1 <= m <= 1024, 0 <= overlap <= 1024; d % 8 == 0;
 * d_rope even, 0 <= d_rope <= d.  No workspace.
 */
LCS_API int csa_compress(const void* x, int x_dtype, int64_t B, int64_t T, int d,
                 const void* x_tail, const float* z_tail, const float* z, const float* bias,
                 int m, int overlap, int d_rope, float rope_theta, int64_t pos0,
                 void* out, int out_dtype, cudaStream_t stream);

/*
 * Token compressor, HCA ("DeepSeek V4 深度解析" §2, HCA paragraph: compression
 * m' = 128, otherwise the same structure as CSA).  As csa_compress with no
 * overlap: entry j pools tokens [m*j, m*j + m).  bias has m entries.
 */
LCS_API int hca_compress(const void* x, int x_dtype, int64_t B, int64_t T, int d,
                 const float* z, const float* bias, int m, int d_rope, float rope_theta,
                 int64_t pos0, void* out, int out_dtype, cudaStream_t stream);

/*
 * Lightning indexer + top-k ("DeepSeek V4 深度解析" §2, CSA step 2: a light,
 * low-rank indexer scores the compressed entries and each query keeps the
 * top-k; "V3 vs V4" page, "FP4 为什么能无损": FP4 QK path, BF16 scores).
 *
 *   score[b,q,s] = sum_{h<H_I} w[b,q,h] * ReLU( qI[b,q,h,:] . kI[b,s,:] ),  s < n_avail
 * computed per head in fp32, summed over heads in the fixed order h = 0..H_I-1
 * with fused multiply-adds; for score_dtype LCS_BF16 the sum is rounded to bf16.
 *   idx[b,q,:] = the k entries with the largest scores (ties -> lower index),
 *                in ascending index order, padded with -1 when n_avail < k.
 * n_avail = N_c when q_pos is NULL (decode), else min(N_c, floor((q_pos+1)/m))
 * (entry j is complete once token m*j+m-1 has arrived).
 *
 *   qI  [B, Q, H_I, d_I]  LCS_F32 (with kI LCS_F32), or LCS_BF16 (with kI LCS_BF16,
 *                         or with kI LCS_FP4: qI is quantised to FP4 per (head,
 *                         32-block) on the fly, scale = E4M3(amax/6))
 *   w   [B, Q, H_I]       fp32
 *   kI  [B, N_c, d_I]     see qI; LCS_FP4 uses the two-plane layout over B*N_c vectors
 *   q_pos [B, Q] int64 or NULL (then Q must be 1)
 *   idx [B, Q, k] int32 (out)
 *   scores [B, Q, N_c] score_dtype, optional output (NULL: kept in the workspace);
 *                         entries s >= n_avail are unspecified
 * score_dtype: LCS_F32 (kI F32 or BF16) or LCS_BF16 (kI FP4).  d_I % 32 == 0,
 * H_I <= 128 (LCS_F32 path) or H_I == 64 (tensor-core paths).  Tensor-core paths:
 * qI and kI start on a 16-byte boundary (else LCS_ERR_INVALID).
 */
LCS_API int csa_index_topk(const void* qI, int qI_dtype, const float* w, const void* kI, int kI_dtype,
                   int64_t B, int64_t Q, int64_t N_c, int H_I, int d_I,
                   const int64_t* q_pos, int m, int k, int score_dtype,
                   int32_t* idx, void* scores, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Compressor with its input projections fused in ("DeepSeek V4 深度解析" §2, CSA step 1:
 * the pooled KV rows and the per-token pooling logits are linear in the token's hidden
 * state).  As csa_compress (hca_compress with overlap 0) on
 *   x[b,t,:] = h[b,t,:] . Wx   and   z[b,t] = h[b,t,:] . wz,
 * each projected value the fp32 fma chain over the hidden dims in order; the projected rows
 * stay on chip.
 *   h [B, T, hidden], h_tail [B, overlap, hidden] or NULL  h_dtype (LCS_F32 or LCS_BF16)
 *   Wx [hidden, d] h_dtype; wz [hidden] fp32; bias [m + overlap] fp32
 *   out [B, T/m, d] out_dtype (LCS_F32 or LCS_BF16)
 * CUDA cores, for small hidden states: LCS_ERR_UNSUPPORTED when one entry's window of hidden
 * and projected rows, (m + overlap) * (hidden + d + 1) floats, exceeds 150 KB.
 */
LCS_API int lcs_compress_proj(const void* h, int h_dtype, int64_t B, int64_t T, int hidden, const void* h_tail,
                 const void* Wx, int d, const float* wz, const float* bias, int m, int overlap,
                 int d_rope, float rope_theta, int64_t pos0, void* out, int out_dtype, cudaStream_t stream);

/*
 * Lightning indexer + top-k with the query projection fused in ("DeepSeek V4 深度解析" §2,
 * CSA step 2: the index heads and the per-head weights come from the query token's hidden
 * state).  As csa_index_topk on fp32 keys with
 *   qI[b,q,:,:] = h[b,q,:] . W_qI   (reshaped [H_I, d_I])   and   w[b,q,:] = h[b,q,:] . W_w,
 * each the fp32 fma chain over the hidden dims in order, then the fp32 score chains.
 *   h [B, Q, hidden] fp32; W_qI [hidden, H_I * d_I] fp32; W_w [hidden, H_I] fp32;
 *   kI [B, N_c, d_I] fp32; q_pos, m, k, idx, scores, ws as csa_index_topk (LCS_F32 scores).
 * hidden + H_I * (d_I + 1) <= 12288, H_I <= 128, d_I <= 256.
 */
LCS_API int csa_index_topk_proj(const float* h, int hidden, const float* W_qI, const float* W_w, const float* kI,
                 int64_t B, int64_t Q, int64_t N_c, int H_I, int d_I, const int64_t* q_pos, int m, int k,
                 int32_t* idx, float* scores, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Top-k alone over a given score array (the selection of csa_index_topk).
 *   scores [B, Q, N_c] LCS_F32 or LCS_BF16; q_pos/m as for csa_index_topk;
 *   idx [B, Q, k] int32 (out).
 */
LCS_API int lcs_topk(const void* scores, int score_dtype, int64_t B, int64_t Q, int64_t N_c,
             const int64_t* q_pos, int m, int k, int32_t* idx,
             void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * CSA sparse attention ("DeepSeek V4 深度解析" §2, CSA step 3: the selected
 * compressed entries together with the most recent W raw tokens; HCA
 * paragraph: shared-KV multi-query attention).
 *
 * For query (b,q) and every head h:
 *   rows R = { comp[b, idx[b,q,i]] : idx != -1 }  followed by the window rows
 *   o[b,q,h,:] = sum_{r in R} softmax_r( scale * q[b,q,h,:] . K_r ) * V_r
 * one softmax over all of R; K_r is the whole D-dim row, V_r its first d_v dims.
 * Window: every row of win[b] when q_pos is NULL (decode, Q == 1); else the rows
 * r with win_pos0[b] + r in [q_pos[b,q] - W + 1, q_pos[b,q]].
 *
 *   q    [B, Q, H, D]   LCS_F32 with kv LCS_F32; LCS_BF16 with kv LCS_BF16 or LCS_KV_FP8
 *   comp [B, N_c, row]  kv_dtype (row = D elements, or 656 bytes for LCS_KV_FP8)
 *   win  [B, Tw, row]   kv_dtype
 *   idx  [B, Q, k]      int32 selection: valid entries first, then -1 padding (the form
 *                       csa_index_topk returns); the first -1 ends the selection.  An
 *                       index >= N_c also ends it and records LCS_ERR_DEVICE.
 *   q_pos [B, Q], win_pos0 [B]  int64 device arrays, or both NULL (decode)
 *   out  [B, Q, H, d_v] out_dtype (LCS_F32 for f32 kv, LCS_BF16 otherwise)
 *   lse  [B, Q, H]      fp32 natural-log sum of exp(scale*q.K) over R, or NULL
 * Tensor-core paths: H == 64, D == 576, d_v == 512.  F32 path: H <= 64, D <= 128.
 * An empty R (no selected entry, no window row) gives o = 0 and lse = -inf.
 * Only rows of R contribute: rows of comp and win outside R may hold anything, NaN
 * included (a cache that fills as the sequence grows).  Tensor-core paths load runs of
 * consecutive rows by TMA: comp and win start on a 16-byte boundary (else
 * LCS_ERR_INVALID), and B*N_c, B*Tw stay below 2^31 (else LCS_ERR_UNSUPPORTED); both
 * are checked before anything is enqueued.
 */
LCS_API int csa_attend(const void* q, int q_dtype, const void* comp, const void* win, int kv_dtype,
               int64_t B, int64_t Q, int64_t N_c, int64_t Tw, const int32_t* idx, int k,
               const int64_t* q_pos, const int64_t* win_pos0, int W, int H, int D, int d_v,
               float scale, void* out, int out_dtype, float* lse,
               void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * HCA dense attention ("DeepSeek V4 深度解析" §2, HCA paragraph: no sparse
 * selection, dense attention over the compressed entries; show-notes glossary,
 * HCA: the query does not pick tokens).  As csa_attend with
 *   R = { comp[b, j] : j < n_avail }  followed by the window rows,
 * n_avail = N_c when q_pos is NULL, else min(N_c, floor((q_pos+1)/m)).
 */
LCS_API int hca_attend(const void* q, int q_dtype, const void* comp, const void* win, int kv_dtype,
               int64_t B, int64_t Q, int64_t N_c, int64_t Tw,
               const int64_t* q_pos, const int64_t* win_pos0, int m, int W, int H, int D, int d_v,
               float scale, void* out, int out_dtype, float* lse,
               void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * csa_attend without a workspace argument.  The pages describe no such call:
 * it exists for callers that cannot hand the library any device memory --
 * e.g. a serving engine that reserved nearly all of HBM for its KV-cache pool
 * at start-up (a later allocation would fail or fragment the pool), or a host
 * program that links only this library and keeps no device allocator.
 *
 * Arguments, layouts, results and host-side validation are those of
 * csa_attend, with (ws, ws_bytes) replaced by
 *   status_out  optional device int (NULL = not wanted) that receives, in
 *               stream order, this call's device status (0 or a LCS_ERR_*
 *               code, as lcs_status would report it).
 * Scratch: a fixed library-owned device array of LCS_NOALLOC_SCRATCH_BYTES per
 * device (256-byte aligned) holding the status word and the split partials.
 * A problem whose scratch exceeds it returns LCS_ERR_TOO_LARGE before anything
 * is enqueued; on a 148-SM B200 every shape csa_attend accepts fits.
 * The call itself makes no cudaMalloc / cudaFree and no allocating library
 * call; it clears the status word (cudaMemsetAsync) before its kernels run.
 * The first call on each device looks the array up with cudaGetSymbolAddress
 * (with that device current), which may make the CUDA runtime load the
 * module that holds the array; make that first call before any stream
 * capture starts.  The lookup is repeated when the device's context has
 * changed since (a cudaDeviceReset destroys the context and the module with
 * it); make the first call after such a reset before any capture as well.
 * Returns LCS_ERR_CUDA if the lookup fails.
 * All calls on one device share the array: calls that overlap in time (other
 * streams, other host threads) race on it and must be serialised by the caller.
 */
#define LCS_NOALLOC_SCRATCH_BYTES (20u << 20)
LCS_API int csa_attend_noalloc(const void* q, int q_dtype, const void* comp, const void* win, int kv_dtype,
               int64_t B, int64_t Q, int64_t N_c, int64_t Tw, const int32_t* idx, int k,
               const int64_t* q_pos, const int64_t* win_pos0, int W, int H, int D, int d_v,
               float scale, void* out, int out_dtype, float* lse,
               int* status_out, cudaStream_t stream);

/*
 * Fused decode step: one new token per request, one call.
 *   mode LCS_MODE_CSA: csa_index_topk -> csa_attend (q_pos = NULL, window = all Tw rows)
 *   mode LCS_MODE_HCA: hca_attend (indexer arguments ignored, may be NULL)
 * Arguments as in those calls with Q = 1.  idx_out [B, k] (optional) receives the
 * selection.  The stages are chained on `stream` with programmatic dependent
 * launch; nothing returns to the host between them.
 */
LCS_API int decode_fused(int mode, int64_t B,
                 const void* q, int q_dtype, const void* comp, const void* win, int kv_dtype,
                 int64_t N_c, int64_t Tw, int H, int D, int d_v, float scale,
                 const void* qI, int qI_dtype, const float* w, const void* kI, int kI_dtype,
                 int H_I, int d_I, int k, int score_dtype,
                 void* out, int out_dtype, float* lse, int32_t* idx_out,
                 void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Decode-time cache update ("DeepSeek V4 深度解析" §4, KV-cache management for the
 * mixed attention: a state cache holding the sliding window and the raw tokens not yet
 * enough to compress, and a compressed cache of CSA and HCA entries).  Appends one new
 * token to each request; request b's token sits at position t = pos[b] (the number of
 * tokens the request had before), and pos[b] < 0 appends nothing to request b.
 *   state cache:  raw    [B, 128, D + d_I] x_dtype  ring of the last 128 raw (un-rotated)
 *                        tokens, KV row then index-key row, slot t % 128;
 *                 logits [B, 3, 128] fp32  ring of the tokens' pooling logits (z, zI, zh);
 *                 win    [B, 128, row] win_dtype  the window: slot t % 128 receives the
 *                        token's KV row rotated at position t (the rows csa_attend reads);
 *   compressed cache, written when an entry's last token arrives:
 *                 comp [B, N_c, row] kv_dtype   CSA entry j = t/4 when (t+1) % 4 == 0: tokens
 *                        4j-2 .. 4j+3 (those >= 0) pooled with softmax(z + bias[0..5]), then
 *                        rotated at position t (as csa_compress with m = 4, overlap 2);
 *                 kI   [B, N_c, d_I] or FP4 planes (kI_dtype)  index key j, pooled the same
 *                        way from the index-key rows with zI and biasI, no rotation;
 *                 hca  [B, N_h, row] kv_dtype   HCA entry h = t/128 when (t+1) % 128 == 0:
 *                        tokens 128h .. 128h+127 pooled with softmax(zh + biash[0..127]),
 *                        rotated at position t (as hca_compress with m' = 128).
 *   x [B, D], kx [B, d_I]  x_dtype (LCS_F32 or LCS_BF16) the new token's raw rows;
 *   z, zI, zh [B] fp32; bias [6], biasI [6], biash [128] fp32.
 * Storage: kv_dtype and win_dtype LCS_F32, LCS_BF16 or LCS_KV_FP8 (content D - d_rope a
 * multiple of 128; quantised exactly as lcs_quant_kv_fp8 quantises the fp32 entry);
 * kI_dtype LCS_F32, LCS_BF16 or LCS_FP4 (as lcs_quant_fp4).  The rings are read only at
 * slots of tokens already appended.  An entry index >= N_c or >= N_h is not written and
 * records LCS_ERR_DEVICE in the status word of ws (>= 256 bytes, 256-byte aligned).
 * D % 8 == 0, d_I % 32 == 0, d_rope even.
 */
LCS_API int lcs_cache_append(int64_t B, const int64_t* pos, const void* x, const void* kx, int x_dtype,
                 const float* z, const float* zI, const float* zh,
                 const float* bias, const float* biasI, const float* biash,
                 int D, int d_rope, int d_I, float rope_theta, void* raw, float* logits,
                 void* win, int win_dtype, void* comp, void* kI, void* hca, int64_t N_c, int64_t N_h,
                 int kv_dtype, int kI_dtype, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Context parallelism for long requests: the compressed entries (and index keys) of every
 * request are split over G ranks, rank r holding the S entries [offset, offset + S).  One
 * decode step is, on every rank: csa_index_topk over the rank's entries (local top-k, local
 * indices), lcs_cp_candidates, an all-gather of the candidates in rank order, lcs_cp_select,
 * csa_attend over the rank's share of the selection (with lse; the window rows on the rank
 * that holds them, Tw = 0 elsewhere), an all-gather of (o, lse) in rank order, and
 * lcs_attn_merge.  The result equals the unsplit step ("DeepSeek V4 深度解析" §2, CSA steps
 * 2-3): every global top-k entry is in the top-k of its own shard, and candidates gathered in
 * rank order are in global-index order, so the selection and its tie rule are unchanged; one
 * softmax over disjoint row sets is the log-sum-exp merge of the parts.
 *
 * lcs_cp_candidates: scores [B, S] (LCS_F32 or LCS_BF16; csa_index_topk's scores output),
 *   idx_local [B, k] (its selection) -> cand_score [B, k] fp32 and cand_idx [B, k] int32
 *   global index offset + local; -1 entries become (-inf, -1).
 * lcs_cp_select: cand_score, cand_idx [G, B, k] (all ranks' candidates, rank r at r) ->
 *   idx_global [B, k] the global top-k (ascending, -1 padded, ties -> lower index) and
 *   idx_local [B, k] the entries of [offset, offset + S) among them, as local indices
 *   (ascending, -1 padded: csa_attend's selection form).  Workspace: lcs_workspace_size(
 *   LCS_OP_CP_SELECT, B, G, 0, 0, k, ...).
 * lcs_attn_merge: o [G, rows, d_v] fp32 and lse [G, rows] fp32 (rank r's normalised
 *   attention output and natural-log sum of exp; -inf for an empty row set) -> out
 *   [rows, d_v] (LCS_F32 or LCS_BF16) = sum_r exp(lse_r - L) o_r with L = log sum_r
 *   exp(lse_r), summed in rank order; lse_out [rows] = L (or NULL).
 */
LCS_API int lcs_cp_candidates(const void* scores, int score_dtype, int64_t B, int64_t S, const int32_t* idx_local,
                 int k, int64_t offset, float* cand_score, int32_t* cand_idx, cudaStream_t stream);
LCS_API int lcs_cp_select(const float* cand_score, const int32_t* cand_idx, int G, int64_t B, int k,
                 int64_t offset, int64_t S, int32_t* idx_global, int32_t* idx_local,
                 void* ws, size_t ws_bytes, cudaStream_t stream);
LCS_API int lcs_attn_merge(const float* o, const float* lse, int G, int64_t rows, int d_v, void* out,
                 int out_dtype, float* lse_out, cudaStream_t stream);

/*
 * Grouped output projection ("DeepSeek V4 深度解析" §2, HCA paragraph: both use a
 * grouped output projection to cut compute; "V3 vs V4" page: 输出端分组投影).
 * The H heads of each token are split into G groups of H/G consecutive heads;
 *   y_g = o[t, heads of g, :] (flattened, (H/G)*d_v) . Wg[g]   -> d_g dims
 *   y[t] = concat_g(y_g) . Wo                                   -> hidden dims
 *   o [T, H, d_v], Wg [G, (H/G)*d_v, d_g], Wo [G*d_g, hidden], y [T, hidden]; fp32.
 * H % G == 0; (H/G)*d_v <= 4096; G*d_g <= 1024.  No workspace.
 */
LCS_API int group_oproj(const float* o, int64_t T, int H, int d_v, const float* Wg, int G, int d_g,
                const float* Wo, int hidden, float* y, cudaStream_t stream);

/*
 * Rotate-half RoPE in place on the last d_rope dims of n rows at positions
 * pos[n] (int64, device): pair (c+i, c+i+d_rope/2), c = d - d_rope, angle
 * pos * rope_theta^(-2i/d_rope).  rows LCS_F32 or LCS_BF16 [n, d].
 */
LCS_API int lcs_rope(void* rows, int dtype, int64_t n, int d, int d_rope, float rope_theta,
             const int64_t* pos, cudaStream_t stream);

/*
 * Cache writers for the two quantised formats ("DeepSeek V4 深度解析" §2 last
 * paragraph and §4).
 *   lcs_quant_kv_fp8: x [n, d_c + d_r] fp32 -> LCS_KV_FP8 rows [n, d_c + 2 d_r + 4 d_c/128]:
 *     per 128-block scale = the smallest power of two >= amax/448 (amax/448 in fp32;
 *     1 when amax is 0), code = E4M3(x/scale), round to nearest even; the d_r RoPE
 *     dims rounded to bf16.  The power-of-two scale makes code*scale exact in bf16.
 *   lcs_quant_fp4: x [n, d] fp32 -> LCS_FP4 planes (out: n*d/2 + n*d/32 bytes):
 *     per 32-block scale = E4M3(amax/6) (1 when that is 0), code = E2M1(x/scale).
 * d_c % 128 == 0, d % 32 == 0.
 */
LCS_API int lcs_quant_kv_fp8(const float* x, int64_t n, int d_c, int d_r, void* out, cudaStream_t stream);
LCS_API int lcs_quant_fp4(const float* x, int64_t n, int d, void* out, cudaStream_t stream);

/*
 * Workspace bytes for op (LCS_OP_*) at the given sizes (unused sizes ignored):
 *   LCS_OP_INDEX_TOPK: B, Q, N_c, k, score_dtype     LCS_OP_TOPK: B, Q, N_c, k
 *   LCS_OP_ATTEND: B, Q, H, d_v (+ N_c, Tw, k for the split plan)
 *   LCS_OP_CP_SELECT: B, Q = G (ranks), k
 *   LCS_OP_DECODE: everything (both stages)
 * Returns a negative value for invalid sizes.  The first 256 bytes hold the
 * status word; the workspace must be 256-byte aligned.
 */
LCS_API int64_t lcs_workspace_size(int op, int64_t B, int64_t Q, int64_t N_c, int64_t Tw, int k,
                           int H, int d_v, int score_dtype);

/*
 * Synchronises `stream`, returns the first device-side error recorded in the
 * workspace's status word since the last call (LCS_OK if none) and clears it.
 */
LCS_API int lcs_status(void* ws, cudaStream_t stream);

/* Clears the status word (enqueued on stream). */
LCS_API int lcs_clear_status(void* ws, cudaStream_t stream);

/*
 * Self-test of the bounded waits every pipelined kernel uses (the pages describe no
 * such call).  Clears the status word of ws, then one CTA waits on an mbarrier that
 * nothing completes: the wait gives up after budget_us microseconds (1..1e6) and
 * records LCS_ERR_TIMEOUT, detail 901, in the status word; a second wait in the same
 * CTA must then give up at once (detail 902 is not recorded: the first error stays).
 * The kernel returns normally and the context stays usable.
 *   ws   device workspace (>= 256 bytes, 256-byte aligned)
 *   out  4 device int64: [first wait succeeded (0/1), its ns, second wait succeeded, its ns]
 * Returns LCS_ERR_INVALID for bad arguments, LCS_ERR_CUDA without a device; the
 * results are in ws and out once the stream reaches the kernel.
 */
LCS_API int lcs_selftest_wait(int budget_us, void* ws, size_t ws_bytes, long long* out, cudaStream_t stream);

/* Static description of a status code. */
LCS_API const char* lcs_error_string(int code);

/*
 * Profiling hook: when n >= 2 events are registered, decode_fused and
 * csa_index_topk record events[0] before their first stage and events[i] after
 * stage i (i >= 1, up to n-1) on the call's stream (decode_fused CSA: index,
 * top-k, attention; HCA: attention; csa_index_topk: index, top-k).  Stages are
 * then launched without programmatic overlap.  Pass n = 0 to stop.  Not
 * thread-safe.
 */
LCS_API int lcs_set_stage_events(cudaEvent_t const* events, int n);

#ifdef __cplusplus
}
#endif
#endif /* LCS_H */
