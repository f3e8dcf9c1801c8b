/*
 * dsa_b200.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention path.
 *
 * The path has four steps, each one entry point:
 *
 *   csa_compress        CSA: pool every m consecutive cache rows into one entry
 *   dsa_indexer_logits  lightning indexer: one score per (query row, cached key)
 *   dsa_topk            per query row, the k best-scoring visible keys
 *   dsa_sparse_mla      MQA-mode MLA attention over the selected latent rows
 *
 * and two variants of the last step for DeepSeek-V4's compressed attention:
 *
 *   csa_core_attention  CSA: the selected compressed entries plus a window and a sink of raw rows
 *   hca_attention       HCA: dense attention over every visible heavily compressed entry
 *
 * and the step before the path, which makes the indexer's inputs:
 *
 *   dsa_indexer_prepare     indexer queries, head weights and keys from the hidden
 *                           states and the query latent; keys written into the cache
 *   dsa_indexer_key_append  the key-cache write alone, for keys already projected
 *
 * Conventions shared by every entry point
 *   - Every data pointer is a DEVICE pointer owned by the caller.  The library
 *     never allocates or frees device memory; scratch space, where a step
 *     needs some, is a caller-provided workspace whose size the matching
 *     *_workspace_size() function returns (dsa_sparse_mla_noalloc instead
 *     uses a fixed scratch array in the library's own device memory).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on that stream and returns; it
 *     never synchronizes, except dsa_get_device_error().
 *   - Every call returns a dsa_status_t.  Arguments are validated on the host
 *     before anything is launched: an invalid argument returns
 *     DSA_ERR_INVALID_ARG, a shape or type combination for which no kernel is
 *     built returns DSA_ERR_UNSUPPORTED, and nothing is enqueued in either
 *     case.  A failed launch returns DSA_ERR_CUDA.  dsa_last_error() gives a
 *     one-line reason for the most recent failure on the calling thread.
 *   - Kernels that wait on asynchronous copies bound every wait; a wait that
 *     runs out records a device error instead of hanging, readable with
 *     dsa_get_device_error().
 *   - Tensor layouts are dense, row-major, innermost dimension last, with no
 *     padding unless a leading dimension argument says otherwise.
 *   - Nothing is thrown across this interface.
 *
 * Sources are cited by page title and section.  "DSA article" below is
 * "DeepSeek-V3.2稀疏注意力机制原理与TPU适配" (trdm.cn); "V4 CSA summary" is the
 * xhh.club summary of DeepSeek-V4's compressed sparse attention.
 */
#ifndef DSA_B200_H
#define DSA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer ... */
    DSA_ERR_UNSUPPORTED = 2,    /* valid, but no kernel is built for this shape/type */
    DSA_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
    DSA_ERR_DEVICE_TIMEOUT = 4  /* a kernel gave up a bounded wait (see dsa_get_device_error) */
} dsa_status_t;

typedef enum {
    DSA_FP32 = 0,
    DSA_BF16 = 1,
    DSA_FP8_E4M3 = 2,           /* OCP e4m3 "fn": bias 7, max 448, no infinities */
    DSA_FP4_E2M1 = 3            /* OCP e2m1: bias 1, values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their
                                   negatives; two per byte, the lower dim in the low nibble */
} dsa_dtype_t;

/* Library version (major*10000 + minor*100 + patch). */
DSA_API int dsa_version(void);

/* One-line reason for the most recent non-DSA_OK status on this thread. */
DSA_API const char* dsa_last_error(void);

/* Number of kernels this library has launched from the calling thread since
 * the process started (a plain counter, for benchmarks and tests). */
DSA_API uint64_t dsa_launch_count(void);

/*
 * csa_compress -- CSA token compression.
 *   dst[b, i, :] = (1/m) * sum_{r<m} src[b, m*i + r, :]
 * Every m consecutive rows of a cache become one "super entry" (V4 CSA
 * summary: 4 tokens -> 1; "解密DeepSeek-V4 ..." section 4.3: average pooling or
 * a small network -- average pooling is what is built).  Used on both the
 * MLA latent cache (D = 576) and the indexer key cache (D = 128), and with
 * m = 128 for HCA ("DeepSeek-V4 技术报告深度解析": m' = 128).
 *
 *   src    [batch, len, dim]   of `dtype` (DSA_BF16 or DSA_FP32)
 *   dst    [batch, len/m, dim] of `dtype`
 * The sum is formed exactly (double precision) and rounded once to the
 * storage type, round-to-nearest-even (exact as long as the m values of a
 * column span fewer than about 45 binary orders of magnitude).  len must be
 * a multiple of m; m in [1, 1024]; src and dst must not overlap; both
 * 16-byte aligned.
 */
DSA_API dsa_status_t csa_compress(const void* src, dsa_dtype_t dtype, int batch, int len, int dim, int m,
                          void* dst, void* stream);

/*
 * dsa_indexer_logits -- lightning-indexer scores (DSA article, section 1.3,
 * 闪电索引器; section 3, Step 2 "compute mqa logits").
 *   logits[t, s] = sum_{j<n_heads} w[t, j] * ReLU( sum_{d<head_dim} q[t, j, d] * k[b, s, d] )
 * for every key s <= row_pos[t] of cache b = row_batch[t].  The keys are
 * shared by all indexer heads (MQA style); w is per query row and head.
 *
 *   q          [rows, n_heads, head_dim]  of q_dtype (DSA_FP32 or DSA_BF16)
 *   w          [rows, n_heads] fp32
 *   k          [batch, ctx_len, head_dim] of k_dtype (DSA_FP32, DSA_BF16 or DSA_FP8_E4M3), or
 *              [batch, ctx_len, head_dim / 2] bytes of DSA_FP4_E2M1 code pairs
 *   k_scale    [batch, ctx_len] fp32, one dequantisation scale per fp8 / fp4 key
 *              row (stored key = code * scale); must be NULL unless k is fp8 or fp4
 *   row_batch  [rows] int32, cache of each query row, in [0, batch)
 *   row_pos    [rows] int32, last visible key of each row, in [0, ctx_len):
 *              prefill rows use their own position (causal), decode rows use
 *              ctx_len-1
 *   logits     [rows, ld_logits] fp32, ld_logits >= ctx_len.  Entries
 *              s <= row_pos[t] are written; entries beyond row_pos[t] are
 *              left untouched (dsa_topk never reads them).
 * Accumulation is fp32.  Supported: head_dim in {32, 64, 128}; q and k of the
 * same floating type, or bf16 q with fp8 k; n_heads <= 128; fp4 keys (V4 CSA
 * summary: the V4 indexer keys are FP4) with bf16 q, n_heads = 64 and
 * head_dim = 128.  fp8 key codes must be finite (0x7F and 0xFF, the e4m3 NaNs,
 * are not valid codes).  With fp8 or fp4 keys the products are formed in f16:
 * every code is exact in f16, and so is every bf16 query value with
 * 2^-14 <= |q| <= 65504 (smaller ones are rounded to f16's subnormal grid,
 * an error below 2^-25 each; larger ones are not supported).
 */
DSA_API dsa_status_t dsa_indexer_logits(const void* q, dsa_dtype_t q_dtype, const float* w,
                                const void* k, dsa_dtype_t k_dtype, const float* k_scale,
                                const int32_t* row_batch, const int32_t* row_pos,
                                int rows, int batch, int ctx_len, int n_heads, int head_dim,
                                float* logits, int64_t ld_logits, void* stream);

/* Workspace bytes dsa_topk needs for these sizes (0 = none). */
DSA_API size_t dsa_topk_workspace_size(int rows, int ctx_len, int k);

/*
 * dsa_topk -- per-row top-k selection (DSA article, section 1.3: keep only
 * the key-value entries of the top-k index scores; section 3, Step 3: when
 * the visible context is no longer than k, every token is kept).
 *
 *   logits     [rows, ld] fp32; row t is read at s = 0 .. row_pos[t]
 *   row_pos    [rows] int32, last visible key of each row
 *   idx        [rows, k] int32 output: the selected key positions in
 *              ascending position order, then -1 in every unused slot
 *              (a row with n = row_pos+1 <= k visible keys selects all n).
 * Order of scores: larger first; equal scores (with -0.0 == +0.0) go to the
 * lower position; -inf is the lowest score.  The selection is exact and
 * deterministic.  NaN scores are not supported.  k in [1, 8192];
 * ctx_len <= ld; ctx_len <= 327680 (a row is held on chip by at most 8 SMs).
 */
DSA_API dsa_status_t dsa_topk(const float* logits, int64_t ld, const int32_t* row_pos, int rows, int ctx_len,
                      int k, int32_t* idx, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes dsa_sparse_mla needs for these sizes (0 = none). */
DSA_API size_t dsa_sparse_mla_workspace_size(int rows, int k, int n_heads, int d_qk, int d_v, dsa_dtype_t dtype);

/*
 * dsa_sparse_mla -- attention over the selected latent rows only, MLA in
 * MQA mode (DSA article, section 1.3 细粒度稀疏注意力; section 1.4: every
 * latent KV entry is shared by all query heads; section 3, Step 4: decode
 * reads only the selected KV rows, index_mask drops the rest).
 *   z_s        = scale * q[t, h, :] . c_s[0:d_qk]           for s in idx[t, :], s >= 0
 *   out[t,h,:] = sum_s softmax_s(z) * c_s[0:d_v]
 *   lse[t,h]   = log sum_s exp(z_s)
 * where c_s is latent row s of cache b = row_batch[t].
 *
 *   q          [rows, n_heads, d_qk] of dtype (DSA_BF16 or DSA_FP32)
 *   kv         contiguous cache [batch, ctx_len, d_qk] when page_table is NULL;
 *              paged cache [num_pages, page_size, d_qk] otherwise, with
 *              c_s = kv[page_table[b, s / page_size], s % page_size, :]
 *   page_table [batch, ctx_len / page_size] int32 physical page ids in
 *              [0, num_pages), or NULL (then page_size and num_pages are ignored);
 *              an id outside the range is skipped and reported by
 *              dsa_get_device_error
 *   row_batch  [rows] int32
 *   idx        [rows, k] int32 key positions in [0, ctx_len); -1 = unused
 *              slot (skipped).  Order within a row does not matter.
 *   out        [rows, n_heads, d_v] of dtype (bf16 rounded to nearest even)
 *   lse        [rows, n_heads] fp32 natural-log sum of exp of the scaled
 *              logits; -inf (and out = 0) for a row with no selected key.
 * Supported: (d_qk, d_v) = (576, 512) bf16 with n_heads = 128, or
 * d_qk, d_v <= 64 multiples of 32 in fp32 or bf16 with n_heads a multiple of 8.
 */
DSA_API dsa_status_t dsa_sparse_mla(const void* q, const void* kv, dsa_dtype_t dtype,
                            const int32_t* page_table, int page_size, int num_pages,
                            const int32_t* row_batch, const int32_t* idx, int k,
                            int rows, int batch, int ctx_len, int n_heads, int d_qk, int d_v,
                            float scale, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * csa_core_attention -- CSA core attention with the window and attention-sink
 * segments ("DeepSeek V4 发布：1.6T 参数、百万上下文…", section on CSA: the
 * window KV and the compressed KV are concatenated and attended together;
 * CSA pipeline "compress -> index selection -> core attention" in
 * "DeepSeek-V4 技术报告深度解析"; "解密DeepSeek-V4 预览版…" section 4.3 and
 * "打破幻觉与成本魔咒：DeepSeek-V4 …" section 3.3.2: local dependencies are
 * kept by sliding-window attention together with an attention sink).  Slot
 * s of query row t holds
 *   s <  k:            the selected compressed entry idx[t, s] of kv, exactly
 *                      as in dsa_sparse_mla (-1 = unused slot);
 *   k <= s < k+window: the raw (uncompressed) cache row
 *                      p = win_pos[t] - window + 1 + (s - k) of kv_win,
 *                      unused when p < 0;
 *   k+window <= s < k+window+n_sink:
 *                      the sink: raw row j = s - k - window of kv_win (the
 *                      sequence's first rows), used only when
 *                      j < win_pos[t] - window + 1, i.e. before the window's
 *                      first row (so no raw row is attended twice, and none
 *                      after the query),
 * and attention runs over all used slots together:
 *   out[t,h,:] = sum_s softmax_s(scale * q[t,h,:] . c_s[0:d_qk]) * c_s[0:d_v].
 * A raw row is not deduplicated against a compressed entry that covers it:
 * the two are different vectors.
 *
 *   kv_win   [batch, win_len, d_qk] contiguous raw cache of dtype, 16-byte
 *            aligned (the bf16 tensor-core path)
 *   win_pos  [rows] int32 raw position of each query (its window ends there);
 *            win_pos[t] >= win_len is skipped and reported by
 *            dsa_get_device_error
 *   window   rows per window, >= 0
 *   n_sink   sink rows, 0 <= n_sink <= win_len (0: no sink; window = n_sink
 *            = 0: plain dsa_sparse_mla); k >= 0 and k + window + n_sink >= 1;
 *            idx may be NULL when k = 0; kv_win and win_pos are needed when
 *            window + n_sink > 0
 * Other arguments, layouts, results and errors are those of dsa_sparse_mla;
 * the workspace is dsa_sparse_mla_workspace_size(rows, k + window + n_sink, ...).
 * The pages give neither the window size nor the number of sink rows: the
 * caller chooses both.  The sink is read as the sequence's first raw rows,
 * the form that pairs a sink with a sliding window (a learned per-head
 * logit is another reading; the pages define neither).
 */
DSA_API dsa_status_t csa_core_attention(const void* q, const void* kv, dsa_dtype_t dtype,
                            const int32_t* page_table, int page_size, int num_pages,
                            const int32_t* row_batch, const int32_t* idx, int k,
                            int rows, int batch, int ctx_len,
                            const void* kv_win, const int32_t* win_pos, int win_len, int window,
                            int n_sink, int n_heads, int d_qk, int d_v, float scale, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * hca_attention -- HCA, heavily compressed attention ("DeepSeek-V4
 * 技术报告深度解析": m' = 128, no sparse selection; "DeepSeek V4 发布…": every
 * query sees all compressed KV, dense attention).  Dense MQA attention over
 * every visible entry of a compressed latent cache (from csa_compress with
 * m = 128):
 *   out[t,h,:] = sum_{s <= row_last[t]} softmax_s(scale * q[t,h,:] . c_s[0:d_qk]) * c_s[0:d_v]
 * with c_s entry s of cache b = row_batch[t].
 *
 *   kv        [batch, ctx_len, d_qk] contiguous compressed cache
 *   row_last  [rows] int32: last visible entry of each row (ctx_len - 1 in
 *             decode; -1: none visible, out = 0 and lse = -inf); entries
 *             past ctx_len - 1 are not read
 * Other arguments, layouts and errors are those of dsa_sparse_mla; the
 * workspace is dsa_sparse_mla_workspace_size(rows, ctx_len, ...).
 */
DSA_API dsa_status_t hca_attention(const void* q, const void* kv, dsa_dtype_t dtype,
                            const int32_t* row_batch, const int32_t* row_last,
                            int rows, int batch, int ctx_len, int n_heads, int d_qk, int d_v,
                            float scale, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the fixed device scratch that dsa_sparse_mla_noalloc uses. */
#define DSA_MLA_NOALLOC_SCRATCH_BYTES ((size_t)20 << 20)

/*
 * dsa_sparse_mla_noalloc -- dsa_sparse_mla without a workspace argument; it
 * allocates nothing, by any route.  The method itself has no counterpart:
 * this is an interface for callers that may not allocate device memory
 * while they run a step, such as a serving engine that hands nearly all of
 * HBM to its paged KV cache up front and keeps cudaMalloc/cudaFree (which
 * can block and synchronize the device) out of its decode loop, or a plain C
 * caller with no device allocator of its own.
 *
 * Arguments, layouts, results and errors are those of dsa_sparse_mla.  The
 * partial results of a split key list go to a static scratch array of
 * DSA_MLA_NOALLOC_SCRATCH_BYTES in the library's device memory (one copy per
 * device), whose address is looked up on the first call on each device: make
 * that first call before any stream capture.  Sizes whose partials do not
 * fit return DSA_ERR_INVALID_ARG with the byte counts in dsa_last_error()
 * and enqueue nothing (on a 148-SM B200 every size fits).  No part of the
 * scratch needs clearing between calls.  Calls that overlap in time on one
 * device -- from two streams or two threads -- race on the scratch and give
 * undefined results; calls in order on one stream are safe.
 */
DSA_API dsa_status_t dsa_sparse_mla_noalloc(const void* q, const void* kv, dsa_dtype_t dtype,
                            const int32_t* page_table, int page_size, int num_pages,
                            const int32_t* row_batch, const int32_t* idx, int k,
                            int rows, int batch, int ctx_len, int n_heads, int d_qk, int d_v,
                            float scale, void* out, float* lse, void* stream);

/* Workspace bytes dsa_indexer_prepare needs for these sizes on the current
 * device (0 when tokens == 0). */
DSA_API size_t dsa_indexer_prepare_workspace_size(int tokens, int n_heads, int d_c, int d_model);

/*
 * dsa_indexer_prepare -- the indexer's inputs for `tokens` new tokens (DSA
 * article, section 3, Step 1: the query latent is RMS-normalised and
 * projected up, the result split into a part with and a part without rotary
 * position encoding, the former turned by apply_rotary_emb, and weights_proj
 * gives the per-head weights; section 1.3: a learned linear map takes query
 * and key to 128 dims), in three launches: the latent's norm, the three
 * projections on the tensor cores, the key-cache write:
 *
 *   q_out[t, j, :] = RoPE( W_qb[j*128 .. j*128+127] . RMSNorm(c_q[t]) )
 *   w_out[t, :]    = W_w . h[t]
 *   key row        = RoPE( W_k . h[t] ), written to row slot[t] of the cache
 *
 *   RMSNorm(x)  = x / sqrt(mean(x^2) + eps) * q_norm_weight
 *   RoPE        turns dims (2i, 2i+1), i < d_rope/2, of every 128-dim head by
 *               the angle whose cosine / sine are rope_cos / rope_sin[pos[t], i]:
 *               (a, b) -> (a cos - b sin, a sin + b cos); dims >= d_rope carry
 *               no position.
 *
 *   c_q           [tokens, d_c] bf16: the low-rank query latent (before its norm)
 *   q_norm_weight [d_c] fp32, the norm's gain; eps >= 0
 *   wq_b          [n_heads * 128, d_c] bf16 (row-major, out x in)
 *   h             [tokens, d_model] bf16 hidden states
 *   wk            [128, d_model] bf16;  w_proj [n_heads, d_model] bf16
 *   rope_cos, rope_sin  [max_pos, d_rope / 2] fp32 (may be NULL when d_rope = 0)
 *   pos           [tokens] int32 position of each token, in [0, max_pos) when d_rope > 0
 *   slot          [tokens] int64 cache row of each token's key, in [0, cache_rows),
 *                 or -1: the key is not stored
 *   q_out         [tokens, n_heads, 128] bf16;  w_out [tokens, n_heads] fp32
 *   k_cache       [cache_rows, 128] of k_dtype: DSA_BF16 (rounded to nearest even),
 *                 DSA_FP8_E4M3 (codes) or DSA_FP4_E2M1 ([cache_rows, 64] code pairs,
 *                 element 2j in the low nibble); k_scale [cache_rows] fp32 for fp8 /
 *                 fp4 (NULL for bf16): scale = amax / 448 (fp8) or amax / 6 (fp4) of
 *                 the rotated row (1 for an all-zero row), code = the nearest code of
 *                 value / scale, ties to even, saturating at the largest finite code;
 *                 all of it in binary32 with every operation rounded on its own
 *   workspace     dsa_indexer_prepare_workspace_size() bytes, 256-byte aligned; no
 *                 part of it needs to hold anything on entry (it carries the scaled
 *                 latent and 1/RMS of each token and the fp32 partial sums of the
 *                 key and weight projections, which the last kernel adds up in a
 *                 fixed order)
 * The projections multiply bf16 operands with fp32 accumulation; the norm's
 * gain is applied to c_q in bf16 (c_q * gain rounded once) and 1/RMS (fp32)
 * to the product.  head_dim must be 128; d_c and d_model multiples of 64,
 * d_c <= 16384;
 * n_heads <= 256; d_rope even and <= 128.  c_q, h, the weights,
 * q_norm_weight and q_out 16-byte aligned.  Rows of other tokens in the cache
 * are not touched.  A token whose position or slot is out of range is
 * skipped and recorded in the device error word (dsa_get_device_error()
 * then returns DSA_ERR_INVALID_ARG).
 */
DSA_API dsa_status_t dsa_indexer_prepare(const void* c_q, const float* q_norm_weight, float eps, const void* wq_b,
                                         const void* h, const void* wk, const void* w_proj, const float* rope_cos,
                                         const float* rope_sin, int max_pos, int d_rope, const int32_t* pos,
                                         const int64_t* slot, int tokens, int d_c, int d_model, int n_heads,
                                         int head_dim, void* q_out, float* w_out, void* k_cache, dsa_dtype_t k_dtype,
                                         float* k_scale, int64_t cache_rows, void* workspace, size_t workspace_bytes,
                                         void* stream);

/*
 * dsa_indexer_key_append -- the key-cache write of dsa_indexer_prepare alone,
 * for n key rows that are already projected (for instance the pooled keys
 * of csa_compress): row r of k (fp32 or bf16, [n, 128]) is turned by RoPE at
 * pos[r] (dims below d_rope) and written to cache row slot[r] (-1: skipped)
 * in the cache's format, with the same rounding rules.  head_dim must be
 * 128; k and k_cache 16-byte aligned.
 */
DSA_API dsa_status_t dsa_indexer_key_append(const void* k, dsa_dtype_t k_in_dtype, const float* rope_cos,
                                            const float* rope_sin, int max_pos, int d_rope, const int32_t* pos,
                                            const int64_t* slot, int n, int head_dim, void* k_cache,
                                            dsa_dtype_t k_dtype, float* k_scale, int64_t cache_rows, void* stream);

/*
 * dsa_get_device_error -- synchronizes `stream`, then reads and clears the
 * library's device error word on the current device.  Returns DSA_OK when
 * no kernel recorded an error, DSA_ERR_DEVICE_TIMEOUT when a kernel gave up
 * a bounded wait, DSA_ERR_INVALID_ARG when a kernel met an index, position
 * or slot out of range and skipped it, DSA_ERR_CUDA when the synchronization
 * itself failed.
 */
DSA_API dsa_status_t dsa_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_H */
