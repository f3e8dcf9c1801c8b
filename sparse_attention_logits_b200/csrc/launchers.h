// Internal host launchers of the DSA library (C++ linkage, not exported in
// the public header).  Arguments have been validated by the entry points.
#pragma once

#include "common.cuh"

namespace dsa {

cudaError_t launch_csa_compress(const Launch& L, const void* src, dsa_dtype_t dtype, int batch, int len, int dim,
                                int m, void* dst);

cudaError_t launch_indexer_simt(const Launch& L, const void* q, dsa_dtype_t q_dtype, const float* w, const void* k,
                                dsa_dtype_t k_dtype, const float* k_scale, const int32_t* row_batch,
                                const int32_t* row_pos, int rows, int batch, int ctx_len, int n_heads,
                                int head_dim, float* logits, int64_t ld);

bool indexer_tc_supported(dsa_dtype_t q_dtype, dsa_dtype_t k_dtype, int n_heads, int head_dim);
cudaError_t launch_indexer_tc(const Launch& L, const void* q, dsa_dtype_t k_dtype, const float* w, const void* k,
                              const float* k_scale, const int32_t* row_batch, const int32_t* row_pos, int rows,
                              int batch, int ctx_len, float* logits, int64_t ld);

cudaError_t launch_topk(const Launch& L, const float* logits, int64_t ld, const int32_t* row_pos, int rows,
                        int ctx_len, int k, int32_t* idx, void* workspace, size_t ws_bytes);
size_t topk_workspace_bytes(int rows, int ctx_len, int k);
bool topk_supported(int ctx_len);

// Optional parts of a sparse-attention call beyond the selected rows:
//  - a window segment: slots [k, k + window) of row t are the raw cache rows
//    pos2[t] - window + 1 .. pos2[t] of kv2 [batch, len2, d_qk] (positions
//    below 0 are unused slots);
//  - a sink segment: slots [k + window, k + window + n_sink) are the raw
//    rows 0 .. n_sink - 1 of kv2, each used only when it lies before the
//    window's first position pos2[t] - window + 1 (so no raw row is
//    attended twice, and none after the query);
//  - dense mode (idx == NULL): slot s < k is key s when s <= row_last[t].
struct KvExtra {
    const void* kv2 = nullptr;
    const int32_t* pos2 = nullptr;
    int len2 = 0, window = 0, n_sink = 0;
    const int32_t* row_last = nullptr;
};

bool mla_simt_supported(int d_qk, int d_v, int n_heads);
cudaError_t launch_mla_simt(const Launch& L, const void* q, const void* kv, dsa_dtype_t dtype,
                            const int32_t* page_table, int page_size, int num_pages, const int32_t* row_batch,
                            const int32_t* idx,
                            int k, int rows, int batch, int ctx_len, int n_heads, int d_qk, int d_v, float scale,
                            void* out, float* lse, const KvExtra& x = KvExtra());

bool mla_tc_supported(dsa_dtype_t dtype, int n_heads, int d_qk, int d_v);
size_t mla_tc_workspace_bytes(int rows, int k, int num_sms);
cudaError_t launch_mla_tc(const Launch& L, const void* q, const void* kv, const int32_t* page_table, int page_size,
                          int num_pages, const int32_t* row_batch, const int32_t* idx, int k, int rows, int batch,
                          int ctx_len, float scale, void* out, float* lse, void* workspace, size_t ws_bytes,
                          const KvExtra& x = KvExtra());

// Preparation of the indexer's inputs (validated arguments of
// dsa_indexer_prepare).
struct PrepareArgs {
    const void* c_q;          // [T, d_c] bf16
    const float* gamma;       // [d_c]
    float eps;
    const void* wq_b;         // [n_heads * 128, d_c] bf16
    const void* h;            // [T, d_model] bf16
    const void* wk;           // [128, d_model] bf16
    const void* w_proj;       // [n_heads, d_model] bf16
    const float* rope_cos;    // [max_pos, d_rope / 2]
    const float* rope_sin;
    int max_pos, d_rope;
    const int32_t* pos;       // [T]
    const int64_t* slot;      // [T]
    int T, d_c, d_model, n_heads;
    void* q_out;              // [T, n_heads, 128] bf16
    float* w_out;             // [T, n_heads]
    void* k_cache;
    dsa_dtype_t k_fmt;
    float* k_scale;
    int64_t cache_rows;
};
size_t indexer_prepare_workspace_bytes(int T, int n_heads, int d_c, int d_model, int num_sms);
int indexer_prepare_max_dc();
cudaError_t launch_indexer_prepare(const Launch& L, const PrepareArgs& a, void* workspace, size_t ws_bytes);
cudaError_t launch_key_append(const Launch& L, const void* k, dsa_dtype_t k_in, int n, const int32_t* pos,
                              const int64_t* slot, const float* rope_cos, const float* rope_sin, int max_pos,
                              int d_rope, void* cache, dsa_dtype_t fmt, float* k_scale, int64_t cache_rows);
}  // namespace dsa
