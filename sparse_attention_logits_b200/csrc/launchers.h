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
//  - dense mode (idx == NULL): slot s < k is key s when s <= row_last[t].
struct KvExtra {
    const void* kv2 = nullptr;
    const int32_t* pos2 = nullptr;
    int len2 = 0, window = 0;
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

}  // namespace dsa
