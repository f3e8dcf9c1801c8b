// Lightning-indexer scores on CUDA cores (FFMA), for fp32 inputs and small
// head dims ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", section 1.3 闪电索引器):
//   logits[t, s] = sum_j w[t, j] * ReLU(q[t, j, :] . k[b, s, :])
//
// One thread per key: the key row sits in registers, the query row's
// n_heads x D block and its weights in shared memory (read as broadcasts).
// Tiles past the row's last visible key are skipped entirely; keys beyond it
// are not written.  The bf16/fp8 configurations of the path run on the
// tensor-core kernel instead.
#include "common.cuh"
#include "launchers.h"

namespace dsa {

template <int D, typename QT, typename KT>
__global__ void __launch_bounds__(256) indexer_simt_kernel(
    const QT* __restrict__ q, const float* __restrict__ w, const KT* __restrict__ k,
    const float* __restrict__ k_scale, const int32_t* __restrict__ row_batch,
    const int32_t* __restrict__ row_pos, int batch, int ctx_len, int n_heads, float* __restrict__ logits, int64_t ld,
    unsigned* err) {
    extern __shared__ float sm[];
    float* qs = sm;                       // [n_heads][D]
    float* ws = sm + n_heads * D;         // [n_heads]
    const int t = blockIdx.x;
    const int pos = row_pos[t];
    const int s0 = blockIdx.y * blockDim.x;
    if (s0 > pos) return;                 // nothing visible in this tile
    const int b = row_batch[t];
    if (b < 0 || b >= batch) {
        if (threadIdx.x == 0) record_error(err, DEV_ERR_BAD_INDEX);
        return;
    }
    for (int i = threadIdx.x; i < n_heads * D; i += blockDim.x)
        qs[i] = to_f32(q[(int64_t)t * n_heads * D + i]);
    for (int i = threadIdx.x; i < n_heads; i += blockDim.x) ws[i] = w[(int64_t)t * n_heads + i];
    __syncthreads();
    const int s = s0 + threadIdx.x;
    if (s > pos || s >= ctx_len) return;
    const int64_t krow = (int64_t)b * ctx_len + s;
    float kr[D];
#pragma unroll
    for (int d = 0; d < D; ++d) kr[d] = to_f32(k[krow * D + d]);
    float acc = 0.f;
    for (int j = 0; j < n_heads; ++j) {
        const float* qj = qs + j * D;
        float dot = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) dot = fmaf(qj[d], kr[d], dot);
        acc = fmaf(ws[j], fmaxf(dot, 0.f), acc);
    }
    if (k_scale) acc *= k_scale[krow];
    logits[(int64_t)t * ld + s] = acc;
}

template <int D, typename QT, typename KT>
static cudaError_t launch_t(const Launch& L, const void* q, const float* w, const void* k, const float* k_scale,
                            const int32_t* rb, const int32_t* rp, int rows, int batch, int ctx, int H, float* logits,
                            int64_t ld) {
    dim3 grid(rows, ceil_div(ctx, 256));
    size_t smem = (size_t)(H * D + H) * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(indexer_simt_kernel<D, QT, KT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    indexer_simt_kernel<D, QT, KT><<<grid, 256, smem, L.stream>>>(
        (const QT*)q, w, (const KT*)k, k_scale, rb, rp, batch, ctx, H, logits, ld, L.err);
    count_launch();
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_d(const Launch& L, const void* q, dsa_dtype_t qt, const float* w, const void* k,
                            dsa_dtype_t kt, const float* ks, const int32_t* rb, const int32_t* rp, int rows,
                            int batch, int ctx, int H, float* logits, int64_t ld) {
    if (qt == DSA_FP32 && kt == DSA_FP32)
        return launch_t<D, float, float>(L, q, w, k, ks, rb, rp, rows, batch, ctx, H, logits, ld);
    if (qt == DSA_BF16 && kt == DSA_BF16)
        return launch_t<D, __nv_bfloat16, __nv_bfloat16>(L, q, w, k, ks, rb, rp, rows, batch, ctx, H, logits, ld);
    if (qt == DSA_BF16 && kt == DSA_FP8_E4M3)
        return launch_t<D, __nv_bfloat16, __nv_fp8_e4m3>(L, q, w, k, ks, rb, rp, rows, batch, ctx, H, logits, ld);
    return cudaErrorInvalidValue;
}

cudaError_t launch_indexer_simt(const Launch& L, const void* q, dsa_dtype_t q_dtype, const float* w,
                                const void* k, dsa_dtype_t k_dtype, const float* k_scale,
                                const int32_t* row_batch, const int32_t* row_pos, int rows, int batch,
                                int ctx_len, int n_heads, int head_dim, float* logits, int64_t ld) {
    if (rows == 0 || ctx_len == 0) return cudaSuccess;
    switch (head_dim) {
    case 32: return launch_d<32>(L, q, q_dtype, w, k, k_dtype, k_scale, row_batch, row_pos, rows, batch, ctx_len, n_heads, logits, ld);
    case 64: return launch_d<64>(L, q, q_dtype, w, k, k_dtype, k_scale, row_batch, row_pos, rows, batch, ctx_len, n_heads, logits, ld);
    case 128: return launch_d<128>(L, q, q_dtype, w, k, k_dtype, k_scale, row_batch, row_pos, rows, batch, ctx_len, n_heads, logits, ld);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dsa
