// Sparse MLA (MQA mode) on CUDA cores, for fp32 inputs and small latent
// sizes ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", sections 1.3 细粒度稀疏注意力
// and 1.4): attention of every query head over the selected latent rows
// only, every row shared by all heads, value = first d_v latent dims.
//
// One CTA per (query row, group of 8 heads); one warp per head.  The
// selected rows are gathered 16 at a time into shared memory (fp32) and read
// by all 8 warps; each lane owns d_qk/32 query dims and d_v/32 output dims.
// Online softmax in base 2 (scores pre-multiplied by scale*log2(e)).
#include "common.cuh"
#include "launchers.h"

namespace dsa {

namespace {
constexpr int MLA_SIMT_HEADS = 8;
constexpr int MLA_SIMT_TILE = 16;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
}  // namespace

template <typename T, int QPL, int VPL>
__global__ void __launch_bounds__(256) mla_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ kv, const int32_t* __restrict__ page_table, int page_size,
    int pages_per_seq, int num_pages, const int32_t* __restrict__ row_batch, const int32_t* __restrict__ idx, int k,
    int batch, int ctx_len, int n_heads, float scale, T* __restrict__ out, float* __restrict__ lse, unsigned* err,
    const T* __restrict__ kv2, const int32_t* __restrict__ pos2, int len2, int window, int n_sink,
    const int32_t* __restrict__ row_last) {
    pdl_wait();
    constexpr int DK = QPL * 32, DV = VPL * 32;
    __shared__ float tile[MLA_SIMT_TILE][DK];
    __shared__ int valid[MLA_SIMT_TILE];
    const int t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y * MLA_SIMT_HEADS + warp;
    int b = row_batch[t];
    const bool row_ok = b >= 0 && b < batch;
    if (!row_ok) {
        if (threadIdx.x == 0) record_error(err, DEV_ERR_BAD_INDEX);
        b = 0;
    }
    const float zscale = scale * LOG2E;

    float qr[QPL];
#pragma unroll
    for (int i = 0; i < QPL; ++i) qr[i] = to_f32(q[((int64_t)t * n_heads + h) * DK + lane + 32 * i]);
    float acc[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
    float m = -INFINITY, l = 0.f;

    const int32_t* sel = idx ? idx + (int64_t)t * k : nullptr;
    const int last = idx ? 0 : row_last[t];
    const int wfirst = window + n_sink > 0 ? pos2[t] - window + 1 : 0;   // the window's first raw position
    const int ktot = k + window + n_sink;
    for (int j0 = 0; j0 < ktot; j0 += MLA_SIMT_TILE) {
        __syncthreads();
        // gather up to 16 slots (warp w loads slots w and w+8): selected keys
        // (or every visible key in dense mode), then the window rows, then
        // the sink rows that lie before the window
        for (int r = warp; r < MLA_SIMT_TILE; r += 8) {
            const int j = j0 + r;
            if (j >= k && j < ktot) {
                const int s = j - k < window ? wfirst + (j - k) : (j - k - window < wfirst ? j - k - window : -1);
                const bool ok = row_ok && s >= 0 && s < len2;
                if (s >= len2) record_error(err, DEV_ERR_BAD_INDEX);
                const int64_t row = (int64_t)b * len2 + s;
                for (int d = lane; d < DK; d += 32) tile[r][d] = ok ? to_f32(kv2[row * DK + d]) : 0.f;
                if (lane == 0) valid[r] = ok;
                continue;
            }
            int s = j < k ? (sel ? sel[j] : (j <= last ? j : -1)) : -1;
            bool ok = row_ok && s >= 0 && s < ctx_len;
            if (s >= ctx_len) record_error(err, DEV_ERR_BAD_INDEX);
            int64_t row = 0;
            if (ok && page_table) {
                const int pg = page_table[(int64_t)b * pages_per_seq + s / page_size];
                if (pg < 0 || pg >= num_pages) {
                    record_error(err, DEV_ERR_BAD_INDEX);
                    ok = false;
                } else {
                    row = (int64_t)pg * page_size + s % page_size;
                }
            } else if (ok) {
                row = (int64_t)b * ctx_len + s;
            }
            for (int d = lane; d < DK; d += 32) tile[r][d] = ok ? to_f32(kv[row * DK + d]) : 0.f;
            if (lane == 0) valid[r] = ok;
        }
        __syncthreads();
#pragma unroll 1
        for (int r = 0; r < MLA_SIMT_TILE; ++r) {
            if (!valid[r]) continue;
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < QPL; ++i) dot = fmaf(qr[i], tile[r][lane + 32 * i], dot);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            const float z = dot * zscale;
            const float mn = fmaxf(m, z);
            const float corr = exp2f(m - mn);      // 0 on the first key (m = -inf)
            const float p = exp2f(z - mn);
            l = l * corr + p;
#pragma unroll
            for (int i = 0; i < VPL; ++i) acc[i] = fmaf(p, tile[r][lane + 32 * i], acc[i] * corr);
            m = mn;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) store_out(out + ((int64_t)t * n_heads + h) * DV + lane + 32 * i, acc[i] * inv);
    if (lane == 0) lse[(int64_t)t * n_heads + h] = l > 0.f ? (m + log2f(l)) * LN2 : -INFINITY;
}

template <typename T, int QPL, int VPL>
static cudaError_t launch_t(const Launch& L, const void* q, const void* kv, const int32_t* pt, int page_size,
                            int pages_per_seq, int num_pages, const int32_t* rb, const int32_t* idx, int k, int rows, int batch,
                            int ctx, int H, float scale, void* out, float* lse, const KvExtra& x) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rows, H / MLA_SIMT_HEADS);
    cfg.blockDim = dim3(256);
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, mla_simt_kernel<T, QPL, VPL>, (const T*)q, (const T*)kv, pt, page_size,
                                             pages_per_seq, num_pages, rb, idx, k, batch, ctx, H, scale, (T*)out, lse,
                                             L.err, (const T*)x.kv2, x.pos2, x.len2, x.kv2 ? x.window : 0,
                                             x.kv2 ? x.n_sink : 0, x.row_last);
    count_launch();
    return e;
}

template <typename T>
static cudaError_t launch_dims(const Launch& L, const void* q, const void* kv, const int32_t* pt, int page_size,
                               int pps, int npages, const int32_t* rb, const int32_t* idx, int k, int rows, int batch, int ctx,
                               int H, int dqk, int dv, float scale, void* out, float* lse, const KvExtra& x) {
    if (dqk == 32 && dv == 32) return launch_t<T, 1, 1>(L, q, kv, pt, page_size, pps, npages, rb, idx, k, rows, batch, ctx, H, scale, out, lse, x);
    if (dqk == 64 && dv == 64) return launch_t<T, 2, 2>(L, q, kv, pt, page_size, pps, npages, rb, idx, k, rows, batch, ctx, H, scale, out, lse, x);
    if (dqk == 64 && dv == 32) return launch_t<T, 2, 1>(L, q, kv, pt, page_size, pps, npages, rb, idx, k, rows, batch, ctx, H, scale, out, lse, x);
    if (dqk == 576 && dv == 512) return launch_t<T, 18, 16>(L, q, kv, pt, page_size, pps, npages, rb, idx, k, rows, batch, ctx, H, scale, out, lse, x);
    return cudaErrorInvalidValue;
}

bool mla_simt_supported(int d_qk, int d_v, int n_heads) {
    if (n_heads % MLA_SIMT_HEADS) return false;
    return (d_qk == 32 && d_v == 32) || (d_qk == 64 && (d_v == 64 || d_v == 32)) || (d_qk == 576 && d_v == 512);
}

cudaError_t launch_mla_simt(const Launch& L, const void* q, const void* kv, dsa_dtype_t dtype, const int32_t* page_table,
                            int page_size, int num_pages, const int32_t* row_batch, const int32_t* idx, int k, int rows, int batch,
                            int ctx_len, int n_heads, int d_qk, int d_v, float scale, void* out, float* lse,
                            const KvExtra& x) {
    if (rows == 0) return cudaSuccess;
    const int pps = page_table ? ctx_len / page_size : 0;
    if (dtype == DSA_FP32)
        return launch_dims<float>(L, q, kv, page_table, page_size, pps, num_pages, row_batch, idx, k, rows, batch, ctx_len,
                                  n_heads, d_qk, d_v, scale, out, lse, x);
    return launch_dims<__nv_bfloat16>(L, q, kv, page_table, page_size, pps, num_pages, row_batch, idx, k, rows, batch,
                                      ctx_len, n_heads, d_qk, d_v, scale, out, lse, x);
}

}  // namespace dsa
