// CSA token compression: each m consecutive cache rows -> their mean
// (V4 CSA summary: every 4 tokens become one entry; "解密DeepSeek-V4 ..."
// section 4.3: pooling of the m consecutive KV pairs).
//
// HBM-bound streaming kernel.  Each thread owns one 16-byte vector of one
// output row and reads the same vector of the m source rows: all loads and
// stores are 16-byte and coalesced across the warp.  The sum of m bf16 values
// is formed in double, where it is exact for the magnitudes a cache holds, and
// rounded once (cvt.rn) to the storage type, so the result is the
// correctly-rounded mean.  fp64 throughput is irrelevant here: the kernel
// moves (m+1)*16 bytes per 8 additions.
#include "common.cuh"
#include "launchers.h"

namespace dsa {

__device__ __forceinline__ uint16_t f64_to_bf16_rn_bits(double x) {
    uint16_t r;
    asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(x));
    return r;
}

// bf16: 8 elements (16 B) per vector.
__global__ void __launch_bounds__(256) csa_compress_bf16_vec(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                             int64_t n_out_rows, int vec_per_row, int m) {
    const int64_t total = n_out_rows * vec_per_row;
    const double inv_m = 1.0 / (double)m;
    const bool pow2 = (m & (m - 1)) == 0;
    for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = v / vec_per_row;
        const int c = (int)(v - r * vec_per_row);
        double acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0;
        const uint4* s = src + (r * m) * vec_per_row + c;
        for (int j = 0; j < m; ++j) {
            uint4 x = __ldcs(s + (int64_t)j * vec_per_row);   // streamed once
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] += (double)__uint_as_float(w[e] << 16);
                acc[2 * e + 1] += (double)__uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            double lo = pow2 ? acc[2 * e] * inv_m : acc[2 * e] / (double)m;
            double hi = pow2 ? acc[2 * e + 1] * inv_m : acc[2 * e + 1] / (double)m;
            o[e] = (uint32_t)f64_to_bf16_rn_bits(lo) | ((uint32_t)f64_to_bf16_rn_bits(hi) << 16);
        }
        __stcs(dst + v, make_uint4(o[0], o[1], o[2], o[3]));
    }
}

// fp32: 4 elements (16 B) per vector.
__global__ void __launch_bounds__(256) csa_compress_f32_vec(const float4* __restrict__ src, float4* __restrict__ dst,
                                                            int64_t n_out_rows, int vec_per_row, int m) {
    const int64_t total = n_out_rows * vec_per_row;
    const bool pow2 = (m & (m - 1)) == 0;
    const double inv_m = 1.0 / (double)m;
    for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = v / vec_per_row;
        const int c = (int)(v - r * vec_per_row);
        double a0 = 0, a1 = 0, a2 = 0, a3 = 0;
        const float4* s = src + (r * m) * vec_per_row + c;
        for (int j = 0; j < m; ++j) {
            float4 x = __ldcs(s + (int64_t)j * vec_per_row);
            a0 += x.x; a1 += x.y; a2 += x.z; a3 += x.w;
        }
        float4 o;
        o.x = (float)(pow2 ? a0 * inv_m : a0 / m);
        o.y = (float)(pow2 ? a1 * inv_m : a1 / m);
        o.z = (float)(pow2 ? a2 * inv_m : a2 / m);
        o.w = (float)(pow2 ? a3 * inv_m : a3 / m);
        __stcs(dst + v, o);
    }
}

cudaError_t launch_csa_compress(const Launch& L, const void* src, dsa_dtype_t dtype, int batch, int len,
                                int dim, int m, void* dst) {
    const int64_t n_out_rows = (int64_t)batch * (len / m);
    const int elems_per_vec = dtype == DSA_BF16 ? 8 : 4;
    const int vec_per_row = dim / elems_per_vec;
    const int64_t total = n_out_rows * vec_per_row;
    if (total == 0) return cudaSuccess;
    // Enough resident warps to keep HBM busy: 8 CTAs of 256 threads per SM,
    // grid-stride over the rest.
    int64_t want = (total + 255) / 256;
    int grid = (int)(want < (int64_t)L.num_sms * 8 ? want : (int64_t)L.num_sms * 8);
    if (dtype == DSA_BF16)
        csa_compress_bf16_vec<<<grid, 256, 0, L.stream>>>((const uint4*)src, (uint4*)dst, n_out_rows, vec_per_row, m);
    else
        csa_compress_f32_vec<<<grid, 256, 0, L.stream>>>((const float4*)src, (float4*)dst, n_out_rows, vec_per_row, m);
    count_launch();
    return cudaGetLastError();
}

}  // namespace dsa
