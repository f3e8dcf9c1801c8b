// Per-query top-k selection ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", section 1.3
// and section 3 Step 3): the k visible keys with the largest index score,
// lower position first among equal scores, every visible key when no more
// than k are visible.
//
// Exact radix select on order-preserving 32-bit keys, one CTA of 1024
// threads per query row:
//   1. four 8-bit digit passes, most significant first, each a shared-memory
//      histogram of the keys that still match the digits chosen so far; the
//      digit holding the k-th largest key is found by a suffix scan, which
//      yields the exact k-th key T and the number of keys above it;
//   2. an ordered compaction: every key > T, plus the first (in position
//      order) keys equal to T until k are taken.  Threads own contiguous
//      position ranges and a block-wide scan gives each its output offset,
//      so the output is in ascending position order and deterministic.
// The scores of a row (<= 1 MB) stay L2-resident between passes.
#include "common.cuh"
#include "launchers.h"

namespace dsa {

namespace {
constexpr int TOPK_THREADS = 1024;

// Exclusive scan over the CTA (1024 threads = 32 warps); also returns the total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = warp_sums[lane];
        uint32_t inc = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        warp_sums[lane] = inc - s;     // exclusive prefix of warp totals
        if (lane == 31) warp_sums[32] = inc;
    }
    __syncthreads();
    uint32_t r = warp_sums[warp] + x - v;
    *total = warp_sums[32];
    __syncthreads();
    return r;
}
}  // namespace

__global__ void __launch_bounds__(TOPK_THREADS, 1) topk_radix_kernel(
    const float* __restrict__ logits, int64_t ld, const int32_t* __restrict__ row_pos, int ctx_len, int k,
    int32_t* __restrict__ idx) {
    __shared__ uint32_t hist[256];
    __shared__ uint32_t warp_sums[33];
    __shared__ uint32_t s_digit, s_above;
    const int t = blockIdx.x;
    const int tid = threadIdx.x;
    const float* x = logits + (int64_t)t * ld;
    int32_t* out = idx + (int64_t)t * k;
    int n = row_pos[t] + 1;
    if (n > ctx_len) n = ctx_len;
    if (n < 0) n = 0;

    if (n <= k) {                                   // keep-all rule
        for (int i = tid; i < k; i += TOPK_THREADS) out[i] = i < n ? i : -1;
        return;
    }

    // ---- 1. radix select of the k-th largest key ----
    uint32_t prefix = 0u, himask = 0u;
    uint32_t remaining = (uint32_t)k;               // still to take among keys matching `prefix`
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += TOPK_THREADS) {
            uint32_t key = score_key(__ldg(x + i));
            if (((key ^ prefix) & himask) == 0u) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            const int lane = tid;
            uint32_t h[8];
            uint32_t mine = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) { h[b] = hist[lane * 8 + b]; mine += h[b]; }
            // exclusive suffix sum over lanes: counts in bins above this lane's bins
            uint32_t incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += y;
            }
            uint32_t cum = incl - mine;
#pragma unroll
            for (int b = 7; b >= 0; --b) {
                if (cum < remaining && cum + h[b] >= remaining) { s_digit = (uint32_t)(lane * 8 + b); s_above = cum; }
                cum += h[b];
            }
        }
        __syncthreads();
        prefix |= s_digit << shift;
        himask |= 255u << shift;
        remaining -= s_above;
        __syncthreads();
    }
    const uint32_t T = prefix;                      // the k-th largest key; `remaining` keys == T to take

    // ---- 2. ordered compaction ----
    const int seg = (n + TOPK_THREADS - 1) / TOPK_THREADS;
    const int lo = min(n, tid * seg), hi = min(n, lo + seg);
    uint32_t gt = 0, eq = 0;
    for (int i = lo; i < hi; ++i) {
        uint32_t key = score_key(__ldg(x + i));
        gt += key > T;
        eq += key == T;
    }
    uint32_t tot;
    const uint32_t eq_before = block_excl_scan(eq, warp_sums, &tot);
    const uint32_t take_eq = eq_before >= remaining ? 0u : min(eq, remaining - eq_before);
    const uint32_t off = block_excl_scan(gt + take_eq, warp_sums, &tot);
    uint32_t j = off, e = 0;
    for (int i = lo; i < hi; ++i) {
        uint32_t key = score_key(__ldg(x + i));
        if (key > T) {
            out[j++] = i;
        } else if (key == T) {
            if (e < take_eq) out[j++] = i;
            ++e;
        }
    }
}

cudaError_t launch_topk(const Launch& L, const float* logits, int64_t ld, const int32_t* row_pos, int rows,
                        int ctx_len, int k, int32_t* idx, void* /*workspace*/, size_t /*ws_bytes*/) {
    if (rows == 0) return cudaSuccess;
    topk_radix_kernel<<<rows, TOPK_THREADS, 0, L.stream>>>(logits, ld, row_pos, ctx_len, k, idx);
    count_launch();
    return cudaGetLastError();
}

size_t topk_workspace_bytes(int /*rows*/, int /*ctx_len*/, int /*k*/) { return 0; }

}  // namespace dsa
