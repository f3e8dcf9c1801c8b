// Per-query top-k selection ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", section 1.3
// and section 3 Step 3): the k visible keys with the largest index score,
// lower position first among equal scores, every visible key when no more
// than k are visible.
//
// Exact radix select on order-preserving 32-bit keys.  One thread-block
// cluster of CL CTAs (1..8) handles one query row; CTA r of the cluster owns
// a contiguous slice of the row, loaded once into shared memory as keys.
//   1. three digit passes (11, 11, 10 bits, most significant first): every
//      CTA histograms the keys of its slice that still match the digits
//      chosen so far; the CTAs add up each other's histograms through
//      distributed shared memory and each finds, by a suffix scan, the digit
//      that holds the k-th largest key.  After the last pass every CTA knows
//      the exact k-th key T and how many keys equal to T must be taken.
//   2. ordered compaction: every key > T, plus the first keys == T in
//      position order until k are taken.  Per-CTA counts are exchanged
//      through distributed shared memory, so the output of the whole row is
//      in ascending position order and deterministic.
// -0.0 is mapped to +0.0 before the key map, so the two zeros tie.
#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"

namespace dsa {

using namespace sm100;

namespace {

constexpr int TOPK_THREADS = 1024;
static_assert(TOPK_THREADS == 32 * 32, "the bin search sums over exactly 32 warps");
constexpr int NBINS = 2048;                    // 11-bit digits
constexpr int SLICE_CAP = 40960;               // keys per CTA kept in shared memory (160 KB)
constexpr int MAX_PASSES = 3;                  // 11 + 10 + 10 bits: the range is exact after three passes
constexpr int CAND_CAP = 1024;                 // candidates ranked directly after the first pass
// hist, merged (scan scratch), one cluster-wide histogram per pass, scratch,
// candidate buffer, candidates' source CTAs, per-CTA counts (rank 0)
constexpr int MAX_CL = 16;                     // CTAs per row (16 needs the non-portable cluster size)
constexpr int SMEM_FIXED = ((2 + MAX_PASSES) * NBINS + 64 + 32 + 2 * CAND_CAP + 32 + 3 * MAX_CL + 16) * 4;
// the per-pass range totals (MAX_PASSES x MAX_CL words) fit in the last 16 + 32 words of the fixed part
static_assert((2 + MAX_PASSES) * NBINS + 40 + 8 + 16 + 2 * CAND_CAP + 3 * MAX_CL + MAX_PASSES * MAX_CL <=
              SMEM_FIXED / 4, "fixed shared-memory layout");
// Alignment of the vector accesses, by construction: the base is rounded up
// to 128 B in the kernel (the launch reserves exactly that rounding room,
// SMEM_ROUND), the key slice starts SMEM_FIXED bytes after it, and every
// 16-byte access of the slice is at a multiple of 4 keys (the slice length
// `per` and every walk's start are multiples of 4); the cluster histograms
// read with 8-byte loads start at even words of an 8-byte aligned array.
constexpr int SMEM_ROUND = 128;
static_assert(SMEM_FIXED % 16 == 0, "the key slice must start 16-byte aligned");
static_assert((2 * NBINS * 4) % 8 == 0 && NBINS % 2 == 0, "cluster histograms: 8-byte aligned pairs");

template <int CL>
__device__ __forceinline__ void cl_sync() {
    if (CL > 1) cluster_sync_all();
    else __syncthreads();
}

template <int CL>
__device__ __forceinline__ uint32_t cl_rank() {
    return CL > 1 ? cluster_ctarank() : 0u;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint2 ld_cluster_v2(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared::cluster.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void red_cluster_add(uint32_t addr, uint32_t v) {
    asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Atomic add on a shared-memory word of any CTA of the cluster (or of this
// CTA); returns the old value.
__device__ __forceinline__ uint32_t atom_add_cluster(uint32_t addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.relaxed.cluster.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

}  // namespace

template <int CL>
__global__ void __launch_bounds__(TOPK_THREADS, 1) topk_cluster_kernel(
    const float* __restrict__ logits, int64_t ld, const int32_t* __restrict__ row_pos, int ctx_len, int k,
    int32_t* __restrict__ idx) {
    extern __shared__ uint8_t tk_smem_raw[];
    // the runtime's placement of dynamic shared memory is not relied upon:
    // the base is rounded up here (the launch reserves the slack)
    uint32_t* tk_smem = (uint32_t*)(((uintptr_t)tk_smem_raw + SMEM_ROUND - 1) & ~(uintptr_t)(SMEM_ROUND - 1));
    uint32_t* hist = tk_smem;                    // [NBINS]   this CTA's histogram
    uint32_t* merged = hist + NBINS;             // [NBINS]   scratch for the suffix scan
    uint32_t* cl_hist = merged + NBINS;          // [MAX_PASSES][NBINS] cluster-wide histograms: CTA r holds the
                                                 // merged counts of its own range of bins (NBINS / CL of them)
    uint32_t* warp_sums = cl_hist + MAX_PASSES * NBINS;   // [33]
    uint32_t* shared_res = warp_sums + 40;       // digit, count above
    uint32_t* cta_counts = shared_res + 8;       // gt, eq of this CTA (read by peers), key range, and [4..7]: the
                                                 // threshold, keys equal to it to take, this CTA's offsets (from rank 0)
    uint32_t* cand_n = cta_counts + 8;           // candidate count (rank 0's is used)
    uint32_t* cand = cta_counts + 16;            // [CAND_CAP] candidate keys (rank 0's is used)
    uint32_t* cand_src = cand + CAND_CAP;        // [CAND_CAP] the CTA each candidate comes from (rank 0's)
    uint32_t* cta_cnt = cand_src + CAND_CAP;     // [3][MAX_CL] per-CTA keys above the bin, candidates > T, == T (rank 0's)
    uint32_t* rtot = cta_cnt + 3 * MAX_CL;       // [MAX_PASSES][MAX_CL] cluster-wide keys in each CTA's bin range
    uint32_t* keys = tk_smem + (SMEM_FIXED / 4); // [slice]

    pdl_wait();                     // the scores of the previous kernel are visible from here on
    pdl_launch_dependents();
    const int row = blockIdx.x / CL;
    const uint32_t rank = cl_rank<CL>();
    const int tid = threadIdx.x;
    const float* x = logits + (int64_t)row * ld;
    int32_t* out = idx + (int64_t)row * k;
    int n = row_pos[row] + 1;
    if (n > ctx_len) n = ctx_len;
    if (n < 0) n = 0;

    if (n <= k) {                                // keep-all rule (uniform over the cluster)
        if (rank == 0)
            for (int i = tid; i < k; i += TOPK_THREADS) out[i] = i < n ? i : -1;
        return;
    }

    // ---- load this CTA's slice as order-preserving keys ----
    const int per = ((n + CL - 1) / CL + 3) & ~3;
    const int lo = min(n, (int)rank * per), hi = min(n, lo + per);
    const int cnt = hi - lo;
    // 8 independent 16-byte loads in flight per thread (one memory round trip
    // for a 32K-key slice); scalar path for rows that are not 16-byte aligned.
    // The key range of the slice is taken on the way.
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    if ((((uintptr_t)(x + lo)) & 15u) == 0u) {
        const float4* x4 = (const float4*)(x + lo);
        const int n4 = cnt >> 2;
        for (int i0 = tid; i0 < n4; i0 += 8 * TOPK_THREADS) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u * TOPK_THREADS < n4) v[u] = __ldg(x4 + i0 + u * TOPK_THREADS);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u * TOPK_THREADS < n4) {
                    const uint4 q = make_uint4(score_key(v[u].x), score_key(v[u].y), score_key(v[u].z),
                                               score_key(v[u].w));
                    *(uint4*)(keys + 4 * (i0 + u * TOPK_THREADS)) = q;
                    kmin = min(min(kmin, min(q.x, q.y)), min(q.z, q.w));
                    kmax = max(max(kmax, max(q.x, q.y)), max(q.z, q.w));
                }
        }
        for (int i = 4 * n4 + tid; i < cnt; i += TOPK_THREADS) {
            const uint32_t key = score_key(__ldg(x + lo + i));
            keys[i] = key;
            kmin = min(kmin, key);
            kmax = max(kmax, key);
        }
    } else {
        for (int i0 = tid; i0 < cnt; i0 += 8 * TOPK_THREADS) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u * TOPK_THREADS < cnt) v[u] = __ldg(x + lo + i0 + u * TOPK_THREADS);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u * TOPK_THREADS < cnt) {
                    const uint32_t key = score_key(v[u]);
                    keys[i0 + u * TOPK_THREADS] = key;
                    kmin = min(kmin, key);
                    kmax = max(kmax, key);
                }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if ((tid & 31) == 0) {
        merged[tid >> 5] = kmin;
        merged[32 + (tid >> 5)] = kmax;
    }
    if (CL > 1) {
        for (int i = tid; i < MAX_PASSES * NBINS; i += TOPK_THREADS) cl_hist[i] = 0u;
        if (tid < MAX_PASSES * MAX_CL) rtot[tid] = 0u;
    }
    if (tid == 0) *cand_n = 0u;
    if (tid < 3 * MAX_CL) cta_cnt[tid] = 0u;
    __syncthreads();
    // the slice is padded with copies of its first key up to a multiple of 4
    // (cnt4), so that every walk below reads 16 bytes per lane
    const int cnt4 = (cnt + 3) & ~3;
    for (int i = cnt + tid; i < cnt4; i += TOPK_THREADS) keys[i] = keys[0];
    if (tid < 32) {                              // this CTA's key range: warp 0 reduces the 32 warps' ranges
        uint32_t a = merged[tid], b = merged[32 + tid];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
            b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
        }
        if (tid == 0) {
            cta_counts[2] = a;
            cta_counts[3] = b;
        }
    }
    // every CTA's key range published, its cluster histograms zeroed
    cl_sync<CL>();

    // ---- 1. select the exact k-th largest key ----
    // Adaptive range narrowing: the candidate keys lie in [lo, hi]; each pass
    // buckets (key - lo) >> s into at most NBINS bins (s chosen from the
    // range's width), finds the bucket that holds the remaining-th largest
    // candidate and shrinks [lo, hi] to it.  Bucketing by the actual range
    // spreads keys over the bins even when all scores share one exponent.
    if (tid < 32) {                              // the cluster's key range: lane r reads CTA r's, in parallel
        uint32_t a = 0xFFFFFFFFu, b = 0u;
        if (tid < CL) {
            if (CL > 1) {
                const uint32_t base = mapa_shared(smem_u32(cta_counts), (uint32_t)tid);
                a = ld_cluster_u32(base + 8);
                b = ld_cluster_u32(base + 12);
            } else {
                a = cta_counts[2];
                b = cta_counts[3];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
            b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
        }
        if (tid == 0) {
            shared_res[4] = a;
            shared_res[5] = b;
        }
    }
    __syncthreads();
    uint32_t lo_key = shared_res[4], hi_key = shared_res[5], remaining = (uint32_t)k;
    // candidate path: rank 0 hands every CTA its output offset and its share
    // of the keys equal to the threshold, so no later cluster exchange is needed
    bool offsets_known = false;
    uint32_t eq_before_given = 0u, out_before_given = 0u;
#pragma unroll 1
    for (int pass = 0; pass < MAX_PASSES && lo_key != hi_key; ++pass) {
        const uint32_t width = hi_key - lo_key;
        const int s_bits = 32 - __clz(width) - 11;        // (width >> s) < NBINS
        const int sh = s_bits > 0 ? s_bits : 0;
        for (int i = tid; i < NBINS; i += TOPK_THREADS) hist[i] = 0u;
        __syncthreads();
        for (int i = 4 * tid; i < cnt; i += 4 * TOPK_THREADS) {
            const uint4 q = *(const uint4*)(keys + i);
            const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i + u < cnt && kq[u] >= lo_key && kq[u] <= hi_key) atomicAdd(&hist[(kq[u] - lo_key) >> sh], 1u);
        }
        __syncthreads();
        // cluster-wide histogram: thread t owns bins 2t and 2t+1.  With a
        // cluster, CTA r holds the merged counts of bins [r OWN, (r+1) OWN):
        // every CTA adds its counts into the owner of each range, and its
        // count per range into every CTA's range totals, so one cluster
        // barrier suffices and no CTA is the target of all the traffic.  After
        // it, every CTA finds (from the totals) the range that holds the
        // remaining-th largest key and reads only that range's merged bins.
        const int lane = tid & 31, warp = tid >> 5;
        uint32_t h0, h1, above_r = 0u;
        if (CL > 1) {
            constexpr int OWN = NBINS / CL;                  // >= 128: a warp's 64 bins lie in one range
            static_assert(NBINS % CL == 0 && OWN % 64 == 0, "bin ranges");
            uint32_t* ch = cl_hist + pass * NBINS;
            const uint32_t owner = (uint32_t)(64 * warp) / OWN;
            const uint32_t dst = mapa_shared(smem_u32(ch + 2 * tid), owner);
            if (hist[2 * tid]) red_cluster_add(dst, hist[2 * tid]);
            if (hist[2 * tid + 1]) red_cluster_add(dst + 4, hist[2 * tid + 1]);
            uint32_t wsum = hist[2 * tid] + hist[2 * tid + 1];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
            if (lane < CL && wsum) red_cluster_add(mapa_shared(smem_u32(rtot + pass * MAX_CL + owner), (uint32_t)lane), wsum);
            cl_sync<CL>();                       // all additions landed
            // the range R that holds the remaining-th key from the top (the
            // same decision in every warp and CTA): keys in ranges above each
            // range by a suffix sum over the lanes
            const uint32_t tq = lane < CL ? rtot[pass * MAX_CL + lane] : 0u;
            uint32_t sq = tq;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_down_sync(0xffffffffu, sq, o);
                if (lane + o < 32) sq += y;
            }
            const uint32_t abv = sq - tq;
            const uint32_t hit = __ballot_sync(0xffffffffu, lane < CL && abv < remaining && remaining <= sq);
            const int R = hit ? __ffs(hit) - 1 : 0;
            above_r = __shfl_sync(0xffffffffu, abv, R);
            h0 = h1 = 0u;
            if (2 * tid >= R * OWN && 2 * tid < (R + 1) * OWN) {
                const uint2 v = ld_cluster_v2(mapa_shared(smem_u32(ch + 2 * tid), (uint32_t)R));
                h0 = v.x;
                h1 = v.y;
            }
        } else {
            h0 = hist[2 * tid];
            h1 = hist[2 * tid + 1];
        }
        // keys in bins above each thread's pair (the pairs of higher
        // threads, plus the ranges above R): a suffix sum within the warp,
        // then over the 32 warps
        const uint32_t hs = h0 + h1;
        uint32_t suf = hs;                       // this lane's pair and the pairs of higher lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += y;
        }
        if (lane == 0) warp_sums[warp] = suf;
        __syncthreads();
        const uint32_t wt = warp_sums[lane];
        uint32_t ws = wt;                        // warps >= lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, ws, o);
            if (lane + o < 32) ws += y;
        }
        const uint32_t above = above_r + __shfl_sync(0xffffffffu, ws - wt, warp) + (suf - hs);
        if (above < remaining && above + h1 >= remaining) {
            shared_res[0] = 2u * tid + 1u;
            shared_res[1] = above;
            shared_res[6] = h1;
        } else if (above + h1 < remaining && above + h1 + h0 >= remaining) {
            shared_res[0] = 2u * tid;
            shared_res[1] = above + h1;
            shared_res[6] = h0;
        }
        __syncthreads();
        const uint32_t bin = shared_res[0], bin_cnt = shared_res[6];
        remaining -= shared_res[1];
        const uint32_t new_lo = lo_key + (bin << sh);
        const uint32_t span = sh == 0 ? 0u : ((1u << sh) - 1u);
        hi_key = (hi_key - new_lo > span) ? new_lo + span : hi_key;
        lo_key = new_lo;
        __syncthreads();                         // shared_res / merged are reused by the next pass
        if (pass == 0 && lo_key != hi_key && bin_cnt <= (uint32_t)CAND_CAP) {
            // Few keys are left in the chosen range (typically tens): gather
            // them into rank 0's buffer and find the remaining-th largest by
            // counting, for each candidate, the candidates above it.
            const uint32_t n_addr = CL > 1 ? mapa_shared(smem_u32(cand_n), 0u) : smem_u32(cand_n);
            const uint32_t c_addr = CL > 1 ? mapa_shared(smem_u32(cand), 0u) : smem_u32(cand);
            const uint32_t s_addr = CL > 1 ? mapa_shared(smem_u32(cand_src), 0u) : smem_u32(cand_src);
            {
                // this CTA's keys in bins above the chosen one: all of them are taken
                uint32_t a = (2u * tid > bin ? hist[2 * tid] : 0u) + (2u * tid + 1u > bin ? hist[2 * tid + 1] : 0u);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                const uint32_t ab_addr =
                    CL > 1 ? mapa_shared(smem_u32(cta_cnt + rank), 0u) : smem_u32(cta_cnt + rank);
                if (lane == 0 && a) atom_add_cluster(ab_addr, a);
            }
            for (int b0 = warp * 128; b0 < cnt; b0 += 128 * (TOPK_THREADS / 32)) {
                const int i = b0 + 4 * lane;
                uint32_t kq[4] = {0u, 0u, 0u, 0u};
                if (i < cnt) {
                    const uint4 q = *(const uint4*)(keys + i);
                    kq[0] = q.x; kq[1] = q.y; kq[2] = q.z; kq[3] = q.w;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const bool c_ok = i + u < cnt && kq[u] >= lo_key && kq[u] <= hi_key;
                    const uint32_t m = __ballot_sync(0xffffffffu, c_ok);
                    if (m == 0u) continue;
                    const int leader = __ffs(m) - 1;
                    uint32_t base = 0u;
                    if (lane == leader) base = atom_add_cluster(n_addr, (uint32_t)__popc(m));
                    base = __shfl_sync(0xffffffffu, base, leader);
                    if (c_ok) {
                        const uint32_t pos = 4u * (base + __popc(m & ((1u << lane) - 1u)));
                        st_cluster_u32(c_addr + pos, kq[u]);
                        st_cluster_u32(s_addr + pos, rank);
                    }
                }
            }
            cl_sync<CL>();                       // every candidate has landed in rank 0's buffer
            if (rank == 0) {
                const uint32_t nc = *cand_n;
                if ((uint32_t)tid < nc) {
                    const uint32_t key = cand[tid];
                    uint32_t gt = 0u, ge = 0u;
                    for (uint32_t j = 0; j < nc; ++j) {
                        const uint32_t kj = cand[j];
                        gt += kj > key ? 1u : 0u;
                        ge += kj >= key ? 1u : 0u;
                    }
                    if (gt < remaining && remaining <= ge) {   // every thread holding that key agrees
                        shared_res[4] = key;
                        shared_res[5] = remaining - gt;
                    }
                }
                __syncthreads();
                // count each CTA's candidates above and equal to the threshold
                const uint32_t t_key = shared_res[4];
                if ((uint32_t)tid < nc) {
                    const uint32_t key = cand[tid], src = cand_src[tid];
                    if (key > t_key) atomicAdd(&cta_cnt[MAX_CL + src], 1u);
                    else if (key == t_key) atomicAdd(&cta_cnt[2 * MAX_CL + src], 1u);
                }
                __syncthreads();
                if (tid == 0) {
                    // ranks own contiguous slices in position order: CTA r's
                    // selected keys follow those of ranks < r
                    const uint32_t rem_eq = shared_res[5];
                    uint32_t eqb = 0u, outb = 0u;
                    for (uint32_t r = 0; r < (uint32_t)CL; ++r) {
                        const uint32_t dst = CL > 1 ? mapa_shared(smem_u32(cta_counts + 4), r) : smem_u32(cta_counts + 4);
                        st_cluster_u32(dst, t_key);
                        st_cluster_u32(dst + 4, rem_eq);
                        st_cluster_u32(dst + 8, eqb);
                        st_cluster_u32(dst + 12, outb);
                        const uint32_t e = cta_cnt[2 * MAX_CL + r];
                        const uint32_t take = eqb >= rem_eq ? 0u : min(e, rem_eq - eqb);
                        outb += cta_cnt[r] + cta_cnt[MAX_CL + r] + take;
                        eqb += e;
                    }
                }
            }
            cl_sync<CL>();                       // the last remote access of the kernel
            lo_key = cta_counts[4];
            remaining = cta_counts[5];
            eq_before_given = cta_counts[6];
            out_before_given = cta_counts[7];
            offsets_known = true;
            hi_key = lo_key;
            break;
        }
    }
    const uint32_t T = lo_key;                   // the k-th largest key; `remaining` keys == T to take

    // ---- 2. ordered compaction ----
    // Warp w owns a contiguous run of the slice and walks it 128 keys at a
    // time, lane l on the 4 consecutive keys 4l..4l+3 of each step (16-byte
    // loads); warp scans of the lanes' counts give every selected key its rank.
    const int warp = tid >> 5, lane = tid & 31;
    const int chunk = (((cnt + 127) / 128) + 31) / 32 * 128;        // keys per warp, multiple of 128
    const int wlo = min(cnt, warp * chunk), whi = min(cnt, wlo + chunk);
    uint32_t gt_w = 0, eq_w = 0;
    for (int base = wlo; base < whi; base += 128) {
        const int i = base + 4 * lane;
        uint32_t g = 0, e = 0;
        if (i < whi) {
            const uint4 q = *(const uint4*)(keys + i);
            const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                g += (i + u < whi && kq[u] > T) ? 1u : 0u;
                e += (i + u < whi && kq[u] == T) ? 1u : 0u;
            }
        }
        gt_w += g;
        eq_w += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt_w += __shfl_xor_sync(0xffffffffu, gt_w, o);
        eq_w += __shfl_xor_sync(0xffffffffu, eq_w, o);
    }
    uint32_t* wgt = merged;                      // per-warp counts and offsets (scratch)
    uint32_t* weq = merged + 32;
    uint32_t* wout = merged + 64;
    uint32_t* wtake = merged + 96;
    if (lane == 0) {
        wgt[warp] = gt_w;
        weq[warp] = eq_w;
    }
    __syncthreads();
    // CTA totals, and the counts of the cluster's lower-ranked CTAs
    uint32_t eq_before_cta = eq_before_given, out_before_cta = out_before_given;
    if (CL > 1 && !offsets_known) {
        if (warp == 0) {
            uint32_t g = wgt[lane], e = weq[lane];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                g += __shfl_xor_sync(0xffffffffu, g, o);
                e += __shfl_xor_sync(0xffffffffu, e, o);
            }
            if (lane == 0) {
                cta_counts[0] = g;
                cta_counts[1] = e;
            }
        }
        cl_sync<CL>();
        if (tid == 0) {
            uint32_t eqb = 0, outb = 0;
            for (uint32_t r = 0; r < rank; ++r) {
                const uint32_t base = mapa_shared(smem_u32(cta_counts), r);
                const uint32_t g = ld_cluster_u32(base), e = ld_cluster_u32(base + 4);
                const uint32_t take = eqb >= remaining ? 0u : min(e, remaining - eqb);
                outb += g + take;
                eqb += e;
            }
            shared_res[2] = eqb;
            shared_res[3] = outb;
        }
        __syncthreads();
        eq_before_cta = shared_res[2];
        out_before_cta = shared_res[3];
    }
    if (warp == 0) {
        // exclusive scans over the 32 warps (in position order)
        const uint32_t e = weq[lane], g = wgt[lane];
        uint32_t eq_incl = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, eq_incl, o);
            if (lane >= o) eq_incl += y;
        }
        const uint32_t eqb = eq_before_cta + eq_incl - e;
        const uint32_t take = eqb >= remaining ? 0u : min(e, remaining - eqb);
        const uint32_t sel = g + take;
        uint32_t sel_incl = sel;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, sel_incl, o);
            if (lane >= o) sel_incl += y;
        }
        wout[lane] = out_before_cta + sel_incl - sel;
        wtake[lane] = take;
    }
    __syncthreads();
    uint32_t j = wout[warp], eq_seen = 0;
    const uint32_t take = wtake[warp];
    for (int base = wlo; base < whi; base += 128) {
        const int i = base + 4 * lane;
        uint32_t kq[4] = {0u, 0u, 0u, 0u};
        if (i < whi) {
            const uint4 q = *(const uint4*)(keys + i);
            kq[0] = q.x; kq[1] = q.y; kq[2] = q.z; kq[3] = q.w;
        }
        uint32_t gm = 0, em = 0;                 // per-lane bit masks of its 4 keys
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            gm |= (i + u < whi && kq[u] > T) ? (1u << u) : 0u;
            em |= (i + u < whi && kq[u] == T) ? (1u << u) : 0u;
        }
        // equal keys before this lane (in position order), then the lane's own
        uint32_t e_incl = __popc(em);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, e_incl, o);
            if (lane >= o) e_incl += y;
        }
        uint32_t e_before = eq_seen + e_incl - __popc(em);
        uint32_t sm = gm;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if ((em >> u) & 1u) {
                if (e_before < take) sm |= 1u << u;
                ++e_before;
            }
        uint32_t s_incl = __popc(sm);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, s_incl, o);
            if (lane >= o) s_incl += y;
        }
        uint32_t o_at = j + s_incl - __popc(sm);
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if ((sm >> u) & 1u) out[o_at++] = lo + i + u;
        j += __shfl_sync(0xffffffffu, s_incl, 31);
        eq_seen += __shfl_sync(0xffffffffu, e_incl, 31);
    }
    if (CL > 1 && !offsets_known) cl_sync<CL>();   // peers are done reading our counts
}

namespace {

// Cluster size: at least enough CTAs to hold a row in shared memory, and,
// when there are few rows, as many more (up to 8) as keep every SM busy --
// a decode batch of 32 rows would otherwise leave most SMs idle.  Many rows
// that fit one SM each are selected one CTA per row (no cross-CTA traffic).
// 16-CTA clusters of topk_cluster_kernel<16> (slices of 16,384 keys) that the
// current device can hold at once (0 if none or the query fails); looked up
// once per device.
int max_active_16() {
    static std::atomic<int> cache[kMaxDevices] = {};
    return device_cached(cache, [] {
        const size_t smem = SMEM_ROUND + SMEM_FIXED + (size_t)16384 * 4;
        int n = 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16);
        cfg.blockDim = dim3(TOPK_THREADS);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaFuncSetAttribute(topk_cluster_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(topk_cluster_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel<16>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        return n;
    });
}

int choose_cluster(int rows, int ctx_len, int num_sms) {
    const int need = (ctx_len + SLICE_CAP - 1) / SLICE_CAP;
    int cl = 1;
    while (cl < need && cl < 8) cl <<= 1;
    while (cl < 8 && (int64_t)rows * cl * 2 <= num_sms && ctx_len / (cl * 2) >= 4096) cl <<= 1;
    // very long rows and very few of them: 16 CTAs per row, when the GPU can
    // hold all rows' 16-CTA clusters at once
    if (cl == 8 && (int64_t)rows * 16 <= num_sms && ctx_len / 16 >= 8192 && rows <= max_active_16()) cl = 16;
    return cl;
}

template <int CL>
cudaError_t launch_cl(const Launch& L, const float* logits, int64_t ld, const int32_t* row_pos, int rows, int ctx_len,
                      int k, int32_t* idx) {
    const int per = ((ctx_len + CL - 1) / CL + 3) & ~3;
    const size_t smem = SMEM_ROUND + SMEM_FIXED + (size_t)per * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel<CL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (CL > 8) {
        e = cudaFuncSetAttribute(topk_cluster_kernel<CL>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)rows * CL);
    cfg.blockDim = dim3(TOPK_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<CL>, logits, ld, row_pos, ctx_len, k, idx);
    count_launch();
    return e;
}

}  // namespace

bool topk_supported(int ctx_len) { return ctx_len <= 8 * SLICE_CAP; }

cudaError_t launch_topk(const Launch& L, const float* logits, int64_t ld, const int32_t* row_pos, int rows,
                        int ctx_len, int k, int32_t* idx, void* /*workspace*/, size_t /*ws_bytes*/) {
    if (rows == 0) return cudaSuccess;
    switch (choose_cluster(rows, ctx_len, L.num_sms)) {
    case 1: return launch_cl<1>(L, logits, ld, row_pos, rows, ctx_len, k, idx);
    case 2: return launch_cl<2>(L, logits, ld, row_pos, rows, ctx_len, k, idx);
    case 4: return launch_cl<4>(L, logits, ld, row_pos, rows, ctx_len, k, idx);
    case 8: return launch_cl<8>(L, logits, ld, row_pos, rows, ctx_len, k, idx);
    default: return launch_cl<16>(L, logits, ld, row_pos, rows, ctx_len, k, idx);
    }
}


size_t topk_workspace_bytes(int /*rows*/, int /*ctx_len*/, int /*k*/) { return 0; }

}  // namespace dsa
