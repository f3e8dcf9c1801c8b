// Sparse MLA (MQA mode) on the 5th-generation tensor cores
// ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", sections 1.3 细粒度稀疏注意力 and 1.4,
// section 3 Step 4): for every query row t and each of its 128 heads,
// attention over the selected latent rows only; one 576-d latent row is
// shared by all heads (512 latent + 64 rope dims); the value is its first
// 512 dims.
//
// Why a 2-CTA cluster: the output accumulator of one query row is
// 128 heads x 512 dims fp32 = 256 KB, exactly the tensor memory of one SM.
// So the work of a (query row, key split) is split by role across the two
// SMs of a cluster:
//
//   score CTA (rank 0)  Q [128 x 576] lives in TMEM (A operand of the MMA).
//                       Per chunk of 64 selected keys: gather the 576-d rows
//                       into 128-B-swizzled shared memory (cp.async), S = Q K^T
//                       (tcgen05, M=128 heads, N=64 keys, K=576) into one of
//                       three TMEM buffers, online softmax in base 2 with lazy
//                       rescaling (the running max moves only when a score
//                       exceeds it by more than 2^8), P rounded to bf16 and
//                       sent with its per-head rescale factors into the value
//                       CTA's shared memory by 16-byte st.async remote stores.
//   value CTA (rank 1)  gathers the first 512 dims of the same rows (the MMA
//                       reads them as an MN-major B operand), rescales O only
//                       for chunks whose max moved, accumulates
//                       O += P V (M=128, N=2x256, K=64) in its 512 TMEM
//                       columns, and at the end writes O / l and
//                       lse = ln(sum exp) -- or, when the key list is split
//                       over several clusters, normalised bf16 partials and
//                       their lse, which mla_combine_kernel merges in fp32
//                       (rounding a partial to bf16 costs at most one more
//                       bf16 ulp of the output).
//
// Two splits per row (decode with few rows): both pairs of a row form one
// 4-CTA cluster (ranks 0-1 split 0, ranks 2-3 split 1) and their value CTAs
// merge the splits themselves: each sends the 256 columns that the other
// finalises (raw fp32, DSMEM stores) as soon as both gather regions are
// drained, then they swap (max, sum) per head and each writes its half of
// out = (a O_0 + a' O_1) / (a l_0 + a' l_1).  This replaces the partials in
// global memory and the merge launch whenever all rows' 4-CTA clusters fit
// on the GPU at once.
//
// Warps (both CTAs): 0-15 gather producers (cp.async, 4 rows each); 16-23
// softmax (score CTA: two threads per head, 32 keys each) or 16-19 rescale +
// epilogue (value CTA, one thread per head / TMEM lane); 24 MMA issuer and
// TMEM owner.  Every wait is bounded; the two CTAs only exchange
// data through bulk copies and mbarrier arrivals that the receiver waits on.
#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"
#include "tensor_map.h"

namespace dsa {

using namespace sm100;

namespace {

constexpr int H = 128;              // query heads = MMA M
constexpr int DK = 576;             // latent + rope
constexpr int DV = 512;             // value dims
constexpr int NK = 64;              // keys per chunk
constexpr int PWARPS = 16;          // gather producer warps: cp.async throughput grows with the copies in flight
constexpr int ROWS_PER_PW = NK / PWARPS;
constexpr int SWARP0 = PWARPS;      // first of the 8 softmax warps (score CTA) / 8 rescale-epilogue warps (value CTA)
constexpr int MWARP = PWARPS + 8;   // MMA issuer, TMEM owner (its warpgroup's other 3 warps are spare)
constexpr int THREADS = 32 * (PWARPS + 12);     // 7 warpgroups
// Register split (per thread) after launch at THREADS x 72: producer and MMA
// warpgroups give registers back, the softmax warpgroups take them.
constexpr int REGS_LOW = 56, REGS_SOFTMAX = 104, REGS_LAUNCH = 72;
static_assert(PWARPS * 32 * REGS_LOW + 8 * 32 * REGS_SOFTMAX + 4 * 32 * REGS_LAUNCH <= REGS_LAUNCH * THREADS,
              "register split exceeds launch");
constexpr int KBLK = DK / 64;       // 9 dim blocks of 64 (128 B per row) per gathered row
constexpr int VBLK = DV / 64;       // the value CTA gathers the first 8
constexpr int KSTAGE = NK * DK * 2; // 73728 B: one chunk's rows, [dim block][64 rows x 128 B]
constexpr int SSTAGES = 3;          // score CTA: gather ring of full rows
constexpr int VSTAGES = 2;          // value CTA: gather ring of value rows (KSTAGE-sized slots)
constexpr int REGION = SSTAGES * KSTAGE;   // 221184: the role-specific part of shared memory
constexpr int QBYTES = H * DK * 2;  // 147456: the Q tile
constexpr int Q_OFF = KSTAGE;       // Q is staged in score stages 1-2, so chunk 0 is gathered into stage 0 at once
static_assert(Q_OFF + QBYTES == REGION, "Q staging fills score stages 1 and 2");
constexpr int EPI_BUF = 4096;       // epilogue: per-warp output staging tile (32 heads x 128 B), two per warp
constexpr int PBYTES = H * NK * 2;  // 16384: P [128 heads x 64 keys] bf16
constexpr int PSLOTS = 4;           // P ring depth (score CTA may run this many chunks ahead)
constexpr int ABYTES = H * 4;       // rescale factor per head
constexpr int SBYTES = 2 * H * 4;   // final running max and sum per head
// value CTA: its V ring, then the P ring and the rescale factors that the
// score CTA stores into it (st.async), inside the same region
constexpr int PBUF_OFF = VSTAGES * KSTAGE;
constexpr int ABUF_OFF = PBUF_OFF + PSLOTS * PBYTES;
static_assert(ABUF_OFF + PSLOTS * ABYTES <= REGION, "value CTA layout");
// the same offsets in every CTA: final statistics, scratch of the pair
// meetings and fused merge, barriers (remote accesses use mapa)
constexpr int SBUF_OFF = REGION;
constexpr int XBUF_OFF = SBUF_OFF + SBYTES;
constexpr int BARS_OFF = XBUF_OFF + 4 * H * 4;
constexpr int S_COL = 320;          // score CTA: Q in TMEM columns [0, 288), S buffers at 320, 384, 448
constexpr int TMEM_COLS = 512;
constexpr float RESCALE_LOG2 = 8.f; // lazy rescale threshold (P <= 2^8 between rescales)
constexpr float LN2 = 0.6931471805599453f;

struct Bars {                       // same offset in both CTAs of a cluster
    uint64_t full[SSTAGES];         // a stage's gathered rows have landed (cp.async arrivals)
    uint64_t empty[SSTAGES];        // the MMA is done reading a stage (score stages 1-2: first, Q has left)
    uint64_t sfull[3], sempty[3], pempty[PSLOTS], qready, statready, statack;
    // value CTA: P slot landed / rescaled, PV of chunk c done (ring of PSLOTS, so
    // that a parity wait never aliases), all PV done, final statistics landed
    uint64_t pfull[PSLOTS], ready[PSLOTS], odone[PSLOTS], ofinal, statfull;
    uint64_t qfull;                 // score CTA: the Q tile has landed in shared memory
    uint64_t cfree, cstat, crecv;   // fused two-split merge (value CTAs): the other split's gather region is
                                    // drained / its statistics / its share of O have landed here
    int mdone[4];                   // score CTA: per quarter, last chunk whose running maximum is published
    uint32_t tmem;
    int abort;
};

struct MlaParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* kv;
    const int32_t* page_table;
    const int32_t* row_batch;
    const int32_t* idx;             // [rows, k]; NULL: dense mode (slot s is key s up to row_last[t])
    const int32_t* row_last;
    const __nv_bfloat16* kv2;       // window segment: raw cache [batch, len2, DK]
    const int32_t* pos2;            // [rows] raw position of each query
    int len2, window, n_sink;
    __nv_bfloat16* out;
    float* lse;
    __nv_bfloat16* part_o;          // [rows, splits, H, DV] normalised partials when splits > 1
    float* part_lse;                // [rows, splits, H]
    unsigned* err;
    int page_size, pages_per_seq, num_pages;
    int k, ktot, rows, batch, ctx, splits, per_split;   // ktot = k + window + n_sink slots per row
    int fuse2;                      // two key splits per row in one 4-CTA cluster, merged in the kernel
    float scale_log2;
};

struct Work {
    int t, split, slot0, slot_end, nchunks, b;
    bool b_ok;
};

__device__ __forceinline__ Work work_of(const MlaParams& p) {
    Work w;
    const int item = blockIdx.x >> 1;
    w.t = item / p.splits;
    w.split = item - w.t * p.splits;
    w.slot0 = w.split * p.per_split;
    w.slot_end = min(p.ktot, w.slot0 + p.per_split);
    w.nchunks = (w.slot_end - w.slot0 + NK - 1) / NK;
    w.b = __ldg(p.row_batch + w.t);
    w.b_ok = w.b >= 0 && w.b < p.batch;
    return w;
}

// Key position held by slot `slot` of this row (-1: unused), before range
// checks: selected (or, in dense mode, every visible) key for slot < k, raw
// window position for k <= slot < k + window, raw sink position (only before
// the window's first position) for k + window <= slot < ktot.
// EXT = false compiles the plain selected-rows path (no window, sink or
// dense mode) exactly as lean as it was before those existed.
template <bool EXT>
__device__ __forceinline__ int slot_key(const MlaParams& p, const Work& w, int slot) {
    if (!EXT) return __ldg(p.idx + (int64_t)w.t * p.k + slot);
    if (slot < p.k) {
        if (p.idx) return __ldg(p.idx + (int64_t)w.t * p.k + slot);
        return slot <= __ldg(p.row_last + w.t) ? slot : -1;
    }
    const int first = __ldg(p.pos2 + w.t) - p.window + 1;     // the window's first raw position
    const int j = slot - p.k;
    if (j < p.window) return first + j < 0 ? -1 : first + j;
    return j - p.window < first ? j - p.window : -1;        // sink row j - window
}

// Row to gather for a slot: >= 0 a row of kv, <= -2 the row -2 - r of the
// window cache kv2, -1 nothing (unused or invalid slot; the copy writes zeros).
template <bool EXT>
__device__ __forceinline__ int64_t key_row(const MlaParams& p, const Work& w, int slot) {
    if (!w.b_ok || slot >= w.slot_end) return -1;
    const int s = slot_key<EXT>(p, w, slot);
    if (s < 0) return -1;
    if (EXT && slot >= p.k) {
        if (s >= p.len2) {
            record_error(p.err, DEV_ERR_BAD_INDEX);
            return -1;
        }
        return -2 - ((int64_t)w.b * p.len2 + s);
    }
    if (s >= p.ctx) {
        record_error(p.err, DEV_ERR_BAD_INDEX);
        return -1;
    }
    if (p.page_table) {
        const int pg = __ldg(p.page_table + (int64_t)w.b * p.pages_per_seq + s / p.page_size);
        if (pg < 0 || pg >= p.num_pages) {
            record_error(p.err, DEV_ERR_BAD_INDEX);
            return -1;
        }
        return (int64_t)pg * p.page_size + s % p.page_size;
    }
    return (int64_t)w.b * p.ctx + s;
}

// 2^x on the MUFU unit (ex2.approx, flush-to-zero): relative error ~2^-22,
// far below the bf16 rounding that P goes through next; -inf -> +0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Key position of a slot for the softmax's validity mask (-1 past the end of
// this split's slots).  It is loaded one chunk ahead and only compared (with
// slot_limit) in the next iteration, so the load latency stays hidden.
template <bool EXT>
__device__ __forceinline__ int slot_index(const MlaParams& p, const Work& w, int slot) {
    return slot < w.slot_end ? slot_key<EXT>(p, w, slot) : -1;
}

// Exclusive bound of valid key positions for a slot: the same decision as
// key_row, without its error reports and page lookups.
template <bool EXT>
__device__ __forceinline__ int slot_limit(const MlaParams& p, int slot) {
    return !EXT || slot < p.k ? p.ctx : p.len2;
}

// Stores into another CTA's shared memory (cluster address from mapa).
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Offset of 16-byte chunk `c` of row `r` in a [rows x 128 B] 128-B-swizzled block.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// Gather of the selected rows with cp.async, 16 bytes per copy: warp w owns
// rows [4w, 4w+4) of every chunk (one index lookup per lane, resolved one
// chunk ahead) and its lanes walk those rows with consecutive lanes on
// consecutive 16-byte pieces.  Many producer warps are used because the copy
// throughput of an SM grows with the number of copies its threads keep in
// flight.
//
// Ring of NST stages, chunk c in stage c % NST.  Score CTA (NST = 3): stages
// 1 and 2 first hold the Q tile, and their empty barrier's first phase is the
// release of Q (after its copy to TMEM), so their gathers wait one phase
// more than stage 0's, which starts at once.
template <int NB, bool EXT, int NST>   // NB: dim blocks gathered per row (9: full 576-d rows; 8: the 512 value dims)
__device__ __forceinline__ void gather_rows(const MlaParams& p, const Work& w, uint8_t* gbuf, Bars* bars, int warp,
                                            int lane, volatile int* abort_flag) {
    constexpr int RC = NB * 8;                           // 16-byte pieces per row
    constexpr bool Q_IN_RING = NB == KBLK;               // score CTA
    const int my_slot = warp * ROWS_PER_PW + (lane % ROWS_PER_PW);
    int64_t next_row = key_row<EXT>(p, w, w.slot0 + my_slot);
    for (int c = 0; c < w.nchunks; ++c) {
        const int st = c % NST;
        const uint32_t par = (uint32_t)((c / NST) & 1) ^ ((Q_IN_RING && st > 0) ? 0u : 1u);
        if (!mbar_wait(&bars->empty[st], par, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag)) break;
        const int myrow_lo = (int)next_row;     // row indices (and the window encoding) fit in 31 bits
        uint8_t* base = gbuf + (size_t)st * KSTAGE;
#pragma unroll
        for (int i = lane; i < ROWS_PER_PW * RC; i += 32) {
            const int rl = i / RC, ci = i - rl * RC;
            const int row = __shfl_sync(0xffffffffu, myrow_lo, rl);
            const int r = warp * ROWS_PER_PW + rl;
            const __nv_bfloat16* src;
            if (EXT)
                src = row >= 0 ? p.kv + (int64_t)row * DK + ci * 8
                    : row <= -2 ? p.kv2 + (int64_t)(-2 - row) * DK + ci * 8 : p.kv;
            else
                src = row >= 0 ? p.kv + (int64_t)row * DK + ci * 8 : p.kv;
            cp_async_16(base + (ci >> 3) * (NK * 128) + sw128(r, ci & 7), src, row != -1 ? 16u : 0u);
        }
        cp_async_arrive_noinc(&bars->full[st]);
        // look up the next chunk's row while this chunk's copies are in flight
        if (c + 1 < w.nchunks) next_row = key_row<EXT>(p, w, w.slot0 + (c + 1) * NK + my_slot);
    }
}

// Dense mode (every key of a contiguous range, no index list): the 64 keys
// of a chunk are consecutive cache rows, so one thread loads them with TMA
// tiles of 64 rows x 64 dims straight into the 128-B-swizzled stage layout
// (NB tiles per chunk) instead of gathering them row by row.  Rows past the
// cache are zero-filled by the tensor map; rows past the row's last visible
// key are masked by the softmax (their P is 0).  Same stage ring and
// barriers as gather_rows; each stage's full barrier counts the bytes.
template <int NB, int NST>
__device__ __forceinline__ void dense_loads(const MlaParams& p, const Work& w, const CUtensorMap* kv_map,
                                            uint8_t* gbuf, Bars* bars, volatile int* abort_flag) {
    constexpr bool Q_IN_RING = NB == KBLK;               // score CTA
    const int row_base = w.b_ok ? w.b * p.ctx + w.slot0 : 0;
    int issued = 0;
    for (int c = 0; c < w.nchunks; ++c) {
        const int st = c % NST;
        const uint32_t par = (uint32_t)((c / NST) & 1) ^ ((Q_IN_RING && st > 0) ? 0u : 1u);
        if (!mbar_wait(&bars->empty[st], par, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag)) break;
        mbar_arrive_expect_tx(&bars->full[st], NB * NK * 128);
        uint8_t* base = gbuf + (size_t)st * KSTAGE;
        for (int b = 0; b < NB; ++b) tma_load_2d(base + b * (NK * 128), kv_map, b * 64, row_base + c * NK, &bars->full[st]);
        ++issued;
    }
    // after an abort, let the tiles already requested land before the CTA exits
    if (*abort_flag)
        for (int j = issued > NST ? issued - NST : 0; j < issued; ++j)
            mbar_wait(&bars->full[j % NST], (j / NST) & 1, p.err, DEV_ERR_TIMEOUT_TMA, nullptr);
}

}  // namespace

// EXT: window / sink / dense slots; DENSE (implies EXT): every key of a
// contiguous range, loaded with TMA tiles (kv_map) instead of row gathers.
template <bool EXT, bool DENSE>
__global__ void __launch_bounds__(THREADS, 1) mla_tc_kernel(const __grid_constant__ CUtensorMap q_map,
                                                          const __grid_constant__ CUtensorMap o_map,
                                                          const __grid_constant__ CUtensorMap kv_map,
                                                          const MlaParams p) {
    pdl_wait();                     // the indices of the previous kernel are visible from here on
    pdl_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* gbuf = smem;                                   // K (score CTA) or V (value CTA) stages
    uint8_t* pbuf = smem + PBUF_OFF;                        // value CTA: [PSLOTS][PBYTES]
    float* abuf = (float*)(smem + ABUF_OFF);                // value CTA: [PSLOTS][H]
    float* sbuf = (float*)(smem + SBUF_OFF);                // [2*H]: running max, running sum
    float* xbuf = (float*)(smem + XBUF_OFF);                // [2][2][H]: partial maxima / sums of the two halves
                                                            // of a head (score CTA)
    Bars* bars = (Bars*)(smem + BARS_OFF);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a (query row, key split) is a pair of CTAs: role 0 = score CTA, role 1 =
    // value CTA; with the fused two-split merge the cluster holds both splits
    // of a row (ranks 0-1: split 0, ranks 2-3: split 1)
    const uint32_t role = cluster_ctarank() & 1u;
    const Work w = work_of(p);

    if (threadIdx.x == 0) {
        if (role == 0) {
            // Q [128 heads x 576] of this row first (it needs no load of the
            // row's batch index): 9 boxes of 128 rows x 64 dims, 128-byte
            // swizzled, into gather stages 1-2 (not yet in use)
            mbar_init(&bars->qfull, 1);
            fence_mbar_init();
            tma_prefetch_desc(&q_map);
            mbar_arrive_expect_tx(&bars->qfull, QBYTES);
            for (int b = 0; b < KBLK; ++b)
                tma_load_2d(gbuf + Q_OFF + b * (H * 128), &q_map, b * 64, w.t * H, &bars->qfull);
        }
        for (int i = 0; i < SSTAGES; ++i) {
            mbar_init(&bars->full[i], DENSE ? 1 : PWARPS * 32);
            mbar_init(&bars->empty[i], 1);
        }
        for (int i = 0; i < 3; ++i) {
            mbar_init(&bars->sfull[i], 1);
            mbar_init(&bars->sempty[i], 4);     // the softmax group of this S buffer
        }
        for (int i = 0; i < PSLOTS; ++i) {
            mbar_init(&bars->pempty[i], 1);
            mbar_init(&bars->pfull[i], 1);
            mbar_init(&bars->ready[i], 4);
            mbar_init(&bars->odone[i], 1);
        }
        mbar_init(&bars->qready, 8);
        mbar_init(&bars->statready, 8);
        mbar_init(&bars->statack, 4);
        mbar_init(&bars->ofinal, 1);
        mbar_init(&bars->statfull, 1);
        bars->abort = 0;
        for (int i = 0; i < 4; ++i) bars->mdone[i] = -1;
        mbar_init(&bars->cfree, 1);
        mbar_init(&bars->cstat, H);
        mbar_init(&bars->crecv, 8 * 32);
        if (role == 1) {
            // arm the first phase of each P slot and the final-statistics slot
            for (int i = 0; i < PSLOTS && i < w.nchunks; ++i) mbar_arrive_expect_tx(&bars->pfull[i], PBYTES + ABYTES);
            mbar_arrive_expect_tx(&bars->statfull, SBYTES);
        }
        fence_mbar_init();
        if (role == 1) tma_prefetch_desc(&o_map);
    }
    if (warp == MWARP) {
        tmem_alloc(&bars->tmem, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    cluster_sync_all();                 // both CTAs' barriers exist before any remote traffic
    tc_fence_after();
    const uint32_t tmem = bars->tmem;
    const uint32_t peer = cluster_ctarank() ^ 1u;
    if (threadIdx.x == 0 && !w.b_ok) record_error(p.err, DEV_ERR_BAD_INDEX);

    if (warp < PWARPS) {
        // ------------------------------------------------ gather producers ----
        regs_dec<REGS_LOW>();
        // Warp w owns rows [8w, 8w+8) of every chunk: lane l resolves one of
        // them once per chunk (one index load per lane, all in flight
        // together); the copy loop then walks the warp's rows with consecutive
        // lanes on consecutive 16-byte pieces of a row.  Several warps are
        // used because each keeps only a bounded number of copies in flight.
        if (DENSE) {
            if (warp == 0 && elect_one()) {
                if (role == 0) dense_loads<KBLK, SSTAGES>(p, w, &kv_map, gbuf, bars, abort_flag);
                else dense_loads<VBLK, VSTAGES>(p, w, &kv_map, gbuf, bars, abort_flag);
            }
        } else if (role == 0) {
            gather_rows<KBLK, EXT, SSTAGES>(p, w, gbuf, bars, warp, lane, abort_flag);
        } else {
            gather_rows<VBLK, EXT, VSTAGES>(p, w, gbuf, bars, warp, lane, abort_flag);
        }
    } else if (warp < SWARP0 + 8) {
      regs_inc<REGS_SOFTMAX>();
      if (role == 0) {
        // ------------------------------------- score CTA: Q load + softmax ----
        // Two groups of 4 warps take alternate chunks: group g = chunk & 1
        // (warps SWARP0 + 4g .. +3; chunk c's S is in buffer c mod 3).  Thread
        // (quarter, lane) of a group owns head h = 32*quarter + lane (its TMEM
        // lane) and all 64 keys of its group's chunks, so a chunk needs no
        // meeting between warps.  The only sequential part of the online
        // softmax is the running maximum: chunk c takes m(c-1) from the other
        // group's warp of the same quarter (published in shared memory, with a
        // per-quarter chunk counter), decides lazily whether it moves (only
        // when a score exceeds it by 2^8) and publishes m(c); the exponentials,
        // the packing and the transfer of P then overlap the other group's
        // chunk.  Each group keeps its own running sum relative to the maximum
        // it last used; the two are brought to the final maximum at the end.
        // P rows (and the head's rescale factor) go straight into the value
        // CTA's P slot with st.async, whose bytes are counted on the value
        // CTA's barrier for that slot, so the score CTA keeps no P ring.
        const int sw = warp - SWARP0, grp = sw >> 2, quarter = sw & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        float* mpub = xbuf;                                  // [2][H]: m(c) of the last chunk of group c & 1
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->qfull, 0, p.err, DEV_ERR_TIMEOUT_TMA, abort_flag));
        if (ok) {   // Q row h -> TMEM lane h; group g writes the 16-column groups [9g, 9g + 9)
#pragma unroll 1
            for (int g = 9 * grp; g < 9 * grp + 9; ++g) {
                const uint8_t* row = gbuf + Q_OFF + (g >> 1) * (H * 128) + h * 128;
                uint32_t words[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 x = ld_shared_v4(row + ((((g & 1) * 4 + v) ^ (h & 7)) << 4));
                    words[4 * v] = x.x; words[4 * v + 1] = x.y; words[4 * v + 2] = x.z; words[4 * v + 3] = x.w;
                }
                tmem_st16(tmem + lane_base + g * 16, words);
            }
            tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->qready);
        float m_own = -INFINITY, l_own = 0.f;     // this group's sum, relative to the maximum it last used
        const uint32_t peer_pbuf = mapa_shared(smem_u32(pbuf), peer);    // the value CTA's P ring
        const uint32_t peer_abuf = mapa_shared(smem_u32(abuf), peer);    // and its rescale factors
        // key positions of this lane's two keys (lane, 32 + lane) of the
        // group's next chunk, loaded one group chunk ahead
        int s_lo = grp < w.nchunks ? slot_index<EXT>(p, w, w.slot0 + grp * NK + lane) : -1;
        int s_hi = grp < w.nchunks ? slot_index<EXT>(p, w, w.slot0 + grp * NK + 32 + lane) : -1;
        for (int c = grp; c < w.nchunks; c += 2) {
            const int sb = c % 3;
            const int slot0 = w.slot0 + c * NK;
            const uint32_t vm_lo = __ballot_sync(0xffffffffu, w.b_ok && s_lo >= 0 && s_lo < slot_limit<EXT>(p, slot0 + lane));
            const uint32_t vm_hi =
                __ballot_sync(0xffffffffu, w.b_ok && s_hi >= 0 && s_hi < slot_limit<EXT>(p, slot0 + 32 + lane));
            if (c + 2 < w.nchunks) {
                s_lo = slot_index<EXT>(p, w, slot0 + 2 * NK + lane);
                s_hi = slot_index<EXT>(p, w, slot0 + 2 * NK + 32 + lane);
            }
            float sv[64];
            ok = ok && __all_sync(0xffffffffu,
                                  mbar_wait(&bars->sfull[sb], (c / 3) & 1, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag));
            if (!ok) break;
            tc_fence_after();
            tmem_ld32(tmem + lane_base + S_COL + sb * NK, *reinterpret_cast<float(*)[32]>(sv));
            tmem_ld32(tmem + lane_base + S_COL + sb * NK + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->sempty[sb]);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                sv[j] = ((vm_lo >> j) & 1u) ? sv[j] * p.scale_log2 : -INFINITY;
                sv[32 + j] = ((vm_hi >> j) & 1u) ? sv[32 + j] * p.scale_log2 : -INFINITY;
            }
            float mx[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) mx[j] = fmaxf(fmaxf(sv[4 * j], sv[4 * j + 1]), fmaxf(sv[4 * j + 2], sv[4 * j + 3]));
#pragma unroll
            for (int w2 = 8; w2 >= 1; w2 >>= 1)
#pragma unroll
                for (int j = 0; j < w2; ++j) mx[j] = fmaxf(mx[j], mx[j + w2]);
            const float mc = mx[0];
            // the running maximum after chunk c - 1 (the other group's chunk)
            float m_prev = -INFINITY;
            if (c > 0) {
                bool got = true;
                if (lane == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    for (uint32_t it = 0; ld_acquire_cta(&bars->mdone[quarter]) < c - 1; ++it) {
                        if ((it & 63u) == 63u) {
                            if (*abort_flag) { got = false; break; }
                            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                                record_error(p.err, DEV_ERR_TIMEOUT_PEER);
                                *abort_flag = 1;
                                got = false;
                                break;
                            }
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                if (!ok) break;
                __syncwarp();                       // orders lane 0's acquire before the other lanes' reads
                m_prev = ((volatile float*)mpub)[((c - 1) & 1) * H + h];
            }
            float m_new = m_prev, alpha = 1.f;
            if (mc > -INFINITY) {
                if (m_prev == -INFINITY) {
                    m_new = mc;
                } else if (mc > m_prev + RESCALE_LOG2) {
                    alpha = exp2f(m_prev - mc);
                    m_new = mc;
                }
            }
            ((volatile float*)mpub)[(c & 1) * H + h] = m_new;
            __syncwarp();                           // every lane's value is written before lane 0 publishes
            if (lane == 0) st_release_cta(&bars->mdone[quarter], c);
            if (m_new != m_own) {
                l_own = m_own == -INFINITY ? 0.f : l_own * exp2f(m_own - m_new);
                m_own = m_new;
            }
            // the slot's previous P has been consumed by the value CTA's MMA
            const int pb = c % PSLOTS, pu = c / PSLOTS;
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars->pempty[pb], (pu & 1) ^ 1, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag));
            if (!ok) break;
            // exp2 of (score - running max): at most 2^8 (lazy rescale); -inf for
            // unused keys, which ex2 maps to +0.  P row h (128 B, 128-B-swizzled
            // K-major tile) and the head's rescale factor: 128 x 128 + 128 x 4
            // bytes per chunk, the count the value CTA expects on pfull[pb]
            const float mr = m_new == -INFINITY ? 0.f : m_new;
            const uint32_t rbar = mapa_shared(smem_u32(&bars->pfull[pb]), peer);
            const uint32_t prow = peer_pbuf + (uint32_t)(pb * PBYTES + (h >> 3) * 1024);
            float ls[8];
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) {            // 16-byte piece q8: keys 8 q8 .. 8 q8 + 7
                uint32_t pk[4];
                float s2 = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 pr = __floats2bfloat162_rn(fast_exp2(sv[8 * q8 + 2 * e] - mr),
                                                                    fast_exp2(sv[8 * q8 + 2 * e + 1] - mr));
                    s2 += __low2float(pr) + __high2float(pr);
                    pk[e] = *(const uint32_t*)&pr;
                }
                ls[q8] = s2;
                st_async_v4(prow + sw128(h & 7, q8), pk[0], pk[1], pk[2], pk[3], rbar);
            }
            st_async_b32(peer_abuf + (uint32_t)(pb * ABYTES + h * 4), __float_as_uint(alpha), rbar);
#pragma unroll
            for (int w2 = 4; w2 >= 1; w2 >>= 1)
#pragma unroll
                for (int j = 0; j < w2; ++j) ls[j] += ls[j + w2];
            l_own += ls[0];
        }
        // final statistics -> value CTA: the last chunk's running maximum and
        // the two groups' sums brought to it.  Every softmax warp reaches the
        // barrier below (the loop has no unbounded wait), aborted or not.
        float* gstat = xbuf + 2 * H;                          // [2][H]: group 1's (m, l)
        if (grp == 1) {
            gstat[h] = m_own;
            gstat[H + h] = l_own;
        }
        named_bar_sync(1, 256);
        if (grp == 0 && ok && !*abort_flag) {
            const float m1 = gstat[h], l1 = gstat[H + h];
            const float mf = fmaxf(m_own, m1);        // the last chunk's maximum: the largest one used
            const float l0s = m_own == -INFINITY ? 0.f : l_own * exp2f(m_own - mf);
            const float l1s = m1 == -INFINITY ? 0.f : l1 * exp2f(m1 - mf);
            sbuf[h] = mf;
            sbuf[H + h] = l0s + l1s;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->statready);
        if (warp == SWARP0 && lane == 0 && !*abort_flag) {
            if (mbar_wait(&bars->statready, 0, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag))
                bulk_copy_s2cluster(mapa_shared(smem_u32(sbuf), peer), sbuf, SBYTES,
                                    mapa_shared(smem_u32(&bars->statfull), peer));
        }
        // stay alive until the value CTA has read the statistics and its last
        // MMA commits (which arrive on our P-slot barriers) have landed
        mbar_wait(&bars->statack, 0, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag);
        for (int c = max(0, w.nchunks - PSLOTS); c < w.nchunks; ++c)
            mbar_wait(&bars->pempty[c % PSLOTS], (c / PSLOTS) & 1, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag);
      } else {
        // --------------------------- value CTA: rescale of O, then epilogue ----
        // Warps SWARP0..SWARP0+3 (one thread per head / TMEM lane) apply the
        // per-chunk rescale factors to O before its next PV MMA.  At the end
        // all 8 warps write O / l: warp SWARP0 + 4*colhalf + quarter takes
        // heads [32*quarter, +32) and columns [256*colhalf, +256), in tiles of
        // 32 heads x 128 B staged in 128-byte-swizzled shared memory (the
        // drained gather region) and stored with TMA.
        const int sw = warp - SWARP0, quarter = sw & 3, colhalf = sw >> 2;
        const int h = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        if (colhalf == 0) {
            for (int c = 0; c < w.nchunks && ok; ++c) {
                const int pb = c % PSLOTS, pu = c / PSLOTS;
                // P and the rescale factors arrive as st.async stores from the
                // score CTA (release at cluster scope): acquire at cluster scope
                ok = mbar_wait_cluster(&bars->pfull[pb], pu & 1, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag);
                if (!ok) break;
                if (warp == SWARP0 && lane == 0 && c + PSLOTS < w.nchunks)
                    mbar_arrive_expect_tx(&bars->pfull[pb], PBYTES + ABYTES);     // arm this slot's next use
                const float alpha = abuf[pb * H + h];
                if (c > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    // O must hold all of chunk c-1 (P of chunk c arriving means
                    // the PV MMA of chunk c-4 is done, so this parity is unambiguous)
                    const int pc = c - 1;
                    ok = mbar_wait(&bars->odone[pc % PSLOTS], (pc / PSLOTS) & 1, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int j = 0; j < DV / 32; ++j) {
                        float v[32];
                        tmem_ld32(tmem + lane_base + j * 32, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] *= alpha;
                        tmem_st32(tmem + lane_base + j * 32, v);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->ready[pb]);
            }
        }
        if (ok) ok = mbar_wait(&bars->ofinal, 0, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag);
        if (p.fuse2) {
            // Fused two-split merge, first half: once both value CTAs' gather
            // regions are drained, each sends the columns that the other split
            // finalises (split s finalises [256 s, +256)), unscaled, into the
            // other's region; the weights need the final statistics, which
            // are swapped afterwards.  Tiles of 32 heads x 32 columns are laid
            // out [8 pieces][32 lanes][16 B], so that one remote store of a
            // warp covers 512 contiguous bytes.
            const uint32_t oth = cluster_ctarank() ^ 2u;
            if (ok && sw == 0 && lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&bars->cfree), oth));
            ok = __all_sync(0xffffffffu, ok) &&
                 __all_sync(0xffffffffu, mbar_wait_cluster(&bars->cfree, 0, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag));
            if (ok) {
                tc_fence_after();
                const int send0 = (1 - w.split) * 256 + colhalf * 128;
                const uint32_t rdst =
                    mapa_shared(smem_u32(gbuf + (quarter * 2 + colhalf) * 4 * 4096 + lane * 16), oth);
#pragma unroll 1
                for (int j = 0; j < 4; ++j) {
                    float v[32];
                    tmem_ld32(tmem + lane_base + send0 + j * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int ci = 0; ci < 8; ++ci)
                        st_cluster_v4(rdst + j * 4096 + ci * 512, v[4 * ci], v[4 * ci + 1], v[4 * ci + 2], v[4 * ci + 3]);
                }
                mbar_arrive_remote(mapa_shared(smem_u32(&bars->crecv), oth));
            }
        }
        if (ok) ok = mbar_wait(&bars->statfull, 0, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag);
        float m = -INFINITY, l = 0.f;
        if (ok) {
            m = sbuf[h];
            l = sbuf[H + h];
        }
        __syncwarp();
        if (colhalf == 0 && lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&bars->statack), peer));
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const float lse = l > 0.f ? (m + log2f(l)) * LN2 : -INFINITY;
            uint8_t* stage = gbuf + sw * 2 * EPI_BUF;
            uint8_t* srow = stage + lane * 128;
            if (p.fuse2) {
                // Fused two-split merge, second half: swap the per-head
                // statistics, then out = (a O_own + a' O_other) / (a l + a' l')
                // on this split's columns, with a = 2^(m - max(m, m')).
                const uint32_t oth = cluster_ctarank() ^ 2u;
                if (colhalf == 0) {
                    st_cluster_f32(mapa_shared(smem_u32(xbuf + h), oth), m);
                    st_cluster_f32(mapa_shared(smem_u32(xbuf + H + h), oth), l);
                    mbar_arrive_remote(mapa_shared(smem_u32(&bars->cstat), oth));
                }
                bool got = __all_sync(0xffffffffu,
                                      mbar_wait_cluster(&bars->cstat, 0, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag));
                if (got) {
                    const float mo = xbuf[h], lo = xbuf[H + h];
                    const float mm = fmaxf(m, mo);
                    const float a = m == -INFINITY ? 0.f : exp2f(m - mm);
                    const float ao = mo == -INFINITY ? 0.f : exp2f(mo - mm);
                    const float ll = a * l + ao * lo;
                    const float so = ll > 0.f ? a / ll : 0.f, sr = ll > 0.f ? ao / ll : 0.f;
                    const int keep0 = w.split * 256 + colhalf * 128;
                    const int tile0 = (quarter * 2 + colhalf) * 4;     // this warp's 4 received tiles
                    got = __all_sync(0xffffffffu,
                                     mbar_wait_cluster(&bars->crecv, 0, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag));
                    if (got) {
#pragma unroll 1
                        for (int jj = 0; jj < 2; ++jj) {
                            // bf16 tile of 32 heads x 64 columns, staged in the
                            // received tile 2jj once the whole warp has read it
                            uint8_t* tbuf = gbuf + (tile0 + 2 * jj) * 4096;
#pragma unroll 1
                            for (int e = 0; e < 2; ++e) {
                                const int j = 2 * jj + e;
                                float v[32];
                                tmem_ld32(tmem + lane_base + keep0 + j * 32, v);
                                tmem_ld_wait();
                                const uint8_t* rrow = gbuf + (tile0 + j) * 4096 + lane * 16;
#pragma unroll
                                for (int ci = 0; ci < 8; ++ci) {
                                    const uint4 x = ld_shared_v4(rrow + ci * 512);
                                    v[4 * ci] = fmaf(v[4 * ci], so, __uint_as_float(x.x) * sr);
                                    v[4 * ci + 1] = fmaf(v[4 * ci + 1], so, __uint_as_float(x.y) * sr);
                                    v[4 * ci + 2] = fmaf(v[4 * ci + 2], so, __uint_as_float(x.z) * sr);
                                    v[4 * ci + 3] = fmaf(v[4 * ci + 3], so, __uint_as_float(x.w) * sr);
                                }
                                if (e == 0) __syncwarp();                 // all lanes are done reading tile 2jj
#pragma unroll
                                for (int ci = 0; ci < 4; ++ci) {
                                    uint32_t o[4];
#pragma unroll
                                    for (int q = 0; q < 4; ++q) {
                                        const __nv_bfloat162 x =
                                            __floats2bfloat162_rn(v[8 * ci + 2 * q], v[8 * ci + 2 * q + 1]);
                                        o[q] = *(const uint32_t*)&x;
                                    }
                                    st_shared_v4(tbuf + lane * 128 + (((4 * e + ci) ^ (lane & 7)) << 4), o[0], o[1],
                                                 o[2], o[3]);
                                }
                            }
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_2d(&o_map, tbuf, keep0 + jj * 64, w.t * H + quarter * 32);
                                bulk_commit_group();
                            }
                        }
                        if (w.split == 0 && colhalf == 0)
                            p.lse[(int64_t)w.t * H + h] = ll > 0.f ? (mm + log2f(ll)) * LN2 : -INFINITY;
                    }
                }
            } else {
                // bf16 tiles of 32 heads x 64 columns: the output, or (key list
                // split over several clusters) this split's normalised partial
                const int row0 = (p.splits == 1 ? w.t * H : (w.t * p.splits + w.split) * H) + quarter * 32;
#pragma unroll 1
                for (int j = 0; j < 4; ++j) {
                    const int col = colhalf * 256 + j * 64;
                    float v[32], u[32];
                    tmem_ld32(tmem + lane_base + col, v);
                    tmem_ld32(tmem + lane_base + col + 32, u);
                    tmem_ld_wait();
                    if (j >= 2) {                       // the store that read this buffer two tiles ago is done
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
                    }
                    uint8_t* buf = srow + (j & 1) * EPI_BUF;
                    uint32_t o[32];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const __nv_bfloat162 x = __floats2bfloat162_rn(v[2 * e] * inv, v[2 * e + 1] * inv);
                        const __nv_bfloat162 y = __floats2bfloat162_rn(u[2 * e] * inv, u[2 * e + 1] * inv);
                        o[e] = *(const uint32_t*)&x;
                        o[16 + e] = *(const uint32_t*)&y;
                    }
#pragma unroll
                    for (int ci = 0; ci < 8; ++ci)
                        st_shared_v4(buf + ((ci ^ (lane & 7)) << 4), o[4 * ci], o[4 * ci + 1], o[4 * ci + 2], o[4 * ci + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&o_map, stage + (j & 1) * EPI_BUF, col, row0);
                        bulk_commit_group();
                    }
                }
                if (colhalf == 0) {
                    if (p.splits == 1) p.lse[(int64_t)w.t * H + h] = lse;
                    else p.part_lse[((int64_t)w.t * p.splits + w.split) * H + h] = lse;
                }
            }
            if (lane == 0) bulk_wait_group<0>();
            __syncwarp();
        }
      }
    } else {
      if (warp == MWARP) {
        // ----------------------------------------------------- MMA issuer ----
        if (elect_one()) {
            if (role == 0) {
                constexpr uint32_t idesc = idesc_bf16_f32(H, NK, 0, 0);
                const uint32_t kbase = smem_u32(gbuf);
                bool ok = mbar_wait(&bars->qready, 0, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag);
                tc_fence_after();
                if (ok) {
                    // Q is in TMEM: gather stages 1 and 2 are free for their first chunks
                    mbar_arrive(&bars->empty[1]);
                    mbar_arrive(&bars->empty[2]);
                }
                for (int c = 0; c < w.nchunks && ok; ++c) {
                    const int st = c % SSTAGES, sb = c % 3;
                    ok = mbar_wait(&bars->sempty[sb], ((c / 3) & 1) ^ 1, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag) &&
                         mbar_wait(&bars->full[st], (c / SSTAGES) & 1, p.err, DEV_ERR_TIMEOUT_TMA, abort_flag);
                    if (!ok) break;
                    fence_proxy_async_smem();
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk) {
                        const uint32_t boff = (uint32_t)(st * KSTAGE + (kk >> 2) * (NK * 128) + (kk & 3) * 32);
                        mma_ts(tmem + S_COL + sb * NK, tmem + kk * 8, desc_sw128(kbase + boff, 1024), idesc, kk > 0);
                    }
                    mma_commit(&bars->empty[st]);
                    if (ok) mma_commit(&bars->sfull[sb]);
                }
            } else {
                constexpr uint32_t idesc = idesc_bf16_f32(H, 256, 0, 1);
                const uint32_t vbase = smem_u32(gbuf), pbase = smem_u32(pbuf);
                bool ok = true;
                for (int c = 0; c < w.nchunks && ok; ++c) {
                    const int st = c & 1, pb = c % PSLOTS, par = (c >> 1) & 1;
                    ok = mbar_wait(&bars->ready[pb], (c / PSLOTS) & 1, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag);
                    ok = ok && mbar_wait(&bars->full[st], par, p.err, DEV_ERR_TIMEOUT_TMA, abort_flag);
                    if (!ok) break;
                    fence_proxy_async_smem();
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < NK / 16; ++kk) {
                        const uint64_t adesc = desc_sw128(pbase + pb * PBYTES + kk * 32, 1024);
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const uint32_t boff = (uint32_t)(st * KSTAGE + half * 4 * (NK * 128) + kk * 16 * 128);
                            mma_ss(tmem + half * 256, adesc, desc_sw128_mn(vbase + boff, NK * 128, 1024), idesc,
                                   (c > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    mma_commit(&bars->empty[st]);
                    mma_commit_multicast(&bars->pempty[pb], (uint16_t)(0x3u << (cluster_ctarank() & 2u)));
                    mma_commit(&bars->odone[pb]);
                }
                if (ok) mma_commit(&bars->ofinal);
            }
        }
    }

    }

    tc_fence_before();
    __syncthreads();
    if (warp == MWARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Merge of split partials: out = sum_s exp(lse_s - lse) * O_s, lse = log sum_s exp(lse_s),
// in fp32 from the bf16 partials.
__global__ void __launch_bounds__(128) mla_combine_kernel(const __nv_bfloat16* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int splits,
                                                          __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    pdl_wait();
    const int t = blockIdx.x, h = blockIdx.y;
    const int d = threadIdx.x * 4;
    float mx = -INFINITY;
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, __ldg(part_lse + ((int64_t)t * splits + s) * H + h));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (mx > -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const int64_t pr = ((int64_t)t * splits + s) * H + h;
            const float ls = __ldg(part_lse + pr);
            if (ls == -INFINITY) continue;
            const float wgt = __expf(ls - mx);
            den += wgt;
            const uint2 raw = __ldg((const uint2*)(part_o + pr * DV + d));
            const float2 a = __bfloat1622float2(*(const __nv_bfloat162*)&raw.x);
            const float2 b = __bfloat1622float2(*(const __nv_bfloat162*)&raw.y);
            acc.x = fmaf(wgt, a.x, acc.x); acc.y = fmaf(wgt, a.y, acc.y);
            acc.z = fmaf(wgt, b.x, acc.z); acc.w = fmaf(wgt, b.y, acc.w);
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 pk = make_uint2(*(uint32_t*)&lo, *(uint32_t*)&hi);
    *(uint2*)(out + ((int64_t)t * H + h) * DV + d) = pk;
    if (threadIdx.x == 0) lse[(int64_t)t * H + h] = den > 0.f ? mx + __logf(den) : -INFINITY;
}

// ------------------------------------------------------------------ host --

namespace {

// 1024 B of room to round the base up to 1024 (128-B swizzle atoms), the
// region, the statistics and pair scratch, the barrier block
constexpr size_t MLA_SMEM = 1024 + (size_t)BARS_OFF + 1024;
static_assert(sizeof(Bars) <= 1024, "barrier block");
static_assert(MLA_SMEM <= 232448, "above the 227 KB of shared memory a CTA may use");

int choose_splits(int rows, int k, int num_sms) {
    const int clusters = num_sms / 2;
    const int max_split = (k + NK - 1) / NK;
    int s = rows >= clusters ? 1 : clusters / rows;
    if (s > max_split) s = max_split;
    return s < 1 ? 1 : s;
}

// How many 4-CTA clusters of mla_tc_kernel can be resident at once on the
// current device (0 if the query fails); looked up once per device.
int max_active_quads() {
    static std::atomic<int> cache[kMaxDevices] = {};
    return device_cached(cache, [] {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(4);
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = MLA_SMEM;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 4;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        // both kernel variants have the same shape; the attribute must be set on the one queried
        if (cudaFuncSetAttribute(mla_tc_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)MLA_SMEM) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, mla_tc_kernel<false, false>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        return n;
    });
}

}  // namespace

bool mla_tc_supported(dsa_dtype_t dtype, int n_heads, int d_qk, int d_v) {
    return dtype == DSA_BF16 && n_heads == H && d_qk == DK && d_v == DV;
}

size_t mla_tc_workspace_bytes(int rows, int k, int num_sms) {
    const int s = choose_splits(rows, k, num_sms);
    if (s == 1) return 0;
    return (size_t)rows * s * H * (DV * sizeof(__nv_bfloat16) + sizeof(float));
}

cudaError_t launch_mla_tc(const Launch& L, const void* q, const void* kv, const int32_t* page_table, int page_size,
                          int num_pages, const int32_t* row_batch, const int32_t* idx, int k, int rows, int batch,
                          int ctx_len, float scale, void* out, float* lse, void* workspace, size_t ws_bytes,
                          const KvExtra& x) {
    if (rows == 0) return cudaSuccess;
    MlaParams p;
    p.q = (const __nv_bfloat16*)q;
    p.kv = (const __nv_bfloat16*)kv;
    p.page_table = page_table;
    p.row_batch = row_batch;
    p.idx = idx;
    p.row_last = x.row_last;
    p.kv2 = (const __nv_bfloat16*)x.kv2;
    p.pos2 = x.pos2;
    p.len2 = x.len2;
    p.window = x.kv2 ? x.window : 0;
    p.n_sink = x.kv2 ? x.n_sink : 0;
    p.out = (__nv_bfloat16*)out;
    p.lse = lse;
    p.err = L.err;
    p.page_size = page_table ? page_size : 1;
    p.pages_per_seq = page_table ? ctx_len / page_size : 0;
    p.num_pages = page_table ? num_pages : 0;
    p.k = k;
    p.ktot = k + p.window + p.n_sink;
    p.rows = rows;
    p.batch = batch;
    p.ctx = ctx_len;
    p.splits = choose_splits(rows, p.ktot, L.num_sms);
    const int per = (p.ktot + p.splits - 1) / p.splits;
    p.per_split = (per + NK - 1) / NK * NK;
    p.splits = (p.ktot + p.per_split - 1) / p.per_split;       // no empty split
    p.scale_log2 = scale * 1.4426950408889634f;
    p.part_o = nullptr;
    p.part_lse = nullptr;
    const bool ext = p.window > 0 || p.n_sink > 0 || !p.idx;
    // every key of a contiguous cache range (no index list, window, sink or
    // page table): TMA tiles instead of row gathers
    const bool dense = !p.idx && p.window == 0 && p.n_sink == 0 && !page_table;
    auto kern = dense ? mla_tc_kernel<true, true> : ext ? mla_tc_kernel<true, false> : mla_tc_kernel<false, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)MLA_SMEM);
    if (e != cudaSuccess) return e;
    // Two splits per row: merge them inside a 4-CTA cluster when all rows'
    // clusters are resident in one wave (no partials in global memory, no
    // merge launch); otherwise split partials go to the workspace.
    p.fuse2 = (p.splits == 2 && rows <= max_active_quads()) ? 1 : 0;
    if (p.splits > 1 && !p.fuse2) {
        const size_t need = (size_t)rows * p.splits * H * (DV * sizeof(__nv_bfloat16) + sizeof(float));
        if (!workspace || ws_bytes < need || (uintptr_t)workspace % 16) return cudaErrorInvalidValue;
        p.part_o = (__nv_bfloat16*)workspace;
        p.part_lse = (float*)(p.part_o + (size_t)rows * p.splits * H * DV);
    }
    // Q as [rows*128, 576] bf16 in boxes of 128 heads x 64 dims; the output as
    // [rows*128, 512] bf16 in boxes of 32 heads x 64 columns, or the partials
    // as [rows*splits*128, 512] fp32 in boxes of 32 heads x 32 columns
    CUtensorMap q_map, o_map, kv_map;
    bool ok = make_map_sw128(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, DK, (uint64_t)rows * H, 64, H);
    // dense mode: the cache as [batch * ctx, 576] in tiles of 64 rows x 64 dims
    kv_map = q_map;
    if (dense) ok = ok && make_map_sw128(&kv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kv, DK, (uint64_t)batch * ctx_len, 64, NK);
    if (p.splits == 1 || p.fuse2)
        ok = ok && make_map_sw128(&o_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, DV, (uint64_t)rows * H, 64, 32);
    else
        ok = ok && make_map_sw128(&o_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.part_o, DV,
                                  (uint64_t)rows * p.splits * H, 64, 32);
    if (!ok) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2u * (unsigned)rows * (unsigned)p.splits);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = MLA_SMEM;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.fuse2 ? 4 : 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, q_map, o_map, kv_map, p);
    count_launch();
    if (e != cudaSuccess) return e;
    if (p.splits > 1 && !p.fuse2) {
        cudaLaunchConfig_t c2 = {};
        c2.gridDim = dim3(rows, H);
        c2.blockDim = dim3(128);
        c2.stream = L.stream;
        cudaLaunchAttribute a2[1] = {pdl_attr()};
        c2.attrs = a2;
        c2.numAttrs = 1;
        e = cudaLaunchKernelEx(&c2, mla_combine_kernel, (const __nv_bfloat16*)p.part_o, (const float*)p.part_lse, p.splits,
                               (__nv_bfloat16*)out, lse);
        count_launch();
    }
    return e;
}

}  // namespace dsa
