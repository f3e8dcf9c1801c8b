// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05)
// ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", section 1.3 闪电索引器 and section 3
// Step 2; xhh.club DeepSeek-V4 CSA summary: 64 heads x 128 dims, ReLU-weighted
// sum):
//   logits[t, s] = sum_{j<64} w[t, j] * ReLU(q[t, j, :] . k[b, s, :])
//
// Per work unit (a group of NQ query rows x a tile of 128 cached keys; two
// such tiles, 256 keys, for fp8 / fp4 keys in decode):
//   D[128 keys, NQ*64 (query,head)] = K_tile[128 x 128] . Q[NQ*64 x 128]^T
// one tcgen05.mma chain per tile (M=128, N=NQ*64, K=128) with the fp32
// accumulator in TMEM, then an epilogue in which each thread owns one key of
// each tile (one TMEM lane) and reduces its NQ*64 columns to NQ scores: ReLU,
// times w, sum over heads (times the key's dequantisation scale for fp8 /
// fp4 keys).  Scores are written coalesced (32 consecutive keys per warp
// store).
//
// Warp roles (512 threads, one CTA per SM, persistent):
//   warp 0      TMA producer: key tiles (ring of STAGES), query tiles (x2)
//   warp 1      MMA issuer (one thread); allocates / frees TMEM
//   warps 4-7   fp8 / fp4 only: widen e4m3 / e2m1 key codes to f16 straight into TMEM
//               (the MMA then reads its A operand from TMEM, which keeps
//               shared-memory traffic below the HBM rate), and convert each
//               query tile from bf16 to f16 in shared memory once it lands:
//               the fp8 path multiplies in f16 (one hardware conversion per
//               two keys instead of four instructions to reach bf16).  Every
//               e4m3 value is exact in f16; a bf16 query value is exact in f16
//               when 2^-14 <= |q| <= 65504, and a smaller one is rounded to
//               f16's subnormal grid (error below 2^-25)
//   warps 8-11  epilogue for query columns [0, 128)
//   warps 12-15 epilogue for query columns [128, 256) (NQ = 4 only)
//
// Decode (NQ = 1): units are the flattened (row, key tile) space split into
// equal contiguous ranges, one per CTA -- the kernel streams the key cache
// once at HBM rate.  Single-sequence prefill (NQ = 4): CTAs take groups of 4
// query rows in a zig-zag order (causal work grows with the position) and
// every visible key tile of each group; fully invisible tiles are never
// loaded.
#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"
#include "tensor_map.h"

namespace dsa {

using namespace sm100;

namespace {

constexpr int KT = 128;      // keys per tile = MMA M
constexpr int DI = 128;      // indexer head dim = MMA K
constexpr int HI = 64;       // indexer heads
constexpr int THREADS = 512;

// Key formats: KF_BF16, KF_FP8 (e4m3 codes, one byte per dim) and KF_FP4
// (e2m1 codes, two dims per byte, low nibble first).  fp8 and fp4 keys carry
// one fp32 dequantisation scale per key row and are widened to f16 in TMEM.
enum { KF_BF16 = 0, KF_FP8 = 1, KF_FP4 = 2 };

template <int NQ, int KF>
struct Cfg {
    static constexpr bool FP8 = KF != KF_BF16;      // narrow keys: widened into TMEM, scaled in the epilogue
    static constexpr int N = NQ * HI;
    // Narrow-key decode takes 256 keys per unit (two 128-key MMA tiles behind one
    // TMA box, one widening pass, one MMA commit and one epilogue hand-off): every
    // hand-off of the unit pipeline costs about the same per unit whatever its
    // size, so a 16 KB fp8 / 8 KB fp4 unit of 128 keys left the stream at half
    // the rate the same ring reaches when nothing else runs.
    static constexpr int SUB = (FP8 && NQ == 1) ? 2 : 1;            // 128-key MMA tiles per unit
    static constexpr int KTU = SUB * KT;                             // keys per unit
    static constexpr int STAGES = KF == KF_FP4 ? (SUB == 2 ? 12 : 16) : KF == KF_FP8 ? (SUB == 2 ? 6 : 8) : (NQ == 1 ? 6 : 3);
    static constexpr int KBYTES = KF == KF_FP4 ? KTU * DI / 2 : KF == KF_FP8 ? KTU * DI : KTU * DI * 2;  // one unit
    static constexpr int QBYTES = N * DI * 2;                        // one query tile (bf16)
    static constexpr int ACC_COLS = SUB * N;
    // accumulator ring: bf16 decode has 4 (two epilogue groups take alternate
    // tiles, so the per-tile epilogue never throttles the key stream), narrow-key
    // decode 2 units of two tiles each
    static constexpr int NACC = NQ == 1 ? 4 / SUB : 2;
    static constexpr int A_COL0 = NACC * ACC_COLS;                  // fp8: f16 key tiles in TMEM
    static constexpr int A_COLS = SUB * DI / 2;                      // 128 f16 = 64 columns per tile
    // fp8: ring of widened key tiles in TMEM (as deep as the columns allow,
    // so that the widening warps can run ahead of the MMA)
    static constexpr int NA = FP8 ? (512 - NACC * ACC_COLS) / A_COLS < 4 ? (512 - NACC * ACC_COLS) / A_COLS : 4 : 2;
    static_assert(KTU <= 256, "one TMA box per unit (at most 256 rows)");
    static constexpr int TMEM_NEED = NACC * ACC_COLS + (FP8 ? NA * A_COLS : 0);
    static_assert(!FP8 || NA >= 2, "fp8 needs at least two widened key tiles in TMEM");
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int EPI_WARPS = 8;     // NQ = 1: two groups of 4 on alternate tiles; NQ = 4: two column halves
    static constexpr int NBARS = 2 * STAGES + 4 + 2 * NACC + 2 * NA + 2;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * KBYTES + 2 * (size_t)QBYTES + NBARS * 8 + 16;
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(TMEM_NEED <= 512, "TMEM budget");
    static_assert(N % 16 == 0 && N <= 256, "MMA N");
};

struct Params {
    const float* w;
    const float* k_scale;
    const int32_t* row_batch;
    const int32_t* row_pos;
    float* logits;
    int64_t ld;
    int rows, batch, ctx;
    unsigned* err;
};

struct Unit {
    int t0;        // first query row of the group
    int tile;      // key tile index
    bool first;    // first unit of a query group (load / wait the query tile)
    bool last;     // last unit of a query group (release the query tile)
};

__device__ __forceinline__ int last_visible(const Params& p, int t) {
    int pos = __ldg(p.row_pos + t);
    return pos < p.ctx - 1 ? pos : p.ctx - 1;     // may be < 0 (nothing visible)
}

// Deterministic schedule, walked identically by every warp role (units of
// KTU keys).
template <int NQ, int KTU>
struct Sched {
    // flat (NQ == 1)
    int64_t u, u_end;
    int tpr, last_t;
    // zig-zag groups (NQ == 4)
    int groups, round, g, tile, ntiles;

    __device__ void init(const Params& p) {
        if (NQ == 1) {
            tpr = (p.ctx + KTU - 1) / KTU;
            const int64_t total = (int64_t)p.rows * tpr;
            u = total * blockIdx.x / gridDim.x;
            u_end = total * (blockIdx.x + 1) / gridDim.x;
            last_t = -1;
        } else {
            groups = (p.rows + NQ - 1) / NQ;
            round = -1;
            g = -1;
            tile = ntiles = 0;
        }
    }

    __device__ bool next(const Params& p, Unit& out) {
        if (NQ == 1) {
            while (u < u_end) {
                const int t = (int)(u / tpr), j = (int)(u - (int64_t)t * tpr);
                const int nt = last_visible(p, t) / KTU + 1;         // 0 if nothing visible
                if (last_visible(p, t) < 0 || j >= nt) {             // rest of this row is invisible
                    u = (int64_t)(t + 1) * tpr;
                    continue;
                }
                out.t0 = t;
                out.tile = j;
                out.first = t != last_t;
                last_t = t;
                out.last = (j + 1 >= nt) || (u + 1 >= u_end);
                ++u;
                return true;
            }
            return false;
        } else {
            while (true) {
                if (tile < ntiles) {
                    out.t0 = g * NQ;
                    out.tile = tile;
                    out.first = tile == 0;
                    out.last = tile + 1 == ntiles;
                    ++tile;
                    return true;
                }
                ++round;
                if ((int64_t)round * gridDim.x >= groups) return false;
                g = (round & 1) ? (round + 1) * (int)gridDim.x - 1 - (int)blockIdx.x
                                : round * (int)gridDim.x + (int)blockIdx.x;
                if (g >= groups) { ntiles = 0; tile = 0; continue; }
                int mp = -1;
                for (int r = 0; r < NQ; ++r)
                    if (g * NQ + r < p.rows) mp = max(mp, last_visible(p, g * NQ + r));
                ntiles = mp < 0 ? 0 : mp / KTU + 1;
                tile = 0;
            }
        }
    }
};

// e4m3 pair (low byte = first element) -> f16 pair, exact for every finite
// code (an e4m3 value has at most 4 significant bits and lies within f16's
// range).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
    return h2;
}

// e2m1 pair (low nibble = first element) -> f16 pair, exact (an e2m1 value
// has at most 2 significant bits and lies within f16's range).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "r"(byte));
    return h2;
}

// bf16 pair -> f16 pair (round to nearest even; exact for 2^-14 <= |x| <= 65504).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(__uint_as_float(v & 0xFFFF0000u)), "f"(__uint_as_float(v << 16)));
    return r;
}

// Instruction descriptor, kind::f16 with f16 A and B, f32 accumulator.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace

template <int NQ, int KF>
__global__ void __launch_bounds__(THREADS, 1) indexer_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                                                                const __grid_constant__ CUtensorMap tmap_q,
                                                                const Params p) {
    using C = Cfg<NQ, KF>;
    constexpr bool FP8 = C::FP8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* kbuf = smem;                                            // [STAGES][KBYTES]
    uint8_t* qbuf = kbuf + (size_t)C::STAGES * C::KBYTES;            // [2][QBYTES]
    uint64_t* bars = (uint64_t*)(qbuf + 2 * (size_t)C::QBYTES);
    uint64_t* kfull = bars;                       // [STAGES]
    uint64_t* kempty = kfull + C::STAGES;         // [STAGES]
    uint64_t* qfull = kempty + C::STAGES;         // [2]
    uint64_t* qempty = qfull + 2;                 // [2]
    uint64_t* accfull = qempty + 2;               // [NACC]
    uint64_t* accempty = accfull + C::NACC;       // [NACC]
    uint64_t* afull = accempty + C::NACC;         // [NA] (fp8)
    uint64_t* aempty = afull + C::NA;             // [NA] (fp8)
    uint64_t* qconv = aempty + C::NA;             // [2]  (fp8) the query tile is in f16
    uint32_t* tmem_slot = (uint32_t*)(qconv + 2);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], FP8 ? 4 : 1);       // fp8: the 4 converter warps free the stage
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], 1);
            mbar_init(&qconv[i], 4);
        }
        for (int i = 0; i < C::NA; ++i) {
            mbar_init(&afull[i], 4);
            mbar_init(&aempty[i], 1);
        }
        for (int i = 0; i < C::NACC; ++i) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], NQ == 1 ? 4 : C::EPI_WARPS);   // the warps that read accumulator i
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();                     // inputs written by earlier kernels are visible from here on
    pdl_launch_dependents();

    Sched<NQ, C::KTU> sch;
    Unit un;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ----
        if (elect_one()) {
            sch.init(p);
            const uint64_t pol_stream = l2_policy_evict_first();
            int i = 0, qe = -1;
            while (sch.next(p, un)) {
                if (un.first) {
                    ++qe;
                    const int qb = qe & 1;
                    if (!mbar_wait(&qempty[qb], ((qe >> 1) & 1) ^ 1, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag)) break;
                    mbar_arrive_expect_tx(&qfull[qb], C::QBYTES);
                    uint8_t* qdst = qbuf + (size_t)qb * C::QBYTES;
                    tma_load_2d(qdst, &tmap_q, 0, un.t0 * HI, &qfull[qb]);
                    tma_load_2d(qdst + C::N * 128, &tmap_q, 64, un.t0 * HI, &qfull[qb]);
                }
                const int st = i % C::STAGES;
                if (!mbar_wait(&kempty[st], ((i / C::STAGES) & 1) ^ 1, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag)) break;
                mbar_arrive_expect_tx(&kfull[st], C::KBYTES);
                const int b = __ldg(p.row_batch + un.t0);
                const int row = b * p.ctx + un.tile * C::KTU;
                uint8_t* kdst = kbuf + (size_t)st * C::KBYTES;
                if (NQ == 1) {       // decode: every key is read once -> stream it past L2
                    tma_load_2d_hint(kdst, &tmap_k, 0, row, &kfull[st], pol_stream);
                    if (!FP8) tma_load_2d_hint(kdst + KT * 128, &tmap_k, 64, row, &kfull[st], pol_stream);
                } else {             // prefill: every key tile is re-read by later query groups
                    tma_load_2d(kdst, &tmap_k, 0, row, &kfull[st]);
                    if (!FP8) tma_load_2d(kdst + KT * 128, &tmap_k, 64, row, &kfull[st]);
                }
                ++i;
            }
            if (*abort_flag) {
                // let the copies already issued land before the CTA exits
                for (int j = (i > C::STAGES ? i - C::STAGES : 0); j < i; ++j)
                    mbar_wait(&kfull[j % C::STAGES], (j / C::STAGES) & 1, p.err, DEV_ERR_TIMEOUT_TMA, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        if (elect_one()) {
            sch.init(p);
            constexpr uint32_t idesc = FP8 ? idesc_f16_f32(KT, C::N) : idesc_bf16_f32(KT, C::N, 0, 0);
            const uint32_t kbase = smem_u32(kbuf), qbase = smem_u32(qbuf);
            int i = 0, qe = -1;
            bool ok = true;
            while (ok && sch.next(p, un)) {
                if (un.first) {
                    ++qe;
                    ok = FP8 ? mbar_wait(&qconv[qe & 1], (qe >> 1) & 1, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag)
                             : mbar_wait(&qfull[qe & 1], (qe >> 1) & 1, p.err, DEV_ERR_TIMEOUT_TMA, abort_flag);
                    if (!ok) break;
                }
                const int st = i % C::STAGES, acc = i % C::NACC, ab = i % C::NA;
                if (FP8) {
                    ok = mbar_wait(&afull[ab], (i / C::NA) & 1, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag);
                } else {
                    ok = mbar_wait(&kfull[st], (i / C::STAGES) & 1, p.err, DEV_ERR_TIMEOUT_TMA, abort_flag);
                }
                if (!ok) break;
                ok = mbar_wait(&accempty[acc], ((i / C::NACC) & 1) ^ 1, p.err, DEV_ERR_TIMEOUT_PEER, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * C::ACC_COLS;
                const uint32_t qaddr = qbase + (uint32_t)((qe & 1) * C::QBYTES);
#pragma unroll
                for (int kk = 0; kk < DI / 16; ++kk) {
                    const uint32_t koff = (uint32_t)((kk >> 2) * (C::N * 128) + (kk & 3) * 32);
                    const uint64_t bdesc = desc_sw128(qaddr + koff, 1024);
                    if (FP8) {
#pragma unroll
                        for (int sb = 0; sb < C::SUB; ++sb)          // the unit's 128-key tiles
                            mma_ts(d + sb * C::N, tmem + C::A_COL0 + ab * C::A_COLS + sb * (DI / 2) + kk * 8, bdesc,
                                   idesc, kk > 0);
                    } else {
                        const uint32_t aoff = (uint32_t)(st * C::KBYTES + (kk >> 2) * (KT * 128) + (kk & 3) * 32);
                        mma_ss(d, desc_sw128(kbase + aoff, 1024), bdesc, idesc, kk > 0);
                    }
                }
                if (FP8) mma_commit(&aempty[ab]);
                else mma_commit(&kempty[st]);
                mma_commit(&accfull[acc]);
                if (un.last) mma_commit(&qempty[qe & 1]);
                ++i;
            }
        }
    } else if (FP8 && warp >= 4 && warp < 8) {
        // ------------------------- fp8 -> f16 key widening into TMEM ----
        const int quarter = warp & 3;
        const int r0 = quarter * 32 + lane;                 // key row of a 128-key tile = TMEM lane
        sch.init(p);
        int i = 0, qe = -1;
        while (sch.next(p, un)) {
            if (un.first) {
                // the new query tile: bf16 -> f16 in place (8 x 16 bytes per thread)
                ++qe;
                if (!mbar_wait(&qfull[qe & 1], (qe >> 1) & 1, p.err, DEV_ERR_TIMEOUT_TMA, abort_flag)) break;
                uint4* qv = (uint4*)(qbuf + (size_t)(qe & 1) * C::QBYTES);
#pragma unroll 4
                for (int c = threadIdx.x - 128; c < C::QBYTES / 16; c += 128) {
                    uint4 x = qv[c];
                    x.x = bf16x2_to_f16x2(x.x);
                    x.y = bf16x2_to_f16x2(x.y);
                    x.z = bf16x2_to_f16x2(x.z);
                    x.w = bf16x2_to_f16x2(x.w);
                    qv[c] = x;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&qconv[qe & 1]);
            }
            const int st = i % C::STAGES, ab = i % C::NA;
            if (!mbar_wait(&kfull[st], (i / C::STAGES) & 1, p.err, DEV_ERR_TIMEOUT_TMA, abort_flag)) break;
            if (!mbar_wait(&aempty[ab], ((i / C::NA) & 1) ^ 1, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag)) break;
            tc_fence_after();
#pragma unroll 1
            for (int sb = 0; sb < C::SUB; ++sb) {
            // tile sb of the unit: smem rows sb*128 + r, TMEM columns [64 sb, +64) of the slot
            const int r = sb * KT + r0;
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + C::A_COL0 + ab * C::A_COLS + sb * (DI / 2);
            if (KF == KF_FP4) {
                // a 64-byte row of e2m1 pairs (64-byte swizzle: chunk c of row r
                // sits at chunk c ^ ((r >> 1) & 3)); 16 bytes -> 32 dims -> 16 columns
                const uint8_t* src = kbuf + (size_t)st * C::KBYTES + r * 64;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 x = *(const uint4*)(src + ((c ^ ((r >> 1) & 3)) << 4));
                    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
                    uint32_t words[16];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) words[4 * e + bb] = e2m1x2_to_f16x2((xs[e] >> (8 * bb)) & 0xFFu);
                    tmem_st16(taddr + c * 16, words);
                }
            } else {
            const uint8_t* src = kbuf + (size_t)st * C::KBYTES + r * 128;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t words[32];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int c = half * 4 + c4;                         // 16-byte chunk of the row
                    const uint4 x = *(const uint4*)(src + ((c ^ (r & 7)) << 4));
                    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        words[c4 * 8 + 2 * e] = e4m3x2_to_f16x2((uint16_t)(xs[e] & 0xFFFFu));
                        words[c4 * 8 + 2 * e + 1] = e4m3x2_to_f16x2((uint16_t)(xs[e] >> 16));
                    }
                }
                uint32_t lo[16], hi[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) { lo[m] = words[m]; hi[m] = words[16 + m]; }
                tmem_st16(taddr + half * 32, lo);
                tmem_st16(taddr + half * 32 + 16, hi);
            }
            }
            }
            tmem_st_wait();
            __syncwarp();
            tc_fence_before();
            if (lane == 0) {
                mbar_arrive(&kempty[st]);
                mbar_arrive(&afull[ab]);
            }
            ++i;
        }
    } else if (warp >= 8 && warp < 8 + C::EPI_WARPS) {
        // --------------------------------------------------- epilogue ----
        // NQ = 1: warp group eg = (warp - 8) / 4 takes the units i with
        // i % 2 == eg; NQ = 4: group eg takes query columns [128 eg, +128).
        const int quarter = warp & 3;
        const int eg = (warp - 8) >> 2;
        sch.init(p);
        int i = 0;
        while (sch.next(p, un)) {
            if (NQ == 1 && (i & 1) != eg) { ++i; continue; }
            const int acc = i % C::NACC;
            // the keys' row and (fp8 / fp4) dequantisation scales are loaded
            // before the wait for the accumulator, so their latency is hidden;
            // thread (quarter, lane) owns key quarter*32 + lane of each 128-key tile
            const int b = __ldg(p.row_batch + un.t0);
            const bool b_ok = b >= 0 && b < p.batch;
            const int key0 = un.tile * C::KTU + quarter * 32 + lane;     // key of tile sb: key0 + 128 sb
            float ks[C::SUB];
#pragma unroll
            for (int sb = 0; sb < C::SUB; ++sb) {
                ks[sb] = 1.f;
                if (FP8 && b_ok && key0 + sb * KT < p.ctx) ks[sb] = __ldg(p.k_scale + (int64_t)b * p.ctx + key0 + sb * KT);
            }
            if (!mbar_wait(&accfull[acc], (i / C::NACC) & 1, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag)) break;
            tc_fence_after();
            const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + acc * C::ACC_COLS;
            constexpr int QPW = NQ == 1 ? 1 : 2;           // query rows per epilogue warp
            static_assert(C::SUB == 1 || QPW == 1, "two-tile units only with one query row per warp");
            float score[QPW], score1 = 0.f;                 // score1: the unit's second tile
#pragma unroll 1
            for (int sb = 0; sb < C::SUB; ++sb) {           // one tile at a time (register budget)
#pragma unroll
            for (int qq = 0; qq < QPW; ++qq) {
                const int qi = NQ == 1 ? 0 : eg * 2 + qq;  // query within the group
                const int t = min(un.t0 + qi, p.rows - 1);
                const float4* wr = (const float4*)(p.w + (int64_t)t * HI);
                // four independent partial sums (the weights are read as float4)
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
                if (C::SUB == 1) {
                    float v0[32], v1[32];
                    tmem_ld32(tbase + qi * HI, v0);
                    tmem_ld32(tbase + qi * HI + 32, v1);
                    tmem_ld_wait();
#pragma unroll
                    for (int h4 = 0; h4 < 8; ++h4) {
                        const float4 wa = __ldg(wr + h4), wb = __ldg(wr + 8 + h4);
                        s4[0] = fmaf(wa.x, fmaxf(v0[4 * h4], 0.f), s4[0]);
                        s4[1] = fmaf(wa.y, fmaxf(v0[4 * h4 + 1], 0.f), s4[1]);
                        s4[2] = fmaf(wa.z, fmaxf(v0[4 * h4 + 2], 0.f), s4[2]);
                        s4[3] = fmaf(wa.w, fmaxf(v0[4 * h4 + 3], 0.f), s4[3]);
                        s4[0] = fmaf(wb.x, fmaxf(v1[4 * h4], 0.f), s4[0]);
                        s4[1] = fmaf(wb.y, fmaxf(v1[4 * h4 + 1], 0.f), s4[1]);
                        s4[2] = fmaf(wb.z, fmaxf(v1[4 * h4 + 2], 0.f), s4[2]);
                        s4[3] = fmaf(wb.w, fmaxf(v1[4 * h4 + 3], 0.f), s4[3]);
                    }
                } else {
                    // two-tile units: the 64 head columns in two loads of 32
                    // (register budget), the same four partial sums
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        float v[32];
                        tmem_ld32(tbase + sb * C::N + qi * HI + hf * 32, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int h4 = 0; h4 < 8; ++h4) {
                            const float4 wa = __ldg(wr + hf * 8 + h4);
                            s4[0] = fmaf(wa.x, fmaxf(v[4 * h4], 0.f), s4[0]);
                            s4[1] = fmaf(wa.y, fmaxf(v[4 * h4 + 1], 0.f), s4[1]);
                            s4[2] = fmaf(wa.z, fmaxf(v[4 * h4 + 2], 0.f), s4[2]);
                            s4[3] = fmaf(wa.w, fmaxf(v[4 * h4 + 3], 0.f), s4[3]);
                        }
                    }
                }
                const float sc = (s4[0] + s4[1]) + (s4[2] + s4[3]);
                if (sb == 0) score[qq] = sc;
                else score1 = sc;
            }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            if (!b_ok && lane == 0) record_error(p.err, DEV_ERR_BAD_INDEX);
#pragma unroll
            for (int sb = 0; sb < C::SUB; ++sb) {
#pragma unroll
            for (int qq = 0; qq < QPW; ++qq) {
                const int t = un.t0 + (NQ == 1 ? 0 : eg * 2 + qq);
                const float sc = sb == 0 ? score[qq] : score1;
                const int key = key0 + sb * KT;
                if (b_ok && t < p.rows && key <= last_visible(p, t))
                    p.logits[(int64_t)t * p.ld + key] = FP8 ? sc * ks[sb] : sc;
            }
            }
            ++i;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host --

namespace {

template <int NQ, int KF>
cudaError_t launch_cfg(const Launch& L, const void* q, const void* k, const Params& p) {
    using C = Cfg<NQ, KF>;
    CUtensorMap mk, mq;
    const uint64_t krows = (uint64_t)p.batch * p.ctx;
    bool ok = KF == KF_FP4 ? make_map_swizzled(&mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k, DI / 2, krows, 64, C::KTU,
                                               CU_TENSOR_MAP_SWIZZLE_64B)
            : KF == KF_FP8 ? make_map_sw128(&mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k, DI, krows, 128, C::KTU)
                  : make_map_sw128(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, DI, krows, 64, KT);
    ok = ok && make_map_sw128(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, DI, (uint64_t)p.rows * HI, 64, NQ * HI);
    if (!ok) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<NQ, KF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::SMEM);
    if (e != cudaSuccess) return e;
    int64_t units;
    if (NQ == 1) units = (int64_t)p.rows * ((p.ctx + C::KTU - 1) / C::KTU);
    else units = (p.rows + NQ - 1) / NQ;
    const int grid = (int)(units < L.num_sms ? units : L.num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, indexer_tc_kernel<NQ, KF>, mk, mq, p);
    count_launch();
    return e;
}

}  // namespace

bool indexer_tc_supported(dsa_dtype_t q_dtype, dsa_dtype_t k_dtype, int n_heads, int head_dim) {
    return q_dtype == DSA_BF16 && (k_dtype == DSA_BF16 || k_dtype == DSA_FP8_E4M3 || k_dtype == DSA_FP4_E2M1) &&
           n_heads == HI &&
           head_dim == DI;
}

cudaError_t launch_indexer_tc(const Launch& L, const void* q, dsa_dtype_t k_dtype, const float* w, const void* k,
                              const float* k_scale, const int32_t* row_batch, const int32_t* row_pos, int rows,
                              int batch, int ctx_len, float* logits, int64_t ld) {
    if (rows == 0 || ctx_len == 0) return cudaSuccess;
    Params p{w, k_scale, row_batch, row_pos, logits, ld, rows, batch, ctx_len, L.err};
    if (k_dtype == DSA_FP8_E4M3) return launch_cfg<1, KF_FP8>(L, q, k, p);
    if (k_dtype == DSA_FP4_E2M1) return launch_cfg<1, KF_FP4>(L, q, k, p);
    // Groups of 4 query rows share a key tile only when every row reads the
    // same cache (one sequence): then the MMA N grows to 256 and each key
    // tile is reused for 4 queries.
    if (batch == 1 && rows >= 4 * L.num_sms) return launch_cfg<4, KF_BF16>(L, q, k, p);
    return launch_cfg<1, KF_BF16>(L, q, k, p);
}

}  // namespace dsa
