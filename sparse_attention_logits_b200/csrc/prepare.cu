// Preparation of the lightning indexer's inputs and the write of new keys
// into its key cache ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", section 3,
// Step 1: the query latent is RMS-normalised and projected up, split into a
// part with and a part without rotary position encoding, the former turned by
// apply_rotary_emb, and weights_proj gives the per-head weights; section 1.3:
// a separate learned linear map takes queries and keys to 128 dims):
//
//   q_I[t, j, :] = RoPE( W_qb[j] . RMSNorm(c_q[t]) )        [T, H, 128] bf16
//   w[t, :]      = W_w . h[t]                               [T, H]      fp32
//   k_I[t, :]    = RoPE( W_k . h[t] )  -> key cache row slot[t] (bf16, or
//                  fp8 e4m3 / fp4 e2m1 codes with one fp32 scale per row)
//
// prepare_norm_kernel -- one warp per token: the token's sum of squares of
// c_q (fp32) gives 1/RMS, and c_q * gain is rounded once to bf16 into the
// workspace; every query tile then reads that operand as it is, instead of
// each of them scaling the same latent again.
//
// indexer_prepare_kernel -- all three projections in one launch on the
// tcgen05 tensor cores, launched right after the norm kernel (programmatic
// dependent launch).  Every CTA computes one tile of 128 tokens x 64
// features (up to 256 when there are many tokens)
// D = A . B^T (M = 128 tokens, N = 64 or 256 features, K streamed 64 at a time
// through a 4-stage TMA ring of one or two 64-wide chunks per stage, fp32
// accumulator in TMEM):
//   query tiles  A = the scaled latent, B = rows of W_qb.  The weight boxes of
//                the first ring's worth of stages are requested before the
//                norm kernel has finished (they do not depend on it); the
//                epilogue multiplies by 1/RMS, turns the rotary pairs (the
//                tile's cosine / sine rows are staged in shared memory while
//                the main loop runs) and stores bf16 q_I.
//   key/weight tiles  A = h, B = as many 64-row blocks of [W_k ; W_w] as a
//                query tile is wide (up to 256 rows, so that with many
//                tokens h crosses into the SMs once per token tile), with K
//                split over S CTAs when the token count is small (so that the long
//                d_model reduction is spread over as many SMs as the query
//                tiles use).  Each writes its fp32 partial tile to the
//                workspace.
// Warp roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer (and
// TMEM owner), warps 4-7 epilogue (warp 4+q owns TMEM lanes 32q .. 32q+31 =
// tokens of the tile).
//
// prepare_finish_kernel -- launched right after (programmatic dependent
// launch), one warp per token: its slot, position and rotary factors are
// read before the projections finish; then it adds the S partials in split
// order (the result does not depend on scheduling), writes the head
// weights, turns the key's rotary pairs and writes the key row in the
// cache's format.
//
// key_append_kernel -- the key-cache write alone for keys that are already
// projected (for instance compressed CSA keys): one warp per key row, lane l
// holding dims 4l .. 4l+3.
//
// The cache write is decided in binary32 with every operation rounded on
// its own (no fused multiply-add): rotary pairs (a c - b s, a s + b c), scale
// = amax / 448 (fp8) or amax / 6 (fp4), 1 for an all-zero row, code = the
// nearest code of x / scale (ties to even, saturating), by the hardware
// conversion instructions.
#include "common.cuh"
#include "launchers.h"
#include "sm100.cuh"
#include "tensor_map.h"

namespace dsa {

using namespace sm100;

namespace {

constexpr int PT = 128;                         // tokens per tile (MMA M)
constexpr int PN = 64;                          // features per key / weight tile, and per query tile for few tokens
constexpr int PK = 64;                          // reduction elements per stage (one 128-byte row)
constexpr int A_BYTES = PT * PK * 2;            // 16 KB (stage room; a 64-token box fills half)
constexpr int PTHREADS = 256;
constexpr int KDIM = 128;                       // indexer head dim (key row length)
// Shared-memory layout for a ring of STG stages of NSUB reduction chunks
// each (A boxes then B boxes): stages, barriers / TMEM address / flags, then
// (query tiles with rotary columns, when it fits) the tile's cosine and sine
// rows, [d_rope / 2][128 tokens] each.  Three variants: few tokens (the grid
// fits on the SMs at one CTA each): query tiles 64 wide, two chunks per
// stage (256 contiguous bytes of every weight row per stage, half the
// hand-offs); many tokens: query tiles 256 wide, one chunk per stage (each
// latent tile feeds four times the features: half the bytes an SM takes in
// per multiply-add); in between: 64-wide tiles, one chunk per stage, two
// CTAs per SM (no staged rotary rows).
template <int STG, int NSUB, int QN>
struct Ring {
    static constexpr int B_ROOM = QN * PK * 2;                                 // one B box (query tiles are QN wide)
    static constexpr size_t SLOT = (size_t)NSUB * (A_BYTES + B_ROOM);          // one stage: NSUB A boxes, NSUB B boxes
    static constexpr size_t BAR_OFF = (size_t)STG * SLOT;
    static constexpr size_t TAB_OFF = (BAR_OFF + (2 * STG + 1) * 8 + 16 + 15) & ~(size_t)15;
    static constexpr size_t SMEM_BASE = 1024 + TAB_OFF;
    static_assert(TAB_OFF % 16 == 0, "table alignment");
};
constexpr size_t SMEM_LIMIT = 227 * 1024;
constexpr int MAX_DC = 16384;

struct KeyOut {
    void* cache;          // [cache_rows, 128] bf16 / [cache_rows, 128] e4m3 / [cache_rows, 64] e2m1 pairs
    float* scale;         // [cache_rows] (fp8 / fp4)
    const float* cos;     // [max_pos, d_rope / 2]
    const float* sin;
    int64_t cache_rows;
    int d_rope, max_pos, fmt;   // fmt: DSA_BF16, DSA_FP8_E4M3 or DSA_FP4_E2M1
};

struct NormParams {
    const __nv_bfloat16* c_q;   // [T, d_c]
    const float* gamma;         // [d_c]
    __nv_bfloat16* cqn;         // [T, d_c] c_q * gain, rounded once
    float* inv_rms;             // [T]
    float eps;
    int T, d_c;
};

struct PrepParams {
    const int32_t* pos;   // [T]
    const int64_t* slot;  // [T]
    __nv_bfloat16* q_out; // [T, H, 128]
    float* w_out;         // [T, H]
    float* ws;            // [S][n_tt * 128][kwc] partial sums of the key / weight tiles
    const float* inv_rms; // [T] (norm kernel)
    KeyOut ko;
    int T, n_heads;
    int n_tt, n_qf, n_kwf, n_kwt, S, kc_q, kc_kw, kwc;   // n_kwf 64-row blocks of [W_k ; W_w] in n_kwt tiles
    int a_bytes;          // bytes of one A box (64 or 128 token rows)
    int tab;              // query tiles stage their rotary rows in shared memory
    unsigned* err;
};

struct Job {
    bool q;          // query tile (else key / weight tile)
    int tt, f, s;    // token tile, feature tile, split
    int c0, c1;      // reduction chunks [c0, c1)
};

// Key / weight tiles come first in the grid: they are the longer ones.
__device__ __forceinline__ Job job_of(const PrepParams& p, int b) {
    Job j;
    const int kw = p.n_tt * p.n_kwt * p.S;
    if (b < kw) {
        j.q = false;
        j.tt = b / (p.n_kwt * p.S);
        const int r = b - j.tt * p.n_kwt * p.S;
        j.f = r / p.S;
        j.s = r - j.f * p.S;
        j.c0 = (int)((int64_t)p.kc_kw * j.s / p.S);
        j.c1 = (int)((int64_t)p.kc_kw * (j.s + 1) / p.S);
    } else {
        b -= kw;
        j.q = true;
        j.tt = b / p.n_qf;
        j.f = b - j.tt * p.n_qf;
        j.s = 0;
        j.c0 = 0;
        j.c1 = p.kc_q;
    }
    return j;
}

__device__ __forceinline__ void rope_pair(float& a, float& b, float c, float s) {
    const float ac = __fmul_rn(a, c), bs = __fmul_rn(b, s), as = __fmul_rn(a, s), bc = __fmul_rn(b, c);
    a = __fsub_rn(ac, bs);
    b = __fadd_rn(as, bc);
}

// Two binary32 values -> e4m3 pair, `lo` in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two binary32 values -> e2m1 pair, `lo` in the low nibble.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// One warp writes one key row: lane l holds dims 4l .. 4l+3 (binary32),
// already turned by the rotary pairs; stored at row `row` of the cache in
// its format.
__device__ __forceinline__ void write_key_row(float (&x)[4], int lane, int64_t row, const KeyOut& o) {
    if (o.fmt == DSA_BF16) {
        __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
        uint2 u;
        u.x = *(uint32_t*)&a;
        u.y = *(uint32_t*)&b;
        ((uint2*)o.cache)[row * (KDIM / 4) + lane] = u;
        return;
    }
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const bool fp8 = o.fmt == DSA_FP8_E4M3;
    const float sc = amax > 0.f ? __fdiv_rn(amax, fp8 ? 448.f : 6.f) : 1.f;
    float y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = __fdiv_rn(x[e], sc);
    if (fp8) {
        const uint32_t w = f32x2_to_e4m3x2(y[0], y[1]) | (f32x2_to_e4m3x2(y[2], y[3]) << 16);
        ((uint32_t*)o.cache)[row * (KDIM / 4) + lane] = w;
    } else {
        const uint32_t w = f32x2_to_e2m1x2(y[0], y[1]) | (f32x2_to_e2m1x2(y[2], y[3]) << 8);
        ((uint16_t*)o.cache)[row * (KDIM / 4) + lane] = (uint16_t)w;
    }
    if (lane == 0) o.scale[row] = sc;
}

// The rotary pairs of dims below d_rope of lane l's dims 4l .. 4l+3 turned at
// position `ps`, then the row written.
__device__ __forceinline__ void store_key_row(float (&x)[4], int lane, int ps, int64_t row, const KeyOut& o) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int d0 = 4 * lane + 2 * e;
        if (d0 < o.d_rope) {
            const int64_t ti = (int64_t)ps * (o.d_rope >> 1) + (d0 >> 1);
            rope_pair(x[2 * e], x[2 * e + 1], __ldg(o.cos + ti), __ldg(o.sin + ti));
        }
    }
    write_key_row(x, lane, row, o);
}

}  // namespace

// One warp per token: 1/RMS of the latent and the latent times the gain,
// rounded once to bf16 (the projection kernel's A operand of query tiles).
__global__ void __launch_bounds__(256) prepare_norm_kernel(const NormParams n) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= n.T) return;
    const uint4* src = (const uint4*)(n.c_q + (int64_t)t * n.d_c);
    uint4* dst = (uint4*)(n.cqn + (int64_t)t * n.d_c);
    const float4* g4 = (const float4*)n.gamma;
    const int nv = n.d_c / 8;
    float ss0 = 0.f, ss1 = 0.f;
    for (int base = lane; base < nv; base += 32 * 8) {
        // eight 16-byte pieces of the row (and their gains) requested together
        uint4 xv[8];
        float4 ga[8], gb[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = base + 32 * k;
            if (i < nv) {
                xv[k] = __ldg(src + i);
                ga[k] = __ldg(g4 + 2 * i);
                gb[k] = __ldg(g4 + 2 * i + 1);
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = base + 32 * k;
            if (i >= nv) break;
            const float g[8] = {ga[k].x, ga[k].y, ga[k].z, ga[k].w, gb[k].x, gb[k].y, gb[k].z, gb[k].w};
            uint32_t xs[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(xs[e] << 16), hi = __uint_as_float(xs[e] & 0xFFFF0000u);
                ss0 = fmaf(lo, lo, ss0);
                ss1 = fmaf(hi, hi, ss1);
                const __nv_bfloat162 v = __floats2bfloat162_rn(lo * g[2 * e], hi * g[2 * e + 1]);
                xs[e] = *(const uint32_t*)&v;
            }
            dst[i] = make_uint4(xs[0], xs[1], xs[2], xs[3]);
        }
    }
    float ss = ss0 + ss1;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    if (lane == 0) n.inv_rms[t] = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)n.d_c), n.eps)));
}

template <int STG, int NSUB, int QN>
__global__ void __launch_bounds__(PTHREADS, 2) indexer_prepare_kernel(const __grid_constant__ CUtensorMap tm_cq,
                                                                      const __grid_constant__ CUtensorMap tm_h,
                                                                      const __grid_constant__ CUtensorMap tm_wqb,
                                                                      const __grid_constant__ CUtensorMap tm_wk,
                                                                      const __grid_constant__ CUtensorMap tm_ww,
                                                                      const PrepParams p) {
    using R = Ring<STG, NSUB, QN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = (uint64_t*)(smem + R::BAR_OFF);                      // [STG] stage landed
    uint64_t* empty = full + STG;                                          // [STG] stage consumed by the MMA
    uint64_t* accfull = empty + STG;                                       // accumulator complete
    uint32_t* tmem_slot = (uint32_t*)(accfull + 1);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
    float* tab = (float*)(smem + R::TAB_OFF);                              // [2][d_rope / 2][PT]: cos, then sin

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Job jb = job_of(p, blockIdx.x);
    const int nch = jb.c1 - jb.c0;                  // reduction chunks of 64
    const int nst = (nch + NSUB - 1) / NSUB;        // stages (the last may hold fewer chunks)
    // key / weight tiles: 64-row blocks [blk0, blk0 + nblk) of [W_k ; W_w] (QN / 64 at most)
    const int blk0 = jb.q ? 0 : jb.f * (QN / PN);
    const int nblk = jb.q ? 0 : min(QN / PN, p.n_kwf - blk0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < STG; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(accfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, QN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Only the query tiles' latent operand and 1/RMS come from the norm
    // kernel; the weights, h, positions and rotary tables
    // are inputs that the kernels before it had finished writing when it
    // started (it waits for them before letting this grid start), so they
    // are read before pdl_wait().
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ----
        if (elect_one()) {
            const CUtensorMap* am = jb.q ? &tm_cq : &tm_h;
            const uint32_t b_bytes = (uint32_t)(jb.q ? QN : nblk * PN) * PK * 2;
            tma_prefetch_desc(am);
            if (jb.q) {
                tma_prefetch_desc(&tm_wqb);
            } else {
                tma_prefetch_desc(&tm_wk);
                tma_prefetch_desc(&tm_ww);
            }
            // B of one chunk: QN rows of W_qb, or the tile's 64-row blocks of [W_k ; W_w]
            auto load_b = [&](uint8_t* dst, int kx, uint64_t* bar) {
                if (jb.q) {
                    tma_load_2d(dst, &tm_wqb, kx, jb.f * QN, bar);
                } else {
                    for (int bb = 0; bb < nblk; ++bb) {
                        const int blk = blk0 + bb;
                        tma_load_2d(dst + bb * PN * 128, blk < 2 ? &tm_wk : &tm_ww, kx, (blk < 2 ? blk : blk - 2) * PN,
                                    bar);
                    }
                }
            };
            // query tiles: the weight boxes of the first ring's worth of
            // stages before waiting for the norm kernel, then their latent boxes
            const int npre = jb.q ? min(STG, nst) : 0;
            for (int i = 0; i < npre; ++i) {
                const int ns = min(NSUB, nch - i * NSUB);
                mbar_arrive_expect_tx(&full[i], (uint32_t)ns * ((uint32_t)p.a_bytes + b_bytes));
                for (int j = 0; j < ns; ++j)
                    load_b(smem + i * R::SLOT + NSUB * A_BYTES + j * R::B_ROOM, (jb.c0 + i * NSUB + j) * PK, &full[i]);
            }
            if (jb.q) pdl_wait();
            for (int i = 0; i < npre; ++i) {
                const int ns = min(NSUB, nch - i * NSUB);
                for (int j = 0; j < ns; ++j)
                    tma_load_2d(smem + i * R::SLOT + j * A_BYTES, am, (jb.c0 + i * NSUB + j) * PK, jb.tt * PT,
                                &full[i]);
            }
            int i = npre;
            for (; i < nst; ++i) {
                const int st = i % STG;
                if (!mbar_wait(&empty[st], ((i / STG) & 1) ^ 1, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag)) break;
                const int ns = min(NSUB, nch - i * NSUB);
                mbar_arrive_expect_tx(&full[st], (uint32_t)ns * ((uint32_t)p.a_bytes + b_bytes));
                uint8_t* dst = smem + st * R::SLOT;
                for (int j = 0; j < ns; ++j) {
                    const int kx = (jb.c0 + i * NSUB + j) * PK;
                    tma_load_2d(dst + j * A_BYTES, am, kx, jb.tt * PT, &full[st]);
                    load_b(dst + NSUB * A_BYTES + j * R::B_ROOM, kx, &full[st]);
                }
            }
            if (*abort_flag) {
                for (int j = (i > STG ? i - STG : 0); j < i; ++j)
                    mbar_wait(&full[j % STG], (j / STG) & 1, p.err, DEV_ERR_TIMEOUT_TMA, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        if (elect_one()) {
            const uint32_t idesc = idesc_bf16_f32(PT, jb.q ? QN : nblk * PN, 0, 0);
            const uint32_t base = smem_u32(smem);
            bool ok = true;
            for (int i = 0; i < nst; ++i) {
                const int st = i % STG;
                ok = mbar_wait(&full[st], (i / STG) & 1, p.err, DEV_ERR_TIMEOUT_TMA, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const int ns = min(NSUB, nch - i * NSUB);
                for (int j = 0; j < ns; ++j) {
                    const uint32_t a = base + (uint32_t)(st * R::SLOT + j * A_BYTES);
                    const uint32_t b = base + (uint32_t)(st * R::SLOT + NSUB * A_BYTES + j * R::B_ROOM);
#pragma unroll
                    for (int kk = 0; kk < PK / 16; ++kk)
                        mma_ss(tmem, desc_sw128(a + kk * 32, 1024), desc_sw128(b + kk * 32, 1024), idesc,
                               (i > 0 || j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&empty[st]);
            }
            if (ok) mma_commit(accfull);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------ epilogue ----
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;                  // token of the tile = TMEM lane
        const int t = jb.tt * PT + r;
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
        if (jb.q) {
            const int col0 = jb.f * QN, o = col0 % KDIM;    // first feature, its dim in the head
            const bool rot = o < p.ko.d_rope;
            const int half = p.ko.d_rope >> 1;
            const int ps = t < p.T ? __ldg(p.pos + t) : 0;
            const bool pos_ok = !rot || (ps >= 0 && ps < p.ko.max_pos);
            if (rot && p.tab && t < p.T && pos_ok) {
                // this token's cosine / sine row while the main loop runs; the
                // thread reads back only its own column, so no barrier is needed
                const float* cr = p.ko.cos + (int64_t)ps * half;
                const float* sr = p.ko.sin + (int64_t)ps * half;
#pragma unroll 8
                for (int i = 0; i < half; ++i) {
                    tab[i * PT + r] = __ldg(cr + i);
                    tab[(half + i) * PT + r] = __ldg(sr + i);
                }
            }
            pdl_wait();                                     // 1/RMS of the norm kernel
            const float inv = t < p.T ? __ldcg(p.inv_rms + t) : 0.f;
            const bool ok = mbar_wait(accfull, 0, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag);
            if (ok) tc_fence_after();
            if (ok && t < p.T && !pos_ok) record_error(p.err, DEV_ERR_BAD_INDEX);
#pragma unroll 1
            for (int hh = 0; hh < QN / 32 && ok; ++hh) {
                float v[32];
                tmem_ld32(taddr + hh * 32, v);
                tmem_ld_wait();
                if (t >= p.T || !pos_ok) continue;
#pragma unroll
                for (int c = 0; c < 32; ++c) v[c] *= inv;
                const int o32 = (col0 + hh * 32) % KDIM;                // dim in the head of this block's first column
                if (o32 < p.ko.d_rope) {
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const int d = o32 + c;                          // dim within the head
                        if (d < p.ko.d_rope) {
                            float cs, sn;
                            if (p.tab) {
                                cs = tab[(d >> 1) * PT + r];
                                sn = tab[(half + (d >> 1)) * PT + r];
                            } else {
                                const int64_t ti = (int64_t)ps * half + (d >> 1);
                                cs = __ldg(p.ko.cos + ti);
                                sn = __ldg(p.ko.sin + ti);
                            }
                            rope_pair(v[c], v[c + 1], cs, sn);
                        }
                    }
                }
                uint4* dst = (uint4*)(p.q_out + (int64_t)t * p.n_heads * KDIM + col0 + hh * 32);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * c + 2 * e], v[8 * c + 2 * e + 1]);
                        w[e] = *(uint32_t*)&b2;
                    }
                    dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        } else {
            // partial tile of this split -> workspace (rows past T hold zeros)
            const bool ok = mbar_wait(accfull, 0, p.err, DEV_ERR_TIMEOUT_MMA, abort_flag);
            if (ok) {
                tc_fence_after();
                float4* dst = (float4*)(p.ws + ((int64_t)jb.s * p.n_tt * PT + t) * p.kwc + blk0 * PN);
#pragma unroll 1
                for (int hh = 0; hh < 2 * nblk; ++hh) {
                    float v[32];
                    tmem_ld32(taddr + hh * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        dst[hh * 8 + c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, QN);
    }
}

// One warp per token (eight per CTA).
__global__ void __launch_bounds__(256) prepare_finish_kernel(const PrepParams p) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    // inputs first (the projections do not write them): slot, position and
    // this lane's rotary factors (dims 4 lane .. 4 lane + 3: pairs 2 lane, 2 lane + 1)
    int64_t sl = -1;
    int ps = 0;
    bool pos_ok = true;
    const int half = p.ko.d_rope >> 1;
    float cs[2] = {1.f, 1.f}, sn[2] = {0.f, 0.f};
    if (t < p.T) {
        sl = __ldg(p.slot + t);
        ps = half > 0 ? __ldg(p.pos + t) : 0;
        pos_ok = half == 0 || (ps >= 0 && ps < p.ko.max_pos);
        if (sl >= 0 && pos_ok) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                if (2 * lane + e < half) {
                    cs[e] = __ldg(p.ko.cos + (int64_t)ps * half + 2 * lane + e);
                    sn[e] = __ldg(p.ko.sin + (int64_t)ps * half + 2 * lane + e);
                }
            }
        }
    }
    pdl_wait();                     // the partials of the projection kernel are visible from here on
    pdl_launch_dependents();
    if (t >= p.T) return;
    const int64_t split_stride = (int64_t)p.n_tt * PT * p.kwc;
    const float* src = p.ws + (int64_t)t * p.kwc;
    float4 a = __ldcg((const float4*)src + lane);
#pragma unroll 4
    for (int sp = 1; sp < p.S; ++sp) {
        const float4 b = __ldcg((const float4*)(src + sp * split_stride) + lane);
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
    }
    for (int j = lane; j < p.n_heads; j += 32) {
        float acc = __ldcg(src + KDIM + j);
#pragma unroll 4
        for (int sp = 1; sp < p.S; ++sp) acc += __ldcg(src + sp * split_stride + KDIM + j);
        p.w_out[(int64_t)t * p.n_heads + j] = acc;
    }
    if (sl < 0) return;                                   // token not stored
    if (sl >= p.ko.cache_rows || !pos_ok) {
        if (lane == 0) record_error(p.err, DEV_ERR_BAD_INDEX);
        return;
    }
    float x[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 2; ++e)
        if (2 * lane + e < half) rope_pair(x[2 * e], x[2 * e + 1], cs[e], sn[e]);
    write_key_row(x, lane, sl, p.ko);
}

__global__ void __launch_bounds__(256) key_append_kernel(const void* k, int k_fp32, int n, const int32_t* pos,
                                                         const int64_t* slot, const KeyOut o, unsigned* err) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps) {
        const int64_t sl = __ldg(slot + r);
        if (sl < 0) continue;
        const int ps = o.d_rope > 0 ? __ldg(pos + r) : 0;
        if (sl >= o.cache_rows || (o.d_rope > 0 && (ps < 0 || ps >= o.max_pos))) {
            if (lane == 0) record_error(err, DEV_ERR_BAD_INDEX);
            continue;
        }
        float x[4];
        if (k_fp32) {
            const float4 v = __ldg((const float4*)k + (int64_t)r * (KDIM / 4) + lane);
            x[0] = v.x;
            x[1] = v.y;
            x[2] = v.z;
            x[3] = v.w;
        } else {
            const uint2 u = __ldg((const uint2*)k + (int64_t)r * (KDIM / 4) + lane);
            x[0] = __uint_as_float(u.x << 16);
            x[1] = __uint_as_float(u.x & 0xFFFF0000u);
            x[2] = __uint_as_float(u.y << 16);
            x[3] = __uint_as_float(u.y & 0xFFFF0000u);
        }
        store_key_row(x, lane, ps, sl, o);
    }
}

// ------------------------------------------------------------------ host --

namespace {

struct PrepShape {
    int n_tt, qn, n_qf, n_kwf, n_kwt, S, kc_q, kc_kw, kwc;
    size_t cqn_off, inv_off, ws_bytes;   // workspace: partials | scaled latent | 1/RMS
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Tiles and the split of the d_model reduction.  When the tiles alone fill
// the GPU (two CTAs per SM) nothing is split; otherwise each key / weight
// tile is split into about as many chunks as a query tile has, as far as
// the free CTA slots allow.
PrepShape prep_shape(int T, int n_heads, int d_c, int d_model, int num_sms) {
    PrepShape s;
    s.n_tt = ceil_div(T, PT);
    // 256-wide query tiles when they alone give at least one CTA per SM
    const bool wide = (n_heads * KDIM) % 256 == 0 && s.n_tt * (n_heads * KDIM / 256) >= num_sms;
    s.qn = wide ? 256 : PN;
    s.n_qf = n_heads * KDIM / s.qn;
    s.n_kwf = KDIM / PN + ceil_div(n_heads, PN);
    s.kc_q = d_c / PK;
    s.kc_kw = d_model / PK;
    s.kwc = s.n_kwf * PN;
    s.n_kwt = ceil_div(s.n_kwf, s.qn / PN);           // key / weight tiles as wide as the query tiles
    const int slots = 2 * num_sms;
    const int base = s.n_tt * (s.n_qf + s.n_kwt);
    int S = 1;
    if (base < slots) {
        S = ceil_div(s.kc_kw, s.kc_q > 0 ? s.kc_q : 1);
        const int room = (slots - s.n_tt * s.n_qf) / (s.n_tt * s.n_kwt);
        if (S > room) S = room;
        if (S > 16) S = 16;
        if (S < 1) S = 1;
    }
    if (S > s.kc_kw) S = s.kc_kw;
    s.S = S;
    s.cqn_off = align256((size_t)S * s.n_tt * PT * s.kwc * sizeof(float));
    s.inv_off = align256(s.cqn_off + (size_t)T * d_c * 2);
    s.ws_bytes = s.inv_off + (size_t)T * sizeof(float);
    return s;
}

}  // namespace

int indexer_prepare_max_dc() { return MAX_DC; }

size_t indexer_prepare_workspace_bytes(int T, int n_heads, int d_c, int d_model, int num_sms) {
    if (T <= 0) return 0;
    return prep_shape(T, n_heads, d_c, d_model, num_sms).ws_bytes;
}

cudaError_t launch_indexer_prepare(const Launch& L, const PrepareArgs& a, void* workspace, size_t ws_bytes) {
    if (a.T == 0) return cudaSuccess;
    const PrepShape s = prep_shape(a.T, a.n_heads, a.d_c, a.d_model, L.num_sms);
    if (ws_bytes < s.ws_bytes) return cudaErrorInvalidValue;
    uint8_t* ws = (uint8_t*)workspace;
    NormParams n;
    n.c_q = (const __nv_bfloat16*)a.c_q;
    n.gamma = a.gamma;
    n.cqn = (__nv_bfloat16*)(ws + s.cqn_off);
    n.inv_rms = (float*)(ws + s.inv_off);
    n.eps = a.eps;
    n.T = a.T;
    n.d_c = a.d_c;
    CUtensorMap m_cq, m_h, m_wqb, m_wk, m_ww;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint32_t a_rows = a.T <= 64 ? 64 : PT;     // rows past the box feed accumulator rows never stored
    bool ok = make_map_sw128(&m_cq, BF, 2, n.cqn, a.d_c, a.T, PK, a_rows);
    ok = ok && make_map_sw128(&m_h, BF, 2, a.h, a.d_model, a.T, PK, a_rows);
    ok = ok && make_map_sw128(&m_wqb, BF, 2, a.wq_b, a.d_c, (uint64_t)a.n_heads * KDIM, PK, (uint32_t)s.qn);
    ok = ok && make_map_sw128(&m_wk, BF, 2, a.wk, a.d_model, KDIM, PK, PN);
    ok = ok && make_map_sw128(&m_ww, BF, 2, a.w_proj, a.d_model, a.n_heads, PK, PN);
    if (!ok) return cudaErrorInvalidValue;
    PrepParams p;
    p.pos = a.pos;
    p.slot = a.slot;
    p.q_out = (__nv_bfloat16*)a.q_out;
    p.w_out = a.w_out;
    p.ws = (float*)workspace;
    p.inv_rms = n.inv_rms;
    p.ko = KeyOut{a.k_cache, a.k_scale, a.rope_cos, a.rope_sin, a.cache_rows, a.d_rope, a.max_pos, (int)a.k_fmt};
    p.T = a.T;
    p.n_heads = a.n_heads;
    p.n_tt = s.n_tt;
    p.n_qf = s.n_qf;
    p.n_kwf = s.n_kwf;
    p.n_kwt = s.n_kwt;
    p.S = s.S;
    p.kc_q = s.kc_q;
    p.kc_kw = s.kc_kw;
    p.kwc = s.kwc;
    p.a_bytes = (int)a_rows * PK * 2;
    p.err = L.err;
    const int grid = s.n_tt * (s.n_qf + s.n_kwt * s.S);
    const bool deep = s.qn == PN && grid <= L.num_sms;
    // the rotary rows of a query tile in shared memory with one CTA per SM
    // (few or many tokens), when they fit beside the ring
    const size_t tab_bytes = (size_t)PT * a.d_rope * sizeof(float);
    const size_t base_smem = s.qn == 256 ? Ring<4, 1, 256>::SMEM_BASE
                           : deep        ? Ring<4, 2, PN>::SMEM_BASE
                                         : Ring<4, 1, PN>::SMEM_BASE;
    p.tab = (s.qn == 256 || deep) && a.d_rope > 0 && base_smem + tab_bytes <= SMEM_LIMIT;
    const size_t smem = base_smem + (p.tab ? tab_bytes : 0);
    auto kern = s.qn == 256 ? indexer_prepare_kernel<4, 1, 256>
              : deep        ? indexer_prepare_kernel<4, 2, PN>
                            : indexer_prepare_kernel<4, 1, PN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = L.stream;
    cfg.gridDim = dim3(ceil_div(a.T, 8));
    cfg.blockDim = dim3(256);
    e = cudaLaunchKernelEx(&cfg, prepare_norm_kernel, n);
    count_launch();
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(PTHREADS);
    cfg.dynamicSmemBytes = smem;
    e = cudaLaunchKernelEx(&cfg, kern, m_cq, m_h, m_wqb, m_wk, m_ww, p);
    count_launch();
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(ceil_div(a.T, 8));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    e = cudaLaunchKernelEx(&cfg, prepare_finish_kernel, p);
    count_launch();
    return e;
}

cudaError_t launch_key_append(const Launch& L, const void* k, dsa_dtype_t k_in, int n, const int32_t* pos,
                              const int64_t* slot, const float* rope_cos, const float* rope_sin, int max_pos,
                              int d_rope, void* cache, dsa_dtype_t fmt, float* k_scale, int64_t cache_rows) {
    if (n == 0) return cudaSuccess;
    const KeyOut o{cache, k_scale, rope_cos, rope_sin, cache_rows, d_rope, max_pos, (int)fmt};
    const int warps_per_block = 8;
    int grid = ceil_div(n, warps_per_block);
    if (grid > 8 * L.num_sms) grid = 8 * L.num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 * warps_per_block);
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, key_append_kernel, k, k_in == DSA_FP32 ? 1 : 0, n, pos, slot, o,
                                             L.err);
    count_launch();
    return e;
}

}  // namespace dsa
