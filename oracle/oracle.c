/*
 * CPU oracle for the DSA / CSA sparse-attention path.  TEST INFRASTRUCTURE
 * ONLY: this file is built and called by the test-suite, by the smoke check
 * and by the CPU baseline leg of the benchmark.  The product (the CUDA
 * library) never links, loads or calls it, and it shares no code with it.
 *
 * Plain C, every quantity in double precision, loops written in the order of
 * the definitions.  OpenMP only splits independent rows / keys over threads.
 *
 * What it computes (sources are the pages' titles and sections):
 *
 *  oracle_csa_compress   CSA token compression: each m consecutive KV rows
 *                        become one entry, their average ("解密DeepSeek-V4 ..."
 *                        section 4.3; "DeepSeek-V4 技术报告深度解析", CSA step 1;
 *                        xhh.club DeepSeek-V4 CSA summary: 4 tokens -> 1).
 *                        Result rounded to bf16 (nearest-even) because the
 *                        compressed caches are stored in bf16.
 *  oracle_index_scores   lightning-indexer score
 *                        I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s])
 *                        ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", section 1.3,
 *                        闪电索引器; the printed formula is lost in the page
 *                        text, the weighted-ReLU form is the one the page's
 *                        prose and the V4 summary describe). Keys after the
 *                        query's position are invisible (-inf).
 *  oracle_topk           top-k selection: the k visible keys with the
 *                        highest score, lower index first on equal scores;
 *                        every visible key when there are at most k of them
 *                        (same article, section 3, Step 3).
 *  oracle_sparse_mla     attention restricted to the selected latent rows,
 *                        MQA mode: one latent row is shared by all query
 *                        heads, value = first D_V dims of the latent (same
 *                        article, sections 1.3 细粒度稀疏注意力, 1.4 and 3 Step 4).
 *
 *
 * and the step before the path, the preparation of the indexer's inputs
 * ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", section 3, Step 1: low-rank
 * projections, RMSNorm of the query latent, the split into parts with and
 * without rotary position encoding, apply_rotary_emb, weights_proj; section
 * 1.3: a separate learned linear map takes query and key to 128 dims):
 *
 *  oracle_rms_norm       x / sqrt(mean(x^2) + eps) * gamma, per row.
 *  oracle_rope           rotary position encoding of the first d_rope dims
 *                        of each head: pair (2i, 2i+1) turned by the angle
 *                        whose cosine and sine the table gives at (pos, i).
 *  oracle_indexer_prepare  q_I = RoPE(W_qb . RMSNorm(c_q)) per head,
 *                        w = W_w . h, k_I = RoPE(W_k . h), in double.
 *  oracle_fp8_e4m3_encode / oracle_fp4_e2m1_encode  round a binary32 value
 *                        to the nearest code, ties to the even code,
 *                        saturating at the largest finite magnitude.
 *  oracle_key_rows_f32   the key-cache write in binary32 arithmetic (the
 *                        precision in which the stored codes are decided):
 *                        RoPE with separately rounded products and sums,
 *                        then per row scale = amax / qmax and code =
 *                        encode(x / scale).
 *
 * Parity pins (tests/test_oracle_pins.py) check each function against closed
 * forms, brute force, hand-computed fixtures and library routines.  The one
 * point left unpinned is whether the lost index-score formula carried an
 * extra positive constant factor; it cannot change the selected set.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ODT_FP32 = 0, ODT_BF16 = 1, ODT_FP8_E4M3 = 2, ODT_FP4_E2M1 = 3 };
enum { ORACLE_MAX_DIM = 1024 };

/* ---- element formats --------------------------------------------------- */

/* bf16 = the upper 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP fp8 E4M3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
 * exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities. */
double oracle_fp8_e4m3_to_double(uint8_t code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 0xF, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* OCP fp4 E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent 0 is
 * subnormal (m/2 * 2^0); no infinities or NaNs.  The 8 magnitudes are
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6.  `code` is one 4-bit code (low nibble). */
double oracle_fp4_e2m1_to_double(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? (double)m / 2.0 : ldexp(1.0 + (double)m / 2.0, e - 1);
    return s ? -v : v;
}

/* Round a double to the nearest bf16 (ties to even), directly from double:
 * find the spacing of bf16 numbers around x (8 significant bits in the
 * normal range, 2^-133 below 2^-126), round x/spacing to the nearest even
 * integer and scale back.  The result is exactly representable in bf16, so
 * the final narrowing through binary32 is exact. */
uint16_t oracle_double_to_bf16_rne(double x)
{
    if (isnan(x))
        return 0x7FC0;
    if (x == 0.0)
        return signbit(x) ? 0x8000 : 0x0000;
    int e;
    (void)frexp(x, &e);                 /* |x| in [2^(e-1), 2^e) */
    int q = e - 8;                      /* spacing exponent for 8 significant bits */
    if (q < -133)
        q = -133;                       /* bf16 subnormal spacing */
    double n = nearbyint(ldexp(x, -q)); /* default mode: nearest, ties to even */
    double y = ldexp(n, q);
    if (fabs(y) >= ldexp(1.0, 128))
        return x > 0 ? 0x7F80 : 0xFF80; /* overflow to infinity */
    float f = (float)y;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (y == 0.0)
        u = signbit(x) ? 0x80000000u : 0u;
    return (uint16_t)(u >> 16);
}

static double load_elem(const void* p, int dtype, int64_t i)
{
    switch (dtype) {
    case ODT_FP32: return (double)((const float*)p)[i];
    case ODT_BF16: return oracle_bf16_to_double(((const uint16_t*)p)[i]);
    case ODT_FP8_E4M3: return oracle_fp8_e4m3_to_double(((const uint8_t*)p)[i]);
    case ODT_FP4_E2M1: {   /* two codes per byte, element 2j in the low nibble */
        uint8_t byte = ((const uint8_t*)p)[i >> 1];
        return oracle_fp4_e2m1_to_double((i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF));
    }
    default: return NAN;
    }
}

/* ---- CSA compression --------------------------------------------------- */

/* dst[b,i,d] = (1/m) * sum_{r<m} src[b, m*i + r, d]; src [B, L, D], dst
 * [B, L/m, D], both of type `dtype` (bf16 or fp32).  The sum is formed in
 * double left to right, then scaled, then rounded once to the storage type. */
void oracle_csa_compress(const void* src, int dtype, int B, int L, int D, int m, void* dst)
{
    int Lc = L / m;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < Lc; ++i)
            for (int d = 0; d < D; ++d) {
                double sum = 0.0;
                for (int r = 0; r < m; ++r)
                    sum += load_elem(src, dtype, ((int64_t)b * L + (int64_t)m * i + r) * D + d);
                double mean = sum / (double)m;
                int64_t o = ((int64_t)b * Lc + i) * D + d;
                if (dtype == ODT_BF16)
                    ((uint16_t*)dst)[o] = oracle_double_to_bf16_rne(mean);
                else
                    ((float*)dst)[o] = (float)mean;
            }
}

/* ---- lightning indexer -------------------------------------------------- */

/* For each requested query row t = row_ids[n]:
 *   out[n, s] = sum_j w[t,j] * max(0, sum_d q[t,j,d] * k[b,s,d])   for s <= row_pos[t]
 *   out[n, s] = -inf                                               for s >  row_pos[t]
 * with b = row_batch[t].  q [rows, H_I, D_I] (fp32 or bf16), w [rows, H_I]
 * fp32, k [B, L, D_I] (fp32, bf16 or fp8 codes, or fp4 code pairs).  For fp8
 * and fp4 keys the stored value is code * k_scale[b, s] (one scale per key
 * row). */
void oracle_index_scores(const void* q, int q_dtype, const float* w,
                         const void* k, int k_dtype, const float* k_scale,
                         const int32_t* row_batch, const int32_t* row_pos,
                         int B, int L, int H_I, int D_I,
                         const int32_t* row_ids, int n_rows, double* out)
{
    (void)B;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int n = 0; n < n_rows; ++n)
        for (int s = 0; s < L; ++s) {
            int t = row_ids[n];
            int b = row_batch[t];
            double* o = out + (int64_t)n * L + s;
            if (s > row_pos[t]) {
                *o = -INFINITY;
                continue;
            }
            double kv[ORACLE_MAX_DIM];
            if (D_I > ORACLE_MAX_DIM) {
                *o = NAN;
                continue;
            }
            int64_t krow = (int64_t)b * L + s;
            double ks = (k_dtype == ODT_FP8_E4M3 || k_dtype == ODT_FP4_E2M1) ? (double)k_scale[krow] : 1.0;
            for (int d = 0; d < D_I; ++d)
                kv[d] = load_elem(k, k_dtype, krow * D_I + d) * ks;
            double score = 0.0;
            for (int j = 0; j < H_I; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D_I; ++d)
                    dot += load_elem(q, q_dtype, ((int64_t)t * H_I + j) * D_I + d) * kv[d];
                double relu = dot > 0.0 ? dot : 0.0;
                score += (double)w[(int64_t)t * H_I + j] * relu;
            }
            *o = score;
        }
}

/* ---- top-k ---------------------------------------------------------------- */

typedef struct { double v; int32_t s; } scored_t;

static int by_score_desc_then_index(const void* a, const void* b)
{
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s > y->s) - (x->s < y->s);
}

/* scores [n_rows, ld] (row n holds the scores of query row_ids[n]); the
 * visible keys of row n are s = 0 .. pos[n].  Writes idx [n_rows, k]: the
 * selected keys in rank order (score descending, index ascending on equal
 * scores), then -1 in the unused slots when fewer than k keys are visible.
 * Equal scores compare equal, so -0.0 and +0.0 tie and go by index. */
void oracle_topk(const double* scores, int64_t ld, const int32_t* pos, int n_rows,
                 int k, int32_t* idx)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_rows; ++n) {
        int nvis = pos[n] + 1;
        scored_t* tmp = (scored_t*)malloc(sizeof(scored_t) * (size_t)(nvis > 0 ? nvis : 1));
        for (int s = 0; s < nvis; ++s) {
            tmp[s].v = scores[(int64_t)n * ld + s];
            tmp[s].s = s;
        }
        qsort(tmp, (size_t)nvis, sizeof(scored_t), by_score_desc_then_index);
        int keep = nvis < k ? nvis : k;
        for (int i = 0; i < k; ++i)
            idx[(int64_t)n * k + i] = i < keep ? tmp[i].s : -1;
        free(tmp);
    }
}

/* ---- sparse MLA (MQA mode) ------------------------------------------------ */

/* For each requested query row t = row_ids[n] and head h:
 *   z_s  = scale * sum_{d<D_K} q[t,h,d] * c[s,d]       for s in idx[t] (idx >= 0)
 *   p_s  = exp(z_s - max z) / sum_s' exp(z_s' - max z)
 *   out[n,h,:] = sum_s p_s * c[s, 0:D_V]
 *   lse[n,h]   = max z + log sum_s exp(z_s - max z)
 * where c[s] is latent row s of sequence b = row_batch[t]:
 *   contiguous cache  kv [B, L, D_K]:            c[s] = kv[b, s]
 *   paged cache       kv [pages, page_size, D_K]: c[s] = kv[page_table[b, s/page_size], s%page_size]
 * idx [rows, k] holds key positions (-1 = unused slot).  probs, if not NULL,
 * receives p [n_rows, H, k] in slot order (0 for unused slots).  A row with no
 * selected key gets out = 0 and lse = -inf. */
void oracle_sparse_mla(const void* q, const void* kv, int dtype,
                       const int32_t* page_table, int page_size, int pages_per_seq,
                       const int32_t* row_batch, const int32_t* idx, int k,
                       int B, int L, int H, int D_K, int D_V, double scale,
                       const int32_t* row_ids, int n_rows,
                       double* out, double* lse, double* probs)
{
    (void)B;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int n = 0; n < n_rows; ++n)
        for (int h = 0; h < H; ++h) {
            int t = row_ids[n];
            int b = row_batch[t];
            const int32_t* sel = idx + (int64_t)t * k;
            double* z = (double*)malloc(sizeof(double) * (size_t)k);
            int64_t* rowoff = (int64_t*)malloc(sizeof(int64_t) * (size_t)k);
            double qv[ORACLE_MAX_DIM];
            for (int d = 0; d < D_K && d < ORACLE_MAX_DIM; ++d)
                qv[d] = load_elem(q, dtype, ((int64_t)t * H + h) * D_K + d);
            double zmax = -INFINITY;
            for (int i = 0; i < k; ++i) {
                int s = sel[i];
                if (s < 0 || s >= L) {
                    z[i] = -INFINITY;
                    rowoff[i] = -1;
                    continue;
                }
                int64_t r = page_table
                    ? (int64_t)page_table[(int64_t)b * pages_per_seq + s / page_size] * page_size + s % page_size
                    : (int64_t)b * L + s;
                rowoff[i] = r * D_K;
                double dot = 0.0;
                for (int d = 0; d < D_K; ++d)
                    dot += qv[d] * load_elem(kv, dtype, rowoff[i] + d);
                z[i] = scale * dot;
                if (z[i] > zmax) zmax = z[i];
            }
            double* o = out + ((int64_t)n * H + h) * D_V;
            for (int d = 0; d < D_V; ++d) o[d] = 0.0;
            double denom = 0.0;
            for (int i = 0; i < k; ++i)
                if (rowoff[i] >= 0) denom += exp(z[i] - zmax);
            for (int i = 0; i < k; ++i) {
                double p = rowoff[i] >= 0 ? exp(z[i] - zmax) / denom : 0.0;
                if (probs) probs[((int64_t)n * H + h) * k + i] = p;
                if (rowoff[i] < 0) continue;
                for (int d = 0; d < D_V; ++d)
                    o[d] += p * load_elem(kv, dtype, rowoff[i] + d);
            }
            lse[(int64_t)n * H + h] = denom > 0.0 ? zmax + log(denom) : -INFINITY;
            free(z);
            free(rowoff);
        }
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- indexer input preparation (DSA article, section 3, Step 1) -------- */

/* RMSNorm of each of the n rows of x [n, d]: x / sqrt(mean(x^2) + eps) * gamma. */
void oracle_rms_norm(const double* x, const double* gamma, int n, int d, double eps, double* out)
{
    for (int r = 0; r < n; ++r) {
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += x[(int64_t)r * d + j] * x[(int64_t)r * d + j];
        double inv = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j) out[(int64_t)r * d + j] = x[(int64_t)r * d + j] * inv * gamma[j];
    }
}

/* Rotary position encoding, in place, of x [n, heads, d]: in every head, dims
 * 2i and 2i+1 (i < d_rope/2) are turned by the angle of row pos[r] of the
 * tables: (a, b) -> (a cos - b sin, a sin + b cos).  The tables are
 * [max_pos, d_rope/2]; dims d_rope .. d-1 carry no position. */
void oracle_rope(double* x, int n, int heads, int d, int d_rope, const int32_t* pos,
                 const float* cos_t, const float* sin_t)
{
    int half = d_rope / 2;
    for (int r = 0; r < n; ++r)
        for (int h = 0; h < heads; ++h) {
            double* v = x + ((int64_t)r * heads + h) * d;
            for (int i = 0; i < half; ++i) {
                double c = cos_t[(int64_t)pos[r] * half + i], s = sin_t[(int64_t)pos[r] * half + i];
                double a = v[2 * i], b = v[2 * i + 1];
                v[2 * i] = a * c - b * s;
                v[2 * i + 1] = a * s + b * c;
            }
        }
}

static double* load_all(const void* p, int dtype, int64_t n)
{
    double* out = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) out[i] = load_elem(p, dtype, i);
    return out;
}

/* out[r, o] = sum_j W[o, j] * x[r, j]  (W [n_out, d] row-major: the linear
 * map of a PyTorch-style weight). */
static void linear(const double* x, const double* W, int n, int d, int n_out, double* out)
{
    #pragma omp parallel for collapse(2) schedule(static)
    for (int r = 0; r < n; ++r)
        for (int o = 0; o < n_out; ++o) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += W[(int64_t)o * d + j] * x[(int64_t)r * d + j];
            out[(int64_t)r * n_out + o] = acc;
        }
}

/* Inputs of the lightning indexer for T tokens, in the order of Step 1:
 *   q_out [T, n_heads, head_dim] = RoPE( W_qb . RMSNorm(c_q; gamma, eps) )
 *   w_out [T, n_heads]           = W_w . h
 *   k_out [T, head_dim]          = RoPE( W_k . h )
 * c_q [T, d_c] is the query latent (the low-rank projection the MLA query
 * shares), h [T, d_model] the hidden states; W_qb [n_heads*head_dim, d_c],
 * W_k [head_dim, d_model], W_w [n_heads, d_model]; act_dtype / w_dtype are
 * the element formats of the activations and of the weights. */
void oracle_indexer_prepare(const void* c_q, const void* h, int act_dtype, const float* gamma, double eps,
                            const void* wq_b, const void* wk, const void* w_proj, int w_dtype,
                            const float* cos_t, const float* sin_t, const int32_t* pos,
                            int T, int d_c, int d_model, int n_heads, int head_dim, int d_rope,
                            double* q_out, double* w_out, double* k_out)
{
    double* c = load_all(c_q, act_dtype, (int64_t)T * d_c);
    double* x = load_all(h, act_dtype, (int64_t)T * d_model);
    double* g = (double*)malloc(sizeof(double) * (size_t)d_c);
    for (int j = 0; j < d_c; ++j) g[j] = gamma[j];
    double* cn = (double*)malloc(sizeof(double) * (size_t)T * d_c + 8);
    oracle_rms_norm(c, g, T, d_c, eps, cn);

    double* W = load_all(wq_b, w_dtype, (int64_t)n_heads * head_dim * d_c);
    linear(cn, W, T, d_c, n_heads * head_dim, q_out);
    free(W);
    oracle_rope(q_out, T, n_heads, head_dim, d_rope, pos, cos_t, sin_t);

    W = load_all(w_proj, w_dtype, (int64_t)n_heads * d_model);
    linear(x, W, T, d_model, n_heads, w_out);
    free(W);

    W = load_all(wk, w_dtype, (int64_t)head_dim * d_model);
    linear(x, W, T, d_model, head_dim, k_out);
    free(W);
    oracle_rope(k_out, T, 1, head_dim, d_rope, pos, cos_t, sin_t);

    free(c); free(x); free(g); free(cn);
}

/* Nearest code of a finite binary32 value among the non-negative codes
 * 0 .. last of a format (ascending in value), ties to the even code (the
 * code's last bit is the mantissa's last bit), the sign bit added after. */
static unsigned encode_nearest_even(float y, int last, int sign_bit, double (*decode)(uint8_t))
{
    double a = fabs((double)y);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= last; ++c) {
        double d = fabs(decode((uint8_t)c) - a);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            bd = d;
            best = c;
        }
    }
    return (unsigned)best | (signbit(y) ? (1u << sign_bit) : 0u);
}

/* E4M3: magnitudes are codes 0 .. 0x7E (0x7F is NaN); above 448 saturates. */
uint8_t oracle_fp8_e4m3_encode(float y) { return (uint8_t)encode_nearest_even(y, 0x7E, 7, oracle_fp8_e4m3_to_double); }

/* E2M1: magnitudes are codes 0 .. 7; above 6 saturates.  Returns one nibble. */
uint8_t oracle_fp4_e2m1_encode(float y) { return (uint8_t)encode_nearest_even(y, 7, 3, oracle_fp4_e2m1_to_double); }

/* The key-cache write, in binary32 (every product and sum rounded on its
 * own, no fused multiply-add): x [n, d] binary32 rows (already projected),
 * RoPE of dims [0, d_rope) at pos[r], then
 *   fmt ODT_BF16:     out [n, d] bf16 bits (nearest-even), no scale
 *   fmt ODT_FP8_E4M3: scale = amax / 448 (1 for a zero row), out [n, d] codes of x / scale
 *   fmt ODT_FP4_E2M1: scale = amax / 6, out [n, d/2] code pairs, element 2j in the low nibble
 * x is overwritten by the rotated values. */
void oracle_key_rows_f32(float* x, int n, int d, int d_rope, const int32_t* pos, const float* cos_t,
                         const float* sin_t, int fmt, void* out, float* scale)
{
    int half = d_rope / 2;
    for (int r = 0; r < n; ++r) {
        float* v = x + (int64_t)r * d;
        for (int i = 0; i < half; ++i) {
            float c = cos_t[(int64_t)pos[r] * half + i], s = sin_t[(int64_t)pos[r] * half + i];
            float a = v[2 * i], b = v[2 * i + 1];
            float ac = a * c, bs = b * s, as = a * s, bc = b * c;
            v[2 * i] = ac - bs;
            v[2 * i + 1] = as + bc;
        }
        if (fmt == ODT_BF16) {
            for (int j = 0; j < d; ++j) ((uint16_t*)out)[(int64_t)r * d + j] = oracle_double_to_bf16_rne((double)v[j]);
            continue;
        }
        float amax = 0.0f;
        for (int j = 0; j < d; ++j) amax = fabsf(v[j]) > amax ? fabsf(v[j]) : amax;
        float qmax = fmt == ODT_FP8_E4M3 ? 448.0f : 6.0f;
        float sc = amax > 0.0f ? amax / qmax : 1.0f;
        scale[r] = sc;
        for (int j = 0; j < d; ++j) {
            float y = v[j] / sc;
            if (fmt == ODT_FP8_E4M3) {
                ((uint8_t*)out)[(int64_t)r * d + j] = oracle_fp8_e4m3_encode(y);
            } else {
                uint8_t* o = (uint8_t*)out + (int64_t)r * (d / 2) + j / 2;
                uint8_t code = oracle_fp4_e2m1_encode(y);
                *o = (j & 1) ? (uint8_t)((*o & 0x0F) | (code << 4)) : (uint8_t)((*o & 0xF0) | code);
            }
        }
    }
}
