// extern "C" entry points of libdsa_b200.so: argument validation, kernel
// selection and the device error word.  Declarations and contracts are in
// include/dsa_b200.h.
#include <stdio.h>
#include <stdarg.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "launchers.h"

namespace {

thread_local char g_last_error[256] = "";
thread_local uint64_t g_launches = 0;

dsa_status_t fail(dsa_status_t st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

dsa_status_t cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return DSA_OK;
    return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// One error word per device; its device address is looked up once per device.
__device__ unsigned g_device_error;

constexpr int kMaxDevices = dsa::kMaxDevices;
// Filled once per device under dsa::init_mutex(): the SM count is stored
// first and the error-word address is then published with release order, so
// a thread that sees the address (acquire) also sees the SM count.
std::atomic<unsigned*> g_err_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

dsa_status_t make_launch(void* stream, dsa::Launch* L) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
    unsigned* err = g_err_ptr[dev].load(std::memory_order_acquire);
    if (!err) {
        std::lock_guard<std::mutex> lock(dsa::init_mutex());
        err = g_err_ptr[dev].load(std::memory_order_relaxed);
        if (!err) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_device_error);
            if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(device error word)");
            int sms = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return cuda_status(e, "cudaDeviceGetAttribute");
            g_num_sms[dev] = sms;
            err = (unsigned*)p;
            g_err_ptr[dev].store(err, std::memory_order_release);
        }
    }
    L->stream = (cudaStream_t)stream;
    L->err = err;
    L->num_sms = g_num_sms[dev];
    return DSA_OK;
}

// Fixed scratch of dsa_sparse_mla_noalloc: the bf16 partial outputs and fp32
// log-sum-exps of a key list split over several clusters.  A (row, split)
// pair takes 128 heads x (512 x 2 + 4) = 131,584 bytes, and the split count is
// chosen so that rows x splits <= SMs / 2, so 20 MiB covers every size on a
// GPU of up to 318 SMs.  No byte of it has to start at zero: each cluster
// writes its whole partial block before the merge kernel, launched after it
// on the same stream, reads it.  One copy per device: calls that overlap on
// one device (two streams, two threads) race on it.
constexpr size_t kMlaScratchBytes = DSA_MLA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_mla_scratch[kMlaScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_mla_scratch on the current device, looked up once per
// device (cudaGetSymbolAddress may load the module, so the first call must
// not happen inside a stream capture).
dsa_status_t mla_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_mla_scratch);
        if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(sparse MLA scratch)");
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return DSA_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
size_t dtype_size(dsa_dtype_t t) { return t == DSA_FP32 ? 4 : t == DSA_BF16 ? 2 : 1; }
bool valid_dtype(dsa_dtype_t t) { return t == DSA_FP32 || t == DSA_BF16 || t == DSA_FP8_E4M3; }
bool valid_key_dtype(dsa_dtype_t t) { return valid_dtype(t) || t == DSA_FP4_E2M1; }

}  // namespace

namespace dsa {
void count_launch(int n) { g_launches += (uint64_t)n; }
std::mutex& init_mutex() {
    static std::mutex mu;
    return mu;
}
}  // namespace dsa

extern "C" {

int dsa_version(void) { return 100; }

uint64_t dsa_launch_count(void) { return g_launches; }

const char* dsa_last_error(void) { return g_last_error; }

dsa_status_t csa_compress(const void* src, dsa_dtype_t dtype, int batch, int len, int dim, int m, void* dst,
                          void* stream) {
    if (!src || !dst) return fail(DSA_ERR_INVALID_ARG, "csa_compress: null pointer");
    if (batch < 0 || len < 0 || dim <= 0 || m < 1 || m > 1024)
        return fail(DSA_ERR_INVALID_ARG, "csa_compress: bad sizes (batch=%d len=%d dim=%d m=%d)", batch, len, dim, m);
    if (len % m) return fail(DSA_ERR_INVALID_ARG, "csa_compress: len=%d not a multiple of m=%d", len, m);
    if (dtype != DSA_BF16 && dtype != DSA_FP32) return fail(DSA_ERR_UNSUPPORTED, "csa_compress: dtype must be bf16 or fp32");
    if ((dim * dtype_size(dtype)) % 16) return fail(DSA_ERR_UNSUPPORTED, "csa_compress: dim*elem_size must be a multiple of 16 bytes");
    if (!aligned(src, 16) || !aligned(dst, 16)) return fail(DSA_ERR_INVALID_ARG, "csa_compress: pointers must be 16-byte aligned");
    const size_t bytes_in = (size_t)batch * len * dim * dtype_size(dtype);
    const size_t bytes_out = bytes_in / m;
    const char* s = (const char*)src; const char* d = (const char*)dst;
    if (bytes_in && s < d + bytes_out && d < s + bytes_in) return fail(DSA_ERR_INVALID_ARG, "csa_compress: src and dst overlap");
    dsa::Launch L;
    dsa_status_t st = make_launch(stream, &L);
    if (st != DSA_OK) return st;
    return cuda_status(dsa::launch_csa_compress(L, src, dtype, batch, len, dim, m, dst), "csa_compress launch");
}

dsa_status_t dsa_indexer_logits(const void* q, dsa_dtype_t q_dtype, const float* w, const void* k,
                                dsa_dtype_t k_dtype, const float* k_scale, const int32_t* row_batch,
                                const int32_t* row_pos, int rows, int batch, int ctx_len, int n_heads,
                                int head_dim, float* logits, int64_t ld_logits, void* stream) {
    if (rows < 0 || batch <= 0 || ctx_len < 0 || n_heads <= 0 || head_dim <= 0)
        return fail(DSA_ERR_INVALID_ARG, "dsa_indexer_logits: bad sizes");
    if (rows == 0 || ctx_len == 0) return DSA_OK;
    if (!q || !w || !k || !row_batch || !row_pos || !logits)
        return fail(DSA_ERR_INVALID_ARG, "dsa_indexer_logits: null pointer");
    if (!valid_dtype(q_dtype) || !valid_key_dtype(k_dtype)) return fail(DSA_ERR_INVALID_ARG, "dsa_indexer_logits: bad dtype");
    if (ld_logits < ctx_len) return fail(DSA_ERR_INVALID_ARG, "dsa_indexer_logits: ld_logits < ctx_len");
    if ((k_dtype == DSA_FP8_E4M3 || k_dtype == DSA_FP4_E2M1) != (k_scale != nullptr))
        return fail(DSA_ERR_INVALID_ARG, "dsa_indexer_logits: k_scale must be given exactly when k is fp8 or fp4");
    const bool combo_ok = (q_dtype == DSA_FP32 && k_dtype == DSA_FP32) || (q_dtype == DSA_BF16 && k_dtype == DSA_BF16) ||
                          (q_dtype == DSA_BF16 && k_dtype == DSA_FP8_E4M3) ||
                          (q_dtype == DSA_BF16 && k_dtype == DSA_FP4_E2M1);
    if (!combo_ok) return fail(DSA_ERR_UNSUPPORTED, "dsa_indexer_logits: unsupported q/k dtype pair");
    if (head_dim != 32 && head_dim != 64 && head_dim != 128)
        return fail(DSA_ERR_UNSUPPORTED, "dsa_indexer_logits: head_dim must be 32, 64 or 128");
    if (n_heads > 128) return fail(DSA_ERR_UNSUPPORTED, "dsa_indexer_logits: n_heads > 128");
    if (k_dtype == DSA_FP4_E2M1 && !dsa::indexer_tc_supported(q_dtype, k_dtype, n_heads, head_dim))
        return fail(DSA_ERR_UNSUPPORTED, "dsa_indexer_logits: fp4 keys need n_heads = 64 and head_dim = 128");
    dsa::Launch L;
    dsa_status_t st = make_launch(stream, &L);
    if (st != DSA_OK) return st;
    if (dsa::indexer_tc_supported(q_dtype, k_dtype, n_heads, head_dim)) {
        if (!aligned(q, 16) || !aligned(k, 16))
            return fail(DSA_ERR_INVALID_ARG, "dsa_indexer_logits: q and k must be 16-byte aligned");
        return cuda_status(dsa::launch_indexer_tc(L, q, k_dtype, w, k, k_scale, row_batch, row_pos, rows, batch,
                                                  ctx_len, logits, ld_logits),
                           "dsa_indexer_logits (tensor-core) launch");
    }
    return cuda_status(dsa::launch_indexer_simt(L, q, q_dtype, w, k, k_dtype, k_scale, row_batch, row_pos, rows,
                                                batch, ctx_len, n_heads, head_dim, logits, ld_logits),
                       "dsa_indexer_logits launch");
}

size_t dsa_topk_workspace_size(int rows, int ctx_len, int k) { return dsa::topk_workspace_bytes(rows, ctx_len, k); }

dsa_status_t dsa_topk(const float* logits, int64_t ld, const int32_t* row_pos, int rows, int ctx_len, int k,
                      int32_t* idx, void* workspace, size_t workspace_bytes, void* stream) {
    if (rows < 0 || ctx_len < 0 || k < 1 || k > 8192) return fail(DSA_ERR_INVALID_ARG, "dsa_topk: bad sizes (k must be in [1, 8192])");
    if (rows == 0) return DSA_OK;
    if (!logits || !row_pos || !idx) return fail(DSA_ERR_INVALID_ARG, "dsa_topk: null pointer");
    if (ld < ctx_len) return fail(DSA_ERR_INVALID_ARG, "dsa_topk: ld < ctx_len");
    if (!dsa::topk_supported(ctx_len)) return fail(DSA_ERR_UNSUPPORTED, "dsa_topk: ctx_len %d above the supported maximum", ctx_len);
    const size_t need = dsa::topk_workspace_bytes(rows, ctx_len, k);
    if (need && (!workspace || workspace_bytes < need))
        return fail(DSA_ERR_INVALID_ARG, "dsa_topk: workspace of %zu bytes needed", need);
    dsa::Launch L;
    dsa_status_t st = make_launch(stream, &L);
    if (st != DSA_OK) return st;
    return cuda_status(dsa::launch_topk(L, logits, ld, row_pos, rows, ctx_len, k, idx, workspace, workspace_bytes),
                       "dsa_topk launch");
}

size_t dsa_sparse_mla_workspace_size(int rows, int k, int n_heads, int d_qk, int d_v, dsa_dtype_t dtype) {
    if (rows <= 0 || k <= 0 || !dsa::mla_tc_supported(dtype, n_heads, d_qk, d_v)) return 0;
    int dev = 0, sms = 0;
    // No device: size for a very large GPU.  The split count grows with the
    // SM count (up to one split per 64 keys), so this bounds every device.
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 1024;
    return dsa::mla_tc_workspace_bytes(rows, k, sms);
}

size_t dsa_indexer_prepare_workspace_size(int tokens, int n_heads, int d_c, int d_model) {
    if (tokens <= 0 || n_heads <= 0 || d_c <= 0 || d_model <= 0) return 0;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 1024;  // no device: size for a large GPU (the most splits)
    return dsa::indexer_prepare_workspace_bytes(tokens, n_heads, d_c, d_model, sms);
}

namespace {

// Checks shared by the two key-cache writers.
dsa_status_t check_key_cache(const char* name, const float* rope_cos, const float* rope_sin, int max_pos, int d_rope,
                             const int32_t* pos, const int64_t* slot, int head_dim, const void* k_cache,
                             dsa_dtype_t k_dtype, const float* k_scale, int64_t cache_rows) {
    if (head_dim != 128) return fail(DSA_ERR_UNSUPPORTED, "%s: head_dim must be 128", name);
    if (d_rope < 0 || d_rope > head_dim || (d_rope & 1))
        return fail(DSA_ERR_INVALID_ARG, "%s: d_rope must be even and in [0, head_dim]", name);
    if (d_rope > 0 && (!rope_cos || !rope_sin || !pos || max_pos < 1))
        return fail(DSA_ERR_INVALID_ARG, "%s: rotary tables, positions and max_pos >= 1 needed when d_rope > 0", name);
    if (!slot || !k_cache || cache_rows < 0) return fail(DSA_ERR_INVALID_ARG, "%s: null slot or cache pointer", name);
    if (k_dtype != DSA_BF16 && k_dtype != DSA_FP8_E4M3 && k_dtype != DSA_FP4_E2M1)
        return fail(DSA_ERR_UNSUPPORTED, "%s: the key cache must be bf16, fp8 or fp4", name);
    if ((k_dtype != DSA_BF16) != (k_scale != nullptr))
        return fail(DSA_ERR_INVALID_ARG, "%s: k_scale must be given exactly when the cache is fp8 or fp4", name);
    if (!aligned(k_cache, 16)) return fail(DSA_ERR_INVALID_ARG, "%s: k_cache must be 16-byte aligned", name);
    return DSA_OK;
}

}  // namespace

dsa_status_t dsa_indexer_prepare(const void* c_q, const float* q_norm_weight, float eps, const void* wq_b,
                                 const void* h, const void* wk, const void* w_proj, const float* rope_cos,
                                 const float* rope_sin, int max_pos, int d_rope, const int32_t* pos,
                                 const int64_t* slot, int tokens, int d_c, int d_model, int n_heads, int head_dim,
                                 void* q_out, float* w_out, void* k_cache, dsa_dtype_t k_dtype, float* k_scale,
                                 int64_t cache_rows, void* workspace, size_t workspace_bytes, void* stream) {
    const char* name = "dsa_indexer_prepare";
    if (tokens < 0 || d_c <= 0 || d_model <= 0 || n_heads <= 0 || head_dim <= 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: bad sizes", name);
    if (tokens == 0) return DSA_OK;
    if (!c_q || !q_norm_weight || !wq_b || !h || !wk || !w_proj || !pos || !q_out || !w_out)
        return fail(DSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (!(eps >= 0.f)) return fail(DSA_ERR_INVALID_ARG, "%s: eps must be >= 0", name);
    dsa_status_t st = check_key_cache(name, rope_cos, rope_sin, max_pos, d_rope, pos, slot, head_dim, k_cache,
                                      k_dtype, k_scale, cache_rows);
    if (st != DSA_OK) return st;
    if (d_c % 64 || d_model % 64) return fail(DSA_ERR_UNSUPPORTED, "%s: d_c and d_model must be multiples of 64", name);
    if (d_c > dsa::indexer_prepare_max_dc())
        return fail(DSA_ERR_UNSUPPORTED, "%s: d_c above %d", name, dsa::indexer_prepare_max_dc());
    if (n_heads > 256) return fail(DSA_ERR_UNSUPPORTED, "%s: n_heads > 256", name);
    if (!aligned(c_q, 16) || !aligned(h, 16) || !aligned(wq_b, 16) || !aligned(wk, 16) || !aligned(w_proj, 16) ||
        !aligned(q_norm_weight, 16) || !aligned(q_out, 16))
        return fail(DSA_ERR_INVALID_ARG, "%s: c_q, h, the weights, q_norm_weight and q_out must be 16-byte aligned", name);
    dsa::Launch L;
    st = make_launch(stream, &L);
    if (st != DSA_OK) return st;
    const size_t need = dsa::indexer_prepare_workspace_bytes(tokens, n_heads, d_c, d_model, L.num_sms);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
        return fail(DSA_ERR_INVALID_ARG, "%s: a 256-byte aligned workspace of %zu bytes is needed", name, need);
    dsa::PrepareArgs a;
    a.c_q = c_q;
    a.gamma = q_norm_weight;
    a.eps = eps;
    a.wq_b = wq_b;
    a.h = h;
    a.wk = wk;
    a.w_proj = w_proj;
    a.rope_cos = rope_cos;
    a.rope_sin = rope_sin;
    a.max_pos = max_pos;
    a.d_rope = d_rope;
    a.pos = pos;
    a.slot = slot;
    a.T = tokens;
    a.d_c = d_c;
    a.d_model = d_model;
    a.n_heads = n_heads;
    a.q_out = q_out;
    a.w_out = w_out;
    a.k_cache = k_cache;
    a.k_fmt = k_dtype;
    a.k_scale = k_scale;
    a.cache_rows = cache_rows;
    return cuda_status(dsa::launch_indexer_prepare(L, a, workspace, workspace_bytes), "dsa_indexer_prepare launch");
}

dsa_status_t dsa_indexer_key_append(const void* k, dsa_dtype_t k_in_dtype, const float* rope_cos,
                                    const float* rope_sin, int max_pos, int d_rope, const int32_t* pos,
                                    const int64_t* slot, int n, int head_dim, void* k_cache, dsa_dtype_t k_dtype,
                                    float* k_scale, int64_t cache_rows, void* stream) {
    const char* name = "dsa_indexer_key_append";
    if (n < 0 || head_dim <= 0) return fail(DSA_ERR_INVALID_ARG, "%s: bad sizes", name);
    if (n == 0) return DSA_OK;
    if (!k) return fail(DSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (k_in_dtype != DSA_FP32 && k_in_dtype != DSA_BF16)
        return fail(DSA_ERR_UNSUPPORTED, "%s: keys must be fp32 or bf16", name);
    dsa_status_t st = check_key_cache(name, rope_cos, rope_sin, max_pos, d_rope, pos, slot, head_dim, k_cache,
                                      k_dtype, k_scale, cache_rows);
    if (st != DSA_OK) return st;
    if (!aligned(k, 16)) return fail(DSA_ERR_INVALID_ARG, "%s: k must be 16-byte aligned", name);
    dsa::Launch L;
    st = make_launch(stream, &L);
    if (st != DSA_OK) return st;
    return cuda_status(dsa::launch_key_append(L, k, k_in_dtype, n, pos, slot, rope_cos, rope_sin, max_pos, d_rope,
                                              k_cache, k_dtype, k_scale, cache_rows),
                       "dsa_indexer_key_append launch");
}

}  // extern "C"

namespace {

// Shared body of dsa_sparse_mla, csa_core_attention and hca_attention: the
// selected (or, with idx NULL, every visible) keys of kv, plus an optional
// window segment of raw rows (x).
dsa_status_t sparse_attention(const char* name, const void* q, const void* kv, dsa_dtype_t dtype,
                              const int32_t* page_table, int page_size, int num_pages, const int32_t* row_batch,
                              const int32_t* idx, int k, int rows, int batch, int ctx_len, int n_heads, int d_qk,
                              int d_v, float scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                              void* stream, const dsa::KvExtra& x) {
    const int window = x.kv2 ? x.window : 0;
    const int n_sink = x.kv2 ? x.n_sink : 0;
    if (rows < 0 || batch <= 0 || ctx_len <= 0 || k < 0 || window < 0 || n_sink < 0 ||
        (int64_t)k + window + n_sink < 1 || (int64_t)k + window + n_sink > (1 << 30) || n_heads <= 0 ||
        d_qk <= 0 || d_v <= 0 || d_v > d_qk)
        return fail(DSA_ERR_INVALID_ARG, "%s: bad sizes", name);
    const bool raw = window + n_sink > 0;                   // a segment of raw rows
    if ((int64_t)batch * ctx_len >= ((int64_t)1 << 31) - 2 ||
        (raw && (int64_t)batch * x.len2 >= ((int64_t)1 << 31) - 2) ||
        (page_table && (int64_t)num_pages * page_size >= ((int64_t)1 << 31) - 2))
        return fail(DSA_ERR_UNSUPPORTED, "%s: a cache holds more than 2^31 - 2 rows", name);
    if (rows == 0) return DSA_OK;
    if (!q || !kv || !row_batch || !out || !lse || (k > 0 && !idx && !x.row_last))
        return fail(DSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (raw && (!x.pos2 || x.len2 <= 0))
        return fail(DSA_ERR_INVALID_ARG, "%s: a window or sink needs win_pos and win_len", name);
    if (dtype != DSA_BF16 && dtype != DSA_FP32) return fail(DSA_ERR_UNSUPPORTED, "%s: dtype must be bf16 or fp32", name);
    if (page_table) {
        if (page_size <= 0 || ctx_len % page_size)
            return fail(DSA_ERR_INVALID_ARG, "%s: ctx_len must be a multiple of page_size", name);
        if (num_pages <= 0) return fail(DSA_ERR_INVALID_ARG, "%s: num_pages must be positive with a page table", name);
    }
    if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "%s: scale must be positive and finite", name);
    const bool tc = dsa::mla_tc_supported(dtype, n_heads, d_qk, d_v);
    if (!tc && !dsa::mla_simt_supported(d_qk, d_v, n_heads))
        return fail(DSA_ERR_UNSUPPORTED, "%s: no kernel for d_qk=%d d_v=%d n_heads=%d", name, d_qk, d_v, n_heads);
    dsa::Launch L;
    dsa_status_t st = make_launch(stream, &L);
    if (st != DSA_OK) return st;
    if (tc) {
        if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(out, 16) || (raw && !aligned(x.kv2, 16)))
            return fail(DSA_ERR_INVALID_ARG, "%s: q, kv, the window cache and out must be 16-byte aligned", name);
        const size_t need = dsa::mla_tc_workspace_bytes(rows, k + window + n_sink, L.num_sms);
        if (need && (!workspace || workspace_bytes < need))
            return fail(DSA_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed", name, need);
        return cuda_status(dsa::launch_mla_tc(L, q, kv, page_table, page_size, num_pages, row_batch, idx, k, rows,
                                              batch, ctx_len, scale, out, lse, workspace, workspace_bytes, x),
                           "sparse attention (tensor-core) launch");
    }
    return cuda_status(dsa::launch_mla_simt(L, q, kv, dtype, page_table, page_size, num_pages, row_batch, idx, k, rows,
                                            batch, ctx_len, n_heads, d_qk, d_v, scale, out, lse, x),
                       "sparse attention launch");
}

}  // namespace

extern "C" {

dsa_status_t dsa_sparse_mla(const void* q, const void* kv, dsa_dtype_t dtype, const int32_t* page_table,
                            int page_size, int num_pages, const int32_t* row_batch, const int32_t* idx, int k, int rows, int batch,
                            int ctx_len, int n_heads, int d_qk, int d_v, float scale, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream) {
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "dsa_sparse_mla: bad sizes (k=%d)", k);
    if (rows > 0 && !idx) return fail(DSA_ERR_INVALID_ARG, "dsa_sparse_mla: null pointer");
    return sparse_attention("dsa_sparse_mla", q, kv, dtype, page_table, page_size, num_pages, row_batch, idx, k, rows,
                            batch, ctx_len, n_heads, d_qk, d_v, scale, out, lse, workspace, workspace_bytes, stream,
                            dsa::KvExtra());
}

dsa_status_t csa_core_attention(const void* q, const void* kv, dsa_dtype_t dtype, const int32_t* page_table,
                                int page_size, int num_pages, const int32_t* row_batch, const int32_t* idx, int k,
                                int rows, int batch, int ctx_len, const void* kv_win, const int32_t* win_pos,
                                int win_len, int window, int n_sink, int n_heads, int d_qk, int d_v, float scale,
                                void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    if (window < 0 || n_sink < 0 || (window + n_sink > 0 && !kv_win))
        return fail(DSA_ERR_INVALID_ARG, "csa_core_attention: bad window or sink");
    if (n_sink > win_len) return fail(DSA_ERR_INVALID_ARG, "csa_core_attention: n_sink above win_len");
    if (rows > 0 && k > 0 && !idx) return fail(DSA_ERR_INVALID_ARG, "csa_core_attention: null pointer");
    dsa::KvExtra x;
    x.kv2 = kv_win;
    x.pos2 = win_pos;
    x.len2 = win_len;
    x.window = window;
    x.n_sink = n_sink;
    return sparse_attention("csa_core_attention", q, kv, dtype, page_table, page_size, num_pages, row_batch, idx, k,
                            rows, batch, ctx_len, n_heads, d_qk, d_v, scale, out, lse, workspace, workspace_bytes,
                            stream, x);
}

dsa_status_t hca_attention(const void* q, const void* kv, dsa_dtype_t dtype, const int32_t* row_batch,
                           const int32_t* row_last, int rows, int batch, int ctx_len, int n_heads, int d_qk, int d_v,
                           float scale, void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    if (rows > 0 && !row_last) return fail(DSA_ERR_INVALID_ARG, "hca_attention: null pointer");
    dsa::KvExtra x;
    x.row_last = row_last;
    return sparse_attention("hca_attention", q, kv, dtype, nullptr, 0, 0, row_batch, nullptr, ctx_len, rows, batch,
                            ctx_len, n_heads, d_qk, d_v, scale, out, lse, workspace, workspace_bytes, stream, x);
}

dsa_status_t dsa_sparse_mla_noalloc(const void* q, const void* kv, dsa_dtype_t dtype, const int32_t* page_table,
                                    int page_size, int num_pages, const int32_t* row_batch, const int32_t* idx, int k,
                                    int rows, int batch, int ctx_len, int n_heads, int d_qk, int d_v, float scale,
                                    void* out, float* lse, void* stream) {
    void* scratch = nullptr;
    if (rows > 0 && k >= 1 && dsa::mla_tc_supported(dtype, n_heads, d_qk, d_v)) {
        dsa::Launch L;
        dsa_status_t st = make_launch(stream, &L);
        if (st != DSA_OK) return st;
        const size_t need = dsa::mla_tc_workspace_bytes(rows, k, L.num_sms);
        if (need > kMlaScratchBytes)
            return fail(DSA_ERR_INVALID_ARG,
                        "dsa_sparse_mla_noalloc: %d rows x k=%d need %zu bytes of scratch, more than its fixed %zu",
                        rows, k, need, kMlaScratchBytes);
        if (need) {
            st = mla_scratch(&scratch);
            if (st != DSA_OK) return st;
        }
    }
    return dsa_sparse_mla(q, kv, dtype, page_table, page_size, num_pages, row_batch, idx, k, rows, batch, ctx_len,
                          n_heads, d_qk, d_v, scale, out, lse, scratch, scratch ? kMlaScratchBytes : 0, stream);
}

dsa_status_t dsa_get_device_error(void* stream) {
    dsa::Launch L;
    dsa_status_t st = make_launch(stream, &L);
    if (st != DSA_OK) return st;
    cudaError_t e = cudaStreamSynchronize(L.stream);
    if (e != cudaSuccess) return cuda_status(e, "dsa_get_device_error: stream synchronize");
    unsigned word = 0;
    e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof word);
    if (e != cudaSuccess) return cuda_status(e, "dsa_get_device_error: read");
    if (word == 0) return DSA_OK;
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_status(e, "dsa_get_device_error: clear");
    if (word & (dsa::DEV_ERR_TIMEOUT_TMA | dsa::DEV_ERR_TIMEOUT_MMA | dsa::DEV_ERR_TIMEOUT_PEER))
        return fail(DSA_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (device error word 0x%x)", word);
    return fail(DSA_ERR_INVALID_ARG, "a kernel met an out-of-range index and skipped it (device error word 0x%x)", word);
}

}  // extern "C"
