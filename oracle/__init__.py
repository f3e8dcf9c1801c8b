"""CPU oracle for the DSA / CSA sparse-attention path -- TEST INFRASTRUCTURE.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA product never imports it, and
it imports nothing from the product.  All arithmetic lives in ``oracle.c``
(plain C, double precision); this module only compiles it with gcc, converts
arrays and marshals arguments.

Functions and the passages they follow are listed in the header of
``oracle.c``.  The two variants of the attention step at the end of this
module (CSA core attention with its window segment, HCA) are compositions of
``sparse_mla``: they only rearrange caches and index lists.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

FP32, BF16, FP8, FP4 = 0, 1, 2, 3

_I32P = ctypes.POINTER(ctypes.c_int32)
_F32P = ctypes.POINTER(ctypes.c_float)
_F64P = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile oracle.c into _build/liboracle.so (gcc, -O2, OpenMP)."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-Wall", "-Wno-unknown-pragmas", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            L.oracle_bf16_to_double.restype = ctypes.c_double
            L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_fp8_e4m3_to_double.restype = ctypes.c_double
            L.oracle_fp8_e4m3_to_double.argtypes = [ctypes.c_uint8]
            L.oracle_fp4_e2m1_to_double.restype = ctypes.c_double
            L.oracle_fp4_e2m1_to_double.argtypes = [ctypes.c_uint8]
            L.oracle_double_to_bf16_rne.restype = ctypes.c_uint16
            L.oracle_double_to_bf16_rne.argtypes = [ctypes.c_double]
            L.oracle_csa_compress.restype = None
            L.oracle_csa_compress.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
            L.oracle_index_scores.restype = None
            L.oracle_index_scores.argtypes = [ctypes.c_void_p, ctypes.c_int, _F32P, ctypes.c_void_p,
                                              ctypes.c_int, _F32P, _I32P, _I32P, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int, _I32P,
                                              ctypes.c_int, _F64P]
            L.oracle_topk.restype = None
            L.oracle_topk.argtypes = [_F64P, ctypes.c_int64, _I32P, ctypes.c_int, ctypes.c_int, _I32P]
            L.oracle_sparse_mla.restype = None
            L.oracle_sparse_mla.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, _I32P,
                                            ctypes.c_int, ctypes.c_int, _I32P, _I32P, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_double, _I32P, ctypes.c_int,
                                            _F64P, _F64P, _F64P]
            L.oracle_rms_norm.restype = None
            L.oracle_rms_norm.argtypes = [_F64P, _F64P, ctypes.c_int, ctypes.c_int, ctypes.c_double, _F64P]
            L.oracle_rope.restype = None
            L.oracle_rope.argtypes = [_F64P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _I32P,
                                      _F32P, _F32P]
            L.oracle_indexer_prepare.restype = None
            L.oracle_indexer_prepare.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, _F32P,
                                                 ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_int, _F32P, _F32P, _I32P]
            L.oracle_indexer_prepare.argtypes += [ctypes.c_int] * 6 + [_F64P, _F64P, _F64P]
            L.oracle_fp8_e4m3_encode.restype = ctypes.c_uint8
            L.oracle_fp8_e4m3_encode.argtypes = [ctypes.c_float]
            L.oracle_fp4_e2m1_encode.restype = ctypes.c_uint8
            L.oracle_fp4_e2m1_encode.argtypes = [ctypes.c_float]
            L.oracle_key_rows_f32.restype = None
            L.oracle_key_rows_f32.argtypes = [_F32P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _I32P, _F32P,
                                              _F32P, ctypes.c_int, ctypes.c_void_p, _F32P]
            L.oracle_max_threads.restype = ctypes.c_int
            L.oracle_max_threads.argtypes = []
            _lib = L
    return _lib


# ---- array marshalling -------------------------------------------------------

def _host(t) -> np.ndarray:
    """Contiguous host numpy view of a tensor/array; bf16 -> raw uint16 bits,
    fp8 -> raw uint8 codes."""
    if isinstance(t, (list, tuple)):
        t = np.asarray(t)
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t)
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.float8_e4m3fn,):
        return t.view(torch.uint8).numpy()
    return t.numpy()


def _dtype_code(t) -> int:
    if isinstance(t, np.ndarray):
        return {np.dtype(np.float32): FP32, np.dtype(np.uint16): BF16, np.dtype(np.uint8): FP8}[t.dtype]
    return {torch.float32: FP32, torch.bfloat16: BF16, torch.uint8: FP8,
            torch.float8_e4m3fn: FP8}[t.dtype]


def _p(a: np.ndarray, typ):
    return a.ctypes.data_as(typ)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(_host(a), dtype=np.int32)


def max_threads() -> int:
    return int(lib().oracle_max_threads())


# ---- element formats -----------------------------------------------------------

def bf16_to_double(bits: int) -> float:
    return float(lib().oracle_bf16_to_double(int(bits) & 0xFFFF))


def fp8_e4m3_to_double(code: int) -> float:
    return float(lib().oracle_fp8_e4m3_to_double(int(code) & 0xFF))


def fp4_e2m1_to_double(code: int) -> float:
    return lib().oracle_fp4_e2m1_to_double(code)


def double_to_bf16_bits(x: float) -> int:
    return int(lib().oracle_double_to_bf16_rne(float(x)))


def fp8_e4m3_encode(y: float) -> int:
    """Nearest e4m3 code of a binary32 value (ties to even, saturating at 448)."""
    return int(lib().oracle_fp8_e4m3_encode(float(y)))


def fp4_e2m1_encode(y: float) -> int:
    """Nearest e2m1 code (one nibble) of a binary32 value (ties to even, saturating at 6)."""
    return int(lib().oracle_fp4_e2m1_encode(float(y)))


# ---- the path -------------------------------------------------------------------

def csa_compress(src, m: int) -> np.ndarray:
    """src [B, L, D] (bf16 or fp32) -> [B, L/m, D] of the same storage type
    (bf16 as raw uint16 bits)."""
    a = _host(src)
    B, L, D = a.shape
    if L % m:
        raise ValueError("L must be a multiple of m")
    out = np.empty((B, L // m, D), dtype=a.dtype)
    lib().oracle_csa_compress(a.ctypes.data, _dtype_code(a), B, L, D, m, out.ctypes.data)
    return out


def index_scores(q_idx, w, k_idx, row_batch, row_pos, k_scale=None, row_ids=None) -> np.ndarray:
    """Index scores of the requested query rows: float64 [n, L].  fp8 keys are
    uint8 [B, L, D_I] codes, fp4 keys uint8 [B, L, D_I/2] code pairs (low
    nibble first), each with k_scale [B, L]."""
    q = _host(q_idx)
    k = _host(k_idx)
    wf = np.ascontiguousarray(_host(w), dtype=np.float32)
    rows, H_I, D_I = q.shape
    B, L, D_I2 = k.shape
    kd = _dtype_code(k)
    if kd == FP8 and 2 * D_I2 == D_I:
        kd = FP4
    else:
        assert D_I2 == D_I
    ks = None
    if kd in (FP8, FP4):
        ks = np.ascontiguousarray(_host(k_scale), dtype=np.float32)
        assert ks.shape == (B, L)
    rb, rp = _i32(row_batch), _i32(row_pos)
    ids = np.arange(rows, dtype=np.int32) if row_ids is None else _i32(row_ids)
    out = np.empty((len(ids), L), dtype=np.float64)
    lib().oracle_index_scores(q.ctypes.data, _dtype_code(q), _p(wf, _F32P), k.ctypes.data, kd,
                              _p(ks, _F32P) if ks is not None else None, _p(rb, _I32P), _p(rp, _I32P),
                              B, L, H_I, D_I, _p(ids, _I32P), len(ids), _p(out, _F64P))
    return out


def topk(scores, pos, k: int) -> np.ndarray:
    """scores [n, ld] (any float type; converted exactly to double), pos [n]:
    last visible key of each row.  Returns int32 [n, k] in rank order, -1 tail."""
    s = np.ascontiguousarray(_host(scores), dtype=np.float64)
    n, ld = s.shape
    p = _i32(pos)
    assert p.shape == (n,)
    if np.any(p >= ld):
        raise ValueError("pos beyond the score row")
    idx = np.empty((n, k), dtype=np.int32)
    lib().oracle_topk(_p(s, _F64P), ld, _p(p, _I32P), n, k, _p(idx, _I32P))
    return idx


def sparse_mla(q, kv, idx, row_batch, scale: float, d_v: int, ctx: int,
               page_table=None, row_ids=None, want_probs: bool = False):
    """Attention of each requested query row over its selected latent rows.

    q [rows, H, D_K]; kv [B, L, D_K] or paged [pages, page, D_K]; idx
    [rows, k] key positions (-1 = unused).  Returns (out [n,H,D_V] f64,
    lse [n,H] f64, probs [n,H,k] f64 or None)."""
    qa, kva = _host(q), _host(kv)
    assert _dtype_code(qa) == _dtype_code(kva)
    rows, H, D_K = qa.shape
    ia = _i32(idx)
    k = ia.shape[1]
    rb = _i32(row_batch)
    if page_table is not None:
        pt = _i32(page_table)
        B, pages_per_seq = pt.shape
        page = kva.shape[1]
        assert pages_per_seq * page == ctx
    else:
        pt, pages_per_seq, page = None, 0, 0
        B = kva.shape[0]
        assert kva.shape[1] == ctx
    ids = np.arange(rows, dtype=np.int32) if row_ids is None else _i32(row_ids)
    n = len(ids)
    out = np.empty((n, H, d_v), dtype=np.float64)
    lse = np.empty((n, H), dtype=np.float64)
    probs = np.empty((n, H, k), dtype=np.float64) if want_probs else None
    lib().oracle_sparse_mla(qa.ctypes.data, kva.ctypes.data, _dtype_code(qa),
                            _p(pt, _I32P) if pt is not None else None, page, pages_per_seq,
                            _p(rb, _I32P), _p(ia, _I32P), k, B, ctx, H, D_K, d_v, float(scale),
                            _p(ids, _I32P), n, _p(out, _F64P), _p(lse, _F64P),
                            _p(probs, _F64P) if probs is not None else None)
    return out, lse, probs


def csa_core_attention(q, kv, idx, row_batch, scale: float, d_v: int, ctx: int, kv_win, win_pos, window: int,
                       page_table=None, n_sink: int = 0):
    """CSA core attention with the window and attention-sink segments
    ("DeepSeek V4 发布：1.6T 参数、百万上下文…", CSA: the window KV and the
    compressed KV are concatenated and take part in core attention together;
    "解密DeepSeek-V4 预览版…" section 4.3 and "打破幻觉与成本魔咒：DeepSeek-V4 …"
    section 3.3.2: CSA keeps local dependencies with sliding-window attention
    and an attention sink).  Slots are the selected compressed entries idx[t]
    of kv, then the raw rows win_pos[t]-window+1 .. win_pos[t] of kv_win
    (negative positions unused), then the sink: raw rows 0 .. n_sink-1 of the
    sequence, each used only if it lies before the window's first position
    (a raw row inside the window is not attended twice).

    Written as that concatenation: one cache [B, ctx + win_len, D] holding the
    (de-paged) compressed cache then the raw cache, and one index list holding
    the selected entries, then ctx + the window positions, then ctx + the
    sink positions; attention over it is sparse_mla.  Returns
    (out [rows,H,D_V] f64, lse [rows,H] f64)."""
    kva = torch.as_tensor(kv)
    if page_table is not None:
        pt = torch.as_tensor(page_table).long()
        B = pt.shape[0]
        kva = kva[pt.reshape(-1)].reshape(B, ctx, kva.shape[-1])
    win = torch.as_tensor(kv_win)
    assert win.dtype == kva.dtype and win.shape[0] == kva.shape[0]
    comb = torch.cat([kva, win], dim=1)
    rows = torch.as_tensor(q).shape[0]
    pos = torch.as_tensor(win_pos).long().view(rows, 1)
    wi = pos - window + 1 + torch.arange(window).view(1, -1)
    wi = torch.where(wi >= 0, wi + ctx, torch.full_like(wi, -1))
    si = torch.arange(n_sink).view(1, -1).expand(rows, n_sink)
    si = torch.where(si < pos - window + 1, si + ctx, torch.full_like(si, -1))
    parts = [] if idx is None else [torch.as_tensor(idx).long()]
    full = torch.cat(parts + [wi, si], dim=1).to(torch.int32)
    out, lse, _ = sparse_mla(q, comb, full, row_batch, scale, d_v, ctx + win.shape[1])
    return out, lse


def hca_attention(q, kv, row_batch, row_last, scale: float, d_v: int):
    """HCA ("DeepSeek-V4 技术报告深度解析": m' = 128, no top-k selection;
    "DeepSeek V4 发布…": each query sees all compressed KV): attention of row t
    over entries 0..row_last[t] of the compressed cache kv [B, L, D], i.e.
    sparse_mla with the index list 0..row_last[t].  Returns (out, lse)."""
    L = torch.as_tensor(kv).shape[1]
    last = torch.as_tensor(row_last).long().view(-1, 1)
    ar = torch.arange(L).view(1, -1)
    idx = torch.where(ar <= last, ar, torch.full_like(ar, -1)).to(torch.int32)
    out, lse, _ = sparse_mla(q, kv, idx, row_batch, scale, d_v, L)
    return out, lse


# ---- preparation of the indexer's inputs (the step before the path) -----------

def rms_norm(x, gamma, eps: float) -> np.ndarray:
    """RMSNorm of each row of x [n, d] (float64 result)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    g = np.ascontiguousarray(np.asarray(gamma, dtype=np.float64))
    n, d = a.shape
    out = np.empty_like(a)
    lib().oracle_rms_norm(_p(a, _F64P), _p(g, _F64P), n, d, float(eps), _p(out, _F64P))
    return out


def rope(x, pos, rope_cos, rope_sin, d_rope: int) -> np.ndarray:
    """Rotary encoding of x [n, heads, d] (float64 copy): pairs (2i, 2i+1),
    i < d_rope/2, of every head turned by the angle of row pos[r] of the
    [max_pos, d_rope/2] cosine / sine tables."""
    a = np.array(np.asarray(x, dtype=np.float64), copy=True, order="C")
    n, heads, d = a.shape
    c = np.ascontiguousarray(_host(rope_cos), dtype=np.float32)
    s = np.ascontiguousarray(_host(rope_sin), dtype=np.float32)
    lib().oracle_rope(_p(a, _F64P), n, heads, d, int(d_rope), _p(_i32(pos), _I32P), _p(c, _F32P), _p(s, _F32P))
    return a


def indexer_prepare(c_q, gamma, eps: float, wq_b, h, wk, w_proj, rope_cos, rope_sin, pos, n_heads: int,
                    d_rope: int):
    """Inputs of the lightning indexer for T tokens (float64):
    q [T, n_heads, head_dim] = RoPE(W_qb . RMSNorm(c_q)), w [T, n_heads] = W_w . h,
    k [T, head_dim] = RoPE(W_k . h).  Activations c_q [T, d_c], h [T, d_model]
    and the weights W_qb [n_heads*head_dim, d_c], W_k [head_dim, d_model],
    W_w [n_heads, d_model] are bf16 or fp32 tensors (all activations one
    type, all weights one type)."""
    cq, hh = _host(c_q), _host(h)
    wqb, wkk, wpj = _host(wq_b), _host(wk), _host(w_proj)
    assert cq.dtype == hh.dtype and wqb.dtype == wkk.dtype == wpj.dtype
    T, d_c = cq.shape
    d_model = hh.shape[1]
    head_dim = wkk.shape[0]
    assert wqb.shape == (n_heads * head_dim, d_c) and wpj.shape == (n_heads, d_model) and hh.shape[0] == T
    g = np.ascontiguousarray(_host(gamma), dtype=np.float32)
    c = np.ascontiguousarray(_host(rope_cos), dtype=np.float32)
    s = np.ascontiguousarray(_host(rope_sin), dtype=np.float32)
    q = np.empty((T, n_heads, head_dim), dtype=np.float64)
    w = np.empty((T, n_heads), dtype=np.float64)
    k = np.empty((T, head_dim), dtype=np.float64)
    lib().oracle_indexer_prepare(cq.ctypes.data, hh.ctypes.data, _dtype_code(cq), _p(g, _F32P), float(eps),
                                 wqb.ctypes.data, wkk.ctypes.data, wpj.ctypes.data, _dtype_code(wqb),
                                 _p(c, _F32P), _p(s, _F32P), _p(_i32(pos), _I32P), T, d_c, d_model, n_heads,
                                 head_dim, int(d_rope), _p(q, _F64P), _p(w, _F64P), _p(k, _F64P))
    return q, w, k


def key_rows_f32(x, pos, rope_cos, rope_sin, d_rope: int, fmt: int):
    """The key-cache write decided in binary32: RoPE of dims [0, d_rope) of
    each row of x [n, d] (separately rounded products and sums), then the
    stored form: fmt BF16 -> (uint16 bits [n, d], None); FP8 -> (codes uint8
    [n, d], scale float32 [n]); FP4 -> (code pairs uint8 [n, d/2], scale).
    x is first rounded to binary32 (exact for bf16 and fp32 inputs)."""
    a = np.array(np.asarray(_to_f32(x)), dtype=np.float32, copy=True, order="C")
    n, d = a.shape
    c = np.ascontiguousarray(_host(rope_cos), dtype=np.float32)
    s = np.ascontiguousarray(_host(rope_sin), dtype=np.float32)
    if fmt == BF16:
        out = np.zeros((n, d), dtype=np.uint16)
    elif fmt == FP8:
        out = np.zeros((n, d), dtype=np.uint8)
    elif fmt == FP4:
        out = np.zeros((n, d // 2), dtype=np.uint8)
    else:
        raise ValueError("fmt must be BF16, FP8 or FP4")
    scale = np.ones(n, dtype=np.float32)
    lib().oracle_key_rows_f32(_p(a, _F32P), n, d, int(d_rope), _p(_i32(pos), _I32P), _p(c, _F32P), _p(s, _F32P),
                              int(fmt), out.ctypes.data, _p(scale, _F32P))
    return out, (None if fmt == BF16 else scale)


def _to_f32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float32)
