"""Python binding of libdsa_b200.so, the sm_100a DeepSeek Sparse Attention path.

Argument marshalling only: every function below checks tensor placement and
dtypes, allocates outputs with torch on the tensors' device when none are
given, and calls the C entry point of the same name on torch's current
stream.  All arithmetic runs in the library's CUDA kernels; there is no CPU
or fallback path.  Importing this package fails loudly when the library has
not been built (``python -m sparse_attention_logits_b200._build``).

Contracts (shapes, layouts, supported sizes) are documented in
``include/dsa_b200.h``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from . import _build

LIB_PATH = _build.LIB_PATH

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m sparse_attention_logits_b200._build` "
        "(nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA, DSA_ERR_DEVICE_TIMEOUT = range(5)
DSA_FP32, DSA_BF16, DSA_FP8_E4M3, DSA_FP4_E2M1 = 0, 1, 2, 3

_STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_CUDA",
                 4: "DSA_ERR_DEVICE_TIMEOUT"}

_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_f32 = ctypes.c_float

_SIGS = {
    "dsa_version": (_i32, []),
    "dsa_launch_count": (ctypes.c_uint64, []),
    "dsa_last_error": (ctypes.c_char_p, []),
    "csa_compress": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "dsa_indexer_logits": (_i32, [_vp, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                                  _i64, _vp]),
    "dsa_topk_workspace_size": (_sz, [_i32, _i32, _i32]),
    "dsa_topk": (_i32, [_vp, _i64, _vp, _i32, _i32, _i32, _vp, _vp, _sz, _vp]),
    "dsa_sparse_mla_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "dsa_sparse_mla": (_i32, [_vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                              _f32, _vp, _vp, _vp, _sz, _vp]),
    "dsa_sparse_mla_noalloc": (_i32, [_vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                      _i32, _f32, _vp, _vp, _vp]),
    "csa_core_attention": (_i32, [_vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i32,
                                  _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz, _vp]),
    "hca_attention": (_i32, [_vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz,
                             _vp]),
    "dsa_indexer_prepare_workspace_size": (_sz, [_i32, _i32, _i32, _i32]),
    "dsa_indexer_prepare": (_i32, [_vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _i32, _i32,
                                   _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _i64, _vp, _sz, _vp]),
    "dsa_indexer_key_append": (_i32, [_vp, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _i32, _i32, _vp, _i32, _vp, _i64,
                                      _vp]),
    "dsa_get_device_error": (_i32, [_vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.dsa_last_error().decode(errors="replace")
        super().__init__(f"{where}: {_STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != DSA_OK:
        raise DSAError(status, where)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DSA_FP32
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DSA_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dev(*ts) -> torch.device:
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (the library takes device pointers)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("tensors on different devices")
    return dev


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def version() -> int:
    return int(_lib.dsa_version())


def launch_count() -> int:
    """Kernels launched by the library from this thread so far."""
    return int(_lib.dsa_launch_count())


def csa_compress(src: torch.Tensor, m: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """src [B, L, D] bf16/fp32 -> [B, L/m, D]: mean of each m consecutive rows."""
    dev = _dev(src, out)
    B, L, D = src.shape
    if out is None:
        out = torch.empty((B, L // m, D), dtype=src.dtype, device=dev)
    with torch.cuda.device(dev):
        _check(_lib.csa_compress(_ptr(src), _dt(src), B, L, D, m, _ptr(out), _stream(dev)), "csa_compress")
    return out


def indexer_logits(q_idx: torch.Tensor, w: torch.Tensor, k_idx: torch.Tensor, row_batch: torch.Tensor,
                   row_pos: torch.Tensor, k_scale: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Index scores [rows, L] fp32 (entries past row_pos untouched).  fp8 keys
    are uint8 [B, L, D] e4m3 codes, fp4 keys uint8 [B, L, D/2] e2m1 code pairs
    (low nibble first), each with k_scale [B, L]."""
    dev = _dev(q_idx, w, k_idx, row_batch, row_pos, k_scale, out)
    rows, H, D = q_idx.shape
    B, L, D2 = k_idx.shape
    kdt = _dt(k_idx)
    if kdt == DSA_FP8_E4M3 and 2 * D2 == D:
        kdt = DSA_FP4_E2M1
    elif D2 != D:
        raise ValueError("q_idx and k_idx head dims differ")
    if out is None:
        out = torch.empty((rows, L), dtype=torch.float32, device=dev)
    ld = out.stride(0) if out.dim() == 2 else L
    with torch.cuda.device(dev):
        _check(_lib.dsa_indexer_logits(_ptr(q_idx), _dt(q_idx), _ptr(w), _ptr(k_idx), kdt, _ptr(k_scale),
                                       _ptr(row_batch), _ptr(row_pos), rows, B, L, H, D, _ptr(out), ld,
                                       _stream(dev)), "dsa_indexer_logits")
    return out


def topk_workspace_size(rows: int, ctx_len: int, k: int) -> int:
    return int(_lib.dsa_topk_workspace_size(rows, ctx_len, k))


def topk(logits: torch.Tensor, row_pos: torch.Tensor, k: int, ctx_len: Optional[int] = None,
         out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Selected key positions [rows, k] int32, ascending, -1 tail."""
    dev = _dev(logits, row_pos, out, workspace)
    rows, ld = logits.shape
    L = ld if ctx_len is None else ctx_len
    if out is None:
        out = torch.empty((rows, k), dtype=torch.int32, device=dev)
    need = topk_workspace_size(rows, L, k)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(_lib.dsa_topk(_ptr(logits), ld, _ptr(row_pos), rows, L, k, _ptr(out), _ptr(workspace), wsb,
                             _stream(dev)), "dsa_topk")
    return out


def sparse_mla_workspace_size(rows: int, k: int, n_heads: int, d_qk: int, d_v: int, dtype: torch.dtype) -> int:
    dt = DSA_FP32 if dtype == torch.float32 else DSA_BF16
    return int(_lib.dsa_sparse_mla_workspace_size(rows, k, n_heads, d_qk, d_v, dt))


def sparse_mla(q: torch.Tensor, kv: torch.Tensor, idx: torch.Tensor, row_batch: torch.Tensor, scale: float,
               d_v: int, ctx_len: int, page_table: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention over the selected latent rows: (out [rows, H, d_v], lse [rows, H] fp32)."""
    dev = _dev(q, kv, idx, row_batch, page_table, out, lse, workspace)
    rows, H, DK = q.shape
    k = idx.shape[1]
    if page_table is not None:
        B = page_table.shape[0]
        num_pages, page_size = kv.shape[0], kv.shape[1]
    else:
        B = kv.shape[0]
        num_pages, page_size = 0, 0
        if kv.shape[1] != ctx_len:
            raise ValueError("kv.shape[1] != ctx_len")
    if out is None:
        out = torch.empty((rows, H, d_v), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((rows, H), dtype=torch.float32, device=dev)
    need = sparse_mla_workspace_size(rows, k, H, DK, d_v, q.dtype)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(_lib.dsa_sparse_mla(_ptr(q), _ptr(kv), _dt(q), _ptr(page_table), page_size, num_pages, _ptr(row_batch),
                                   _ptr(idx), k, rows, B, ctx_len, H, DK, d_v, float(scale), _ptr(out), _ptr(lse),
                                   _ptr(workspace), wsb, _stream(dev)), "dsa_sparse_mla")
    return out, lse


def csa_core_attention(q: torch.Tensor, kv: torch.Tensor, idx: Optional[torch.Tensor], row_batch: torch.Tensor,
                       scale: float, d_v: int, ctx_len: int, kv_win: torch.Tensor, win_pos: torch.Tensor, window: int,
                       page_table: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       n_sink: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """CSA core attention: the selected compressed entries idx of kv plus the
    window of `window` raw rows of kv_win [B, win_len, d_qk] ending at
    win_pos[t] and the sink of the first `n_sink` raw rows (those before the
    window) (out [rows, H, d_v], lse [rows, H] fp32)."""
    dev = _dev(q, kv, idx, row_batch, kv_win, win_pos, page_table, out, lse, workspace)
    rows, H, DK = q.shape
    k = 0 if idx is None else idx.shape[1]
    if page_table is not None:
        B = page_table.shape[0]
        num_pages, page_size = kv.shape[0], kv.shape[1]
    else:
        B = kv.shape[0]
        num_pages, page_size = 0, 0
        if kv.shape[1] != ctx_len:
            raise ValueError("kv.shape[1] != ctx_len")
    if kv_win.shape[0] != B or kv_win.dtype != q.dtype:
        raise ValueError("kv_win must be [B, win_len, d_qk] of q's dtype")
    if out is None:
        out = torch.empty((rows, H, d_v), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((rows, H), dtype=torch.float32, device=dev)
    need = sparse_mla_workspace_size(rows, k + window + n_sink, H, DK, d_v, q.dtype)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(_lib.csa_core_attention(_ptr(q), _ptr(kv), _dt(q), _ptr(page_table), page_size, num_pages,
                                       _ptr(row_batch), _ptr(idx), k, rows, B, ctx_len, _ptr(kv_win), _ptr(win_pos),
                                       kv_win.shape[1], window, n_sink, H, DK, d_v, float(scale), _ptr(out), _ptr(lse),
                                       _ptr(workspace), wsb, _stream(dev)), "csa_core_attention")
    return out, lse


def hca_attention(q: torch.Tensor, kv: torch.Tensor, row_batch: torch.Tensor, row_last: torch.Tensor, scale: float,
                  d_v: int, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """HCA: dense attention of each row over entries 0..row_last[t] of the
    compressed cache kv [B, L, d_qk] (out [rows, H, d_v], lse [rows, H] fp32)."""
    dev = _dev(q, kv, row_batch, row_last, out, lse, workspace)
    rows, H, DK = q.shape
    B, L = kv.shape[0], kv.shape[1]
    if out is None:
        out = torch.empty((rows, H, d_v), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((rows, H), dtype=torch.float32, device=dev)
    need = sparse_mla_workspace_size(rows, L, H, DK, d_v, q.dtype)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(_lib.hca_attention(_ptr(q), _ptr(kv), _dt(q), _ptr(row_batch), _ptr(row_last), rows, B, L, H, DK, d_v,
                                  float(scale), _ptr(out), _ptr(lse), _ptr(workspace), wsb, _stream(dev)),
               "hca_attention")
    return out, lse


def sparse_mla_noalloc(q: torch.Tensor, kv: torch.Tensor, idx: torch.Tensor, row_batch: torch.Tensor, scale: float,
                       d_v: int, ctx_len: int, out: torch.Tensor, lse: torch.Tensor,
                       page_table: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """sparse_mla through the entry point that allocates nothing: the caller
    passes out [rows, H, d_v] and lse [rows, H]; split partials go to the
    library's fixed device scratch (calls overlapping on one device race)."""
    dev = _dev(q, kv, idx, row_batch, page_table, out, lse)
    rows, H, DK = q.shape
    k = idx.shape[1]
    if page_table is not None:
        B = page_table.shape[0]
        num_pages, page_size = kv.shape[0], kv.shape[1]
    else:
        B = kv.shape[0]
        num_pages, page_size = 0, 0
        if kv.shape[1] != ctx_len:
            raise ValueError("kv.shape[1] != ctx_len")
    with torch.cuda.device(dev):
        _check(_lib.dsa_sparse_mla_noalloc(_ptr(q), _ptr(kv), _dt(q), _ptr(page_table), page_size, num_pages,
                                           _ptr(row_batch), _ptr(idx), k, rows, B, ctx_len, H, DK, d_v, float(scale),
                                           _ptr(out), _ptr(lse), _stream(dev)), "dsa_sparse_mla_noalloc")
    return out, lse


def _key_cache_fmt(k_cache: torch.Tensor) -> Tuple[int, int]:
    """(format, rows) of an indexer key cache: bf16 [..., 128], fp8 codes
    (uint8 / float8_e4m3fn) [..., 128] or fp4 code pairs (uint8) [..., 64]."""
    last = k_cache.shape[-1]
    rows = k_cache.numel() // last if last else 0
    if k_cache.dtype == torch.bfloat16 and last == 128:
        return DSA_BF16, rows
    if k_cache.dtype in (torch.uint8, torch.float8_e4m3fn) and last == 128:
        return DSA_FP8_E4M3, rows
    if k_cache.dtype == torch.uint8 and last == 64:
        return DSA_FP4_E2M1, rows
    raise TypeError("key cache must be bf16 [..., 128], fp8 [..., 128] or fp4 pairs uint8 [..., 64]")


def indexer_prepare_workspace_size(tokens: int, n_heads: int, d_c: int, d_model: int) -> int:
    return int(_lib.dsa_indexer_prepare_workspace_size(tokens, n_heads, d_c, d_model))


def indexer_prepare(c_q: torch.Tensor, q_norm_weight: torch.Tensor, wq_b: torch.Tensor, h: torch.Tensor,
                    wk: torch.Tensor, w_proj: torch.Tensor, pos: torch.Tensor, slot: torch.Tensor,
                    k_cache: torch.Tensor, k_scale: Optional[torch.Tensor] = None,
                    rope_cos: Optional[torch.Tensor] = None, rope_sin: Optional[torch.Tensor] = None,
                    eps: float = 1e-6, q_out: Optional[torch.Tensor] = None, w_out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Indexer inputs of T new tokens: (q_out [T, H, 128] bf16, w_out [T, H]
    fp32); each token's key is written to row slot[t] of k_cache (-1: not
    stored).  d_rope = 2 * rope_cos.shape[1] (0 without tables)."""
    dev = _dev(c_q, q_norm_weight, wq_b, h, wk, w_proj, pos, slot, k_cache, k_scale, rope_cos, rope_sin, q_out,
               w_out, workspace)
    T, d_c = c_q.shape
    d_model = h.shape[1]
    head_dim = wk.shape[0]
    H = w_proj.shape[0]
    fmt, rows = _key_cache_fmt(k_cache)
    d_rope = 0 if rope_cos is None else 2 * rope_cos.shape[1]
    max_pos = 0 if rope_cos is None else rope_cos.shape[0]
    if q_out is None:
        q_out = torch.empty((T, H, head_dim), dtype=torch.bfloat16, device=dev)
    if w_out is None:
        w_out = torch.empty((T, H), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(indexer_prepare_workspace_size(T, H, d_c, d_model), 1), dtype=torch.uint8,
                                device=dev)
    wsb = workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(_lib.dsa_indexer_prepare(_ptr(c_q), _ptr(q_norm_weight), float(eps), _ptr(wq_b), _ptr(h), _ptr(wk),
                                        _ptr(w_proj), _ptr(rope_cos), _ptr(rope_sin), max_pos, d_rope, _ptr(pos),
                                        _ptr(slot), T, d_c, d_model, H, head_dim, _ptr(q_out), _ptr(w_out),
                                        _ptr(k_cache), fmt, _ptr(k_scale), rows, _ptr(workspace), wsb,
                                        _stream(dev)), "dsa_indexer_prepare")
    return q_out, w_out


def indexer_key_append(k: torch.Tensor, slot: torch.Tensor, k_cache: torch.Tensor,
                       k_scale: Optional[torch.Tensor] = None, pos: Optional[torch.Tensor] = None,
                       rope_cos: Optional[torch.Tensor] = None, rope_sin: Optional[torch.Tensor] = None) -> None:
    """Write already-projected key rows k [n, 128] (fp32 or bf16) into rows
    slot[r] of the key cache (RoPE of the first 2 * rope_cos.shape[1] dims
    at pos[r] first, when tables are given)."""
    dev = _dev(k, slot, k_cache, k_scale, pos, rope_cos, rope_sin)
    n, head_dim = k.shape
    fmt, rows = _key_cache_fmt(k_cache)
    d_rope = 0 if rope_cos is None else 2 * rope_cos.shape[1]
    max_pos = 0 if rope_cos is None else rope_cos.shape[0]
    with torch.cuda.device(dev):
        _check(_lib.dsa_indexer_key_append(_ptr(k), _dt(k), _ptr(rope_cos), _ptr(rope_sin), max_pos, d_rope,
                                           _ptr(pos), _ptr(slot), n, head_dim, _ptr(k_cache), fmt, _ptr(k_scale),
                                           rows, _stream(dev)), "dsa_indexer_key_append")


def get_device_error(device: Optional[torch.device] = None) -> int:
    """Synchronizes the current stream and returns (and clears) the library's
    device error status; raises DSAError if a kernel recorded an error."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        st = _lib.dsa_get_device_error(_stream(dev))
    _check(st, "dsa_get_device_error")
    return st


def dsa_step(q_idx, w, k_idx, row_batch, row_pos, q, kv, topk_k: int, scale: float, d_v: int,
             k_scale=None, page_table=None, logits=None, idx=None, out=None, lse=None,
             topk_ws=None, mla_ws=None):
    """One pass of the DSA path: indexer scores -> top-k -> sparse MLA.
    Returns (out, lse, idx)."""
    L = k_idx.shape[1]
    logits = indexer_logits(q_idx, w, k_idx, row_batch, row_pos, k_scale=k_scale, out=logits)
    idx = topk(logits, row_pos, topk_k, ctx_len=L, out=idx, workspace=topk_ws)
    out, lse = sparse_mla(q, kv, idx, row_batch, scale, d_v, L, page_table=page_table, out=out, lse=lse,
                          workspace=mla_ws)
    return out, lse, idx
