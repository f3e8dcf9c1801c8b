"""Seeded synthetic workloads for the DSA / CSA sparse-attention path.

This module only *draws inputs*: shapes, seeded random values, the bf16 cast,
the fp8-e4m3 storage format of the indexer keys and the page table. It holds
none of the method's arithmetic (no index score, no selection, no softmax, no
pooling), so that both the CPU oracle (``oracle/``) and the CUDA path can take
their inputs from here without sharing any computation.

Value recipe (same for every workload, one generator, fixed draw order):

    q_I ~ N(0,1)/sqrt(D_I)    indexer queries           [rows, H_I, D_I]
    w   ~ U(0,1)              per-head indexer weights  [rows, H_I]
    k_I ~ N(0,1)/sqrt(D_I)    indexer key cache         [B, L_raw, D_I]
    q   ~ N(0,1)/sqrt(D_K)    MLA queries               [rows, H, D_K]
    kv  ~ N(0,1)/sqrt(D_K)    MLA latent KV cache       [B, L_raw, D_K]
    page_table = randperm(B * L / page)                 (paged caches only)

The pages' sizes: the lightning indexer of DeepSeek-V3.2 uses 64 heads of
128 dims and keeps the top 2048 keys ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配",
sections 1.3 and 3, Steps 2-3); CSA pools every 4 tokens and keeps the top
1024 blocks (xhh.club DeepSeek-V4 CSA summary); MLA runs in MQA mode with a
512-d latent (same article, section 1.4) plus a 64-d rope part.

Floating-point tensors are drawn in fp32 and then cast (round to nearest even)
to the workload's storage type. fp8 indexer keys are stored as e4m3fn codes
with one fp32 scale per key row, ``scale = amax(row) / 448``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str              # "prefill" (causal, one query per cached token) or "decode"
    batch: int             # B: number of sequences / caches
    ctx: int               # L: keys the indexer scores per sequence (after CSA pooling)
    rows: int              # query rows in one step
    idx_heads: int         # H_I
    idx_dim: int           # D_I
    topk: int              # k
    heads: int             # H (MLA query heads, MQA mode: one shared latent)
    d_qk: int              # D_K (latent + rope)
    d_v: int               # D_V (value = first D_V dims of the latent)
    dtype: str             # "fp32" or "bf16": q, kv, q_I storage and MLA output
    idx_key_dtype: str     # "fp32", "bf16", "fp8" or "fp4"
    page_size: int = 0     # 0: contiguous KV cache; else paged MLA KV cache
    compress_m: int = 1    # CSA pooling factor m (raw context = ctx * m)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_qk)

    @property
    def raw_ctx(self) -> int:
        return self.ctx * self.compress_m

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the path, by what they are.
TINY_PREFILL_FP32 = Workload(
    name="tiny_prefill_fp32_L256", mode="prefill", batch=1, ctx=256, rows=256,
    idx_heads=4, idx_dim=32, topk=64, heads=8, d_qk=64, d_v=64,
    dtype="fp32", idx_key_dtype="fp32")
DECODE_32K = Workload(
    name="dsa_decode_bf16_B32_L32768_k2048", mode="decode", batch=32, ctx=32768, rows=32,
    idx_heads=64, idx_dim=128, topk=2048, heads=128, d_qk=576, d_v=512,
    dtype="bf16", idx_key_dtype="bf16")
PREFILL_16K = Workload(
    name="dsa_prefill_bf16_T16384_k2048", mode="prefill", batch=1, ctx=16384, rows=16384,
    idx_heads=64, idx_dim=128, topk=2048, heads=128, d_qk=576, d_v=512,
    dtype="bf16", idx_key_dtype="bf16")
CSA_DECODE_1M = Workload(
    name="csa_decode_bf16_B4_L1048576_m4_k1024", mode="decode", batch=4, ctx=262144, rows=4,
    idx_heads=64, idx_dim=128, topk=1024, heads=128, d_qk=576, d_v=512,
    dtype="bf16", idx_key_dtype="bf16", compress_m=4)
DECODE_128K_FP8_PAGED = Workload(
    name="dsa_decode_fp8idx_paged64_B64_L131072_k2048", mode="decode", batch=64, ctx=131072,
    rows=64, idx_heads=64, idx_dim=128, topk=2048, heads=128, d_qk=576, d_v=512,
    dtype="bf16", idx_key_dtype="fp8", page_size=64)

ALL = [TINY_PREFILL_FP32, DECODE_32K, PREFILL_16K, CSA_DECODE_1M, DECODE_128K_FP8_PAGED]
BY_NAME = {w.name: w for w in ALL}

FP8_E4M3_MAX = 448.0

_TORCH_DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


def _normal(g: torch.Generator, shape, dim: int, device) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    return x.mul_(1.0 / math.sqrt(dim))


def quantize_fp8_rows(x: torch.Tensor):
    """Storage format of fp8 indexer keys: e4m3fn codes (uint8) plus one fp32
    scale per row, scale = amax(row)/448 (1.0 for an all-zero row)."""
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / FP8_E4M3_MAX, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp_(-FP8_E4M3_MAX, FP8_E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.to(torch.float32)


FP4_E2M1_MAX = 6.0
_E2M1_MAG = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def quantize_fp4_rows(x: torch.Tensor):
    """x [..., D] -> (codes uint8 [..., D/2], scale fp32 [...]): e2m1 codes,
    two per byte (dim 2j in the low nibble), with one scale per row,
    scale = amax(row) / 6; each value goes to the nearest e2m1 magnitude
    (ties to the smaller one), saturating at 6."""
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / FP4_E2M1_MAX, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp(-FP4_E2M1_MAX, FP4_E2M1_MAX)
    mags = torch.tensor(_E2M1_MAG, dtype=y.dtype, device=y.device)
    code = (y.abs().unsqueeze(-1) - mags).abs().argmin(dim=-1).to(torch.uint8)
    code = code | torch.where(y < 0, torch.full_like(code, 8), torch.zeros_like(code))
    packed = code[..., 0::2] | (code[..., 1::2] << 4)
    return packed.contiguous(), scale.to(torch.float32)


def row_metadata(w: Workload, rows: Optional[int] = None, device="cpu"):
    """row_batch[r]: which cache query row r reads; row_pos[r]: the last key
    position it may see (keys s <= row_pos[r] are visible)."""
    n = w.rows if rows is None else rows
    if w.mode == "prefill":
        assert w.batch == 1
        rb = torch.zeros(n, dtype=torch.int32)
        rp = torch.arange(n, dtype=torch.int32)
    else:
        rb = torch.arange(n, dtype=torch.int32) % w.batch
        rp = torch.full((n,), w.ctx - 1, dtype=torch.int32)
    return rb.to(device), rp.to(device)


def generate(w: Workload, device="cpu", seed: int = 0, parts=("indexer", "mla")) -> Dict[str, torch.Tensor]:
    """Draw one step's inputs. Tensors are created on ``device`` with a
    ``torch.Generator`` of that device seeded with ``seed`` (host and CUDA
    generators give different streams; each run uses one of them).

    Keys of the result: q_idx, w, k_idx, k_scale (fp8 only), q, kv,
    page_table (paged only), row_batch, row_pos.  For CSA workloads k_idx and
    kv hold the *raw* (unpooled) caches of length ctx*m.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    out: Dict[str, torch.Tensor] = {}
    dt = _TORCH_DT[w.dtype]
    L_raw = w.raw_ctx
    # --- indexer inputs (draw order: q_I, w, k_I) ---
    q_idx = _normal(g, (w.rows, w.idx_heads, w.idx_dim), w.idx_dim, dev)
    wts = torch.rand((w.rows, w.idx_heads), generator=g, dtype=torch.float32, device=dev)
    k_idx = _normal(g, (w.batch, L_raw, w.idx_dim), w.idx_dim, dev)
    if "indexer" in parts:
        out["q_idx"] = q_idx.to(dt)
        out["w"] = wts
        if w.idx_key_dtype == "fp8":
            out["k_idx"], out["k_scale"] = quantize_fp8_rows(k_idx.to(torch.bfloat16).float())
        elif w.idx_key_dtype == "fp4":
            out["k_idx"], out["k_scale"] = quantize_fp4_rows(k_idx.to(torch.bfloat16).float())
        else:
            out["k_idx"] = k_idx.to(_TORCH_DT[w.idx_key_dtype])
    del q_idx, wts, k_idx
    # --- MLA inputs (draw order: q, kv, page_table) ---
    if "mla" in parts:
        q = _normal(g, (w.rows, w.heads, w.d_qk), w.d_qk, dev)
        out["q"] = q.to(dt)
        del q
        if w.page_size:
            assert L_raw % w.page_size == 0
            n_pages = w.batch * L_raw // w.page_size
            kv = _normal(g, (n_pages, w.page_size, w.d_qk), w.d_qk, dev).to(dt)
            perm = torch.randperm(n_pages, generator=g, device=dev).to(torch.int32)
            out["kv"] = kv
            out["page_table"] = perm.view(w.batch, L_raw // w.page_size)
        else:
            out["kv"] = _normal(g, (w.batch, L_raw, w.d_qk), w.d_qk, dev).to(dt)
    rb, rp = row_metadata(w, device=dev)
    out["row_batch"], out["row_pos"] = rb, rp
    return out


def synthetic_scores(rows: int, ctx: int, device="cpu", seed: int = 0, ties: bool = True) -> torch.Tensor:
    """fp32 score matrices for exercising the selection step on its own:
    a mix of continuous values, exact duplicates, zeros of both signs and
    -inf, so that tie-breaking is exercised. Not produced by any scorer."""
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed)
    x = torch.randn((rows, ctx), generator=g, dtype=torch.float32, device=device)
    if ties:
        # round a third of the values to a coarse grid -> many exact duplicates
        sel = torch.rand((rows, ctx), generator=g, device=device) < 0.33
        x = torch.where(sel, torch.round(x * 4.0) / 4.0, x)
        z = torch.rand((rows, ctx), generator=g, device=device)
        x = torch.where(z < 0.05, torch.zeros_like(x), x)
        x = torch.where((z >= 0.05) & (z < 0.08), torch.full_like(x, -0.0), x)
        x = torch.where((z >= 0.08) & (z < 0.09), torch.full_like(x, float("-inf")), x)
    return x


# ---- inputs of the step before the path (the indexer's own projections) -------
#
# Recipe (one generator, fixed draw order): the query latent c_q ~ N(0,1) and
# the hidden states h ~ N(0,1) (bf16); stand-in weights, since no trained ones
# exist here: the norm gain ~ U(0.5, 1.5) (fp32) and every projection
# ~ N(0,1)/sqrt(fan_in) (bf16); positions uniform in [0, max_pos); cache slots
# distinct random rows of the cache, each token's slot -1 (not stored) with
# probability `skip`.  The rotary tables are the usual ones,
# angle(p, i) = p * base^(-2i/d_rope), computed in float64 and rounded to fp32.

@dataclasses.dataclass(frozen=True)
class PrepareShape:
    tokens: int
    d_c: int           # query latent width
    d_model: int       # hidden size
    n_heads: int = 64  # indexer heads
    head_dim: int = 128
    d_rope: int = 64
    max_pos: int = 4096
    cache_rows: int = 8192


def rope_tables(max_pos: int, d_rope: int, base: float = 10000.0):
    """(cos, sin) fp32 [max_pos, d_rope/2]."""
    i = torch.arange(d_rope // 2, dtype=torch.float64)
    theta = base ** (-2.0 * i / d_rope)
    ang = torch.arange(max_pos, dtype=torch.float64).unsqueeze(1) * theta.unsqueeze(0)
    return torch.cos(ang).float().contiguous(), torch.sin(ang).float().contiguous()


def make_prepare_inputs(s: PrepareShape, seed: int = 0, skip: float = 0.1) -> Dict[str, torch.Tensor]:
    g = torch.Generator().manual_seed(seed)
    T = s.tokens
    out = {
        "c_q": torch.randn(T, s.d_c, generator=g).to(torch.bfloat16),
        "h": torch.randn(T, s.d_model, generator=g).to(torch.bfloat16),
        "gamma": (0.5 + torch.rand(s.d_c, generator=g)).float(),
        "wq_b": (torch.randn(s.n_heads * s.head_dim, s.d_c, generator=g) / math.sqrt(s.d_c)).to(torch.bfloat16),
        "wk": (torch.randn(s.head_dim, s.d_model, generator=g) / math.sqrt(s.d_model)).to(torch.bfloat16),
        "w_proj": (torch.randn(s.n_heads, s.d_model, generator=g) / math.sqrt(s.d_model)).to(torch.bfloat16),
        "pos": torch.randint(0, s.max_pos, (T,), generator=g, dtype=torch.int32),
    }
    slot = torch.randperm(s.cache_rows, generator=g)[:T].to(torch.int64)
    drop = torch.rand(T, generator=g) < skip
    out["slot"] = torch.where(drop, torch.full_like(slot, -1), slot)
    if s.d_rope:
        out["rope_cos"], out["rope_sin"] = rope_tables(s.max_pos, s.d_rope)
    return out
