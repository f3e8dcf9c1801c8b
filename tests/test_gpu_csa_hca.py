"""GPU parity of the two variants of the attention step for DeepSeek-V4's
compressed attention, through the C ABI:

  csa_core_attention  the selected compressed entries plus a window of raw
                      cache rows, attended together;
  hca_attention       dense attention over every visible entry of a cache
                      pooled 128:1.

The compressed caches are pooled on the GPU (csa_compress, checked bit-exact
elsewhere) and the oracle runs on those same bytes.  Tolerances are the
attention rule of the parity tests: max-abs 2e-2 for bf16 outputs, 1e-4 for
fp32."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import ATOL_LSE, ATOL_OUT

dsa = pytest.importorskip("sparse_attention_logits_b200")

pytestmark = pytest.mark.gpu


def _caches(B, Lraw, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    raw = (torch.randn(B, Lraw, D, generator=g) / math.sqrt(D)).to(dtype)
    return raw, g


def _pooled(raw_dev, m):
    kvc = dsa.csa_compress(raw_dev, m)
    torch.cuda.synchronize()
    return kvc


def _check(out, lse, ro, rl, dtype):
    key = "bf16" if dtype == torch.bfloat16 else "fp32"
    err = np.abs(out.float().cpu().numpy() - ro).max()
    lerr = np.abs(lse.cpu().numpy() - rl)
    lerr = np.where(np.isneginf(rl) & np.isneginf(lse.cpu().numpy()), 0.0, lerr).max()
    assert err <= ATOL_OUT[key], err
    assert lerr <= ATOL_LSE[key], lerr


# (rows, B, raw length, k, window, window end, page size, dtype, heads, d_qk, d_v, sink rows)
CSA_CASES = {
    "bf16_rows4_split": (4, 4, 4096, 256, 128, "end", 0, torch.bfloat16, 128, 576, 512, 0),
    "bf16_rows32_fused_splits": (32, 4, 4096, 256, 128, "end", 0, torch.bfloat16, 128, 576, 512, 0),
    "bf16_window_clipped": (4, 2, 2048, 192, 128, "early", 0, torch.bfloat16, 128, 576, 512, 0),
    "bf16_window_only": (3, 3, 1024, 0, 100, "end", 0, torch.bfloat16, 128, 576, 512, 0),
    "bf16_paged": (5, 2, 4096, 300, 64, "end", 64, torch.bfloat16, 128, 576, 512, 0),
    "fp32_small_heads": (6, 2, 256, 16, 32, "early", 0, torch.float32, 8, 64, 64, 0),
    # attention sink: the first raw rows beside the window
    "bf16_sink_rows4_split": (4, 4, 4096, 256, 128, "end", 0, torch.bfloat16, 128, 576, 512, 4),
    "bf16_sink_rows32_fused_splits": (32, 4, 4096, 256, 128, "end", 0, torch.bfloat16, 128, 576, 512, 64),
    "bf16_sink_window_overlap": (6, 2, 2048, 192, 128, "overlap", 0, torch.bfloat16, 128, 576, 512, 100),
    "bf16_sink_only": (3, 3, 1024, 0, 0, "overlap", 0, torch.bfloat16, 128, 576, 512, 70),
    "bf16_sink_paged": (5, 2, 4096, 300, 64, "end", 64, torch.bfloat16, 128, 576, 512, 16),
    "fp32_sink_small_heads": (6, 2, 256, 16, 32, "overlap", 0, torch.float32, 8, 64, 64, 20),
}


@pytest.mark.parametrize("case", list(CSA_CASES), ids=list(CSA_CASES))
def test_csa_core_attention_matches_oracle(cuda_device, case):
    rows, B, Lraw, k, W, end, page, dtype, H, DK, DV, S = CSA_CASES[case]
    raw, g = _caches(B, Lraw, DK, dtype, seed=41)
    raw_d = raw.to(cuda_device)
    kvc = _pooled(raw_d, 4)
    Lc = Lraw // 4
    q = (torch.randn(rows, H, DK, generator=g) / math.sqrt(DK)).to(dtype)
    rb = (torch.arange(rows) % B).to(torch.int32)
    if end == "end":
        pos = torch.full((rows,), Lraw - 1, dtype=torch.int32)
    elif end == "early":                    # windows that start before position 0
        pos = torch.tensor([(7 * t) % W for t in range(rows)], dtype=torch.int32)
    else:                                   # sink and window meet, overlap or the query sits inside the sink
        pos = torch.tensor([[0, S // 2, S - 1, S + W - 2, S + W - 1, S + W + 37][t % 6] for t in range(rows)],
                           dtype=torch.int32)
    idx = None
    if k:
        idx = torch.stack([torch.randperm(Lc, generator=g)[:k] for _ in range(rows)]).to(torch.int32)
        idx[:, -5:] = -1                    # a few unused slots
    scale = 1.0 / math.sqrt(DK)
    table = None
    kv_arg = kvc
    if page:
        n_pages = B * Lc // page
        perm = torch.randperm(n_pages, generator=g)
        pages = torch.empty((n_pages, page, DK), dtype=dtype, device=cuda_device)
        pages[perm.to(cuda_device)] = kvc.reshape(n_pages, page, DK)
        table = perm.view(B, Lc // page).to(torch.int32)
        kv_arg = pages
    out, lse = dsa.csa_core_attention(q.to(cuda_device), kv_arg, None if idx is None else idx.to(cuda_device),
                                      rb.to(cuda_device), scale, DV, Lc, raw_d, pos.to(cuda_device), W,
                                      page_table=None if table is None else table.to(cuda_device), n_sink=S)
    assert dsa.get_device_error(cuda_device) == dsa.DSA_OK
    ro, rl = oracle.csa_core_attention(q, kvc.cpu(), idx, rb, scale, DV, Lc, raw, pos, W, n_sink=S)
    _check(out, lse, ro, rl, dtype)


# (rows, B, raw length, row_last rule, dtype, heads, d_qk, d_v)
HCA_CASES = {
    "bf16_decode_rows4": (4, 2, 16384, "all", torch.bfloat16, 128, 576, 512),
    "bf16_decode_rows32_fused_splits": (32, 4, 16384, "all", torch.bfloat16, 128, 576, 512),
    "bf16_causal_prefix": (6, 1, 8192, "prefix", torch.bfloat16, 128, 576, 512),
    "fp32_small_heads": (5, 2, 4096, "prefix", torch.float32, 8, 64, 64),
}


@pytest.mark.parametrize("case", list(HCA_CASES), ids=list(HCA_CASES))
def test_hca_attention_matches_oracle(cuda_device, case):
    rows, B, Lraw, rule, dtype, H, DK, DV = HCA_CASES[case]
    raw, g = _caches(B, Lraw, DK, dtype, seed=43)
    kvc = _pooled(raw.to(cuda_device), 128)
    Lc = Lraw // 128
    q = (torch.randn(rows, H, DK, generator=g) / math.sqrt(DK)).to(dtype)
    rb = (torch.arange(rows) % B).to(torch.int32)
    if rule == "all":
        last = torch.full((rows,), Lc - 1, dtype=torch.int32)
    else:                                   # causal prefill: -1 (nothing complete yet), 0, ..., all
        last = torch.tensor([[-1, 0, 1, Lc // 3, Lc - 2, Lc - 1][t % 6] for t in range(rows)], dtype=torch.int32)
    scale = 1.0 / math.sqrt(DK)
    out, lse = dsa.hca_attention(q.to(cuda_device), kvc, rb.to(cuda_device), last.to(cuda_device), scale, DV)
    dsa.get_device_error(cuda_device)
    ro, rl = oracle.hca_attention(q, kvc.cpu(), rb, last, scale, DV)
    _check(out, lse, ro, rl, dtype)
    if rule != "all":
        none = (last < 0).numpy()
        assert np.all(out.float().cpu().numpy()[none] == 0)
