"""GPU parity at the full sizes of the four large workloads, in the launch
configuration bench.py times: whole batches go through the same library calls
(csa_compress for CSA, indexer -> top-k -> sparse MLA), and sampled query rows
are checked against the oracle, which computes them one by one.

Per sampled row: the index scores (relative 1e-4 of the row's largest
magnitude), the selected set (equal to the oracle's up to near-ties, see
tests/helpers.py) and the attention output and lse on the oracle's indices
(max-abs 2e-2, bf16), the latter taken from a full-batch MLA launch in which
the sampled rows' index lists were replaced by the oracle's.  CSA: the pooled
rows feeding the sampled checks are also compared bit-exactly.

Every oracle input is drawn by the seeded generator (the pooled caches of CSA
are pooled by the oracle itself); nothing the CUDA path computes is fed to it.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import ATOL_LSE, ATOL_OUT, check_index_sets, check_sorted_unique

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_logits_b200")

CASES = [
    (workloads.DECODE_32K, [0, 17, 31]),
    (workloads.PREFILL_16K, [0, 1, 2046, 2047, 2048, 9001, 16383]),
    (workloads.CSA_DECODE_1M, [0, 3]),
    (workloads.DECODE_128K_FP8_PAGED, [5, 62]),
]


def _step(wl, dv):
    """The bench's step on the full batch; returns the pooled caches and results."""
    k_idx, kv = dv["k_idx"], dv["kv"]
    if wl.compress_m > 1:
        k_idx = dsa.csa_compress(k_idx, wl.compress_m)
        kv = dsa.csa_compress(kv, wl.compress_m)
    dev = kv.device
    logits = torch.empty((wl.rows, wl.ctx), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.rows, wl.topk), dtype=torch.int32, device=dev)
    n = dsa.topk_workspace_size(wl.rows, wl.ctx, wl.topk)
    tws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    n = dsa.sparse_mla_workspace_size(wl.rows, wl.topk, wl.heads, wl.d_qk, wl.d_v, dv["q"].dtype)
    mws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    dsa.indexer_logits(dv["q_idx"], dv["w"], k_idx, dv["row_batch"], dv["row_pos"], k_scale=dv.get("k_scale"),
                       out=logits)
    dsa.topk(logits, dv["row_pos"], wl.topk, ctx_len=wl.ctx, out=idx, workspace=tws)
    out, lse = dsa.sparse_mla(dv["q"], kv, idx, dv["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                              page_table=dv.get("page_table"), workspace=mws)
    dsa.get_device_error()
    return k_idx, kv, logits, idx, out, lse, mws


def _oracle_keys(wl, dv, b):
    """Indexer keys of cache b for the oracle (pooled by the oracle for CSA)."""
    raw = dv["k_idx"][b:b + 1]
    if wl.compress_m > 1:
        return oracle.csa_compress(raw, wl.compress_m)
    return oracle._host(raw)


def _oracle_rows(wl, dv, b, keys):
    """The selected latent rows c_s (s in keys) of cache b, as a [1, n, 576]
    cache for the oracle (pooled by the oracle for CSA)."""
    keys = torch.as_tensor(np.asarray(keys, dtype=np.int64), device=dv["kv"].device)
    if wl.compress_m > 1:
        m = wl.compress_m
        raw_ids = (keys[:, None] * m + torch.arange(m, device=keys.device)[None, :]).reshape(-1)
        raw = dv["kv"][b, raw_ids].unsqueeze(0)
        return oracle.csa_compress(raw, m)
    if "page_table" in dv:
        pt = dv["page_table"][b].long()
        rows = dv["kv"][pt[keys // wl.page_size], keys % wl.page_size]
        return oracle._host(rows.unsqueeze(0))
    return oracle._host(dv["kv"][b, keys].unsqueeze(0))


@pytest.mark.parametrize("wl,sample", CASES, ids=[c[0].name for c in CASES])
def test_full_size_sampled_rows(cuda_device, wl, sample):
    dv = workloads.generate(wl, device=cuda_device, seed=0)
    k_pooled, kv_pooled, logits, idx, _, _, mws = _step(wl, dv)
    rb = dv["row_batch"].cpu().numpy()
    rp = dv["row_pos"].cpu().numpy()
    gidx_all = idx.cpu().numpy()
    ref_lists = {}
    for t in sample:
        b, pos = int(rb[t]), int(rp[t])
        keys_b = _oracle_keys(wl, dv, b)
        if wl.compress_m > 1:   # pooling is bit-exact on the blocks this row reads
            blocks = np.random.default_rng(t).integers(0, wl.ctx, 64)
            assert np.array_equal(oracle._host(k_pooled[b, blocks]), keys_b[0, blocks])
        ks = dv["k_scale"][b:b + 1] if "k_scale" in dv else None
        scores = oracle.index_scores(dv["q_idx"][t:t + 1], dv["w"][t:t + 1], keys_b, [0], [pos], k_scale=ks)
        g = logits[t, :pos + 1].double().cpu().numpy()
        scale = max(1e-30, np.abs(scores[0, :pos + 1]).max())
        assert np.abs(g - scores[0, :pos + 1]).max() / scale <= 1e-4, f"row {t}: index scores"
        ref = oracle.topk(scores, [pos], wl.topk)
        check_sorted_unique(gidx_all[t:t + 1], np.array([pos + 1]))
        check_index_sets(gidx_all[t:t + 1], scores, ref, wl.topk)
        ref_lists[t] = ref[0]
    # attention on the oracle's indices, from a full-batch launch
    idx2 = idx.clone()
    for t, ref in ref_lists.items():
        sel = np.sort(ref[ref >= 0])
        row = np.full(wl.topk, -1, dtype=np.int32)
        row[:len(sel)] = sel
        idx2[t] = torch.from_numpy(row).to(idx.device)
    out2, lse2 = dsa.sparse_mla(dv["q"], kv_pooled, idx2, dv["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                                page_table=dv.get("page_table"), workspace=mws)
    dsa.get_device_error()
    for t, ref in ref_lists.items():
        b = int(rb[t])
        sel = ref[ref >= 0]
        rows = _oracle_rows(wl, dv, b, sel)
        local = np.arange(len(sel), dtype=np.int32)[None, :]
        ro, rl, _ = oracle.sparse_mla(dv["q"][t:t + 1], rows, local, [0], wl.softmax_scale, wl.d_v, len(sel))
        err = np.abs(out2[t].float().cpu().numpy() - ro[0]).max()
        lerr = np.abs(lse2[t].cpu().numpy() - rl[0]).max()
        assert err <= ATOL_OUT[wl.dtype], f"row {t}: out max-abs {err:.3g}"
        assert lerr <= ATOL_LSE[wl.dtype], f"row {t}: lse max-abs {lerr:.3g}"
    del dv, k_pooled, kv_pooled, logits, idx, idx2, out2, lse2, mws
    torch.cuda.empty_cache()


V4_WINDOW = 128
V4_SINK = 4


def test_full_size_v4_variants(cuda_device):
    """The 1M-token CSA shapes (4 sequences of 1,048,576 raw tokens) through
    the two variants of the attention step, in the bench's launch
    configuration: CSA core attention over 1024 seeded pooled entries plus a
    128-row window and a 4-row sink of raw rows, and HCA over all 8,192 entries of the 128:1
    pooled cache.  Sampled rows are checked against the oracle, which pools
    the raw seeded rows itself."""
    wl = workloads.CSA_DECODE_1M
    dv = workloads.generate(wl, device=cuda_device, seed=0, parts=("mla",))
    raw = dv["kv"]                                               # [4, 1048576, 576] bf16
    B, Lraw = raw.shape[0], raw.shape[1]
    rows = wl.rows
    rb = dv["row_batch"]
    pos = torch.full((rows,), Lraw - 1, dtype=torch.int32, device=cuda_device)
    # --- CSA core attention: pooled entries + window ---
    kv_c = dsa.csa_compress(raw, wl.compress_m)
    g = torch.Generator().manual_seed(5)
    idx = torch.stack([torch.randperm(wl.ctx, generator=g)[:wl.topk] for _ in range(rows)]).to(torch.int32)
    out, lse = dsa.csa_core_attention(dv["q"], kv_c, idx.to(cuda_device), rb, wl.softmax_scale, wl.d_v, wl.ctx,
                                      raw, pos, V4_WINDOW, n_sink=V4_SINK)
    assert dsa.get_device_error() == dsa.DSA_OK
    for t in (0, rows - 1):
        b = int(rb[t])
        sel = idx[t].long().to(cuda_device)
        raw_ids = (sel[:, None] * wl.compress_m + torch.arange(wl.compress_m, device=cuda_device)[None, :]).reshape(-1)
        pooled = oracle.csa_compress(raw[b, raw_ids].unsqueeze(0), wl.compress_m)            # [1, 1024, 576]
        pooled_t = torch.from_numpy(pooled.view(np.int16)).view(torch.bfloat16)
        # the oracle's raw cache: the sink rows, then the window's rows (the query at its end)
        win = torch.cat([raw[b, :V4_SINK], raw[b, Lraw - V4_WINDOW:]]).unsqueeze(0).cpu()
        ro, rl = oracle.csa_core_attention(dv["q"][t:t + 1].cpu(), pooled_t, torch.arange(wl.topk).view(1, -1), [0],
                                           wl.softmax_scale, wl.d_v, wl.topk, win, [V4_SINK + V4_WINDOW - 1],
                                           V4_WINDOW, n_sink=V4_SINK)
        assert np.abs(out[t].float().cpu().numpy() - ro[0]).max() <= ATOL_OUT["bf16"], f"csa row {t}"
        assert np.abs(lse[t].cpu().numpy() - rl[0]).max() <= ATOL_LSE["bf16"], f"csa row {t} lse"
    del kv_c, out, lse
    # --- HCA: every entry of the 128:1 pooled cache ---
    m_h = 128
    kv_h = dsa.csa_compress(raw, m_h)                                                       # [4, 8192, 576]
    last = torch.full((rows,), Lraw // m_h - 1, dtype=torch.int32, device=cuda_device)
    out, lse = dsa.hca_attention(dv["q"], kv_h, rb, last, wl.softmax_scale, wl.d_v)
    dsa.get_device_error()
    for t in (0, rows - 1):
        b = int(rb[t])
        pooled = oracle.csa_compress(raw[b:b + 1], m_h)                                    # [1, 8192, 576]
        assert np.array_equal(oracle._host(kv_h[b:b + 1]), pooled), f"hca pooling, cache {b}"
        pooled_t = torch.from_numpy(pooled.view(np.int16)).view(torch.bfloat16)
        ro, rl = oracle.hca_attention(dv["q"][t:t + 1].cpu(), pooled_t, [0], [Lraw // m_h - 1], wl.softmax_scale,
                                      wl.d_v)
        assert np.abs(out[t].float().cpu().numpy() - ro[0]).max() <= ATOL_OUT["bf16"], f"hca row {t}"
        assert np.abs(lse[t].cpu().numpy() - rl[0]).max() <= ATOL_LSE["bf16"], f"hca row {t} lse"
    del dv, raw, kv_h, out, lse
    torch.cuda.empty_cache()
