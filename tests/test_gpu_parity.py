"""GPU parity: every step of the path through the C ABI against the CPU oracle,
at sizes the oracle finishes in seconds (several tiles plus ragged tails) and
on the edge cases of each step.

Rules (see tests/helpers.py): compression bit-exact; top-k on given fp32
scores bit-exact; chained indices equal up to near-ties (1e-3 relative of the
k-th score); attention on the oracle's indices within 2e-2 (bf16) / 1e-4
(fp32) max-abs; index scores within 1e-4 of the row's largest magnitude.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import ATOL_LSE, ATOL_OUT, check_index_sets, check_sorted_unique

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_logits_b200")


def _cuda(d, dev):
    return {k: v.to(dev) for k, v in d.items()}


def _logits_close(gpu, ora, pos):
    for r in range(ora.shape[0]):
        n = int(pos[r]) + 1
        o = ora[r, :n]
        g = gpu[r, :n].astype(np.float64)
        scale = max(1e-30, np.abs(o).max())
        err = np.abs(g - o).max() / scale
        assert err <= 1e-4, f"row {r}: relative score error {err:.3g}"


# ------------------------------------------------------------- compress ----

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,L,D,m", [(2, 64, 576, 4), (3, 36, 128, 4), (1, 12, 64, 3), (2, 8, 576, 1), (1, 4096, 128, 4)])
def test_compress_bit_exact(cuda_device, dtype, B, L, D, m):
    g = torch.Generator().manual_seed(B * 1000 + L + D + m)
    src = (torch.randn(B, L, D, generator=g) / D ** 0.5).to(dtype)
    got = dsa.csa_compress(src.to(cuda_device), m).cpu()
    ref = oracle.csa_compress(src, m)
    got_h = oracle._host(got)
    assert got_h.shape == ref.shape
    assert np.array_equal(got_h, ref), f"{(got_h != ref).sum()} elements differ"


# -------------------------------------------------------------- indexer ----

@pytest.mark.parametrize("wl", [
    workloads.TINY_PREFILL_FP32,
    workloads.DECODE_32K.with_(batch=3, rows=3, ctx=1000),              # ragged tail
    workloads.PREFILL_16K.with_(ctx=300, rows=300),                     # causal, ragged, 1 query per tile
    workloads.PREFILL_16K.with_(ctx=1001, rows=1001),                   # causal, 4 queries per tile, ragged
    workloads.DECODE_128K_FP8_PAGED.with_(batch=2, rows=2, ctx=4096 + 64),
    workloads.DECODE_128K_FP8_PAGED.with_(batch=5, rows=5, ctx=777),    # fp8, ragged tail
    workloads.DECODE_128K_FP8_PAGED.with_(batch=3, rows=4, ctx=4096 + 64, idx_key_dtype="fp4"),
    workloads.DECODE_128K_FP8_PAGED.with_(batch=5, rows=5, ctx=777, idx_key_dtype="fp4"),    # fp4, ragged tail
], ids=lambda w: f"{w.name}-{w.idx_key_dtype}-ctx{w.ctx}")
def test_indexer_matches_oracle(cuda_device, wl):
    inp = workloads.generate(wl, parts=("indexer",))
    dv = _cuda(inp, cuda_device)
    got = dsa.indexer_logits(dv["q_idx"], dv["w"], dv["k_idx"], dv["row_batch"], dv["row_pos"],
                             k_scale=dv.get("k_scale")).cpu().numpy()
    ref = oracle.index_scores(inp["q_idx"], inp["w"], inp["k_idx"], inp["row_batch"], inp["row_pos"],
                              k_scale=inp.get("k_scale"))
    _logits_close(got, ref, inp["row_pos"].numpy())


# ---------------------------------------------------------------- top-k ----

@pytest.mark.parametrize("rows,L,k,seed", [(7, 1000, 64, 0), (4, 32768, 2048, 1), (3, 5000, 2048, 2),
                                           (2, 262144, 1024, 3), (5, 300, 300, 4), (3, 129, 1, 5),
                                           (9, 200000, 2048, 6)])
def test_topk_bit_exact_on_given_scores(cuda_device, rows, L, k, seed):
    x = workloads.synthetic_scores(rows, L, seed=seed)
    pos = torch.tensor([L - 1 - (r * 37) % max(1, L // 3) for r in range(rows)], dtype=torch.int32)
    got = dsa.topk(x.to(cuda_device), pos.to(cuda_device), k).cpu().numpy()
    check_sorted_unique(got, pos.numpy() + 1)
    ref = oracle.topk(x, pos, k)
    for r in range(rows):
        assert np.array_equal(np.sort(got[r][got[r] >= 0]), np.sort(ref[r][ref[r] >= 0])), f"row {r}"


def test_topk_rows_not_16_byte_aligned(cuda_device):
    # ld = L + 3: most rows start off a 16-byte boundary, so every CTA of a
    # row's cluster takes the scalar load path (L = 100,001 keys: 8 CTAs per row)
    rows, L, k = 4, 100001, 2048
    x = workloads.synthetic_scores(rows, L + 3, seed=8)
    pos = torch.tensor([L - 1, L - 2, 70000, 5000], dtype=torch.int32)
    got = dsa.topk(x.to(cuda_device), pos.to(cuda_device), k, ctx_len=L).cpu().numpy()
    check_sorted_unique(got, pos.numpy() + 1)
    ref = oracle.topk(x[:, :L], pos, k)
    for r in range(rows):
        assert np.array_equal(got[r][got[r] >= 0], np.sort(ref[r][ref[r] >= 0])), f"row {r}"


@pytest.mark.parametrize("rows,L,ld_pad,k,seed", [(40, 131079, 0, 2048, 21), (80, 50000, 0, 1024, 22),
                                                    (40, 90001, 3, 2048, 23)])
def test_topk_clusters_in_several_waves(cuda_device, rows, L, ld_pad, k, seed):
    # more rows' clusters (2 to 4 CTAs per row) than a B200 holds at once, so the
    # launch runs in waves; ld = L + 3 puts most rows off a 16-byte boundary
    # (the scalar load path)
    x = workloads.synthetic_scores(rows, L + ld_pad, seed=seed)
    pos = torch.tensor([L - 1 - (r * 997) % (L // 2) for r in range(rows)], dtype=torch.int32)
    got = dsa.topk(x.to(cuda_device), pos.to(cuda_device), k, ctx_len=L).cpu().numpy()
    check_sorted_unique(got, pos.numpy() + 1)
    ref = oracle.topk(x[:, :L].contiguous(), pos, k)
    for r in range(rows):
        assert np.array_equal(got[r][got[r] >= 0], np.sort(ref[r][ref[r] >= 0])), f"row {r}"


def test_topk_edge_cases(cuda_device):
    L = 4100
    rows = []
    rows.append(torch.zeros(L))                                      # all equal: lowest positions win
    z = torch.zeros(L); z[1::2] = -0.0; rows.append(z)               # +0 / -0 tie
    rows.append(torch.full((L,), float("-inf")))                     # all -inf
    r = torch.full((L,), 1.0); r[4000:] = 2.0; rows.append(r)        # winners at the tail
    r = torch.arange(L, dtype=torch.float32); rows.append(-r)        # strictly decreasing
    x = torch.stack(rows)
    n = x.shape[0]
    for k, pos in [(1, [L - 1] * n), (2048, [L - 1] * n), (4100, [L - 1] * n), (4200, [L - 1] * n),
                   (64, [0, 1, 63, 64, 65]), (100, [99, 100, 101, 4099, 2000])]:
        p = torch.tensor(pos, dtype=torch.int32)
        got = dsa.topk(x.to(cuda_device), p.to(cuda_device), k).cpu().numpy()
        check_sorted_unique(got, p.numpy() + 1)
        ref = oracle.topk(x, p, k)
        for i in range(n):
            assert np.array_equal(got[i][got[i] >= 0], np.sort(ref[i][ref[i] >= 0])), (k, i)


# ------------------------------------------------------------ sparse MLA ----

def _random_idx(rows, k, ctx, g, pad=0):
    idx = torch.stack([torch.randperm(ctx, generator=g)[:k - pad] for _ in range(rows)]).to(torch.int32)
    if pad:
        idx = torch.cat([idx, torch.full((rows, pad), -1, dtype=torch.int32)], 1)
    return idx


@pytest.mark.parametrize("wl,pad", [
    (workloads.TINY_PREFILL_FP32.with_(ctx=256, rows=40), 5),
    (workloads.DECODE_32K.with_(batch=3, rows=5, ctx=3000), 0),
    (workloads.DECODE_32K.with_(batch=2, rows=3, ctx=2500), 700),
    (workloads.DECODE_128K_FP8_PAGED.with_(batch=2, rows=2, ctx=4096), 13),
    # two key splits per row, merged inside one 4-CTA cluster
    (workloads.DECODE_32K.with_(batch=4, rows=32, ctx=4096), 0),
    # same, with the second split of every row entirely unused slots
    (workloads.DECODE_32K.with_(batch=3, rows=26, ctx=3000), 1500),
], ids=lambda x: getattr(x, "name", str(x)))
def test_sparse_mla_on_given_indices(cuda_device, wl, pad):
    inp = workloads.generate(wl, parts=("mla",))
    g = torch.Generator().manual_seed(7)
    k = min(wl.topk, wl.ctx)
    idx = _random_idx(wl.rows, k, wl.ctx, g, pad)
    dv = _cuda(inp, cuda_device)
    out, lse = dsa.sparse_mla(dv["q"], dv["kv"], idx.to(cuda_device), dv["row_batch"], wl.softmax_scale, wl.d_v,
                              wl.ctx, page_table=dv.get("page_table"))
    ro, rl, _ = oracle.sparse_mla(inp["q"], inp["kv"], idx, inp["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                                  page_table=inp.get("page_table"))
    err = np.abs(out.float().cpu().numpy() - ro).max()
    lerr = np.abs(lse.cpu().numpy() - rl).max()
    assert err <= ATOL_OUT[wl.dtype], err
    assert lerr <= ATOL_LSE[wl.dtype], lerr


@pytest.mark.parametrize("order,rows", [("ascending", 3), ("descending", 3), ("shuffled", 3), ("ascending", 28)])
def test_sparse_mla_running_max_moves(cuda_device, order, rows):
    """Scores that climb by many e-folds across the key list, so the running
    maximum moves again and again (the lazy-rescale path of the kernel).  With
    28 rows each row's two key splits end with maxima far apart, which the
    in-cluster merge of the splits must weigh."""
    wl = workloads.DECODE_32K.with_(batch=2, rows=rows, ctx=4096)
    inp = workloads.generate(wl, parts=("mla",))
    q, kv = inp["q"].float(), inp["kv"].float()
    ramp = torch.arange(wl.ctx, dtype=torch.float32) * 0.02           # rope dims carry the ramp
    kv[:, :, 512:] = ramp.view(1, -1, 1)
    q[:, :, 512:] = 1.0
    q, kv = q.to(torch.bfloat16), kv.to(torch.bfloat16)
    g = torch.Generator().manual_seed(11)
    idx = _random_idx(wl.rows, 2048, wl.ctx, g)
    if order == "ascending":
        idx = idx.sort(dim=1).values
    elif order == "descending":
        idx = idx.sort(dim=1, descending=True).values
    out, lse = dsa.sparse_mla(q.to(cuda_device), kv.to(cuda_device), idx.to(cuda_device),
                              inp["row_batch"].to(cuda_device), wl.softmax_scale, wl.d_v, wl.ctx)
    ro, rl, _ = oracle.sparse_mla(q, kv, idx, inp["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx)
    assert np.abs(out.float().cpu().numpy() - ro).max() <= ATOL_OUT["bf16"]
    assert np.abs(lse.cpu().numpy() - rl).max() <= ATOL_LSE["bf16"]


def test_sparse_mla_all_slots_unused(cuda_device):
    wl = workloads.DECODE_32K.with_(batch=2, rows=2, ctx=512)
    inp = workloads.generate(wl, parts=("mla",))
    idx = torch.full((2, 300), -1, dtype=torch.int32)
    idx[1, 7] = 5
    dv = _cuda(inp, cuda_device)
    out, lse = dsa.sparse_mla(dv["q"], dv["kv"], idx.to(cuda_device), dv["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx)
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(o[0] == 0) and np.all(np.isneginf(l[0]))
    row = inp["kv"][1, 5, :512].float().numpy()
    assert np.abs(o[1] - row[None, :]).max() <= 1e-2


@pytest.mark.parametrize("kd", ["fp8", "fp4", "bf16"])
def test_indexer_partial_visibility(cuda_device, kd):
    # decode rows that see only a prefix of their sequence's keys: the narrow-key
    # path takes keys in units of 256, so prefixes ending inside, at and just past
    # a unit are all present; rows share sequences
    wl = workloads.DECODE_128K_FP8_PAGED.with_(batch=3, rows=8, ctx=777, idx_key_dtype=kd)
    inp = workloads.generate(wl, parts=("indexer",))
    inp["row_pos"] = torch.tensor([776, 0, 127, 255, 256, 511, 600, 1], dtype=torch.int32)
    dv = _cuda(inp, cuda_device)
    got = dsa.indexer_logits(dv["q_idx"], dv["w"], dv["k_idx"], dv["row_batch"], dv["row_pos"],
                             k_scale=dv.get("k_scale")).cpu().numpy()
    ref = oracle.index_scores(inp["q_idx"], inp["w"], inp["k_idx"], inp["row_batch"], inp["row_pos"],
                              k_scale=inp.get("k_scale"))
    _logits_close(got, ref, inp["row_pos"].numpy())


# ----------------------------------------------------------- whole chain ----

@pytest.mark.parametrize("wl", [
    workloads.TINY_PREFILL_FP32,
    workloads.DECODE_32K.with_(batch=4, rows=4, ctx=5000),
    workloads.PREFILL_16K.with_(ctx=1200, rows=1200, topk=256),
    workloads.DECODE_32K.with_(batch=4, rows=4, ctx=5000, idx_key_dtype="fp4"),
], ids=lambda w: f"{w.name}-{w.idx_key_dtype}-ctx{w.ctx}")
def test_chain_matches_oracle(cuda_device, wl):
    inp = workloads.generate(wl)
    dv = _cuda(inp, cuda_device)
    out, lse, idx = dsa.dsa_step(dv["q_idx"], dv["w"], dv["k_idx"], dv["row_batch"], dv["row_pos"], dv["q"], dv["kv"],
                                 wl.topk, wl.softmax_scale, wl.d_v, k_scale=dv.get("k_scale"),
                                 page_table=dv.get("page_table"))
    dsa.get_device_error()
    scores = oracle.index_scores(inp["q_idx"], inp["w"], inp["k_idx"], inp["row_batch"], inp["row_pos"],
                                 k_scale=inp.get("k_scale"))
    ref_idx = oracle.topk(scores, inp["row_pos"], wl.topk)
    gidx = idx.cpu().numpy()
    check_sorted_unique(gidx, inp["row_pos"].numpy() + 1)
    check_index_sets(gidx, scores, ref_idx, wl.topk)
    # attention checked on the oracle's indices
    out2, lse2 = dsa.sparse_mla(dv["q"], dv["kv"], torch.from_numpy(ref_idx).to(cuda_device), dv["row_batch"],
                                wl.softmax_scale, wl.d_v, wl.ctx, page_table=dv.get("page_table"))
    ro, rl, _ = oracle.sparse_mla(inp["q"], inp["kv"], ref_idx, inp["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx)
    assert np.abs(out2.float().cpu().numpy() - ro).max() <= ATOL_OUT[wl.dtype]
    assert np.abs(lse2.cpu().numpy() - rl).max() <= ATOL_LSE[wl.dtype]


def test_index_reuse_across_layers(cuda_device):
    # index reuse between adjacent layers (IndexShare): the second layer runs no
    # indexer or top-k of its own and attends over its own queries and latent
    # cache with the first layer's selection
    wl = workloads.DECODE_32K.with_(batch=3, rows=6, ctx=3000, topk=512)
    l1 = workloads.generate(wl, seed=21)
    l2 = workloads.generate(wl, seed=22)
    d1, d2 = _cuda(l1, cuda_device), _cuda(l2, cuda_device)
    _, _, idx = dsa.dsa_step(d1["q_idx"], d1["w"], d1["k_idx"], d1["row_batch"], d1["row_pos"], d1["q"], d1["kv"],
                             wl.topk, wl.softmax_scale, wl.d_v)
    out2, lse2 = dsa.sparse_mla(d2["q"], d2["kv"], idx, d2["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx)
    dsa.get_device_error()
    gidx = idx.cpu().numpy()
    ro, rl, _ = oracle.sparse_mla(l2["q"], l2["kv"], gidx, l2["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx)
    assert np.abs(out2.float().cpu().numpy() - ro).max() <= ATOL_OUT[wl.dtype]
    assert np.abs(lse2.cpu().numpy() - rl).max() <= ATOL_LSE[wl.dtype]
