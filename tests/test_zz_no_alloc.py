"""dsa_sparse_mla_noalloc: the sparse MLA entry point that allocates nothing
and keeps the partials of a split key list in the library's fixed device
scratch.  It must give what dsa_sparse_mla gives (with a caller workspace)
on the same inputs, call after call, without touching the allocator."""
import numpy as np
import pytest
import torch

import workloads
from helpers import ATOL_LSE, ATOL_OUT

dsa = pytest.importorskip("sparse_attention_logits_b200")

pytestmark = pytest.mark.gpu


def _idx(rows, k, ctx, seed, pad=0):
    g = torch.Generator().manual_seed(seed)
    idx = torch.stack([torch.randperm(ctx, generator=g)[:k - pad] for _ in range(rows)]).to(torch.int32)
    if pad:
        idx = torch.cat([idx, torch.full((rows, pad), -1, dtype=torch.int32)], 1)
    return idx


@pytest.mark.parametrize("wl,k,pad", [
    (workloads.DECODE_32K.with_(batch=4, rows=32, ctx=4096), 2048, 0),          # 2 splits per row
    (workloads.DECODE_128K_FP8_PAGED.with_(batch=2, rows=2, ctx=4096), 2048, 13),  # many splits, paged
    (workloads.DECODE_32K.with_(batch=2, rows=80, ctx=1024), 256, 3),           # no split: scratch unused
], ids=["decode_B4_rows32", "paged_rows2", "rows80_nosplit"])
def test_noalloc_matches_workspace_entry(cuda_device, wl, k, pad):
    inp = workloads.generate(wl, parts=("mla",))
    dv = {n: t.to(cuda_device) for n, t in inp.items()}
    pt = dv.get("page_table")
    rows, H = wl.rows, wl.heads
    out = torch.empty((rows, H, wl.d_v), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((rows, H), dtype=torch.float32, device=cuda_device)
    for call, seed in enumerate((21, 22)):            # two calls in a row, different key lists
        idx = _idx(rows, k, wl.ctx, seed, pad).to(cuda_device)
        ref_o, ref_l = dsa.sparse_mla(dv["q"], dv["kv"], idx, dv["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                                      page_table=pt)
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated(cuda_device)
        dsa.sparse_mla_noalloc(dv["q"], dv["kv"], idx, dv["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                               out, lse, page_table=pt)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated(cuda_device) == before
        assert dsa.get_device_error(cuda_device) == dsa.DSA_OK
        err = (out.float() - ref_o.float()).abs().max().item()
        o_l, r_l = lse.cpu().numpy(), ref_l.cpu().numpy()
        assert np.array_equal(np.isneginf(o_l), np.isneginf(r_l))
        fin = np.isfinite(r_l)
        lerr = float(np.abs(o_l[fin] - r_l[fin]).max()) if fin.any() else 0.0
        assert err <= ATOL_OUT["bf16"], (call, err)
        assert lerr <= ATOL_LSE["bf16"], (call, lerr)
