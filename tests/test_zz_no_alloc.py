"""dsa_sparse_mla_noalloc: the sparse MLA entry point that allocates nothing
and keeps the partials of a split key list in the library's fixed device
scratch.  It must give what dsa_sparse_mla gives (with a caller workspace)
on the same inputs, call after call, without touching any allocator; where
the key list is split over several clusters (the cases that use the fixed
scratch) it is also checked against the oracle directly.

This file is collected last, so that a run that stops at the first failure
has already run every other test."""
import numpy as np
import pytest
import torch

import oracle
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


def _close(out, lse, ref_o, ref_l, what):
    o = out.float().cpu().numpy()
    r = ref_o.float().cpu().numpy() if torch.is_tensor(ref_o) else ref_o
    err = float(np.abs(o - r).max())
    o_l = lse.cpu().numpy()
    r_l = ref_l.cpu().numpy() if torch.is_tensor(ref_l) else ref_l
    assert np.array_equal(np.isneginf(o_l), np.isneginf(r_l)), what
    fin = np.isfinite(r_l)
    lerr = float(np.abs(o_l[fin] - r_l[fin]).max()) if fin.any() else 0.0
    assert err <= ATOL_OUT["bf16"], (what, err)
    assert lerr <= ATOL_LSE["bf16"], (what, lerr)


# (workload, k, -1 slots, scratch used on a 148-SM B200, oracle check)
CASES = {
    # 2 splits per row, merged inside 4-CTA clusters: the scratch is not touched
    "decode_B4_rows32_fused": (workloads.DECODE_32K.with_(batch=4, rows=32, ctx=4096), 2048, 0, False, False),
    # 16 rows x 4 splits of 512 keys: partials in the scratch, merge launch
    "decode_rows16_4splits": (workloads.DECODE_32K.with_(batch=4, rows=16, ctx=8192), 2048, 0, True, True),
    # 2 rows x 32 splits, paged cache, unused slots
    "paged_rows2_32splits": (workloads.DECODE_128K_FP8_PAGED.with_(batch=2, rows=2, ctx=4096), 2048, 13, True,
                             True),
    # 80 rows: one split each, the scratch is not touched
    "rows80_nosplit": (workloads.DECODE_32K.with_(batch=2, rows=80, ctx=1024), 256, 3, False, False),
}


@pytest.mark.parametrize("case", list(CASES), ids=list(CASES))
def test_noalloc_matches_workspace_entry(cuda_device, case):
    wl, k, pad, uses_scratch, vs_oracle = CASES[case]
    inp = workloads.generate(wl, parts=("mla",))
    dv = {n: t.to(cuda_device) for n, t in inp.items()}
    pt = dv.get("page_table")
    rows, H = wl.rows, wl.heads
    out = torch.empty((rows, H, wl.d_v), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((rows, H), dtype=torch.float32, device=cuda_device)
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    # a first call sets up the scratch's address on this device (outside the checks below)
    warm = _idx(rows, k, wl.ctx, 20, pad).to(cuda_device)
    dsa.sparse_mla_noalloc(dv["q"], dv["kv"], warm, dv["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx, out, lse,
                           page_table=pt)
    torch.cuda.synchronize()
    for call, seed in enumerate((21, 22)):            # two calls in a row, different key lists
        idx = _idx(rows, k, wl.ctx, seed, pad).to(cuda_device)
        ref_o, ref_l = dsa.sparse_mla(dv["q"], dv["kv"], idx, dv["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                                      page_table=pt)
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated(cuda_device)
        free_before = torch.cuda.mem_get_info(cuda_device)[0]
        n0 = dsa.launch_count()
        dsa.sparse_mla_noalloc(dv["q"], dv["kv"], idx, dv["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                               out, lse, page_table=pt)
        launched = dsa.launch_count() - n0
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated(cuda_device) == before
        assert torch.cuda.mem_get_info(cuda_device)[0] == free_before     # no cudaMalloc inside the library
        assert dsa.get_device_error(cuda_device) == dsa.DSA_OK
        if sms == 148:
            # split partials (scratch) -> the attention kernel and the merge kernel
            assert launched == (2 if uses_scratch else 1), launched
        _close(out, lse, ref_o, ref_l, (case, call, "vs dsa_sparse_mla"))
        if vs_oracle:
            ro, rl, _ = oracle.sparse_mla(inp["q"], inp["kv"], idx.cpu(), inp["row_batch"], wl.softmax_scale,
                                          wl.d_v, wl.ctx, page_table=inp.get("page_table"))
            _close(out, lse, ro, rl, (case, call, "vs oracle"))

