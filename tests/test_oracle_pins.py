"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to a hand-worked fixture, a closed form,
a library routine (numpy / scipy / torch format conversions), brute force on
tiny inputs or an invariant of the mathematics, chosen so that a dropped
term, a wrong sign, a wrong index or a transposed operand fails at least one.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _num(x):
    return float(x) if not isinstance(x, str) else float(x.replace("inf", "inf"))


# ---------------------------------------------------------------- formats ----

def test_bf16_decode_matches_torch_for_all_codes():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_double(c) for c in codes[::97]])
    r = ref[::97]
    same = (got == r) | (np.isnan(got) & np.isnan(r))
    assert same.all()


def test_fp8_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = np.array([oracle.fp8_e4m3_to_double(c) for c in codes])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    # format landmarks: max normal, min subnormal, one, NaN
    assert oracle.fp8_e4m3_to_double(0x7E) == 448.0
    assert oracle.fp8_e4m3_to_double(0x01) == 2.0 ** -9
    assert oracle.fp8_e4m3_to_double(0x38) == 1.0
    assert math.isnan(oracle.fp8_e4m3_to_double(0x7F))


def _bf16_value(bits):
    u = np.array([bits << 16], dtype=np.uint32)
    return Fraction(float(u.view(np.float32)[0]))


def _is_rne_bf16(x: Fraction, bits: int) -> bool:
    """bits is the bf16 nearest to x, ties to the even code (exact check)."""
    v = _bf16_value(bits)
    up = _bf16_value((bits + 1) & 0xFFFF) if (bits & 0x7FFF) != 0x7F7F else None
    dn = _bf16_value((bits - 1) & 0xFFFF) if (bits & 0x7FFF) != 0 else None
    # neighbours in value order depend on sign
    cands = [c for c in (up, dn) if c is not None]
    d = abs(x - v)
    for c in cands:
        dc = abs(x - c)
        if dc < d:
            return False
        if dc == d and (bits & 1):
            return False
    return True


def test_double_to_bf16_is_round_to_nearest_even():
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(300) / 24.0) + [1.00390625, 1.01171875, -1.00390625, 3e-39, -1e-40]
    for x in xs:
        b = oracle.double_to_bf16_bits(float(x))
        assert _is_rne_bf16(Fraction(float(x)), b), (x, hex(b))


# ----------------------------------------------------------- compression ----

def test_compress_identical_rows_and_identity():
    g = torch.Generator().manual_seed(3)
    row = torch.randn(1, 1, 40, generator=g).to(torch.bfloat16)
    src = row.repeat(2, 8, 1)                       # 8 identical rows per sequence
    out = oracle.csa_compress(src, 4)
    ref = row.view(torch.int16).numpy().view(np.uint16)[0, 0]
    assert (out == ref).all()
    x = torch.randn(2, 12, 7, generator=g).to(torch.bfloat16)
    assert (oracle.csa_compress(x, 1) == x.view(torch.int16).numpy().view(np.uint16)).all()


def test_compress_is_rne_of_exact_mean():
    g = torch.Generator().manual_seed(4)
    x = (torch.randn(2, 16, 24, generator=g) / 24.0).to(torch.bfloat16)
    out = oracle.csa_compress(x, 4)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    for b in range(2):
        for i in range(4):
            for d in range(0, 24, 5):
                exact = sum((_bf16_value(int(xb[b, 4 * i + r, d])) for r in range(4)), Fraction(0)) / 4
                assert _is_rne_bf16(exact, int(out[b, i, d]))


def test_compress_fp32_matches_numpy_mean():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(3, 32, 9, generator=g)
    out = oracle.csa_compress(x, 4)
    ref = x.double().numpy().reshape(3, 8, 4, 9).mean(axis=2)
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=0)


# --------------------------------------------------------------- indexer ----

def test_index_scores_hand_fixture():
    d = _load("index_score_hand.json")
    q = torch.tensor(d["q_idx"], dtype=torch.float32)
    w = torch.tensor(d["w"], dtype=torch.float32)
    k = torch.tensor(d["k_idx"], dtype=torch.float32)
    rb = torch.zeros(2, dtype=torch.int32)
    rp = torch.tensor(d["row_pos"], dtype=torch.int32)
    got = oracle.index_scores(q, w, k, rb, rp)
    exp = np.array([[_num(v) for v in r] for r in d["expected"]])
    assert np.array_equal(got, exp)
    # same fixture in bf16 (all values exact in bf16)
    got16 = oracle.index_scores(q.to(torch.bfloat16), w, k.to(torch.bfloat16), rb, rp)
    assert np.array_equal(got16, exp)


def _rand_indexer(seed, rows=5, B=2, L=37, H=3, D=6):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(rows, H, D, generator=g)
    w = torch.rand(rows, H, generator=g)
    k = torch.randn(B, L, D, generator=g)
    rb = torch.arange(rows, dtype=torch.int32) % B
    rp = torch.randint(0, L, (rows,), generator=g, dtype=torch.int32)
    return q, w, k, rb, rp


def test_index_one_hot_weights_reduce_to_single_head_relu_matmul():
    q, w, k, rb, rp = _rand_indexer(7)
    rows, H, D = q.shape
    for j in range(H):
        wj = torch.zeros_like(w)
        wj[:, j] = 1.0
        got = oracle.index_scores(q, wj, k, rb, rp)
        for t in range(rows):
            kb = k[rb[t]].double().numpy()                      # [L, D]
            dots = kb @ q[t, j].double().numpy()                # library matmul
            ref = np.maximum(dots, 0.0)
            vis = np.arange(kb.shape[0]) <= int(rp[t])
            np.testing.assert_allclose(got[t][vis], ref[vis], rtol=1e-13, atol=1e-15)
            assert np.all(np.isneginf(got[t][~vis]))


def test_index_linear_in_weights_and_positive_scaling():
    q, w, k, rb, rp = _rand_indexer(8)
    g = torch.Generator().manual_seed(9)
    w2 = torch.rand(w.shape, generator=g)
    a = oracle.index_scores(q, w, k, rb, rp)
    b = oracle.index_scores(q, w2, k, rb, rp)
    c = oracle.index_scores(q, w + w2, k, rb, rp)
    fin = np.isfinite(a)
    np.testing.assert_allclose(c[fin], (a + b)[fin], rtol=1e-6, atol=1e-7)
    s = oracle.index_scores(q, w * 4.0, k, rb, rp)            # power of two: exact
    assert np.array_equal(s[fin], 4.0 * a[fin])
    # positive scaling leaves the selection unchanged
    assert np.array_equal(oracle.topk(s, rp, 5), oracle.topk(a, rp, 5))


def test_index_head_permutation_invariance():
    q, w, k, rb, rp = _rand_indexer(10)
    perm = torch.tensor([2, 0, 1])
    a = oracle.index_scores(q, w, k, rb, rp)
    b = oracle.index_scores(q[:, perm], w[:, perm], k, rb, rp)
    fin = np.isfinite(a)
    np.testing.assert_allclose(b[fin], a[fin], rtol=1e-13, atol=1e-15)


def test_index_relu_drops_negative_dots():
    q, w, k, rb, rp = _rand_indexer(11, rows=1, B=1, L=4, H=3, D=6)
    kk = torch.zeros(1, 4, 6)
    kk[0, 0] = -q[0, 0] * 0 - q[0].sum(0)          # negative dot with the sum of heads
    kk[0, 1] = -q[0, 0]                            # head 0 negative
    rpos = torch.tensor([3], dtype=torch.int32)
    got = oracle.index_scores(q, w, kk, rb, rpos)
    d = q[0].double().numpy() @ kk[0].double().numpy().T   # [H, L]
    ref = (w[0].double().numpy()[:, None] * np.maximum(d, 0)).sum(0)
    np.testing.assert_allclose(got[0], ref, rtol=1e-13, atol=1e-15)
    assert got[0, 2] == 0.0 and got[0, 3] == 0.0   # zero keys -> zero score


def test_index_fp8_keys_equal_dequantized_fp32_keys():
    g = torch.Generator().manual_seed(12)
    q = torch.randn(3, 4, 16, generator=g).to(torch.bfloat16)
    w = torch.rand(3, 4, generator=g)
    kf = torch.randn(1, 50, 16, generator=g)
    codes, scale = workloads.quantize_fp8_rows(kf)
    deq = codes.view(torch.float8_e4m3fn).float() * scale[..., None]   # torch decode, fp32 product
    rb = torch.zeros(3, dtype=torch.int32)
    rp = torch.tensor([49, 20, 0], dtype=torch.int32)
    a = oracle.index_scores(q, w, codes, rb, rp, k_scale=scale)
    b = oracle.index_scores(q.float(), w, deq, rb, rp)
    fin = np.isfinite(a)
    assert np.array_equal(np.isfinite(a), np.isfinite(b))
    np.testing.assert_allclose(a[fin], b[fin], rtol=1e-6, atol=1e-9)


def test_fp4_e2m1_decode_matches_the_format_table():
    # OCP e2m1: codes 0-7 are the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (exponent
    # bias 1, one mantissa bit, exponent 0 subnormal); bit 3 is the sign
    table = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        v = oracle.fp4_e2m1_to_double(c)
        assert v == (-1.0 if c & 8 else 1.0) * table[c & 7], c
        assert math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0)


def test_index_fp4_keys_equal_dequantized_fp32_keys():
    g = torch.Generator().manual_seed(13)
    q = torch.randn(3, 4, 16, generator=g).to(torch.bfloat16)
    w = torch.rand(3, 4, generator=g)
    kf = torch.randn(1, 50, 16, generator=g)
    codes, scale = workloads.quantize_fp4_rows(kf)
    assert codes.shape == (1, 50, 8)
    # unpack independently: dim 2j is the low nibble of byte j
    table = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    nib = torch.stack([codes & 0xF, codes >> 4], dim=-1).reshape(1, 50, 16).long()
    val = table[nib & 7] * torch.where(nib >= 8, -1.0, 1.0)
    deq = val * scale[..., None]
    # the quantiser picks the nearest magnitude of the scaled value
    assert (deq - kf).abs().max() <= (scale.max() * 1.0 + 1e-6)
    rb = torch.zeros(3, dtype=torch.int32)
    rp = torch.tensor([49, 20, 0], dtype=torch.int32)
    a = oracle.index_scores(q, w, codes, rb, rp, k_scale=scale)
    b = oracle.index_scores(q.float(), w, deq, rb, rp)
    fin = np.isfinite(a)
    assert np.array_equal(np.isfinite(a), np.isfinite(b))
    np.testing.assert_allclose(a[fin], b[fin], rtol=1e-6, atol=1e-9)


# ------------------------------------------------------------------ top-k ----

def test_topk_hand_fixture():
    d = _load("topk_hand.json")
    for c in d["cases"]:
        s = np.array([[_num(v) for v in c["scores"]]], dtype=np.float64)
        got = oracle.topk(s, [c["pos"]], c["k"])
        assert got[0].tolist() == c["expected"], c["why"]


def _brute_topk(scores, pos, k):
    """Rank counting: key s is kept iff fewer than k visible keys beat it
    (higher score, or equal score and lower index)."""
    n = pos + 1
    sel = []
    for s in range(n):
        beat = sum(1 for t in range(n) if scores[t] > scores[s] or (scores[t] == scores[s] and t < s))
        if beat < k:
            sel.append((beat, s))
    sel.sort()
    return [s for _, s in sel] + [-1] * (k - len(sel))


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_brute_force_on_tiny_inputs(seed):
    x = workloads.synthetic_scores(4, 23, seed=seed).double().numpy()
    if seed == 0:
        x[0] = 0.0                      # an all-zero row
        x[1, ::2] = -0.0
    for pos in (0, 5, 22):
        for k in range(1, 26):
            got = oracle.topk(x, [pos] * 4, k)
            for r in range(4):
                assert got[r].tolist() == _brute_topk(x[r], pos, k)


def test_topk_matches_library_lexsort():
    x = workloads.synthetic_scores(3, 500, seed=42).double().numpy()
    pos = [499, 250, 3]
    got = oracle.topk(x, pos, 64)
    for r in range(3):
        n = pos[r] + 1
        order = np.lexsort((np.arange(n), -x[r, :n]))     # score desc, index asc
        exp = order[:64].tolist() + [-1] * max(0, 64 - n)
        assert got[r].tolist() == exp


# ------------------------------------------------------------ sparse MLA ----

def test_sparse_mla_hand_fixture():
    d = _load("sparse_mla_hand.json")
    q = torch.tensor(d["q"], dtype=torch.float32)
    kv = torch.tensor(d["kv"], dtype=torch.float32)
    idx = torch.tensor(d["idx"], dtype=torch.int32)
    out, lse, probs = oracle.sparse_mla(q, kv, idx, torch.zeros(1, dtype=torch.int32), d["scale"],
                                        d["D_V"], ctx=4, want_probs=True)
    np.testing.assert_allclose(out, np.array(d["expected_out"]), rtol=0, atol=d["tol"])
    np.testing.assert_allclose(lse, np.array(d["expected_lse"]), rtol=0, atol=d["tol"])
    assert np.all(probs[0, :, 2] == 0.0)          # the -1 slot carries no weight


def _dense_causal_attention(q, kv, pos, scale, d_v):
    """Textbook dense attention over every visible key (library softmax)."""
    qd = q.double().numpy()
    kd = kv.double().numpy()
    out = np.zeros((qd.shape[0], qd.shape[1], d_v))
    lse = np.zeros((qd.shape[0], qd.shape[1]))
    for t in range(qd.shape[0]):
        c = kd[: pos[t] + 1]
        z = scale * (qd[t] @ c.T)                 # [H, n]
        out[t] = scipy.special.softmax(z, axis=-1) @ c[:, :d_v]
        lse[t] = scipy.special.logsumexp(z, axis=-1)
    return out, lse


def test_sparse_equals_dense_when_context_fits_in_k():
    # tiny prefill shape family: every row sees at most k keys -> keep all
    w = workloads.TINY_PREFILL_FP32.with_(ctx=48, rows=48, topk=64)
    inp = workloads.generate(w)
    scores = oracle.index_scores(inp["q_idx"], inp["w"], inp["k_idx"], inp["row_batch"], inp["row_pos"])
    idx = oracle.topk(scores, inp["row_pos"], w.topk)
    out, lse, probs = oracle.sparse_mla(inp["q"], inp["kv"], idx, inp["row_batch"], w.softmax_scale,
                                        w.d_v, ctx=w.ctx, want_probs=True)
    dout, dlse = _dense_causal_attention(inp["q"], inp["kv"][0], inp["row_pos"].tolist(), w.softmax_scale, w.d_v)
    np.testing.assert_allclose(out, dout, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, dlse, rtol=0, atol=1e-12)
    np.testing.assert_allclose(probs.sum(-1), 1.0, rtol=0, atol=1e-12)


def test_sparse_mla_invariants():
    g = torch.Generator().manual_seed(20)
    rows, H, D, L, k = 3, 4, 10, 30, 7
    q = torch.randn(rows, H, D, generator=g)
    kv = torch.randn(2, L, D, generator=g)
    rb = torch.tensor([0, 1, 1], dtype=torch.int32)
    idx = torch.stack([torch.randperm(L, generator=g)[:k] for _ in range(rows)]).to(torch.int32)
    out, lse, probs = oracle.sparse_mla(q, kv, idx, rb, 0.3, 6, ctx=L, want_probs=True)
    np.testing.assert_allclose(probs.sum(-1), 1.0, rtol=0, atol=1e-12)
    # slot order does not matter
    perm = torch.randperm(k, generator=g)
    out2, lse2, _ = oracle.sparse_mla(q, kv, idx[:, perm], rb, 0.3, 6, ctx=L)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-13)
    # unused (-1) slots are ignored
    pad = torch.cat([idx, torch.full((rows, 3), -1, dtype=torch.int32)], 1)
    out3, lse3, _ = oracle.sparse_mla(q, kv, pad, rb, 0.3, 6, ctx=L)
    np.testing.assert_allclose(out3, out, rtol=0, atol=1e-13)
    # k = 1: the output is the selected row's value exactly, lse its logit
    out1, lse1, _ = oracle.sparse_mla(q, kv, idx[:, :1], rb, 0.3, 6, ctx=L)
    for t in range(rows):
        row = kv[rb[t], idx[t, 0]].double().numpy()
        assert np.array_equal(out1[t], np.broadcast_to(row[:6], (H, 6)))
        np.testing.assert_allclose(lse1[t], 0.3 * (q[t].double().numpy() @ row), rtol=1e-14)
    # identical value rows -> output equals that value whatever the weights
    kv_c = kv.clone()
    kv_c[:, :, :6] = kv[0, 0, :6]
    outc, _, _ = oracle.sparse_mla(q, kv_c, idx, rb, 0.3, 6, ctx=L)
    np.testing.assert_allclose(outc, np.broadcast_to(kv[0, 0, :6].double().numpy(), outc.shape), rtol=0, atol=1e-14)


def test_paged_cache_equals_contiguous_cache():
    g = torch.Generator().manual_seed(21)
    B, L, D, page, rows, k = 2, 64, 12, 8, 4, 9
    kv = torch.randn(B, L, D, generator=g).to(torch.bfloat16)
    q = torch.randn(rows, 3, D, generator=g).to(torch.bfloat16)
    rb = torch.tensor([0, 1, 0, 1], dtype=torch.int32)
    idx = torch.stack([torch.randperm(L, generator=g)[:k] for _ in range(rows)]).to(torch.int32)
    n_pages = B * L // page
    perm = torch.randperm(n_pages, generator=g)
    table = perm.view(B, L // page).to(torch.int32)
    phys = torch.empty(n_pages, page, D, dtype=torch.bfloat16)
    logical = kv.view(B, L // page, page, D)
    for b in range(B):
        for p in range(L // page):
            phys[table[b, p]] = logical[b, p]
    a, la, _ = oracle.sparse_mla(q, kv, idx, rb, 0.25, 8, ctx=L)
    b_, lb, _ = oracle.sparse_mla(q, phys, idx, rb, 0.25, 8, ctx=L, page_table=table)
    assert np.array_equal(a, b_) and np.array_equal(la, lb)


def test_csa_with_m1_is_dsa():
    w = workloads.TINY_PREFILL_FP32.with_(ctx=40, rows=40, topk=16)
    inp = workloads.generate(w)
    k1 = oracle.csa_compress(inp["k_idx"], 1)
    a = oracle.index_scores(inp["q_idx"], inp["w"], inp["k_idx"], inp["row_batch"], inp["row_pos"])
    b = oracle.index_scores(inp["q_idx"], inp["w"], k1, inp["row_batch"], inp["row_pos"])
    assert np.array_equal(a, b)


# ------------------------------------------- CSA window and HCA (NEXT rows) ----

def _brute_attention(q, vecs, scale, d_v):
    """softmax(scale * q . c) @ c[:d_v] for one row: q [H, D], vecs [n, D] (n >= 1)."""
    z = scale * (q @ vecs.T)                                   # [H, n]
    p = scipy.special.softmax(z, axis=1)
    return p @ vecs[:, :d_v], scipy.special.logsumexp(z, axis=1)


def test_csa_core_attention_is_attention_over_the_concatenated_keys():
    g = torch.Generator().manual_seed(31)
    B, Lc, Lr, H, D, dv, k, W = 2, 20, 80, 3, 12, 8, 5, 6
    q = torch.randn(5, H, D, generator=g)
    kv = torch.randn(B, Lc, D, generator=g)
    raw = torch.randn(B, Lr, D, generator=g)
    rb = torch.tensor([0, 1, 1, 0, 1], dtype=torch.int32)
    pos = torch.tensor([79, 40, 3, 0, 5], dtype=torch.int32)      # rows 2-4: window clipped at position 0
    idx = torch.stack([torch.randperm(Lc, generator=g)[:k] for _ in range(5)]).to(torch.int32)
    idx[1, 2] = -1
    out, lse = oracle.csa_core_attention(q, kv, idx, rb, 0.4, dv, Lc, raw, pos, W)
    for t in range(5):
        b = int(rb[t])
        sel = [kv[b, int(s)] for s in idx[t] if s >= 0]
        win = [raw[b, p] for p in range(int(pos[t]) - W + 1, int(pos[t]) + 1) if p >= 0]
        vecs = torch.stack(sel + win).double().numpy()
        ro, rl = _brute_attention(q[t].double().numpy(), vecs, 0.4, dv)
        np.testing.assert_allclose(out[t], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[t], rl, rtol=0, atol=1e-12)
    # a window of 0 rows is plain sparse attention; no selected entries leaves the window alone
    o0, l0 = oracle.csa_core_attention(q, kv, idx, rb, 0.4, dv, Lc, raw, pos, 0)
    so, sl, _ = oracle.sparse_mla(q, kv, idx, rb, 0.4, dv, Lc)
    np.testing.assert_allclose(o0, so, rtol=0, atol=0)
    ow, lw = oracle.csa_core_attention(q, kv, None, rb, 0.4, dv, Lc, raw, pos, W)
    t = 0
    ro, rl = _brute_attention(q[t].double().numpy(), raw[0, 74:80].double().numpy(), 0.4, dv)
    np.testing.assert_allclose(ow[t], ro, rtol=0, atol=1e-12)


def test_csa_core_attention_sink_is_attention_over_the_union_of_raw_positions():
    # The sink and the window are both raw rows: the attended raw positions
    # are the union {0 .. n_sink-1} u {pos-W+1 .. pos}, clipped to [0, pos],
    # each once; with the selected compressed entries beside them.
    g = torch.Generator().manual_seed(34)
    B, Lc, Lr, H, D, dv, k = 2, 20, 80, 3, 12, 8, 5
    rows = 7
    q = torch.randn(rows, H, D, generator=g)
    kv = torch.randn(B, Lc, D, generator=g)
    raw = torch.randn(B, Lr, D, generator=g)
    rb = torch.tensor([0, 1, 1, 0, 1, 0, 1], dtype=torch.int32)
    # far from the start, window touching the sink, overlapping it, inside it, at position 0
    pos = torch.tensor([79, 9, 7, 5, 2, 0, 40], dtype=torch.int32)
    idx = torch.stack([torch.randperm(Lc, generator=g)[:k] for _ in range(rows)]).to(torch.int32)
    idx[3, 1] = -1
    for W, n_sink in ((6, 4), (0, 4), (6, 0), (3, 12), (1, 1)):
        out, lse = oracle.csa_core_attention(q, kv, idx, rb, 0.4, dv, Lc, raw, pos, W, n_sink=n_sink)
        for t in range(rows):
            b, p_t = int(rb[t]), int(pos[t])
            raw_pos = sorted(set(range(min(n_sink, p_t + 1))) | set(range(max(0, p_t - W + 1), p_t + 1)))
            sel = [kv[b, int(s)] for s in idx[t] if s >= 0]
            vecs = torch.stack(sel + [raw[b, p] for p in raw_pos]).double().numpy()
            ro, rl = _brute_attention(q[t].double().numpy(), vecs, 0.4, dv)
            np.testing.assert_allclose(out[t], ro, rtol=0, atol=1e-12, err_msg=f"W={W} sink={n_sink} t={t}")
            np.testing.assert_allclose(lse[t], rl, rtol=0, atol=1e-12)
    # no sink: the window-only composition, unchanged
    a, la = oracle.csa_core_attention(q, kv, idx, rb, 0.4, dv, Lc, raw, pos, 6)
    b_, lb = oracle.csa_core_attention(q, kv, idx, rb, 0.4, dv, Lc, raw, pos, 6, n_sink=0)
    np.testing.assert_array_equal(a, b_)
    # sink only (no window, no selection): attention over raw rows 0 .. min(n_sink, pos+1)-1
    so, sl = oracle.csa_core_attention(q, kv, None, rb, 0.4, dv, Lc, raw, pos, 0, n_sink=4)
    ro, rl = _brute_attention(q[0].double().numpy(), raw[0, :4].double().numpy(), 0.4, dv)
    np.testing.assert_allclose(so[0], ro, rtol=0, atol=1e-12)
    ro, rl = _brute_attention(q[5].double().numpy(), raw[0, :1].double().numpy(), 0.4, dv)
    np.testing.assert_allclose(so[5], ro, rtol=0, atol=1e-12)


def test_csa_core_attention_paged_equals_contiguous():
    g = torch.Generator().manual_seed(32)
    B, Lc, page, H, D = 2, 16, 4, 2, 8
    kv = torch.randn(B, Lc, D, generator=g)
    raw = torch.randn(B, 30, D, generator=g)
    q = torch.randn(3, H, D, generator=g)
    rb = torch.tensor([1, 0, 1], dtype=torch.int32)
    pos = torch.tensor([29, 10, 2], dtype=torch.int32)
    idx = torch.stack([torch.randperm(Lc, generator=g)[:6] for _ in range(3)]).to(torch.int32)
    perm = torch.randperm(B * Lc // page, generator=g)
    pages = torch.empty(B * Lc // page, page, D)
    pages[perm] = kv.reshape(-1, page, D)
    table = perm.view(B, Lc // page).to(torch.int32)
    a, la = oracle.csa_core_attention(q, kv, idx, rb, 0.5, 8, Lc, raw, pos, 4)
    p, lp = oracle.csa_core_attention(q, pages, idx, rb, 0.5, 8, Lc, raw, pos, 4, page_table=table)
    np.testing.assert_allclose(p, a, rtol=0, atol=0)
    np.testing.assert_allclose(lp, la, rtol=0, atol=0)


def test_hca_attention_is_dense_attention_over_visible_blocks():
    g = torch.Generator().manual_seed(33)
    m, B, Lraw, H, D, dv = 128, 2, 1024, 2, 16, 16
    raw = torch.randn(B, Lraw, D, generator=g).to(torch.bfloat16)
    kvc_bits = oracle.csa_compress(raw, m)                      # [B, 8, D] bf16 codes
    kvc = torch.from_numpy(kvc_bits.view(np.int16)).view(torch.bfloat16)
    # the pooled entry is the mean of its 128 raw rows, rounded once
    mean = raw[1, 3 * m:4 * m].double().mean(0)
    assert torch.equal(kvc[1, 3], mean.to(torch.bfloat16))
    q = torch.randn(4, H, D, generator=g).to(torch.bfloat16)
    rb = torch.tensor([0, 1, 1, 0], dtype=torch.int32)
    last = torch.tensor([7, 7, 2, -1], dtype=torch.int32)       # decode, decode, causal prefix, nothing visible
    out, lse = oracle.hca_attention(q, kvc, rb, last, 0.25, dv)
    for t in range(3):
        vecs = kvc[int(rb[t]), :int(last[t]) + 1].double().numpy()
        ro, rl = _brute_attention(q[t].double().numpy(), vecs, 0.25, dv)
        np.testing.assert_allclose(out[t], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[t], rl, rtol=0, atol=1e-12)
    assert np.all(out[3] == 0) and np.all(np.isneginf(lse[3]))
