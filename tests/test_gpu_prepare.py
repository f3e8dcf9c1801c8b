"""Parity of the indexer-input preparation and the key-cache write (GPU).

dsa_indexer_key_append is compared with the oracle bit for bit: the stored
codes and scales are decided in binary32 on both sides with the same
separately rounded operations (only the sign of a zero code is not compared:
+0 and -0 decode to the same key value).

dsa_indexer_prepare multiplies bf16 operands on the tensor cores with fp32
accumulation, so its outputs are compared with the oracle's float64 values
under bounds derived from the rounding steps:
  q_I   bf16 output (unit roundoff 2^-8, relative) plus the bf16 rounding of
        c_q * gain in the MMA operand (each term off by at most 2^-8 of
        itself, independent signs: standard deviation at most
        2^-8 / sqrt(3) * sqrt(sum of squared terms), bounded by 2^-6 times
        that root, about 7 standard deviations), with a rotary pair's two
        bounds added;
  w     fp32 accumulation only: 1e-5 of the sum of absolute terms;
  keys  bf16 cache: as w plus 2^-8 relative; fp8 / fp4 cache: the scale
        within 1e-4 of amax / qmax of the oracle's rotated key, and every
        code a nearest code of key / scale up to a slack for values near a
        rounding midpoint: the fp32 accumulation error of the key (a random
        walk over d_model roundings, well below 3e-6 of the sum of absolute
        terms, a rotary pair's two sums added) divided by the scale, plus
        1e-3 of the value.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_logits_b200")

FMT = {"bf16": oracle.BF16, "fp8": oracle.FP8, "fp4": oracle.FP4}
E4M3_GRID = np.array([oracle.fp8_e4m3_to_double(c) for c in range(0x7F)])
E2M1_GRID = np.array([oracle.fp4_e2m1_to_double(c) for c in range(8)])
E4M3_ALL = np.array([oracle.fp8_e4m3_to_double(c) for c in range(256)])
E2M1_ALL = np.array([oracle.fp4_e2m1_to_double(c) for c in range(16)])


def _cache(fmt: str, rows: int, dev):
    """A key cache filled with a recognisable pattern (and its scales)."""
    if fmt == "bf16":
        c = torch.full((rows, 128), 0x5A5A, dtype=torch.int16).view(torch.bfloat16)
        return c.to(dev), None
    width = 128 if fmt == "fp8" else 64
    return (torch.full((rows, width), 0x5A, dtype=torch.uint8, device=dev),
            torch.full((rows,), 7.5, dtype=torch.float32, device=dev))


def _zero_sign_free(codes: np.ndarray, fmt: str) -> np.ndarray:
    c = codes.astype(np.uint8).copy()
    if fmt == "fp8":
        c[c == 0x80] = 0
    elif fmt == "fp4":
        lo, hi = c & 0x0F, c >> 4
        lo[lo == 8] = 0
        hi[hi == 8] = 0
        c = lo | (hi << 4)
    return c


def _check_untouched(cache_g, scale_g, slots, fmt, rows):
    keep = np.ones(rows, dtype=bool)
    keep[slots[slots >= 0]] = False
    c = cache_g.view(torch.uint8).cpu().numpy() if fmt != "bf16" else cache_g.view(torch.int16).cpu().numpy()
    ref = 0x5A if fmt != "bf16" else 0x5A5A
    assert (c[keep] == ref).all(), "rows of other tokens were written"
    if scale_g is not None:
        assert (scale_g.cpu().numpy()[keep] == 7.5).all()


# ------------------------------------------------------------ key append --

@pytest.mark.parametrize("fmt", ["bf16", "fp8", "fp4"])
@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d_rope", [0, 64])
def test_key_append_bit_exact(fmt, in_dtype, d_rope):
    dev = torch.device("cuda:0")
    n, rows, max_pos = 301, 1000, 512
    g = torch.Generator().manual_seed(11)
    x = torch.randn(n, 128, generator=g) * torch.exp2(torch.randint(-8, 8, (n, 1), generator=g).float())
    x[5] = 0.0                                       # all-zero row: scale 1
    x[6] *= 1e-3                                     # codes down in the subnormal range
    x[7, :64] = 0.0
    x = x.to(in_dtype)
    pos = torch.randint(0, max_pos, (n,), generator=g, dtype=torch.int32)
    slot = torch.randperm(rows, generator=g)[:n].long()
    slot[::13] = -1
    cos, sin = workloads.rope_tables(max_pos, d_rope) if d_rope else (None, None)
    cache, scale = _cache(fmt, rows, dev)
    dsa.indexer_key_append(x.to(dev), slot.to(dev), cache, scale, pos.to(dev),
                           None if cos is None else cos.to(dev), None if sin is None else sin.to(dev))
    assert dsa.get_device_error() == 0
    want, want_scale = oracle.key_rows_f32(x.float(), pos.numpy(),
                                           cos if cos is not None else np.ones((1, 1), np.float32),
                                           sin if sin is not None else np.zeros((1, 1), np.float32), d_rope, FMT[fmt])
    s = slot.numpy()
    ok = s >= 0
    got = cache.view(torch.uint8).cpu().numpy() if fmt != "bf16" else cache.view(torch.int16).cpu().numpy().view(np.uint16)
    if fmt == "bf16":
        np.testing.assert_array_equal(got[s[ok]], want[ok])
    else:
        np.testing.assert_array_equal(_zero_sign_free(got[s[ok]], fmt), _zero_sign_free(want[ok], fmt))
        np.testing.assert_array_equal(scale.cpu().numpy()[s[ok]], want_scale[ok])
    _check_untouched(cache, scale, s, fmt, rows)


# ---------------------------------------------------------- the fused step --

def _prepare_oracle(inp, shape):
    return oracle.indexer_prepare(inp["c_q"], inp["gamma"], 1e-6, inp["wq_b"], inp["h"], inp["wk"], inp["w_proj"],
                                  inp.get("rope_cos", np.ones((1, 1), np.float32)),
                                  inp.get("rope_sin", np.zeros((1, 1), np.float32)),
                                  inp["pos"].numpy(), shape.n_heads, shape.d_rope)


def _pair_sum(a: np.ndarray, d_rope: int) -> np.ndarray:
    """Bound of a rotated pair: the two dims' bounds added (dims below d_rope)."""
    if d_rope == 0:
        return a
    b = a.copy()
    r = a[..., :d_rope]
    b[..., :d_rope] = r + r.reshape(*r.shape[:-1], -1, 2)[..., ::-1].reshape(r.shape)
    return b


def _check_codes(codes_g, scale_g, k_o, fmt, abs_sum):
    qmax = 448.0 if fmt == "fp8" else 6.0
    amax = np.abs(k_o).max(axis=1)
    want = np.where(amax > 0, amax / qmax, 1.0)
    np.testing.assert_allclose(scale_g, want, rtol=1e-4)
    if fmt == "fp8":
        dec = E4M3_ALL[codes_g]
        grid = E4M3_GRID
    else:
        dec = np.empty((codes_g.shape[0], 128))
        dec[:, 0::2], dec[:, 1::2] = E2M1_ALL[codes_g & 0xF], E2M1_ALL[codes_g >> 4]
        grid = E2M1_GRID
    y = k_o / scale_g[:, None].astype(np.float64)
    ay = np.minimum(np.abs(y), qmax)
    nearest = np.abs(ay[..., None] - grid).min(axis=-1)
    err = np.abs(np.abs(dec) - ay)
    slack = 3e-6 * abs_sum / scale_g[:, None] + 1e-3 * ay
    assert (err <= nearest + slack).all(), float((err - nearest - slack).max())
    assert ((np.sign(dec) == np.sign(y)) | (dec == 0)).all()


def _run_prepare(shape: workloads.PrepareShape, fmt: str, seed: int):
    dev = torch.device("cuda:0")
    inp = workloads.make_prepare_inputs(shape, seed)
    d = {k: v.to(dev) for k, v in inp.items()}
    cache, scale = _cache(fmt, shape.cache_rows, dev)
    q_g, w_g = dsa.indexer_prepare(d["c_q"], d["gamma"], d["wq_b"], d["h"], d["wk"], d["w_proj"], d["pos"],
                                   d["slot"], cache, scale, d.get("rope_cos"), d.get("rope_sin"), eps=1e-6)
    assert dsa.get_device_error() == 0
    _verify(inp, q_g.cpu(), w_g.cpu(), cache, scale, shape, fmt)
    _check_untouched(cache, scale, inp["slot"].numpy(), fmt, shape.cache_rows)


def _verify(inp, q_g, w_g, cache, scale, shape, fmt):
    """GPU outputs of the tokens in `inp` (host inputs of those tokens only:
    c_q, h, pos, slot; the weights whole) against the oracle."""
    q_o, w_o, k_o = _prepare_oracle(inp, shape)
    T, H = inp["c_q"].shape[0], shape.n_heads

    # queries
    cn = oracle.rms_norm(inp["c_q"].double().numpy(), inp["gamma"].numpy(), 1e-6)
    W = inp["wq_b"].double().numpy()
    sq = np.sqrt((cn ** 2) @ (W ** 2).T).reshape(T, H, 128)
    tol_q = 2.0 ** -7 * np.abs(q_o) + 2.0 ** -6 * _pair_sum(sq, shape.d_rope) + 1e-6
    err_q = np.abs(q_g.double().numpy() - q_o)
    assert (err_q <= tol_q).all(), f"q: worst excess {float((err_q - tol_q).max())}"

    # head weights
    hd = np.abs(inp["h"].double().numpy())
    aw = hd @ np.abs(inp["w_proj"].double().numpy()).T
    np.testing.assert_array_less(np.abs(w_g.double().numpy() - w_o), 1e-5 * aw + 1e-6)

    # keys in the cache
    s = inp["slot"].numpy()
    ok = s >= 0
    ak = _pair_sum(hd @ np.abs(inp["wk"].double().numpy()).T, shape.d_rope)
    if fmt == "bf16":
        kg = cache[torch.from_numpy(s[ok]).to(cache.device)].double().cpu().numpy()
        tol_k = 1.01 * 2.0 ** -8 * np.abs(k_o[ok]) + 1e-5 * ak[ok] + 1e-6
        assert (np.abs(kg - k_o[ok]) <= tol_k).all()
    else:
        _check_codes(cache[torch.from_numpy(s[ok]).to(cache.device)].cpu().numpy(),
                     scale[torch.from_numpy(s[ok]).to(scale.device)].cpu().numpy(), k_o[ok], fmt, ak[ok])


@pytest.mark.parametrize("tokens", [1, 64, 200])
@pytest.mark.parametrize("fmt", ["fp8", "fp4", "bf16"])
def test_prepare_v3_sizes(tokens, fmt):
    # query latent 1536, hidden 7168, 64 indexer heads of 128 with a 64-dim rotary part
    _run_prepare(workloads.PrepareShape(tokens, 1536, 7168, cache_rows=4096), fmt, seed=tokens)


@pytest.mark.parametrize("tokens", [64, 200])
def test_prepare_reuses_one_workspace(tokens):
    # Two calls on one workspace that starts out filled with 0xFF bytes: nothing
    # in it is read before this call writes it, so each call gives its own
    # keys and weights.  64 tokens: one CTA per SM, rotary rows staged in shared
    # memory; 200 tokens: two CTAs per SM.
    dev = torch.device("cuda:0")
    shape = workloads.PrepareShape(tokens, 1536, 7168, cache_rows=4096)
    ws = torch.full((dsa.indexer_prepare_workspace_size(tokens, 64, 1536, 7168),), 0xFF, dtype=torch.uint8,
                    device=dev)
    for seed in (31, 32):
        inp = workloads.make_prepare_inputs(shape, seed)
        d = {k: v.to(dev) for k, v in inp.items()}
        cache, scale = _cache("fp8", shape.cache_rows, dev)
        q_g, w_g = dsa.indexer_prepare(d["c_q"], d["gamma"], d["wq_b"], d["h"], d["wk"], d["w_proj"], d["pos"],
                                       d["slot"], cache, scale, d.get("rope_cos"), d.get("rope_sin"), eps=1e-6,
                                       workspace=ws)
        assert dsa.get_device_error() == 0
        _verify(inp, q_g.cpu(), w_g.cpu(), cache, scale, shape, "fp8")
        _check_untouched(cache, scale, inp["slot"].numpy(), "fp8", shape.cache_rows)


@pytest.mark.parametrize("n_heads,d_rope", [(16, 0), (24, 32), (96, 128)])
def test_prepare_other_geometries(n_heads, d_rope):
    # partial head-weight tiles, no / short / full rotary parts, ragged token tiles
    _run_prepare(workloads.PrepareShape(333, 256, 512, n_heads=n_heads, d_rope=d_rope, cache_rows=1024), "fp8",
                 seed=n_heads)


@pytest.mark.parametrize("fmt", ["fp8", "bf16"])
def test_prepare_prefill_many_token_tiles(fmt):
    # enough tiles to fill the GPU: 256-wide query tiles, no split of the d_model
    # reduction, a ragged last token tile (2400 = 18 * 128 + 96)
    _run_prepare(workloads.PrepareShape(2400, 512, 1024, cache_rows=4096), fmt, seed=5)


@pytest.mark.parametrize("n_heads,d_rope", [(96, 128), (200, 32)])
def test_prepare_prefill_wide_key_weight_tiles(n_heads, d_rope):
    # 256-wide tiles: [W_k ; W_w] in one tile of 256 rows (96 heads; rotary rows
    # too long to stage in shared memory) or in tiles of 256 and 128 rows
    # (200 heads, the last weight block partly past the head count)
    _run_prepare(workloads.PrepareShape(2400, 512, 1024, n_heads=n_heads, d_rope=d_rope, cache_rows=4096), "fp8",
                 seed=n_heads + d_rope)


def test_prepare_then_indexer_scores_the_new_keys():
    # the prepared queries / weights and the fp8 cache feed the indexer directly
    dev = torch.device("cuda:0")
    shape = workloads.PrepareShape(64, 1536, 7168, cache_rows=64 * 256)
    inp = workloads.make_prepare_inputs(shape, seed=9, skip=0.0)
    inp["slot"] = (torch.arange(64) * 256 + inp["pos"] % 256).long()       # token t -> its own cache b = t
    inp["pos"] = inp["pos"] % 256
    d = {k: v.to(dev) for k, v in inp.items()}
    cache, scale = _cache("fp8", shape.cache_rows, dev)
    cache.zero_()
    scale.fill_(1.0)
    q_g, w_g = dsa.indexer_prepare(d["c_q"], d["gamma"], d["wq_b"], d["h"], d["wk"], d["w_proj"], d["pos"],
                                   d["slot"], cache, scale, d["rope_cos"], d["rope_sin"], eps=1e-6)
    rb = torch.arange(64, dtype=torch.int32, device=dev)
    rp = d["pos"].clone()
    logits = dsa.indexer_logits(q_g, w_g, cache.view(64, 256, 128), rb, rp, k_scale=scale.view(64, 256))
    t = torch.arange(64)
    got = logits.cpu()[t, inp["pos"].long()]
    # the same score from the stored key: the oracle's index score of the prepared inputs
    ref = oracle.index_scores(q_g.cpu(), w_g.cpu(), cache.view(64, 256, 128).cpu(), rb.cpu(), rp.cpu(),
                              k_scale=scale.view(64, 256).cpu())
    want = ref[t.numpy(), inp["pos"].numpy()]
    np.testing.assert_allclose(got.double().numpy(), want, rtol=2e-3, atol=2e-3)


@pytest.mark.parametrize("case", ["decode", "prefill"])
def test_prepare_full_size_sampled(case):
    # the launch configurations bench.py times: 64 decode tokens appending into the
    # 64 x 131072-row fp8 key cache, and 16384 prefill tokens into a bf16 cache;
    # every output of the sampled tokens is checked (the oracle treats tokens
    # one by one, so it runs on the sample only)
    dev = torch.device("cuda:0")
    if case == "decode":
        T, fmt, rows, max_pos = 64, "fp8", 64 * 131072, 131072
        sample = np.array([0, 1, 31, 62, 63])
    else:
        T, fmt, rows, max_pos = 16384, "bf16", 16384, 16384
        sample = np.array([0, 1, 127, 128, 4095, 8191, 12345, 16383])
    shape = workloads.PrepareShape(T, 1536, 7168, max_pos=max_pos, cache_rows=rows)
    inp = workloads.make_prepare_inputs(shape, seed=77, skip=0.0)
    if case == "decode":
        inp["pos"] = torch.full((T,), max_pos - 1, dtype=torch.int32)
        inp["slot"] = torch.arange(T, dtype=torch.int64) * 131072 + (max_pos - 1)
    else:
        inp["pos"] = torch.arange(T, dtype=torch.int32)
        inp["slot"] = torch.arange(T, dtype=torch.int64)
    d = {k: v.to(dev) for k, v in inp.items()}
    if fmt == "fp8":
        cache = torch.zeros((rows, 128), dtype=torch.uint8, device=dev)
        scale = torch.ones(rows, dtype=torch.float32, device=dev)
    else:
        cache = torch.zeros((rows, 128), dtype=torch.bfloat16, device=dev)
        scale = None
    q_g, w_g = dsa.indexer_prepare(d["c_q"], d["gamma"], d["wq_b"], d["h"], d["wk"], d["w_proj"], d["pos"],
                                   d["slot"], cache, scale, d["rope_cos"], d["rope_sin"], eps=1e-6)
    assert dsa.get_device_error() == 0
    sub = dict(inp)
    for k in ("c_q", "h", "pos", "slot"):
        sub[k] = inp[k][torch.from_numpy(sample)]
    ts = torch.from_numpy(sample).to(dev)
    _verify(sub, q_g[ts].cpu(), w_g[ts].cpu(), cache, scale, shape, fmt)
