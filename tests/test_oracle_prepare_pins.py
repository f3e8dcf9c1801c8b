"""Pins of the oracle's preparation of the indexer inputs (CPU only).

The step before the path ("DeepSeek-V3.2稀疏注意力机制原理与TPU适配", section 3,
Step 1: RMSNorm of the query latent, the up-projection, the split into parts
with and without rotary encoding, apply_rotary_emb, weights_proj) and the
key-cache write (fp8 / fp4 codes with a per-row scale).  Each test ties an
oracle function to the format definitions (OCP E4M3 / E2M1 tables,
round-to-nearest-even), to a library cast (torch), to a hand-worked fixture
or to an invariant of the mathematics (RMSNorm's scale invariance, the
relative-position property of rotary encoding).
"""
import math

import numpy as np
import pytest
import torch

import oracle


# ------------------------------------------------------------ fp8 / fp4 codes --

def test_e4m3_encode_round_trips_every_finite_code():
    for c in list(range(0x00, 0x7F)) + list(range(0x80, 0xFF)):
        assert oracle.fp8_e4m3_encode(oracle.fp8_e4m3_to_double(c)) == c, hex(c)


def test_e4m3_encode_matches_torch_cast_within_range():
    g = torch.Generator().manual_seed(3)
    mags = torch.exp2(torch.empty(4000).uniform_(-12, 8.8, generator=g))
    vals = (mags * torch.where(torch.rand(4000, generator=g) < 0.5, -1.0, 1.0)).float()
    vals = vals[vals.abs() <= 448]
    ref = vals.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.fp8_e4m3_encode(v) for v in vals.numpy()], dtype=np.uint8)
    np.testing.assert_array_equal(got, ref)


def test_e4m3_encode_ties_go_to_the_even_code_and_saturate():
    # 1.0 = 0x38, 1.125 = 0x39, 1.25 = 0x3A: midpoints tie to the even code
    assert oracle.fp8_e4m3_encode(1.0625) == 0x38
    assert oracle.fp8_e4m3_encode(1.1875) == 0x3A
    assert oracle.fp8_e4m3_encode(np.nextafter(np.float32(1.0625), np.float32(2))) == 0x39
    # subnormals: 2^-9 is code 1; 2^-10 ties between 0 and 2^-9 -> 0; 3*2^-10 ties -> code 2
    assert oracle.fp8_e4m3_encode(2.0 ** -9) == 0x01
    assert oracle.fp8_e4m3_encode(2.0 ** -10) == 0x00
    assert oracle.fp8_e4m3_encode(3 * 2.0 ** -10) == 0x02
    # saturation at 448 (0x7E) instead of the NaN code
    assert oracle.fp8_e4m3_encode(464.0) == 0x7E
    assert oracle.fp8_e4m3_encode(1e30) == 0x7E
    assert oracle.fp8_e4m3_encode(-1e30) == 0xFE
    assert oracle.fp8_e4m3_encode(-0.0) == 0x80


def test_e2m1_encode_round_trips_every_code():
    for c in range(16):
        assert oracle.fp4_e2m1_encode(oracle.fp4_e2m1_to_double(c)) == c


def test_e2m1_encode_fixture():
    # magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 are codes 0..7; ties go to the even code
    table = [(0.25, 0), (0.26, 1), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6), (5.01, 7),
             (7.0, 7), (1e9, 7), (-0.75, 0x8 | 2), (-0.0, 0x8), (0.0, 0)]
    for y, code in table:
        assert oracle.fp4_e2m1_encode(y) == code, y


# ------------------------------------------------------------------ RMSNorm --

def test_rms_norm_fixture():
    got = oracle.rms_norm([[3.0, 4.0]], [1.0, 2.0], 0.0)
    r = math.sqrt((9 + 16) / 2)
    np.testing.assert_allclose(got, [[3 / r, 8 / r]], rtol=1e-15)
    np.testing.assert_allclose(oracle.rms_norm([[1.0, 1.0]], [1.0, 1.0], 1.0), [[2 ** -0.5, 2 ** -0.5]],
                               rtol=1e-15)
    np.testing.assert_array_equal(oracle.rms_norm([[0.0, 0.0]], [1.0, 1.0], 1e-6), [[0.0, 0.0]])


def test_rms_norm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 96))
    y = oracle.rms_norm(x, np.ones(96), 0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(axis=1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(oracle.rms_norm(x * 37.5, np.ones(96), 0.0), y, rtol=1e-13)


# ---------------------------------------------------------- rotary encoding --

def _rope_tables(max_pos, d_rope, base=10000.0):
    i = np.arange(d_rope // 2)
    theta = base ** (-2.0 * i / d_rope)
    ang = np.arange(max_pos)[:, None] * theta[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def test_rope_quarter_turn_fixture_pairs_adjacent_dims():
    # pair 0 turned by +90 degrees, pair 1 by 0; dims beyond d_rope untouched
    cos = np.array([[1.0, 1.0], [0.0, 1.0]], dtype=np.float32)
    sin = np.array([[0.0, 0.0], [1.0, 0.0]], dtype=np.float32)
    x = np.array([[[1.0, 0.0, 0.0, 0.0, 5.0, 7.0]]])
    np.testing.assert_array_equal(oracle.rope(x, [1], cos, sin, 4), [[[0.0, 1.0, 0.0, 0.0, 5.0, 7.0]]])
    np.testing.assert_array_equal(oracle.rope(x, [0], cos, sin, 4), x)
    x2 = np.array([[[0.0, 1.0, 2.0, 3.0, 0.0, 0.0]]])
    np.testing.assert_array_equal(oracle.rope(x2, [1], cos, sin, 4), [[[-1.0, 0.0, 2.0, 3.0, 0.0, 0.0]]])


def test_rope_keeps_pair_norms_and_depends_on_relative_position():
    rng = np.random.default_rng(1)
    d, d_rope = 16, 8
    cos, sin = _rope_tables(64, d_rope)
    q = rng.standard_normal((1, 2, d))
    k = rng.standard_normal((1, 2, d))
    a = oracle.rope(q, [9], cos, sin, d_rope)
    pn = lambda v: np.hypot(v[..., 0:d_rope:2], v[..., 1:d_rope:2])
    np.testing.assert_allclose(pn(a), pn(q), rtol=1e-6)
    np.testing.assert_array_equal(a[..., d_rope:], q[..., d_rope:])
    dots = []
    for m, n in [(9, 4), (20, 15), (50, 45)]:
        qa = oracle.rope(q, [m], cos, sin, d_rope)
        ka = oracle.rope(k, [n], cos, sin, d_rope)
        dots.append((qa * ka).sum(axis=-1))
    np.testing.assert_allclose(dots[1], dots[0], rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(dots[2], dots[0], rtol=1e-6, atol=1e-6)
    qa = oracle.rope(q, [9], cos, sin, d_rope)
    ka = oracle.rope(k, [5], cos, sin, d_rope)
    assert np.abs((qa * ka).sum(axis=-1) - dots[0]).max() > 1e-3


# ------------------------------------------------------------ the prepare step --

def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _prepare_inputs(rng, T, d_c, d_model, H, D, d_rope, max_pos=64):
    c_q = _bf16(rng.standard_normal((T, d_c)))
    h = _bf16(rng.standard_normal((T, d_model)))
    gamma = (0.5 + rng.random(d_c)).astype(np.float32)
    wq_b = _bf16(rng.standard_normal((H * D, d_c)) / math.sqrt(d_c))
    wk = _bf16(rng.standard_normal((D, d_model)) / math.sqrt(d_model))
    w_proj = _bf16(rng.standard_normal((H, d_model)) / math.sqrt(d_model))
    cos, sin = _rope_tables(max_pos, max(d_rope, 2))
    return c_q, h, gamma, wq_b, wk, w_proj, cos, sin


def test_prepare_with_permutation_weights():
    rng = np.random.default_rng(2)
    T, H, D, d_model = 3, 2, 8, 5
    d_c = H * D
    c_q, h, gamma, _, _, _, cos, sin = _prepare_inputs(rng, T, d_c, d_model, H, D, 0)
    perm = np.array([5, 11, 0, 3, 14, 9, 1, 7, 15, 2, 12, 6, 10, 4, 13, 8])   # not its own inverse
    P = np.zeros((d_c, d_c), dtype=np.float32)
    P[np.arange(d_c), perm] = 1.0
    Wk = rng.integers(-3, 4, size=(D, d_model)).astype(np.float32)
    Ww = rng.integers(-3, 4, size=(H, d_model)).astype(np.float32)
    q, w, k = oracle.indexer_prepare(c_q, gamma, 0.0, _bf16(P), h, _bf16(Wk), _bf16(Ww), cos, sin,
                                     np.zeros(T, np.int32), H, 0)
    cn = oracle.rms_norm(c_q.double().numpy(), gamma, 0.0)
    np.testing.assert_allclose(q.reshape(T, d_c), cn[:, perm], rtol=1e-15)
    hd = h.double().numpy()
    np.testing.assert_allclose(k, hd @ Wk.T.astype(np.float64), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(w, hd @ Ww.T.astype(np.float64), rtol=1e-14, atol=1e-14)
    # position 0 turns nothing: the same with a rotary part
    q2, _, k2 = oracle.indexer_prepare(c_q, gamma, 0.0, _bf16(P), h, _bf16(Wk), _bf16(Ww), cos, sin,
                                       np.zeros(T, np.int32), H, 2)
    np.testing.assert_array_equal(q2, q)
    np.testing.assert_array_equal(k2, k)


def test_prepare_scores_depend_on_relative_positions_only():
    rng = np.random.default_rng(4)
    T, d_c, d_model, H, D, d_rope = 4, 32, 24, 2, 16, 8
    c_q, h, gamma, wq_b, wk, w_proj, cos, sin = _prepare_inputs(rng, T, d_c, d_model, H, D, d_rope)
    pos = np.array([3, 7, 8, 20], np.int32)

    def scores(p):
        q, _, k = oracle.indexer_prepare(c_q, gamma, 1e-6, wq_b, h, wk, w_proj, cos, sin, p, H, d_rope)
        return np.einsum("thd,ud->thu", q, k)

    s0 = scores(pos)
    # exact up to the binary32 rounding of the cosine / sine tables
    np.testing.assert_allclose(scores(pos + 11), s0, rtol=1e-6, atol=1e-6)
    assert np.abs(scores(pos[[1, 0, 2, 3]]) - s0).max() > 1e-3


def test_prepare_query_is_invariant_to_the_latent_scale():
    rng = np.random.default_rng(5)
    T, d_c, d_model, H, D, d_rope = 2, 32, 24, 2, 16, 8
    c_q, h, gamma, wq_b, wk, w_proj, cos, sin = _prepare_inputs(rng, T, d_c, d_model, H, D, d_rope)
    pos = np.array([1, 6], np.int32)
    q, w, k = oracle.indexer_prepare(c_q, gamma, 0.0, wq_b, h, wk, w_proj, cos, sin, pos, H, d_rope)
    q2, w2, k2 = oracle.indexer_prepare(c_q * 8, gamma, 0.0, wq_b, h, wk, w_proj, cos, sin, pos, H, d_rope)
    np.testing.assert_allclose(q2, q, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(w2, w)
    np.testing.assert_array_equal(k2, k)


# ----------------------------------------------------------- key-cache write --

def test_key_rows_fp8_equal_the_torch_cast_of_the_scaled_row():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((7, 128)) * np.exp2(rng.integers(-6, 6, size=(7, 1)))).astype(np.float32)
    x[3] = 0.0
    codes, scale = oracle.key_rows_f32(x, np.zeros(7, np.int32), np.ones((1, 1), np.float32),
                                       np.zeros((1, 1), np.float32), 0, oracle.FP8)
    amax = np.abs(x).max(axis=1)
    want_scale = np.where(amax > 0, amax / np.float32(448), np.float32(1)).astype(np.float32)
    np.testing.assert_array_equal(scale, want_scale)
    ref = torch.from_numpy(x / want_scale[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, ref)
    # the largest magnitude of every nonzero row is stored as +-448
    top = np.abs(x).argmax(axis=1)
    for r in range(7):
        if amax[r] > 0:
            assert codes[r, top[r]] & 0x7F == 0x7E
    assert scale[3] == 1.0 and not codes[3].any()


def test_key_rows_fp4_pairs_and_nearest_magnitudes():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 128)).astype(np.float32)
    pairs, scale = oracle.key_rows_f32(x, np.zeros(5, np.int32), np.ones((1, 1), np.float32),
                                       np.zeros((1, 1), np.float32), 0, oracle.FP4)
    assert pairs.shape == (5, 64)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for r in range(5):
        np.testing.assert_array_equal(scale[r], np.abs(x[r]).max() / np.float32(6))
        y = (x[r] / scale[r]).astype(np.float64)
        lo = np.array([oracle.fp4_e2m1_to_double(int(b) & 0xF) for b in pairs[r]])
        hi = np.array([oracle.fp4_e2m1_to_double(int(b) >> 4) for b in pairs[r]])
        dec = np.empty(128)
        dec[0::2], dec[1::2] = lo, hi
        dist = np.abs(np.abs(y)[:, None] - grid[None, :]).min(axis=1)
        np.testing.assert_array_equal(np.abs(dec - y), dist)
        assert (np.sign(dec) * np.sign(y) >= 0).all()


def test_key_rows_bf16_and_rotary_part():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((4, 128)).astype(np.float32)
    cos, sin = _rope_tables(32, 64)
    pos = np.array([0, 3, 17, 31], np.int32)
    bits, none = oracle.key_rows_f32(x, pos, cos, sin, 64, oracle.BF16)
    assert none is None
    got = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    want = oracle.rope(x.astype(np.float64)[:, None, :], pos, cos, sin, 64)[:, 0, :]
    # binary32 rotation, then one rounding to bf16
    np.testing.assert_allclose(got, want, rtol=2 ** -8, atol=1e-6)
    np.testing.assert_array_equal(got[:, 64:], torch.from_numpy(x[:, 64:]).bfloat16().double().numpy())
    np.testing.assert_array_equal(got[0], torch.from_numpy(x[0]).bfloat16().double().numpy())
